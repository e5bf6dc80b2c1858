"""The bounds-checked build on valid calls: every kernel of the path runs with
its index checks compiled in, the results still match the fp64 oracle, and no
check fires (the device-wide record stays clear).  A check that fires records
the first failing index and skips the access instead of trapping, so the
record is read back through ssm_bounds_record."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import _abi
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import assert_close, check_scan, to_dev

pytestmark = pytest.mark.gpu


def _record(chk, clear=0):
    code, site, idx, ext = C.c_int32(-1), C.c_int32(-1), C.c_int64(-1), C.c_int64(-1)
    st = chk.ssm_bounds_record(C.byref(code), C.byref(site), C.byref(idx), C.byref(ext), clear)
    assert st == _abi.SSM_OK
    return code.value, site.value, idx.value, ext.value


@pytest.fixture
def checked(monkeypatch):
    chk = _abi.checked_lib()
    assert chk.ssm_check_bounds_enabled() == 1
    _record(chk, clear=1)
    monkeypatch.setattr(_abi, "lib", lambda: chk)       # the package's calls go to the checked build
    yield chk


def test_checked_build_runs_clean(checked):
    # Mamba-2 packed varlen on the tensor-core path (B / C pre-pass + SSD kernel)
    lengths = [130, 0, 64, 1, 77]
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(1201, 1, int(cu[-1]), 4, 64, 2, 128, dtype="bf16", conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    check_scan(oracle.MAMBA2, d, "bf16", what="checked SSD varlen")
    # Mamba-2 on the SIMT path (fp32)
    check_scan(oracle.MAMBA2, W.mamba2_inputs(1202, 2, 70, 3, 40, 3, 32, dtype="f32", conv_state=True), "f32",
               what="checked M2 SIMT")
    # Mamba-1: the time-parallel form (few channels) and the sequential form (enough warps)
    check_scan(oracle.MAMBA1, W.mamba1_inputs(1203, 2, 150, 48, 16, dtype="bf16", conv_state=True), "bf16",
               what="checked M1 time-parallel")
    check_scan(oracle.MAMBA1, W.mamba1_inputs(1204, 8, 40, 1056, 16, dtype="bf16", conv_state=True), "bf16",
               what="checked M1 sequential")
    # decode
    g = W.decode_inputs(1205, 4, 8, 64, 2, 128, nsets=1, dtype="bf16")
    t = to_dev(g, "bf16")
    st, cs = t["state"].clone(), t["conv_state"].clone()
    y = ssm.state_update(oracle.MAMBA2, st, cs, t["x"][0], t["dt"][0], t["A"], t["B"][0], t["C"][0], D=t["D"],
                         z=t["z"][0], dt_bias=t["dt_bias"], conv_w=t["conv_w"])
    torch.cuda.synchronize()
    rs, rc = g["state"].astype(np.float64), g["conv_state"].astype(np.float64)
    ry = oracle.state_update(oracle.MAMBA2, rs, rc, g["x"][0], g["dt"][0], g["A"], g["B"][0], g["C"][0], D=g["D"],
                             z=g["z"][0], dt_bias=g["dt_bias"], conv_w=g["conv_w"])
    assert_close(y.float().cpu().numpy(), ry, "bf16", "checked decode y")
    assert_close(st.cpu().numpy(), rs, "bf16", "checked decode state")
    # backward (Mamba-1, fp32)
    m = W.mamba1_inputs(1206, 1, 50, 16, 4, dtype="f32", conv_state=True)
    tm = to_dev(m, "f32")
    dy = np.random.default_rng(1207).standard_normal(m["x"].shape).astype(np.float32).astype(np.float64)
    gg = ssm.scan_bwd(oracle.MAMBA1, tm["x"], tm["dt"], tm["A"], tm["B"], tm["C"], torch.from_numpy(dy).float().cuda(),
                      D=tm["D"], z=tm["z"], dt_bias=tm["dt_bias"], h0=tm["h0"], conv_w=tm["conv_w"],
                      conv_state_in=tm["conv_state_in"])
    torch.cuda.synchronize()
    rg = oracle.scan_bwd(oracle.MAMBA1, m["x"], m["dt"], m["A"], m["B"], m["C"], dy, D=m["D"], z=m["z"],
                         dt_bias=m["dt_bias"], h0=m["h0"], conv_w=m["conv_w"], conv_state_in=m["conv_state_in"])
    assert_close(gg["dx"].cpu().numpy(), rg["dx"], "f32", "checked backward dx")
    code, site, idx, ext = _record(checked)
    assert code == 0, f"bounds check fired: site {site}, index {idx}, extent {ext}"
