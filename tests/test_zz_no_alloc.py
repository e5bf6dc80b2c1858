"""ssm_scan_fwd_noalloc: the scan for callers that cannot allocate device
memory (graph captures that must not allocate, runtimes that own the memory
pool, plugins handed buffers but no allocator).  It must give the same
results as ssm_scan_fwd with a caller-allocated workspace.

Kept in its own file, collected last, so a failure here comes after every
other test has run.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import _abi, ops
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(t, y, hf, cso):
    """Call the allocation-free entry point through the C ABI."""
    a = ops._scan_args(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], t["z"], t["dt_bias"], t["h0"],
                       hf, t["cu_seqlens"], t["conv_w"], t["conv_b"], t["conv_state_in"], cso, y, True, 0)
    st = _abi.lib().ssm_scan_fwd_noalloc(C.byref(a), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _abi.SSM_OK, _abi.lib().ssm_status_string(st)


def _case(seed):
    # packed varlen Mamba-2 on the tensor-core path: needs the error word, the
    # schedule and the conv'd B / C tiles, well inside the fixed scratch
    lengths = [130, 0, 64, 1, 77]
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(seed, 1, int(cu[-1]), 4, 64, 2, 128, dtype="bf16", conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    return to_dev(d, "bf16")


@pytest.mark.parametrize("call", [0, 1])
def test_noalloc_matches_workspace_entry_point(call):
    """Two calls in a row (different inputs), each against ssm_scan_fwd."""
    t = _case(900 + call)
    need = ssm.scan_workspace_size(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"],
                                   cu_seqlens=t["cu_seqlens"], conv_w=t["conv_w"])
    assert 0 < need <= 4 << 20
    y_ref, h_ref, c_ref = ssm.scan_fwd(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                       dt_bias=t["dt_bias"], h0=t["h0"], cu_seqlens=t["cu_seqlens"],
                                       conv_w=t["conv_w"], conv_b=t["conv_b"], conv_state_in=t["conv_state_in"])
    y = torch.full_like(y_ref, float("nan"))
    hf = torch.full_like(h_ref, float("nan"))
    cso = torch.full_like(c_ref, float("nan"))
    _noalloc(t, y, hf, cso)
    torch.cuda.synchronize()
    # both entry points run the same kernels, which use no atomics and a fixed
    # reduction order, so the results must agree bit for bit (the tolerance
    # the other tests use, max|err|/max|ref| <= 2e-2, is checked as well)
    for got, ref, what in ((y, y_ref, "y"), (hf, h_ref, "h_final"), (cso, c_ref, "conv_state_out")):
        g, r = got.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.all(np.isfinite(g)), what
        assert rel_err(g, r) <= TOL["bf16"], what
        ib = torch.int16 if got.dtype == torch.bfloat16 else torch.int32
        assert torch.equal(got.view(ib), ref.view(ib)), f"{what}: not bit-identical to ssm_scan_fwd"


def test_noalloc_rejects_oversized_workspace():
    """Shapes whose workspace exceeds the fixed scratch are refused up front."""
    d = W.mamba2_inputs(910, 4, 4096, 2, 64, 8, 128, dtype="bf16", conv_state=False)
    t = to_dev(d, "bf16")
    need = ssm.scan_workspace_size(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], conv_w=t["conv_w"])
    assert need > 4 << 20
    y = torch.empty_like(t["x"])
    a = ops._scan_args(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], t["z"], t["dt_bias"], t["h0"],
                       None, None, t["conv_w"], None, None, None, y, True, 0)
    st = _abi.lib().ssm_scan_fwd_noalloc(C.byref(a), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _abi.SSM_ERR_WORKSPACE


def test_noalloc_keeps_rows_whole_when_segment_states_do_not_fit():
    """A fixed-length batch the library would cut into token segments needs
    their states in the workspace (over the fixed scratch here); the no-alloc
    entry point then runs the rows whole, bit for bit like segments=1."""
    d = W.mamba2_inputs(912, 2, 1024, 8, 64, 1, 128, dtype="bf16", conv_state=True)
    t = to_dev(d, "bf16")
    kw = dict(conv_w=t["conv_w"])
    assert ssm.scan_segments(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], z=t["z"], **kw) > 1
    assert ssm.scan_workspace_size(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], **kw) > 4 << 20
    assert ssm.scan_workspace_size(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], segments=1, **kw) <= 4 << 20
    y_ref, h_ref, c_ref = ssm.scan_fwd(oracle.MAMBA2, t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                       dt_bias=t["dt_bias"], h0=t["h0"], conv_w=t["conv_w"], conv_b=t["conv_b"],
                                       conv_state_in=t["conv_state_in"], segments=1)
    y = torch.full_like(y_ref, float("nan"))
    hf = torch.full_like(h_ref, float("nan"))
    cso = torch.full_like(c_ref, float("nan"))
    t["cu_seqlens"] = None
    _noalloc(t, y, hf, cso)
    torch.cuda.synchronize()
    for got, ref, what in ((y, y_ref, "y"), (hf, h_ref, "h_final"), (cso, c_ref, "conv_state_out")):
        ib = torch.int16 if got.dtype == torch.bfloat16 else torch.int32
        assert torch.equal(got.view(ib), ref.view(ib)), f"{what}: not bit-identical to whole rows"
