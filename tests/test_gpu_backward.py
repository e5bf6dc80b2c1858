"""Backward of the conv + scan on the GPU against the fp64 oracle's backward.

The oracle's backward is itself pinned against central finite differences of
the forward oracle (tests/oracle_pins.py); here every gradient the CUDA path
returns is compared with it element by element: dx, dz, ddt, dB, dC (raw,
before the conv), dA, dD, ddt_bias, dh0, dconv_w, dconv_b, dconv_state_in.
"""
import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu
M1, M2 = oracle.MAMBA1, oracle.MAMBA2
NAMES = ("dx", "dz", "ddt", "dB", "dC", "dA", "dD", "ddt_bias", "dh0", "dconv_w", "dconv_b", "dconv_state_in")


def _check(mode, d, dtype, softplus=True, upstream=True, seed=0):
    cu = d.get("cu_seqlens")
    t = to_dev(d, dtype)
    rng = np.random.default_rng(seed)
    y, hf, cs = oracle.scan_fwd(mode, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d.get("D"), z=d.get("z"),
                                dt_bias=d.get("dt_bias"), h0=d.get("h0"), cu_seqlens=cu, conv_w=d.get("conv_w"),
                                conv_b=d.get("conv_b"), conv_state_in=d.get("conv_state_in"), delta_softplus=softplus)
    dy = rng.standard_normal(y.shape)
    dy = W.round_bf16(dy) if dtype == "bf16" else dy.astype(np.float32).astype(np.float64)
    dhf = rng.standard_normal(hf.shape).astype(np.float32).astype(np.float64) if upstream else None
    dcs = None
    if upstream and cs is not None:
        dcs = rng.standard_normal(cs.shape)
        dcs = W.round_bf16(dcs) if dtype == "bf16" else dcs.astype(np.float32).astype(np.float64)
    ref = oracle.scan_bwd(mode, d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d.get("D"), z=d.get("z"),
                          dt_bias=d.get("dt_bias"), h0=d.get("h0"), cu_seqlens=cu, conv_w=d.get("conv_w"),
                          conv_b=d.get("conv_b"), conv_state_in=d.get("conv_state_in"), delta_softplus=softplus,
                          dh_final=dhf, dconv_state_out=dcs)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    got = ssm.scan_bwd(mode, t["x"], t["dt"], t["A"], t["B"], t["C"], torch.from_numpy(dy).to("cuda", tdt),
                       D=t.get("D"), z=t.get("z"), dt_bias=t.get("dt_bias"), h0=t.get("h0"),
                       cu_seqlens=t.get("cu_seqlens"), conv_w=t.get("conv_w"), conv_b=t.get("conv_b"),
                       conv_state_in=t.get("conv_state_in"), delta_softplus=softplus,
                       dh_final=None if dhf is None else torch.from_numpy(dhf).float().cuda(),
                       dconv_state_out=None if dcs is None else torch.from_numpy(dcs).to("cuda", tdt))
    torch.cuda.synchronize()
    for k in NAMES:
        if ref[k] is None:
            assert got[k] is None, k
            continue
        e = rel_err(got[k].cpu().numpy(), ref[k])
        assert e <= TOL[dtype], f"{k}: max|err|/max|ref| = {e:.3e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mamba1(dtype):
    d = W.mamba1_inputs(950, 2, 40, 40, 16, dtype=dtype, conv_bias=True, conv_state=True)
    _check(M1, d, dtype, seed=1)


def test_mamba1_varlen_no_conv_state():
    lengths = [21, 0, 33, 5]
    d = W.mamba1_inputs(951, 1, sum(lengths), 24, 8, dtype="f32", conv_bias=False, conv_state=False,
                        nseqs=len(lengths))
    d["cu_seqlens"] = W.cu_from_lengths(lengths)
    _check(M1, d, "f32", seed=2)


def test_mamba1_no_conv_softplus_off():
    d = W.mamba1_inputs(952, 1, 35, 16, 4, d_conv=0, dtype="f32")
    d["dt"] = np.abs(d["dt"]) * 0.05
    d["dt_bias"] = np.full_like(d["dt_bias"], 0.01)
    _check(M1, d, "f32", softplus=False, upstream=False, seed=3)


@pytest.mark.parametrize("dtype,H,P,G,N", [("f32", 4, 8, 2, 16), ("bf16", 2, 64, 1, 128), ("f32", 2, 4, 2, 256)])
def test_mamba2(dtype, H, P, G, N):
    d = W.mamba2_inputs(953, 2, 37, H, P, G, N, dtype=dtype, conv_bias=True, conv_state=True)
    _check(M2, d, dtype, seed=4)


def test_mamba2_varlen():
    lengths = [18, 0, 31, 3]
    d = W.mamba2_inputs(954, 1, sum(lengths), 4, 8, 2, 16, dtype="f32", conv_bias=True, conv_state=True,
                        nseqs=len(lengths))
    d["cu_seqlens"] = W.cu_from_lengths(lengths)
    _check(M2, d, "f32", seed=5)


def test_mamba2_no_conv():
    d = W.mamba2_inputs(955, 1, 29, 4, 4, 1, 16, d_conv=0, dtype="f32")
    _check(M2, d, "f32", seed=6)
