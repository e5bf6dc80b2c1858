"""The sequence split on the GPU against the oracle's unsplit scan.

R ranks are emulated in one process on one GPU: each rank's SegmentScan runs
its kernels (ssm_split_conv_tail, ssm_scan_fwd, ssm_split_cum_delta,
ssm_split_combine, ssm_split_fixup) on its own token segment, and the two
exchanges are stacks of the ranks' tensors.  No kernel waits on another.
The joined y, every rank's outgoing state and the last rank's conv state are
compared with the oracle's scan of the whole sequence (and of its prefixes).
Segment boundaries are ragged and unequal; the cases cover the Mamba-1
kernel, the tensor-core Mamba-2 kernel (bf16, headdim 64, dstate 128) and the
SIMT Mamba-2 kernel.
"""
import numpy as np
import pytest
import torch

import oracle
from state_space_model_conv1d_b200 import seq_split
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import assert_close, oracle_scan, to_dev

pytestmark = pytest.mark.gpu
M1, M2 = oracle.MAMBA1, oracle.MAMBA2
SEQ = ("x", "z", "dt", "B", "C")


def run_split_gpu(mode, t, bounds):
    R = len(bounds) - 1
    segs = []
    for r in range(R):
        lo, hi = bounds[r], bounds[r + 1]
        s = {k: (None if t.get(k) is None else t[k][:, lo:hi]) for k in SEQ}
        segs.append(seq_split.SegmentScan(mode, r, R, s["x"], s["dt"], t["A"], s["B"], s["C"], D=t["D"], z=s["z"],
                                          dt_bias=t["dt_bias"], h0=t["h0"], conv_w=t.get("conv_w"),
                                          conv_b=t.get("conv_b"), conv_state_in=t.get("conv_state_in")))
    tails = [s.tail() for s in segs]
    tails = None if tails[0] is None else torch.stack(tails)
    pairs = torch.stack([s.scan(tails) for s in segs])
    outs = [s.join(pairs) for s in segs]
    torch.cuda.synchronize()
    f = lambda a: None if a is None else a.float().cpu().numpy().astype(np.float64)
    y = np.concatenate([f(o[0]) for o in outs], axis=1)
    return y, [f(o[1]) for o in outs], f(outs[-1][2])


def _prefix(d, T):
    return {k: (None if v is None else (v[:, :T] if k in SEQ else v)) for k, v in d.items()}


def _check(mode, d, dtype, bounds):
    y, houts, conv_out = run_split_gpu(mode, to_dev(d, dtype), bounds)
    ry, rh, rc = oracle_scan(mode, d)
    assert_close(y, ry, dtype, "y")
    assert_close(houts[-1], rh, dtype, "h_out of the last rank")
    for r in range(len(bounds) - 2):
        _, rhr, _ = oracle_scan(mode, _prefix(d, bounds[r + 1]))
        assert_close(houts[r], rhr, dtype, f"h_out of rank {r}")
    if rc is not None:
        np.testing.assert_array_equal(conv_out, rc)


@pytest.mark.parametrize("dtype,bounds", [("bf16", [0, 100, 229, 300]), ("f32", [0, 64, 131]),
                                          ("bf16", [0, 3, 40, 41 + 64, 170])])
def test_mamba1(dtype, bounds):
    d = W.mamba1_inputs(901, 2, bounds[-1], 96, 16, dtype=dtype, conv_bias=True, conv_state=True)
    _check(M1, d, dtype, bounds)


def test_mamba1_no_gate_no_conv():
    d = W.mamba1_inputs(902, 3, 150, 40, 8, d_conv=0, dtype="f32", with_z=False)
    _check(M1, d, "f32", [0, 50, 51, 150])


@pytest.mark.parametrize("bounds", [[0, 128, 320], [0, 77, 200, 320]])
def test_mamba2_tensor_core_shape(bounds):
    d = W.mamba2_inputs(903, 2, bounds[-1], 4, 64, 2, 128, dtype="bf16", conv_bias=True, conv_state=True)
    _check(M2, d, "bf16", bounds)


@pytest.mark.parametrize("H,G,gate", [(4, 2, True), (6, 1, False), (2, 2, True)])
def test_mamba2_tensor_core_fixup_tiles(H, G, gate):
    """The tensor-core fix-up over several 128-token tiles with a ragged last
    one, one to six heads per group (both accumulator buffers), with and
    without the gate."""
    d = W.mamba2_inputs(915 + H, 2, 701, H, 64, G, 128, dtype="bf16", conv_bias=True, conv_state=True)
    if not gate:
        d["z"] = None
    _check(M2, d, "bf16", [0, 300, 701])


@pytest.mark.parametrize("dtype,P,N,bounds", [("f32", 8, 16, [0, 30, 61, 95, 130]), ("bf16", 48, 64, [0, 90, 200]),
                                              ("f32", 64, 256, [0, 40, 97])])
def test_mamba2_simt_shapes(dtype, P, N, bounds):
    d = W.mamba2_inputs(904, 2, bounds[-1], 4, P, 2, N, dtype=dtype, conv_bias=True, conv_state=True)
    _check(M2, d, dtype, bounds)


def test_single_rank_is_the_plain_scan():
    d = W.mamba2_inputs(905, 2, 96, 4, 8, 2, 16, dtype="f32", conv_bias=True, conv_state=True)
    _check(M2, d, "f32", [0, 96])


def test_mamba2_scalar_fixup_dstate_not_multiple_of_4():
    """dstate 5: the Mamba-2 fix-up's scalar path (no float4 state rows)."""
    d = W.mamba2_inputs(906, 2, 30, 4, 8, 2, 5, dtype="f32", conv_bias=True, conv_state=True)
    _check(M2, d, "f32", [0, 13, 30])


@pytest.mark.parametrize("K", [0, 1])
@pytest.mark.parametrize("shape", ["tensor_core", "simt"])
def test_mamba2_conv_width_0_and_1(K, shape):
    """A Mamba-2 split with no conv history to hand on (width 0 or 1): the
    fix-up stages the raw C (width 0) or its pointwise conv (width 1)."""
    P, N, dtype = (64, 128, "bf16") if shape == "tensor_core" else (16, 24, "f32")
    d = W.mamba2_inputs(907 + K, 2, 130, 4, P, 2, N, d_conv=K, dtype=dtype, conv_bias=K > 0, conv_state=False)
    _check(M2, d, dtype, [0, 13, 70, 130])


@pytest.mark.parametrize("mode,shape", [(M1, None), (M2, "tensor_core"), (M2, "simt")])
def test_rank_with_no_tokens(mode, shape):
    """Without a conv a rank may hold no tokens: it passes the state through
    (its pair is (sum of delta 0, zero state)) and writes no y."""
    if mode == M1:
        d = W.mamba1_inputs(909, 2, 30, 40, 8, d_conv=0, dtype="f32", with_z=True)
        dtype = "f32"
    else:
        P, N, dtype = (64, 128, "bf16") if shape == "tensor_core" else (16, 24, "f32")
        d = W.mamba2_inputs(910, 2, 30, 4, P, 2, N, d_conv=0, dtype=dtype, conv_state=False)
    _check(mode, d, dtype, [0, 13, 13, 30])


@pytest.mark.parametrize("mode,T,U", [(M2, 5000, 40), (M1, 700, 70), (M2, 256, 8), (M2, 257, 3)])
def test_cum_delta_prefix_sums(mode, T, U):
    """ssm_split_cum_delta against the running sum of softplus(dt + dt_bias)
    in fp64: several token blocks of 256 (more than 16, one, and one plus a
    single token), a unit count that is not a multiple of 32; the total alone
    (no cs requested) agrees with the total of the blocked path."""
    from state_space_model_conv1d_b200 import ops
    rng = np.random.default_rng(930 + T + U)
    b = 2
    dt = W.round_bf16(rng.standard_normal((b, T, U)).astype(np.float32))
    bias = rng.uniform(-4.0, -1.0, U).astype(np.float32)
    ref = np.cumsum(np.log1p(np.exp(dt.astype(np.float64) + bias.astype(np.float64))), axis=1)
    dev = torch.from_numpy(dt).to("cuda", torch.bfloat16)
    tb = torch.from_numpy(bias).cuda()
    if mode == M1:
        x = torch.zeros((b, T, U), dtype=torch.bfloat16, device="cuda")
        Bm = torch.zeros((b, T, 4), dtype=torch.bfloat16, device="cuda")
        A = torch.zeros((U, 4), dtype=torch.float32, device="cuda")
    else:
        x = torch.zeros((b, T, U, 8), dtype=torch.bfloat16, device="cuda")
        Bm = torch.zeros((b, T, 1, 16), dtype=torch.bfloat16, device="cuda")
        A = torch.zeros((U,), dtype=torch.float32, device="cuda")
    cs, sd = ops.split_cum_delta(mode, x, dev, A, Bm, Bm, dt_bias=tb)
    _, sd_only = ops.split_cum_delta(mode, x, dev, A, Bm, Bm, dt_bias=tb, cum=False)
    torch.cuda.synchronize()
    got = cs.cpu().numpy().astype(np.float64)
    # softplus on the GPU is within 2e-5 relative of log1p(exp(u)) in each of its regimes
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1.0)) < 5e-5
    np.testing.assert_allclose(sd.cpu().numpy(), ref[:, -1], rtol=5e-5)
    np.testing.assert_allclose(sd_only.cpu().numpy(), sd.cpu().numpy(), rtol=1e-6)
    np.testing.assert_array_equal(sd.cpu().numpy(), got[:, -1].astype(np.float32))


# The combine reads every rank's (sum of delta, h_loc) in place from one
# gathered buffer of packed pairs (rank strides), or from dense stacks; both
# give the same bits, and both the fold H_k = exp(A sum_delta_k) H_{k-1} + h_k
# computed here in fp64 (the combine uses the MUFU exp: 2^-21 relative).
@pytest.mark.parametrize("mode,state", [(M2, (3, 4, 8, 16)), (M1, (3, 24, 16)), (M1, (2, 10, 5))])
@pytest.mark.parametrize("pad", [0, 3])          # rank strides a multiple of 4, or not (copied)
def test_split_combine_strided_pairs(mode, state, pad):
    from state_space_model_conv1d_b200 import ops
    rng = np.random.default_rng(601 + len(state) + state[-1] + pad)
    R, rank = 3, 2
    b = state[0]
    U = state[1]
    A = -rng.uniform(0.1, 1.0, size=(U,) if mode == M2 else state[1:]).astype(np.float32)
    sd = rng.uniform(0.1, 2.0, size=(R, b, U)).astype(np.float32)
    hl = rng.standard_normal((R,) + state).astype(np.float32)
    dev = lambda a: torch.from_numpy(a).cuda()
    h_in, h_out = ops.split_combine(mode, dev(A), dev(sd), dev(hl), rank)
    nsd, nhl = b * U, int(np.prod(state))
    off = (nsd + 3) // 4 * 4
    buf = torch.full((R, off + nhl + pad + 4), float("nan"), dtype=torch.float32, device="cuda")
    buf[:, :nsd] = dev(sd.reshape(R, -1))
    buf[:, off:off + nhl] = dev(hl.reshape(R, -1))
    s_in, s_out = ops.split_combine(mode, dev(A), buf[:, :nsd].unflatten(1, (b, U)),
                                    buf[:, off:off + nhl].unflatten(1, state), rank)
    torch.cuda.synchronize()
    assert torch.equal(s_in, h_in) and torch.equal(s_out, h_out)
    # fp64 fold
    a64 = A.astype(np.float64)
    H = hl[0].astype(np.float64)
    before = np.zeros_like(H)
    for k in range(1, rank + 1):
        before = H
        if mode == M2:
            dec = np.exp(a64[None, :, None, None] * sd[k].astype(np.float64)[:, :, None, None])
        else:
            dec = np.exp(a64[None] * sd[k].astype(np.float64)[:, :, None])
        H = dec * H + hl[k]
    np.testing.assert_allclose(h_in.cpu().numpy(), before, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(h_out.cpu().numpy(), H, rtol=1e-5, atol=1e-5)
