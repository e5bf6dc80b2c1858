"""CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Sizes span several CTA tiles and chunks with ragged tails (channel blocks of
32, token chunks of 32 / 64), plus the degenerate cases: one token, empty
sequences, no gate / skip / bias / initial state, strided views.
"""
import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import TOL, assert_close, check_scan, gpu_scan, oracle_scan, rel_err, to_dev

pytestmark = pytest.mark.gpu
M1, M2 = oracle.MAMBA1, oracle.MAMBA2


# ------------------------------------------------------------------ conv
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 4, 5])
@pytest.mark.parametrize("C_", [64, 20])          # vector path and the element path
def test_conv1d(dtype, K, C_):
    rng = np.random.default_rng(100 + K + C_)
    b, T = 3, 77
    x = W.round_bf16(rng.standard_normal((b, T, C_)).astype(np.float32)) if dtype == "bf16" else \
        rng.standard_normal((b, T, C_)).astype(np.float32)
    w = rng.uniform(-0.5, 0.5, (C_, K)).astype(np.float32)
    bias = rng.uniform(-0.5, 0.5, C_).astype(np.float32)
    st = W.round_bf16(rng.standard_normal((b, C_, max(K - 1, 0))).astype(np.float32)) if K > 1 else None
    t = to_dev(dict(x=x, conv_state_in=st), dtype)
    so = torch.empty_like(t["conv_state_in"]) if K > 1 else None
    out = ssm.conv1d_fwd(t["x"], torch.from_numpy(w).cuda(), torch.from_numpy(bias).cuda(),
                         state_in=t["conv_state_in"], state_out=so, activation=True)
    torch.cuda.synchronize()
    ref, rso = oracle.conv1d_fwd(x, w, b=bias, state_in=st, activation=True)
    assert_close(out.float().cpu().numpy(), ref, dtype, "conv out")
    if K > 1:
        assert_close(so.float().cpu().numpy(), rso, dtype, "conv state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv1d_varlen_inplace_state(dtype):
    rng = np.random.default_rng(7)
    lengths = [40, 0, 1, 2, 70, 33]
    cu = W.cu_from_lengths(lengths)
    tot, C_, K = int(cu[-1]), 48, 4
    x = rng.standard_normal((1, tot, C_)).astype(np.float32)
    st = rng.standard_normal((len(lengths), C_, K - 1)).astype(np.float32)
    if dtype == "bf16":
        x, st = W.round_bf16(x), W.round_bf16(st)
    w = rng.uniform(-0.5, 0.5, (C_, K)).astype(np.float32)
    t = to_dev(dict(x=x, conv_state_in=st, cu_seqlens=cu), dtype)
    state = t["conv_state_in"].clone()
    out = ssm.conv1d_fwd(t["x"], torch.from_numpy(w).cuda(), state_in=state, state_out=state,
                         cu_seqlens=t["cu_seqlens"], activation=False)
    torch.cuda.synchronize()
    ref, rso = oracle.conv1d_fwd(x, w, state_in=st, cu_seqlens=cu, activation=False)
    assert_close(out.float().cpu().numpy(), ref, dtype, "varlen conv out")
    assert_close(state.float().cpu().numpy(), rso, dtype, "in-place conv state")


# --------------------------------------------------------------- Mamba-1
M1_CASES = [
    # (b, T, D, N, K, dtype)
    (1, 64, 16, 4, 4, "f32"),         # the tiny fp32 workload
    (2, 1, 32, 16, 4, "bf16"),        # a single token
    (2, 130, 40, 16, 4, "bf16"),      # ragged channel block and token chunk
    (3, 200, 64, 16, 4, "f32"),
    (2, 97, 96, 8, 3, "bf16"),
    (1, 150, 32, 64, 2, "f32"),       # the widest dstate of the path
    (2, 70, 24, 13, 4, "f32"),        # dstate not a multiple of 4
    (2, 65, 64, 16, 0, "bf16"),       # no conv in front
    (1, 2113, 48, 16, 4, "f32"),      # fp32 over many chunks (66 of 32 tokens) and a ragged tail
    (4, 130, 640, 16, 4, "bf16"),     # time-parallel form with 16-channel blocks (160 CTAs)
    (3, 200, 1000, 32, 3, "f32"),     # the same, dstate 32, a ragged channel block
]


@pytest.mark.parametrize("b,T,D,N,K,dtype", M1_CASES)
def test_mamba1(b, T, D, N, K, dtype):
    d = W.mamba1_inputs(300 + T + D + N, b, T, D, N, d_conv=K, dtype=dtype, conv_bias=True, conv_state=True)
    check_scan(M1, d, dtype, what=f"M1 b{b} T{T} D{D} N{N} K{K}")


def test_mamba1_optional_inputs_absent():
    d = W.mamba1_inputs(310, 2, 90, 32, 16, dtype="bf16", with_h0=False, with_z=False)
    d["D"] = None
    d["dt_bias"] = None
    check_scan(M1, d, "bf16", what="M1 minimal")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mamba1_strided_views(dtype):
    """x and z as non-contiguous views of one projection row (the llama.cpp
    x/z view bug)."""
    d = W.mamba1_inputs(320, 2, 100, 48, 16, dtype=dtype, conv_state=True)
    check_scan(M1, d, dtype, views=True, what="M1 views")


# --------------------------------------------------------------- Mamba-2
M2_CASES = [
    # (b, T, H, P, G, N, K, dtype)
    (2, 1, 4, 64, 2, 128, 4, "bf16"),
    (2, 100, 4, 64, 2, 128, 4, "bf16"),
    (1, 70, 6, 40, 3, 32, 4, "f32"),      # headdim not a multiple of 32
    (2, 65, 4, 32, 1, 16, 3, "f32"),
    (1, 40, 2, 64, 2, 200, 4, "bf16"),    # dstate beyond 128, not a power of two
    (2, 33, 4, 64, 4, 64, 0, "bf16"),     # no conv
    (1, 2081, 2, 64, 1, 128, 4, "f32"),   # fp32 over many chunks and a ragged tail
]


@pytest.mark.parametrize("b,T,H,P,G,N,K,dtype", M2_CASES)
def test_mamba2(b, T, H, P, G, N, K, dtype):
    d = W.mamba2_inputs(400 + T + H + P + N, b, T, H, P, G, N, d_conv=K, dtype=dtype, conv_bias=True,
                        conv_state=True)
    check_scan(M2, d, dtype, what=f"M2 b{b} T{T} H{H} P{P} G{G} N{N}")


# Rows cut into token segments on the tensor-core path: a state-only pass over
# every segment but the last, then one scan CTA per (segment, head) from the
# folded entering state.  Requested counts become runs of whole chunks.
SEG_CASES = [
    # (b, T, H, G, K, segments)
    (2, 300, 4, 2, 4, 2),      # 5 chunks: runs of 3 and 2, the last chunk ragged
    (1, 520, 2, 1, 4, 4),      # 9 chunks: three runs of 3
    (2, 256, 4, 4, 3, 3),      # 4 chunks asked in 3 runs: two runs of 2
    (1, 640, 2, 2, 0, 5),      # no conv in front
    (1, 200, 2, 1, 2, 2),      # conv width 2
    (1, 65, 2, 1, 4, 2),       # the last run is a single token
    (1, 4160, 2, 1, 4, 0),     # 65 chunks, count chosen by the library
]


@pytest.mark.parametrize("b,T,H,G,K,segments", SEG_CASES)
def test_mamba2_segments(b, T, H, G, K, segments):
    d = W.mamba2_inputs(450 + T + H + K, b, T, H, 64, G, 128, d_conv=K, dtype="bf16", conv_bias=True,
                        conv_state=True)
    check_scan(M2, d, "bf16", segments=segments, what=f"M2 segments={segments} b{b} T{T} H{H} G{G} K{K}")


def test_mamba2_segments_match_unsegmented():
    """Segmenting changes only the fp32 rounding of the carried state."""
    d = W.mamba2_inputs(460, 2, 1000, 4, 64, 2, 128, dtype="bf16", conv_bias=True, conv_state=True)
    t = to_dev(d, "bf16")
    y1, h1, c1 = gpu_scan(M2, t, segments=1)
    for nseg in (2, 4, 8):
        y2, h2, c2 = gpu_scan(M2, t, segments=nseg)
        # both sides round X' (the decay-weighted x) to bf16, with different weights
        assert rel_err(y2, y1) <= TOL["bf16"], nseg
        assert rel_err(h2, h1) <= TOL["bf16"], nseg
        assert np.array_equal(c2, c1), nseg


# Packed sequences cut on the device: one run length for all of them, a table
# of (sequence, run) entries built from cu_seqlens, surplus CTA rows idle.
# Empty, one-token and exactly-one-run sequences sit between long ones.
VARLEN_SEG_CASES = [
    # (lengths, H, G, K, segments)
    ([3000, 0, 1, 700, 64, 2049], 2, 1, 4, 2),     # runs of 8 chunks
    ([1000, 1000], 4, 2, 3, 4),                    # runs of 4 chunks, the last 232 tokens
    ([5000], 2, 1, 4, 0),                          # one sequence x 2 heads: cut by the library
    ([130, 4100, 0, 65], 2, 2, 0, 3),              # no conv; runs of 6 chunks
    ([64, 128, 192], 2, 1, 2, 2),                  # runs of one chunk, every sequence ends on a run edge
]


@pytest.mark.parametrize("lengths,H,G,K,segments", VARLEN_SEG_CASES)
def test_mamba2_varlen_segments(lengths, H, G, K, segments):
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(470 + len(lengths) + H + K, 1, int(cu[-1]), H, 64, G, 128, d_conv=K, dtype="bf16",
                        conv_bias=True, conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    check_scan(M2, d, "bf16", segments=segments, what=f"M2 varlen segments={segments} {lengths}")


def test_mamba2_varlen_segments_many_sequences():
    """More sequences than the table pre-pass has threads (its prefix sum
    carries across tiles of 1024 sequences), most of them cut into runs of
    one chunk."""
    rng = np.random.default_rng(491)
    lengths = rng.integers(0, 200, size=2500)
    lengths[rng.integers(0, 2500, size=40)] = 0
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(492, 1, int(cu[-1]), 1, 64, 1, 128, d_conv=4, dtype="bf16", conv_bias=True,
                        conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    t = to_dev(d, "bf16")
    assert ssm.scan_segments(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], z=t["z"], cu_seqlens=t["cu_seqlens"],
                             conv_w=t["conv_w"], segments=2) > len(lengths)
    check_scan(M2, d, "bf16", segments=2, what="M2 varlen segments, 2500 sequences")


def test_mamba2_varlen_segments_bad_cu_seqlens():
    """With the sequences cut on the device, a decreasing cu_seqlens still
    leaves y unwritten and sets the error word (the segment table stays empty)."""
    d = W.mamba2_inputs(494, 1, 600, 2, 64, 1, 128, dtype="bf16", conv_bias=True, nseqs=2)
    t = to_dev(d, "bf16")
    cu = torch.tensor([0, 500, 300], dtype=torch.int32, device="cuda")
    assert ssm.scan_segments(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu, conv_w=t["conv_w"],
                             segments=3) > 1
    y = torch.full(t["x"].shape, 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(ssm.scan_workspace_size(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu,
                                             conv_w=t["conv_w"], segments=3), dtype=torch.uint8, device="cuda")
    ssm.scan_fwd(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu, conv_w=t["conv_w"], y=y, workspace=ws,
                 segments=3)
    assert ssm.workspace_error(ws) == 1
    assert torch.all(y == 7.0)


def test_mamba2_varlen_segments_match_unsegmented():
    lengths = [2500, 3, 0, 900, 1300]
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(480, 1, int(cu[-1]), 4, 64, 2, 128, dtype="bf16", conv_bias=True, conv_state=True,
                        nseqs=len(lengths))
    d["cu_seqlens"] = cu
    t = to_dev(d, "bf16")
    y1, h1, c1 = gpu_scan(M2, t, segments=1)
    for nseg in (2, 5, 9):
        y2, h2, c2 = gpu_scan(M2, t, segments=nseg)
        assert rel_err(y2, y1) <= TOL["bf16"], nseg
        assert rel_err(h2, h1) <= TOL["bf16"], nseg
        assert np.array_equal(c2, c1), nseg


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_mamba2_strided_views(dtype):
    d = W.mamba2_inputs(410, 2, 50, 4, 32, 2, 32, dtype=dtype, conv_state=True)
    check_scan(M2, d, dtype, views=True, what="M2 views")


# ---------------------------------------------------------------- varlen
@pytest.mark.parametrize("mode", [M1, M2])
def test_varlen(mode):
    lengths = [5, 0, 130, 1, 64, 77, 0, 3]
    cu = W.cu_from_lengths(lengths)
    tot = int(cu[-1])
    if mode == M1:
        d = W.mamba1_inputs(500, 1, tot, 40, 16, dtype="bf16", conv_state=True, nseqs=len(lengths))
    else:
        d = W.mamba2_inputs(501, 1, tot, 4, 64, 2, 64, dtype="bf16", conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    check_scan(mode, d, "bf16", what=f"varlen mode {mode}")


def test_varlen_no_leak():
    """Perturbing one packed sequence leaves every other sequence's outputs
    bit-for-bit unchanged."""
    lengths = [50, 70, 40]
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(502, 1, int(cu[-1]), 4, 32, 2, 32, dtype="bf16", conv_state=True, nseqs=3)
    d["cu_seqlens"] = cu
    y1, h1, c1 = gpu_scan(M2, to_dev(d, "bf16"))
    d2 = dict(d)
    d2["x"] = d["x"].copy()
    d2["x"][:, cu[1]:cu[2]] = W.round_bf16(d2["x"][:, cu[1]:cu[2]] + 1.0)
    y2, h2, c2 = gpu_scan(M2, to_dev(d2, "bf16"))
    keep = np.ones(int(cu[-1]), bool)
    keep[cu[1]:cu[2]] = False
    assert np.array_equal(y1[:, keep], y2[:, keep])
    assert np.array_equal(h1[[0, 2]], h2[[0, 2]]) and np.array_equal(c1[[0, 2]], c2[[0, 2]])
    assert not np.array_equal(y1[:, ~keep], y2[:, ~keep])


def test_varlen_bad_cu_seqlens_reported():
    """A decreasing cu_seqlens is caught on the device: the error word reads
    SSM_DEVERR_CU_SEQLENS and no output is written."""
    d = W.mamba2_inputs(503, 1, 40, 2, 32, 1, 16, dtype="bf16", nseqs=2)
    t = to_dev(d, "bf16")
    cu = torch.tensor([0, 30, 20], dtype=torch.int32, device="cuda")
    y = torch.full(t["x"].shape, 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(ssm.scan_workspace_size(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu),
                     dtype=torch.uint8, device="cuda")
    ssm.scan_fwd(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu, y=y, workspace=ws)
    assert ssm.workspace_error(ws) == 1
    assert torch.all(y == 7.0)
    # and a good call on the same workspace clears it
    cu_ok = torch.tensor([0, 20, 40], dtype=torch.int32, device="cuda")
    ssm.scan_fwd(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], cu_seqlens=cu_ok, y=y, workspace=ws)
    assert ssm.workspace_error(ws) == 0


# --------------------------------------------------------------- decode
def _decode_run(mode, d, dtype, nsteps, idx=None):
    t = to_dev(d, dtype)
    state, cs = t["state"].clone(), t["conv_state"].clone()
    ys = []
    for s in range(nsteps):
        ys.append(ssm.state_update(mode, state, cs, t["x"][s], t["dt"][s], t["A"], t["B"][s], t["C"][s],
                                   D=t["D"], z=None if t["z"] is None else t["z"][s], dt_bias=t["dt_bias"],
                                   conv_w=t["conv_w"], conv_b=t["conv_b"], state_batch_indices=idx))
    torch.cuda.synchronize()
    return [y.float().cpu().numpy() for y in ys], state.cpu().numpy(), cs.float().cpu().numpy()


def _decode_oracle(mode, d, nsteps):
    state = d["state"].astype(np.float64).copy()
    cs = d["conv_state"].astype(np.float64).copy()
    ys = []
    for s in range(nsteps):
        ys.append(oracle.state_update(mode, state, cs, d["x"][s], d["dt"][s], d["A"], d["B"][s], d["C"][s], D=d["D"],
                                      z=None if d["z"] is None else d["z"][s], dt_bias=d["dt_bias"],
                                      conv_w=d["conv_w"], conv_b=d["conv_b"]))
    return ys, state, cs


@pytest.mark.parametrize("mode,H,P,G,N,Ls,dtype", [
    (M2, 8, 64, 2, 128, 4, "bf16"),
    (M2, 4, 33, 2, 256, 4, "f32"),    # streaming path with 256 states and an odd headdim
    (M2, 6, 32, 3, 16, 3, "f32"),
    (M2, 4, 16, 1, 10, 5, "f32"),     # dstate not a multiple of 4
    (M1, 300, 1, 1, 16, 4, "bf16"),   # Mamba-1: H is d_inner
    (M1, 64, 1, 1, 8, 3, "f32"),
])
def test_decode(mode, H, P, G, N, Ls, dtype):
    d = W.decode_inputs(600 + H + N, 5, H, P, G, N, conv_state_len=Ls, nsets=3, dtype=dtype, mode=mode,
                        conv_bias=True)
    ys, st, cs = _decode_run(mode, d, dtype, 3)
    rys, rst, rcs = _decode_oracle(mode, d, 3)
    for s in range(3):
        assert_close(ys[s], rys[s], dtype, f"decode y step {s}")
    assert_close(st, rst, dtype, "decode state")
    assert_close(cs, rcs, dtype, "decode conv state")


def test_decode_slots_and_padding():
    """Row r updates slot idx[r]; a negative slot is a padding row whose y is 0
    and which touches no state."""
    d = W.decode_inputs(610, 4, 4, 32, 2, 32, nsets=1, dtype="bf16")
    t = to_dev(d, "bf16")
    slots = 6
    state = torch.randn((slots, 4, 32, 32), device="cuda") * 0.1
    cs = torch.randn((slots, 4 * 32 + 2 * 2 * 32, 4), device="cuda").to(torch.bfloat16)
    idx = torch.tensor([5, -1, 0, 3], dtype=torch.int32, device="cuda")
    s0, c0 = state.clone(), cs.clone()
    y = ssm.state_update(M2, state, cs, t["x"][0], t["dt"][0], t["A"], t["B"][0], t["C"][0], D=t["D"], z=t["z"][0],
                         dt_bias=t["dt_bias"], conv_w=t["conv_w"], state_batch_indices=idx)
    torch.cuda.synchronize()
    assert torch.all(y[1] == 0)
    for untouched in (1, 2, 4):
        assert torch.equal(state[untouched], s0[untouched]) and torch.equal(cs[untouched], c0[untouched])
    for r, sl in ((0, 5), (2, 0), (3, 3)):
        st = s0[sl].double().cpu().numpy()[None].copy()
        cst = c0[sl].float().double().cpu().numpy()[None].copy()
        ry = oracle.state_update(M2, st, cst, d["x"][0][r:r + 1], d["dt"][0][r:r + 1], d["A"], d["B"][0][r:r + 1],
                                 d["C"][0][r:r + 1], D=d["D"], z=d["z"][0][r:r + 1], dt_bias=d["dt_bias"],
                                 conv_w=d["conv_w"])
        assert_close(y[r:r + 1].float().cpu().numpy(), ry, "bf16", f"slot row {r}")
        assert_close(state[sl].cpu().numpy()[None], st, "bf16", f"slot state {sl}")


def test_decode_batch_invariant():
    """Row r's result does not depend on which other rows share the batch."""
    d = W.decode_inputs(620, 8, 8, 64, 2, 64, nsets=1, dtype="bf16")
    t = to_dev(d, "bf16")
    def run(rows):
        state, cs = t["state"][rows].clone(), t["conv_state"][rows].clone()
        y = ssm.state_update(M2, state, cs, t["x"][0][rows], t["dt"][0][rows], t["A"], t["B"][0][rows],
                             t["C"][0][rows], D=t["D"], z=t["z"][0][rows], dt_bias=t["dt_bias"], conv_w=t["conv_w"])
        torch.cuda.synchronize()
        return y, state
    y_all, s_all = run(list(range(8)))
    y_sub, s_sub = run([6, 2])
    assert torch.equal(y_all[[6, 2]], y_sub) and torch.equal(s_all[[6, 2]], s_sub)


@pytest.mark.parametrize("mode", [M1, M2])
def test_prefill_equals_repeated_decode(mode):
    """T decode steps reproduce one forward scan over the same T tokens."""
    T = 9
    if mode == M1:
        d = W.mamba1_inputs(700, 3, T, 64, 16, dtype="f32", conv_state=True)
    else:
        d = W.mamba2_inputs(701, 3, T, 4, 32, 2, 32, dtype="f32", conv_state=True)
    t = to_dev(d, "f32")
    y, hf, cs = gpu_scan(mode, t)
    state = t["h0"].clone()
    conv_state = t["conv_state_in"].clone()
    ys = []
    for s in range(T):
        ys.append(ssm.state_update(mode, state, conv_state, t["x"][:, s], t["dt"][:, s], t["A"], t["B"][:, s],
                                   t["C"][:, s], D=t["D"], z=t["z"][:, s], dt_bias=t["dt_bias"], conv_w=t["conv_w"]))
    torch.cuda.synchronize()
    yd = torch.stack(ys, 1).cpu().numpy()
    assert rel_err(yd, y) <= 1e-5
    assert rel_err(state.cpu().numpy(), hf) <= 1e-5
    assert np.array_equal(conv_state.cpu().numpy(), cs)


@pytest.mark.parametrize("mode", [M1, M2])
def test_split_invariance(mode):
    """Scanning [0, L) equals scanning [0, k) then [k, L) from the returned
    h_final and conv state, across chunk boundaries."""
    L = 150
    if mode == M1:
        d = W.mamba1_inputs(710, 2, L, 32, 16, dtype="f32", conv_state=True)
    else:
        d = W.mamba2_inputs(711, 2, L, 4, 32, 2, 32, dtype="f32", conv_state=True)
    t = to_dev(d, "f32")
    y, hf, cs = gpu_scan(mode, t)
    for k in (1, 63, 64, 100):
        a = {kk: (v[:, :k] if kk in ("x", "z", "dt", "B", "C") else v) for kk, v in t.items()}
        b = {kk: (v[:, k:] if kk in ("x", "z", "dt", "B", "C") else v) for kk, v in t.items()}
        y1, h1, c1 = gpu_scan(mode, a)
        b["h0"] = torch.from_numpy(h1).float().cuda()
        b["conv_state_in"] = torch.from_numpy(c1).float().cuda()
        y2, h2, c2 = gpu_scan(mode, b)
        assert rel_err(np.concatenate([y1, y2], 1), y) <= 1e-5
        assert rel_err(h2, hf) <= 1e-5
        assert np.array_equal(c2, cs)


# ------------------------------------------- Mamba-2 on the tensor-core path
# headdim 64, dstate 128, bf16 activations, conv width <= 4 take the chunked
# tcgen05 kernel (64-token chunks); the cases cross chunk boundaries and end
# on ragged tails.
SSD_CASES = [
    # (b, T, H, G, K)
    (1, 1, 2, 1, 4),
    (2, 64, 4, 2, 4),
    (2, 65, 4, 2, 4),
    (1, 200, 6, 3, 4),
    (2, 130, 4, 4, 3),
    (1, 97, 2, 1, 2),
    (2, 70, 4, 2, 0),       # no conv: B, C and x used as given
]


@pytest.mark.parametrize("b,T,H,G,K", SSD_CASES)
def test_ssd(b, T, H, G, K):
    d = W.mamba2_inputs(800 + T + H + K, b, T, H, 64, G, 128, d_conv=K, dtype="bf16", conv_bias=True,
                        conv_state=True)
    check_scan(M2, d, "bf16", what=f"SSD b{b} T{T} H{H} G{G} K{K}")


def test_ssd_optional_inputs_absent():
    d = W.mamba2_inputs(820, 2, 100, 4, 64, 2, 128, dtype="bf16", with_h0=False, with_z=False)
    d["D"] = None
    d["dt_bias"] = None
    check_scan(M2, d, "bf16", what="SSD minimal")


def test_ssd_strided_views():
    d = W.mamba2_inputs(821, 2, 90, 4, 64, 2, 128, dtype="bf16", conv_state=True)
    check_scan(M2, d, "bf16", views=True, what="SSD views")


def test_ssd_varlen():
    lengths = [63, 0, 1, 64, 65, 200, 2, 130]
    cu = W.cu_from_lengths(lengths)
    d = W.mamba2_inputs(822, 1, int(cu[-1]), 4, 64, 2, 128, dtype="bf16", conv_state=True, nseqs=len(lengths))
    d["cu_seqlens"] = cu
    check_scan(M2, d, "bf16", what="SSD varlen")


def test_ssd_split_invariance():
    """Continuing a sequence from the returned state reproduces one long scan
    (chunk boundaries land in different places in the two runs)."""
    L = 180
    d = W.mamba2_inputs(823, 2, L, 4, 64, 2, 128, dtype="bf16", conv_state=True)
    t = to_dev(d, "bf16")
    y, hf, cs = gpu_scan(M2, t)
    for k in (37, 64, 100):
        a = {kk: (v[:, :k] if kk in ("x", "z", "dt", "B", "C") else v) for kk, v in t.items()}
        b = {kk: (v[:, k:] if kk in ("x", "z", "dt", "B", "C") else v) for kk, v in t.items()}
        y1, h1, c1 = gpu_scan(M2, a)
        b["h0"] = torch.from_numpy(h1).float().cuda()
        b["conv_state_in"] = torch.from_numpy(c1).to(torch.bfloat16).cuda()
        y2, h2, c2 = gpu_scan(M2, b)
        assert rel_err(np.concatenate([y1, y2], 1), y) <= 2e-2
        assert rel_err(h2, hf) <= 2e-2
        assert np.array_equal(c2, cs)


def test_kernel_timing_counts_launches():
    """ssm_kernel_timing brackets each call's dominant kernel with events on the call's stream."""
    d = W.mamba1_inputs(901, 1, 96, 32, 16, dtype="bf16")
    t = to_dev(d, "bf16")
    ssm.kernel_time_ms()
    ssm.kernel_timing(True)
    gpu_scan(M1, t)
    gpu_scan(M1, t)
    ssm.kernel_timing(False)
    ms, n = ssm.kernel_time_ms()
    assert n == 2 and ms > 0.0
    gpu_scan(M1, t)
    assert ssm.kernel_time_ms() == (0.0, 0)
