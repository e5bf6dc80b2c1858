"""Seeded synthetic inputs for the scan, conv and decode paths.

This module only draws random numbers and arranges them; it holds none of the
method's arithmetic.  Both the CUDA path (tests, benchmark) and the fp64
oracle are fed from here, so they always see identical values.

Every array is returned as a numpy float32 array.  When ``dtype == "bf16"``
the activations are quantised to bf16-representable float32 values (round to
nearest, ties to even), so widening them to bf16 on the device and to float64
in the oracle is exact.  Parameters (A, D, dt_bias, conv weights) and states
stay float32.

Recipe (same for every workload unless its entry says otherwise):
  x, z, B, C            ~ N(0, 1)
  dt (raw)              ~ N(0, 1) * dt_sigma        (dt_sigma = 1 by default)
  dt_bias               = log(expm1(u)), u ~ LogUniform[1e-3, 1e-1] per
                          channel / head, so softplus(dt_bias) = u
  A                     = -exp(U(log 1, log 16))    (Mamba-1 per [d, n]; Mamba-2 per head)
  D                     = 1
  conv weight           ~ U(-0.5, 0.5), width 4; conv bias absent unless asked
  h0                    ~ N(0, 0.1^2)
  conv state (carried)  ~ N(0, 1) raw inputs when asked, else absent
Varlen lengths          ~ U{lo..hi} per sequence.
"""
from __future__ import annotations

import dataclasses

import numpy as np

BASE_SEED = 20261202


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Quantise float32 values to the nearest bf16 (ties to even), kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    r = u + np.uint32(0x7FFF)                       # half an ulp of bf16, less one
    r += (u >> np.uint32(16)) & np.uint32(1)        # ties go to the even bf16 value
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _act(rng, shape, dtype, scale=1.0):
    v = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        v *= np.float32(scale)
    return round_bf16(v) if dtype == "bf16" else v


def _dt_bias(rng, n):
    u = np.exp(rng.uniform(np.log(1e-3), np.log(1e-1), size=n))
    return np.log(np.expm1(u)).astype(np.float32)


def _neg_A(rng, shape):
    return (-np.exp(rng.uniform(0.0, np.log(16.0), size=shape))).astype(np.float32)


def varlen_lengths(seed: int, nseqs: int, lo: int, hi: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, size=nseqs).astype(np.int64)


def cu_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    return cu


def mamba1_inputs(seed, batch, seqlen, d_inner, dstate, *, d_conv=4, dtype="bf16", with_h0=True,
                  conv_bias=False, conv_state=False, with_z=True, dt_sigma=1.0, nseqs=None):
    """Mamba-1 scan inputs.  Shapes: x, z, dt [batch, T, d]; B, C [batch, T, n];
    A [d, n]; D, dt_bias [d]; h0 [nseqs, d, n]; conv_w [d, K]; conv_state_in
    [nseqs, d, K-1].  ``nseqs`` defaults to ``batch`` (pass it for packed varlen)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ns = batch if nseqs is None else nseqs
    out = {}
    out["x"] = _act(rng, (batch, seqlen, d_inner), dtype)
    out["z"] = _act(rng, (batch, seqlen, d_inner), dtype) if with_z else None
    out["dt"] = _act(rng, (batch, seqlen, d_inner), dtype, dt_sigma)
    out["B"] = _act(rng, (batch, seqlen, dstate), dtype)
    out["C"] = _act(rng, (batch, seqlen, dstate), dtype)
    out["A"] = _neg_A(rng, (d_inner, dstate))
    out["D"] = np.ones(d_inner, dtype=np.float32)
    out["dt_bias"] = _dt_bias(rng, d_inner)
    out["h0"] = (rng.standard_normal(size=(ns, d_inner, dstate), dtype=np.float32) * np.float32(0.1)) if with_h0 else None
    if d_conv > 0:
        out["conv_w"] = rng.uniform(-0.5, 0.5, size=(d_inner, d_conv)).astype(np.float32)
        out["conv_b"] = rng.uniform(-0.5, 0.5, size=d_inner).astype(np.float32) if conv_bias else None
        out["conv_state_in"] = _act(rng, (ns, d_inner, d_conv - 1), dtype) if (conv_state and d_conv > 1) else None
    else:
        out["conv_w"] = out["conv_b"] = out["conv_state_in"] = None
    return out


def mamba2_inputs(seed, batch, seqlen, nheads, headdim, ngroups, dstate, *, d_conv=4, dtype="bf16",
                  with_h0=True, conv_bias=False, conv_state=False, with_z=True, dt_sigma=1.0, nseqs=None):
    """Mamba-2 scan inputs.  Shapes: x, z [batch, T, H, P]; dt [batch, T, H];
    B, C [batch, T, G, N]; A, D, dt_bias [H]; h0 [nseqs, H, P, N];
    conv_w [H*P + 2*G*N, K] (channel order x | B | C); conv_state_in
    [nseqs, H*P + 2*G*N, K-1]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ns = batch if nseqs is None else nseqs
    cdim = nheads * headdim + 2 * ngroups * dstate
    out = {}
    out["x"] = _act(rng, (batch, seqlen, nheads, headdim), dtype)
    out["z"] = _act(rng, (batch, seqlen, nheads, headdim), dtype) if with_z else None
    out["dt"] = _act(rng, (batch, seqlen, nheads), dtype, dt_sigma)
    out["B"] = _act(rng, (batch, seqlen, ngroups, dstate), dtype)
    out["C"] = _act(rng, (batch, seqlen, ngroups, dstate), dtype)
    out["A"] = _neg_A(rng, (nheads,))
    out["D"] = np.ones(nheads, dtype=np.float32)
    out["dt_bias"] = _dt_bias(rng, nheads)
    out["h0"] = (rng.standard_normal(size=(ns, nheads, headdim, dstate), dtype=np.float32) * np.float32(0.1)) if with_h0 else None
    if d_conv > 0:
        out["conv_w"] = rng.uniform(-0.5, 0.5, size=(cdim, d_conv)).astype(np.float32)
        out["conv_b"] = rng.uniform(-0.5, 0.5, size=cdim).astype(np.float32) if conv_bias else None
        out["conv_state_in"] = _act(rng, (ns, cdim, d_conv - 1), dtype) if (conv_state and d_conv > 1) else None
    else:
        out["conv_w"] = out["conv_b"] = out["conv_state_in"] = None
    return out


def decode_inputs(seed, batch, nheads, headdim, ngroups, dstate, *, d_conv=4, conv_state_len=4, nsets=1,
                  dtype="bf16", mode=2, conv_bias=False, with_z=True, dt_sigma=1.0):
    """Single-token decode inputs.  ``mode=2``: x, z [nsets, batch, H, P];
    dt [nsets, batch, H]; B, C [nsets, batch, G, N]; state [batch, H, P, N]
    (float32, ~N(0, 0.1^2)); conv_state [batch, H*P + 2*G*N, conv_state_len].
    ``mode=1``: H is d_inner, P = G = 1 and x, z, dt [nsets, batch, d],
    B, C [nsets, batch, N], A [d, N], state [batch, d, N]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    if mode == 1:
        d = nheads
        cdim = d
        out["x"] = _act(rng, (nsets, batch, d), dtype)
        out["z"] = _act(rng, (nsets, batch, d), dtype) if with_z else None
        out["dt"] = _act(rng, (nsets, batch, d), dtype, dt_sigma)
        out["B"] = _act(rng, (nsets, batch, dstate), dtype)
        out["C"] = _act(rng, (nsets, batch, dstate), dtype)
        out["A"] = _neg_A(rng, (d, dstate))
        out["D"] = np.ones(d, dtype=np.float32)
        out["dt_bias"] = _dt_bias(rng, d)
        out["state"] = rng.standard_normal(size=(batch, d, dstate), dtype=np.float32) * np.float32(0.1)
    else:
        cdim = nheads * headdim + 2 * ngroups * dstate
        out["x"] = _act(rng, (nsets, batch, nheads, headdim), dtype)
        out["z"] = _act(rng, (nsets, batch, nheads, headdim), dtype) if with_z else None
        out["dt"] = _act(rng, (nsets, batch, nheads), dtype, dt_sigma)
        out["B"] = _act(rng, (nsets, batch, ngroups, dstate), dtype)
        out["C"] = _act(rng, (nsets, batch, ngroups, dstate), dtype)
        out["A"] = _neg_A(rng, (nheads,))
        out["D"] = np.ones(nheads, dtype=np.float32)
        out["dt_bias"] = _dt_bias(rng, nheads)
        out["state"] = rng.standard_normal(size=(batch, nheads, headdim, dstate), dtype=np.float32) * np.float32(0.1)
    if d_conv > 0:
        out["conv_w"] = rng.uniform(-0.5, 0.5, size=(cdim, d_conv)).astype(np.float32)
        out["conv_b"] = rng.uniform(-0.5, 0.5, size=cdim).astype(np.float32) if conv_bias else None
        out["conv_state"] = _act(rng, (batch, cdim, conv_state_len), dtype)
    else:
        out["conv_w"] = out["conv_b"] = out["conv_state"] = None
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named synthetic workload: what it is, with its sizes."""
    name: str
    kind: str              # "mamba1" | "mamba2" | "mamba2_varlen" | "decode"
    dtype: str
    batch: int = 1
    seqlen: int = 0
    d_inner: int = 0
    nheads: int = 0
    headdim: int = 0
    ngroups: int = 1
    dstate: int = 0
    d_conv: int = 4
    chunk: int = 0
    nseqs: int = 0
    len_lo: int = 0
    len_hi: int = 0
    conv_state_len: int = 4
    steps: int = 0
    nsets: int = 1
    state_interval: int = 0   # > 0: intermediate states every this many tokens (prefix caching)
    backward: bool = False    # the step is the backward of the scan (gradients of every input)
    split_ranks: int = 0      # > 0: the tokens of every row are split into this many equal segments, one per rank
    split_rank: int = 0       # the rank whose step is measured (its segment, fix-up included)
    seed: int = BASE_SEED


# The five workloads of the hot path (seeds BASE_SEED + position), then the
# varlen workload again with intermediate-state extraction and the Mamba-1
# layer's backward (same inputs as their forward workloads).
WORKLOADS = {
    "mamba1_tiny_f32": Workload("mamba1_tiny_f32", "mamba1", "f32", batch=1, seqlen=64, d_inner=16, dstate=4,
                                seed=BASE_SEED + 0),
    "mamba1_layer_b8_l2048_d1536_n16": Workload("mamba1_layer_b8_l2048_d1536_n16", "mamba1", "bf16", batch=8,
                                                seqlen=2048, d_inner=1536, dstate=16, seed=BASE_SEED + 1),
    "mamba2_ssd_b4_l4096_h80_p64_g8_n128": Workload("mamba2_ssd_b4_l4096_h80_p64_g8_n128", "mamba2", "bf16",
                                                    batch=4, seqlen=4096, nheads=80, headdim=64, ngroups=8,
                                                    dstate=128, chunk=256, seed=BASE_SEED + 2),
    "mamba2_varlen_16seq_h64_p64_g1_n128": Workload("mamba2_varlen_16seq_h64_p64_g1_n128", "mamba2_varlen", "bf16",
                                                    nheads=64, headdim=64, ngroups=1, dstate=128, nseqs=16,
                                                    len_lo=128, len_hi=8192, chunk=256, seed=BASE_SEED + 3),
    "mamba2_decode_b256_h128_p64_g8_n128": Workload("mamba2_decode_b256_h128_p64_g8_n128", "decode", "bf16",
                                                    batch=256, nheads=128, headdim=64, ngroups=8, dstate=128,
                                                    conv_state_len=4, steps=1000, nsets=8, seed=BASE_SEED + 4),
    # the packed varlen workload again, also storing every sequence's state and
    # conv history after each 512 tokens (prefix-caching extraction)
    "mamba2_varlen_16seq_h64_p64_g1_n128_states512": Workload(
        "mamba2_varlen_16seq_h64_p64_g1_n128_states512", "mamba2_varlen", "bf16", nheads=64, headdim=64, ngroups=1,
        dstate=128, nseqs=16, len_lo=128, len_hi=8192, chunk=256, state_interval=512, seed=BASE_SEED + 3),
    # one rank's step of a two-way token split of the Mamba-2 and Mamba-1
    # workloads (the second rank: scan of its half from zero, then the fold of
    # both ranks' pairs and the fix-up of y)
    "mamba2_ssd_b4_l4096_h80_p64_g8_n128_split2": Workload(
        "mamba2_ssd_b4_l4096_h80_p64_g8_n128_split2", "mamba2", "bf16", batch=4, seqlen=4096, nheads=80, headdim=64,
        ngroups=8, dstate=128, chunk=256, split_ranks=2, split_rank=1, seed=BASE_SEED + 2),
    "mamba1_layer_b8_l2048_d1536_n16_split2": Workload(
        "mamba1_layer_b8_l2048_d1536_n16_split2", "mamba1", "bf16", batch=8, seqlen=2048, d_inner=1536, dstate=16,
        split_ranks=2, split_rank=1, seed=BASE_SEED + 1),
    # one long Mamba-1 sequence (a single-prompt prefill): too few channels x
    # batch rows to fill the GPU with the sequential scan, so the time-parallel
    # (warp-shuffle pair scan) form runs
    "mamba1_seq_b1_l8192_d1536_n16": Workload("mamba1_seq_b1_l8192_d1536_n16", "mamba1", "bf16", batch=1,
                                              seqlen=8192, d_inner=1536, dstate=16, seed=BASE_SEED + 5),
    # one long Mamba-2 sequence (a single-prompt prefill): 80 (row, head) chains
    # for 296 CTA slots, so the rows are cut into token segments scanned at once
    "mamba2_seq_b1_l16384_h80_p64_g8_n128": Workload("mamba2_seq_b1_l16384_h80_p64_g8_n128", "mamba2", "bf16",
                                                     batch=1, seqlen=16384, nheads=80, headdim=64, ngroups=8,
                                                     dstate=128, chunk=256, seed=BASE_SEED + 6),
    # two long packed sequences (4096 to 16384 tokens each): 160 (sequence,
    # head) chains for 296 CTA slots, so the device cuts the sequences into
    # token segments from their cu_seqlens
    "mamba2_varlen_2seq_h80_p64_g8_n128": Workload("mamba2_varlen_2seq_h80_p64_g8_n128", "mamba2_varlen", "bf16",
                                                   nheads=80, headdim=64, ngroups=8, dstate=128, nseqs=2,
                                                   len_lo=4096, len_hi=16384, chunk=256, seed=BASE_SEED + 7),
    # the Mamba-1 layer's backward (same inputs; upstream gradients drawn alongside)
    "mamba1_layer_b8_l2048_d1536_n16_bwd": Workload("mamba1_layer_b8_l2048_d1536_n16_bwd", "mamba1", "bf16", batch=8,
                                                    seqlen=2048, d_inner=1536, dstate=16, backward=True,
                                                    seed=BASE_SEED + 1),
}


def workload_inputs(w: Workload, **overrides):
    """Draw the full inputs of a named workload (numpy, host memory)."""
    if w.kind == "mamba1":
        return mamba1_inputs(w.seed, w.batch, w.seqlen, w.d_inner, w.dstate, d_conv=w.d_conv, dtype=w.dtype,
                             **overrides)
    if w.kind == "mamba2":
        return mamba2_inputs(w.seed, w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate,
                             d_conv=w.d_conv, dtype=w.dtype, **overrides)
    if w.kind == "mamba2_varlen":
        lengths = varlen_lengths(w.seed, w.nseqs, w.len_lo, w.len_hi)
        total = int(lengths.sum())
        d = mamba2_inputs(w.seed + 1000, 1, total, w.nheads, w.headdim, w.ngroups, w.dstate, d_conv=w.d_conv,
                          dtype=w.dtype, nseqs=w.nseqs, **overrides)
        d["cu_seqlens"] = cu_from_lengths(lengths)
        return d
    if w.kind == "decode":
        return decode_inputs(w.seed, w.batch, w.nheads, w.headdim, w.ngroups, w.dstate, d_conv=w.d_conv,
                             conv_state_len=w.conv_state_len, nsets=w.nsets, dtype=w.dtype, **overrides)
    raise ValueError(w.kind)
