"""Independent pins for the fp64 oracle.

Each ``check_*`` function computes an expected value by a route that does not
go through the oracle's loop (a closed form, explicit products, a library
routine, a split of the same input) and raises AssertionError on a mismatch.
They take ``mutant`` so the mutation test can run them against oracle builds
with a planted mistake and show that some pin fails for each.

Passages the pins follow:
  * recurrence and (decay, value) pair with the (1, h0) seed: "Adding Initial
    Value Support to Selective Scan Forward Kernel" (state-spaces/mamba issue
    285), opening post and the running-prefix replies;
  * op shapes, final state as output, conv state of K-1 columns: "ggml : add
    GPU support for Mamba models" (llama.cpp issue 6758), test-backend-ops
    patch and the SSM_CONV / SSM_SCAN discussion;
  * conv as concat + im2col + mul_mat, or mul + sum_rows: same page, the
    replies on reformulating SSM_CONV;
  * groups of heads as contiguous repeat_interleave blocks: "Tensor-parallel
    SSM" (Fast-LLM PR 333), repeat_kv review thread;
  * prefill with h0 equals the step function fed the same state: issue 285,
    closing replies;
  * decode state update and varlen conv: "Clean up SSM ops directory
    structure" (Megatron-LM PR 6444), kernel inventory.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from state_space_model_conv1d_b200 import workloads as W

M1, M2 = oracle.MAMBA1, oracle.MAMBA2


# ---------------------------------------------------------------- helpers
def softplus_np(u):
    """softplus via numpy's logaddexp (a library route, not the oracle's)."""
    return np.logaddexp(0.0, np.asarray(u, dtype=np.float64))


def silu_np(v):
    v = np.asarray(v, dtype=np.float64)
    return v * (0.5 * (1.0 + np.tanh(0.5 * v)))   # x * sigmoid(x), sigmoid via tanh


def conv_im2col(x, w, b=None, state=None, act=True):
    """Causal depthwise conv as concat + im2col + matmul (the llama.cpp
    reformulation), for one sequence x [T, C], w [C, K], state [C, K-1]."""
    T, Cn = x.shape
    K = w.shape[1]
    hist = np.zeros((K - 1, Cn)) if state is None else np.asarray(state, np.float64).T
    full = np.concatenate([hist, np.asarray(x, np.float64)], axis=0)        # [T+K-1, C]
    cols = np.stack([full[t:t + K] for t in range(T)], axis=0)             # [T, K, C]
    out = np.einsum("tkc,ck->tc", cols, np.asarray(w, np.float64))
    if b is not None:
        out = out + np.asarray(b, np.float64)[None, :]
    return silu_np(out) if act else out, full[T:].T.copy() if K > 1 else None


def conv_mul_sumrows(x, w, b=None, state=None, act=True):
    """Same conv as elementwise multiply + row sums (the other reformulation)."""
    T, Cn = x.shape
    K = w.shape[1]
    hist = np.zeros((K - 1, Cn)) if state is None else np.asarray(state, np.float64).T
    full = np.concatenate([hist, np.asarray(x, np.float64)], axis=0)
    out = np.zeros((T, Cn))
    for t in range(T):
        out[t] = (full[t:t + K].T * np.asarray(w, np.float64)).sum(axis=1)
    if b is not None:
        out = out + np.asarray(b, np.float64)[None, :]
    return silu_np(out) if act else out


def _close(a, b, rtol=1e-11, atol=1e-12, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.shape != b.shape:
        raise AssertionError(f"{what}: shape {a.shape} vs {b.shape}")
    with np.errstate(invalid="ignore", over="ignore"):     # a planted mistake may produce inf / nan: it fails below
        err = np.max(np.abs(a - b)) if a.size else 0.0
    ref = np.max(np.abs(b)) if b.size else 0.0
    if not err <= atol + rtol * ref:
        raise AssertionError(f"{what}: max|err| {err:.3e} (max|ref| {ref:.3e})")


def _m1_scan(d, mutant, **kw):
    return oracle.scan_fwd(M1, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d.get("D"), z=d.get("z"),
                           dt_bias=d.get("dt_bias"), h0=d.get("h0"), conv_w=d.get("conv_w"),
                           conv_b=d.get("conv_b"), conv_state_in=d.get("conv_state_in"), mutant=mutant, **kw)


def _m2_scan(d, mutant, **kw):
    return oracle.scan_fwd(M2, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d.get("D"), z=d.get("z"),
                           dt_bias=d.get("dt_bias"), h0=d.get("h0"), conv_w=d.get("conv_w"),
                           conv_b=d.get("conv_b"), conv_state_in=d.get("conv_state_in"), mutant=mutant, **kw)


# ------------------------------------------------------- recurrence pins
def check_A_zero_is_cumsum(mutant=0):
    """A = 0: every decay is 1, so h_t = h0 + cumsum_s(delta_s B_s x_s) and
    y_t = C_t . h_t + D x_t, gated by silu(z_t)."""
    d = W.mamba1_inputs(11, 2, 13, 5, 3, d_conv=0, dtype="f32")
    d["A"] = np.zeros_like(d["A"])
    y, hf, _ = _m1_scan(d, mutant)
    delta = softplus_np(d["dt"].astype(np.float64) + d["dt_bias"][None, None, :])           # [b,T,D]
    inc = delta[..., None] * d["B"][:, :, None, :] * d["x"][..., None]                      # [b,T,D,N]
    h = d["h0"][:, None, :, :] + np.cumsum(inc, axis=1)
    yy = np.einsum("btn,btdn->btd", d["C"].astype(np.float64), h) + d["D"] * d["x"]
    yy = yy * silu_np(d["z"])
    _close(hf, h[:, -1], what="A=0 h_final")
    _close(y, yy, what="A=0 y")
    # Mamba-2 form of the same closed form
    e = W.mamba2_inputs(12, 1, 9, 4, 3, 2, 5, d_conv=0, dtype="f32")
    e["A"] = np.zeros_like(e["A"])
    y2, hf2, _ = _m2_scan(e, mutant)
    delta = softplus_np(e["dt"].astype(np.float64) + e["dt_bias"][None, None, :])            # [b,T,H]
    Bh = np.repeat(e["B"].astype(np.float64), 2, axis=2)                                    # [b,T,H,N]
    Ch = np.repeat(e["C"].astype(np.float64), 2, axis=2)
    inc = delta[..., None, None] * e["x"][..., None] * Bh[:, :, :, None, :]                # [b,T,H,P,N]
    h = e["h0"][:, None] + np.cumsum(inc, axis=1)
    yy = np.einsum("bthn,bthpn->bthp", Ch, h) + e["D"][None, None, :, None] * e["x"]
    yy = yy * silu_np(e["z"])
    _close(hf2, h[:, -1], what="M2 A=0 h_final")
    _close(y2, yy, what="M2 A=0 y")


def check_zero_delta_keeps_h0(mutant=0):
    """dt = 0, dt_bias = 0, softplus off: delta = 0, the state never moves,
    h_T == h0 exactly and y_t = C_t . h0 + D x_t."""
    d = W.mamba1_inputs(13, 2, 11, 6, 4, d_conv=0, dtype="f32", with_z=False)
    d["dt"] = np.zeros_like(d["dt"])
    d["dt_bias"] = np.zeros_like(d["dt_bias"])
    y, hf, _ = _m1_scan(d, mutant, delta_softplus=False)
    if not np.array_equal(hf, d["h0"].astype(np.float64)):
        raise AssertionError("delta=0 must return h0 bit for bit")
    yy = np.einsum("btn,bdn->btd", d["C"].astype(np.float64), d["h0"].astype(np.float64)) + d["D"] * d["x"]
    _close(y, yy, what="delta=0 y")


def check_geometric_fixed_point(mutant=0):
    """Constant delta, x, B and A < 0: h_t = a^t h0 + delta B x (1 - a^t)/(1 - a)
    with a = exp(delta A); for large t it reaches the fixed point
    delta B x / (1 - exp(delta A))."""
    T, Dn, N = 400, 3, 4
    rng = np.random.default_rng(14)
    x0 = rng.standard_normal(Dn)
    B0 = rng.standard_normal(N)
    A = -np.exp(rng.uniform(0, np.log(16), size=(Dn, N)))
    delta = 0.05
    h0 = rng.standard_normal((1, Dn, N)) * 0.1
    d = dict(x=np.broadcast_to(x0, (1, T, Dn)).copy(), dt=np.full((1, T, Dn), delta),
             B=np.broadcast_to(B0, (1, T, N)).copy(), C=rng.standard_normal((1, T, N)),
             A=A, D=np.zeros(Dn), h0=h0)
    y, hf, _ = _m1_scan(d, mutant, delta_softplus=False)
    a = np.exp(delta * A)
    bx = delta * B0[None, :] * x0[:, None]
    t = np.arange(1, T + 1, dtype=np.float64)[:, None, None]
    h_t = a[None] ** t * h0[0][None] + bx[None] * (1 - a[None] ** t) / (1 - a[None])
    yy = np.einsum("tn,tdn->td", d["C"][0], h_t)
    _close(hf[0], h_t[-1], rtol=1e-10, what="geometric h_T")
    _close(y[0], yy, rtol=1e-10, what="geometric y")
    fixed = bx / (1 - a)
    _close(hf[0], fixed, rtol=1e-6, atol=1e-8, what="fixed point")


def _f64(d):
    """float64 copies of every array input (Python-float times float32-scalar
    products would otherwise stay float32 under numpy's promotion rules)."""
    return {k: (np.asarray(v, np.float64) if isinstance(v, np.ndarray) else v) for k, v in d.items()}


def _bruteforce_m1(d, softplus=True):
    """Explicit-product evaluation: h_T = (prod_t a_t) h0 + sum_s (prod_{t>s} a_t) delta_s B_s x_s."""
    d = _f64(d)
    x = d["x"]
    b, T, Dn = x.shape
    N = d["B"].shape[2]
    if d.get("conv_w") is not None:
        xs = np.stack([conv_im2col(x[i], d["conv_w"], d.get("conv_b"),
                                   None if d.get("conv_state_in") is None else d["conv_state_in"][i])[0]
                       for i in range(b)])
    else:
        xs = x
    u = d["dt"].astype(np.float64) + d["dt_bias"][None, None, :]
    delta = softplus_np(u) if softplus else u
    y = np.zeros((b, T, Dn))
    hT = np.zeros((b, Dn, N))
    for i in range(b):
        for c in range(Dn):
            for n in range(N):
                a = [math.exp(delta[i, t, c] * d["A"][c, n]) for t in range(T)]
                for tt in range(T):
                    h = math.prod(a[:tt + 1]) * (d["h0"][i, c, n] if d.get("h0") is not None else 0.0)
                    for s in range(tt + 1):
                        h += math.prod(a[s + 1:tt + 1]) * delta[i, s, c] * d["B"][i, s, n] * xs[i, s, c]
                    y[i, tt, c] += d["C"][i, tt, n] * h
                    if tt == T - 1:
                        hT[i, c, n] = h
            y[i, :, c] += d["D"][c] * xs[i, :, c]
    if d.get("z") is not None:
        y *= silu_np(d["z"])
    return y, hT


def check_bruteforce_m1(mutant=0):
    """L <= 8 against explicit products (a different evaluation order)."""
    for L in (1, 2, 5, 8):
        d = W.mamba1_inputs(20 + L, 2, L, 3, 2, d_conv=4, dtype="f32", conv_bias=True, conv_state=True)
        y, hf, _ = _m1_scan(d, mutant)
        yy, hh = _bruteforce_m1(d)
        _close(hf, hh, rtol=1e-10, what=f"brute h L={L}")
        _close(y, yy, rtol=1e-10, what=f"brute y L={L}")


def check_bruteforce_m2(mutant=0):
    """Mamba-2 at L <= 8: conv over x|B|C by im2col, groups expanded with
    np.repeat (repeat_interleave), explicit products per (head, p, n)."""
    H, P, G, N = 4, 2, 2, 3
    for L in (1, 3, 8):
        d = W.mamba2_inputs(30 + L, 1, L, H, P, G, N, d_conv=4, dtype="f32", conv_bias=True, conv_state=True)
        y, hf, _ = _m2_scan(d, mutant)
        d = _f64(d)
        xr = d["x"][0].reshape(L, H * P)
        raw = np.concatenate([xr, d["B"][0].reshape(L, G * N), d["C"][0].reshape(L, G * N)], axis=1)
        u, _ = conv_im2col(raw, d["conv_w"], d["conv_b"], d["conv_state_in"][0])
        xs = u[:, :H * P].reshape(L, H, P)
        Bh = np.repeat(u[:, H * P:H * P + G * N].reshape(L, G, N), H // G, axis=1)
        Ch = np.repeat(u[:, H * P + G * N:].reshape(L, G, N), H // G, axis=1)
        delta = softplus_np(d["dt"][0].astype(np.float64) + d["dt_bias"][None, :])      # [L,H]
        yy = np.zeros((L, H, P))
        hh = np.zeros((H, P, N))
        for h_ in range(H):
            a = [math.exp(delta[t, h_] * d["A"][h_]) for t in range(L)]
            for p in range(P):
                for n in range(N):
                    for tt in range(L):
                        v = math.prod(a[:tt + 1]) * d["h0"][0, h_, p, n]
                        for s in range(tt + 1):
                            v += math.prod(a[s + 1:tt + 1]) * delta[s, h_] * Bh[s, h_, n] * xs[s, h_, p]
                        yy[tt, h_, p] += Ch[tt, h_, n] * v
                        if tt == L - 1:
                            hh[h_, p, n] = v
        yy += d["D"][None, :, None] * xs
        yy *= silu_np(d["z"][0])
        _close(hf[0], hh, rtol=1e-10, what=f"M2 brute h L={L}")
        _close(y[0], yy, rtol=1e-10, what=f"M2 brute y L={L}")


def check_split_invariance(mutant=0):
    """Scanning [0, L) equals scanning [0, k) and then [k, L) from the returned
    final state and conv state, for every k (the carry the llama.cpp thread
    found broken when the ubatch size changed the output)."""
    L = 12
    for mode in (M1, M2):
        if mode == M1:
            d = W.mamba1_inputs(40, 2, L, 4, 3, dtype="f32", conv_bias=True, conv_state=True)
            run = _m1_scan
        else:
            d = W.mamba2_inputs(41, 2, L, 4, 2, 2, 3, dtype="f32", conv_bias=True, conv_state=True)
            run = _m2_scan
        y, hf, cs = run(d, mutant)
        for k in range(0, L + 1):
            first = {kk: (v[:, :k] if kk in ("x", "z", "dt", "B", "C") and v is not None else v) for kk, v in d.items()}
            second = {kk: (v[:, k:] if kk in ("x", "z", "dt", "B", "C") and v is not None else v) for kk, v in d.items()}
            y1, h1, c1 = run(first, mutant)
            second["h0"], second["conv_state_in"] = h1, c1
            y2, h2, c2 = run(second, mutant)
            _close(np.concatenate([y1, y2], axis=1), y, rtol=1e-12, atol=1e-13, what=f"split y k={k}")
            _close(h2, hf, rtol=1e-12, atol=1e-13, what=f"split h k={k}")
            _close(c2, cs, rtol=0, atol=0, what=f"split conv state k={k}")


def check_m2_reduces_to_m1(mutant=0):
    """Mamba-2 with one head per group and headdim 1 is Mamba-1 with
    A[d, n] = A[h] for every n (and B/C per group = per channel)."""
    H, N, L = 3, 4, 10
    e = W.mamba2_inputs(50, 1, L, H, 1, H, N, d_conv=0, dtype="f32")
    y2, h2, _ = _m2_scan(e, mutant)
    for h_ in range(H):
        d = dict(x=e["x"][:, :, h_:h_ + 1, 0], z=e["z"][:, :, h_:h_ + 1, 0], dt=e["dt"][:, :, h_:h_ + 1],
                 B=e["B"][:, :, h_, :], C=e["C"][:, :, h_, :], A=np.full((1, N), e["A"][h_]),
                 D=e["D"][h_:h_ + 1], dt_bias=e["dt_bias"][h_:h_ + 1], h0=e["h0"][:, h_, :, :])
        y1, h1, _ = _m1_scan(d, mutant)
        _close(y2[:, :, h_, 0], y1[:, :, 0], rtol=1e-13, what="M2->M1 y")
        _close(h2[:, h_, 0, :], h1[:, 0, :], rtol=1e-13, what="M2->M1 h")


def check_prefill_equals_decode(mutant=0):
    """T calls of the single-token update equal one forward over T tokens
    (the step-function equivalence the h0 discussion ends on)."""
    T = 7
    for mode in (M1, M2):
        if mode == M1:
            d = W.mamba1_inputs(60, 3, T, 5, 4, dtype="f32", conv_bias=True, conv_state=True)
            y, hf, cs = _m1_scan(d, mutant)
        else:
            d = W.mamba2_inputs(61, 3, T, 4, 3, 2, 5, dtype="f32", conv_bias=True, conv_state=True)
            y, hf, cs = _m2_scan(d, mutant)
        state = d["h0"].astype(np.float64).copy()
        conv_state = d["conv_state_in"].astype(np.float64).copy()
        ys = []
        for t in range(T):
            ys.append(oracle.state_update(mode, state, conv_state, d["x"][:, t], d["dt"][:, t], d["A"],
                                          d["B"][:, t], d["C"][:, t], D=d["D"], z=d["z"][:, t],
                                          dt_bias=d["dt_bias"], conv_w=d["conv_w"], conv_b=d["conv_b"],
                                          mutant=mutant))
        _close(np.stack(ys, axis=1), y, rtol=1e-12, atol=1e-13, what=f"decode y mode={mode}")
        _close(state, hf, rtol=1e-12, atol=1e-13, what=f"decode state mode={mode}")
        _close(conv_state, cs, rtol=0, atol=0, what=f"decode conv state mode={mode}")


def check_decode_wide_conv_state(mutant=0):
    """A conv state kept K columns wide (rolled left, newest last) gives the
    same outputs as the K-1-column form; its oldest column just drops out."""
    d = W.decode_inputs(62, 4, 4, 3, 2, 5, conv_state_len=4, nsets=1, dtype="f32")
    s1 = d["state"].astype(np.float64).copy()
    c1 = d["conv_state"].astype(np.float64).copy()
    y1 = oracle.state_update(M2, s1, c1, d["x"][0], d["dt"][0], d["A"], d["B"][0], d["C"][0], D=d["D"], z=d["z"][0],
                             dt_bias=d["dt_bias"], conv_w=d["conv_w"], mutant=mutant)
    s2 = d["state"].astype(np.float64).copy()
    c2 = d["conv_state"][:, :, 1:].astype(np.float64).copy()
    y2 = oracle.state_update(M2, s2, c2, d["x"][0], d["dt"][0], d["A"], d["B"][0], d["C"][0], D=d["D"], z=d["z"][0],
                             dt_bias=d["dt_bias"], conv_w=d["conv_w"], mutant=mutant)
    _close(y1, y2, rtol=0, atol=0, what="wide conv state y")
    _close(c1[:, :, 1:], c2, rtol=0, atol=0, what="wide conv state roll")
    raw = np.concatenate([d["x"][0].reshape(4, -1), d["B"][0].reshape(4, -1), d["C"][0].reshape(4, -1)], axis=1)
    _close(c1[:, :, -1], raw, rtol=0, atol=0, what="newest column")


def check_varlen_equals_per_sequence(mutant=0):
    """Packed sequences give exactly the per-sequence results; a zero-length
    sequence returns h0 and its conv state untouched; perturbing one sequence
    changes no other sequence's outputs (no leak across boundaries)."""
    lengths = [5, 0, 9, 1, 4]
    cu = W.cu_from_lengths(lengths)
    tot = int(cu[-1])
    d = W.mamba2_inputs(70, 1, tot, 4, 2, 2, 3, dtype="f32", conv_bias=True, conv_state=True, nseqs=len(lengths))
    y, hf, cs = _m2_scan(d, mutant, cu_seqlens=cu)
    for s, L in enumerate(lengths):
        a, b = cu[s], cu[s + 1]
        sub = {k: (v[:, a:b] if k in ("x", "z", "dt", "B", "C") else v) for k, v in d.items()}
        sub["h0"] = d["h0"][s:s + 1]
        sub["conv_state_in"] = d["conv_state_in"][s:s + 1]
        ys, hs, css = _m2_scan(sub, mutant)
        _close(y[:, a:b], ys, rtol=0, atol=0, what=f"varlen y seq {s}")
        _close(hf[s:s + 1], hs, rtol=0, atol=0, what=f"varlen h seq {s}")
        _close(cs[s:s + 1], css, rtol=0, atol=0, what=f"varlen conv seq {s}")
        if L == 0:
            _close(hf[s], d["h0"][s], rtol=0, atol=0, what="empty sequence keeps h0")
            _close(cs[s], d["conv_state_in"][s], rtol=0, atol=0, what="empty sequence keeps conv state")
    pert = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in d.items()}
    pert["x"][:, cu[2]:cu[3]] += 1.0
    y2, h2, c2 = _m2_scan(pert, mutant, cu_seqlens=cu)
    mask = np.ones(tot, bool)
    mask[cu[2]:cu[3]] = False
    if not np.array_equal(y2[:, mask], y[:, mask]):
        raise AssertionError("perturbing sequence 2 changed another sequence's y")
    keep = [s for s in range(len(lengths)) if s != 2]
    if not (np.array_equal(h2[keep], hf[keep]) and np.array_equal(c2[keep], cs[keep])):
        raise AssertionError("perturbing sequence 2 changed another sequence's state")


def check_intermediate_states_are_prefix_states(mutant=0):
    """Intermediate-state extraction (the conditional slot scatter that prefix
    caching uses): the state and conv history stored for boundary k equal the
    final state and conv state of a separate run over the sequence's first
    (k + 1) * interval tokens; negative and out-of-range slots write nothing,
    and pool rows nobody names keep their contents."""
    interval = 3
    lengths = [7, 0, 9, 3]
    cu = W.cu_from_lengths(lengths)
    tot = int(cu[-1])
    for mode in (M1, M2):
        if mode == M1:
            d = W.mamba1_inputs(75, 1, tot, 4, 3, dtype="f32", conv_bias=True, conv_state=True, nseqs=len(lengths))
            run = _m1_scan
        else:
            d = W.mamba2_inputs(76, 1, tot, 4, 2, 2, 3, dtype="f32", conv_bias=True, conv_state=True, nseqs=len(lengths))
            run = _m2_scan
        stride = 3
        # sequence 0: boundaries at 3, 6 -> slots 4, 0 (third entry unused: 9 > 7)
        # sequence 2: boundaries at 3, 6, 9 -> slots -1 (skip), 9 (out of range: skip), 2
        # sequence 3: boundary at 3 -> slot 5
        slots = np.array([[4, 0, 1], [6, 6, 6], [-1, 9, 2], [5, 3, 3]], dtype=np.int32)
        nslots = 7
        hs_shape = (nslots,) + (d["h0"].shape[1:])
        cdim = d["conv_w"].shape[0]
        rng = np.random.default_rng(77)
        pool_h = rng.standard_normal(hs_shape)
        pool_c = rng.standard_normal((nslots, cdim, d["conv_w"].shape[1] - 1))
        before_h, before_c = pool_h.copy(), pool_c.copy()
        run(d, mutant, cu_seqlens=cu, state_interval=interval, inter_slots=slots, inter_states=pool_h, inter_conv=pool_c)
        written = {}
        for s, L in enumerate(lengths):
            for k in range(stride):
                if (k + 1) * interval <= L and 0 <= slots[s, k] < nslots:
                    written[int(slots[s, k])] = (s, (k + 1) * interval)
        for slot in range(nslots):
            if slot not in written:
                _close(pool_h[slot], before_h[slot], rtol=0, atol=0, what=f"slot {slot} untouched (state)")
                _close(pool_c[slot], before_c[slot], rtol=0, atol=0, what=f"slot {slot} untouched (conv)")
                continue
            s, n = written[slot]
            a = cu[s]
            sub = {k: (v[:, a:a + n] if k in ("x", "z", "dt", "B", "C") else v) for k, v in d.items()}
            sub["h0"] = d["h0"][s:s + 1]
            sub["conv_state_in"] = d["conv_state_in"][s:s + 1]
            _, hp, cp = run(sub, mutant)
            _close(pool_h[slot], hp[0], rtol=0, atol=0, what=f"mode {mode} slot {slot} state = prefix state")
            _close(pool_c[slot], cp[0], rtol=0, atol=0, what=f"mode {mode} slot {slot} conv = prefix conv state")
        if sorted(written) != [0, 2, 4, 5]:
            raise AssertionError(f"unexpected written slots {sorted(written)}")


def check_backward_matches_finite_differences(mutant=0):
    """The backward (reverse mode over the stored trajectory) against central
    finite differences of the forward oracle, for every input: the loss is
    sum(dy*y) + sum(dh_final*h_final) + sum(dconv_state_out*conv_state_out) on
    packed sequences with an empty one, a conv with bias and carried state,
    grouped heads, and softplus on and off."""
    lengths = [5, 0, 4]
    cu = W.cu_from_lengths(lengths)
    tot = int(cu[-1])
    names = {"x": "dx", "z": "dz", "dt": "ddt", "B": "dB", "C": "dC", "A": "dA", "D": "dD", "dt_bias": "ddt_bias",
             "h0": "dh0", "conv_w": "dconv_w", "conv_b": "dconv_b", "conv_state_in": "dconv_state_in"}
    for mode, sp in ((M1, True), (M2, True), (M2, False)):
        if mode == M1:
            d = W.mamba1_inputs(90, 1, tot, 3, 2, d_conv=3, dtype="f32", conv_bias=True, conv_state=True, nseqs=3)
        else:
            d = W.mamba2_inputs(91, 1, tot, 4, 2, 2, 2, d_conv=3, dtype="f32", conv_bias=True, conv_state=True, nseqs=3)
        d = {k: (np.asarray(v, np.float64) if isinstance(v, np.ndarray) else v) for k, v in d.items()}
        if not sp:                         # delta = dt + dt_bias directly: keep it small and positive
            d["dt"] = np.abs(d["dt"]) * 0.1
            d["dt_bias"] = np.full_like(d["dt_bias"], 0.01)
        run = _m1_scan if mode == M1 else _m2_scan
        y, hf, cs = run(d, mutant, cu_seqlens=cu, delta_softplus=sp)
        rng = np.random.default_rng(92)
        dy, dhf, dcs = rng.standard_normal(y.shape), rng.standard_normal(hf.shape), rng.standard_normal(cs.shape)

        def loss():
            y2, h2, c2 = run(d, 0, cu_seqlens=cu, delta_softplus=sp)
            return float(np.sum(dy * y2) + np.sum(dhf * h2) + np.sum(dcs * c2))

        g = oracle.scan_bwd(mode, d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d["D"], z=d["z"], dt_bias=d["dt_bias"],
                            h0=d["h0"], cu_seqlens=cu, conv_w=d["conv_w"], conv_b=d["conv_b"],
                            conv_state_in=d["conv_state_in"], delta_softplus=sp, dh_final=dhf, dconv_state_out=dcs,
                            mutant=mutant)
        eps = 1e-6
        for k, gk in names.items():
            arr = d[k]
            fd = np.zeros_like(arr)
            for i in range(arr.size):
                old = arr.flat[i]
                arr.flat[i] = old + eps
                lp = loss()
                arr.flat[i] = old - eps
                lm = loss()
                arr.flat[i] = old
                fd.flat[i] = (lp - lm) / (2 * eps)
            _close(g[gk], fd, rtol=1e-6, atol=1e-9, what=f"mode {mode} softplus {sp}: {gk} vs finite differences")


# ------------------------------------------------------------ conv pins
def check_conv_impulse(mutant=0):
    """A unit impulse at t = 0 through a conv without activation returns each
    channel's taps reversed in time: out[t, c] = w[c, K-1-t]."""
    K, Cn, T = 4, 5, 6
    rng = np.random.default_rng(80)
    w = rng.uniform(-1, 1, size=(Cn, K))
    x = np.zeros((1, T, Cn))
    x[0, 0, :] = 1.0
    out, st = oracle.conv1d_fwd(x, w, activation=False, mutant=mutant)
    exp = np.zeros((T, Cn))
    for t in range(K):
        exp[t] = w[:, K - 1 - t]
    _close(out[0], exp, rtol=0, atol=0, what="impulse response")
    _close(st[0], np.zeros((Cn, K - 1)), rtol=0, atol=0, what="state after impulse passed")


def check_conv_width_one(mutant=0):
    """K = 1 makes the conv a per-channel scale + bias, then SiLU."""
    rng = np.random.default_rng(81)
    x = rng.standard_normal((2, 7, 3))
    w = rng.standard_normal((3, 1))
    b = rng.standard_normal(3)
    out, st = oracle.conv1d_fwd(x, w, b=b, activation=True, mutant=mutant)
    _close(out, silu_np(x * w[:, 0] + b), rtol=1e-13, what="K=1")
    if st is not None:
        raise AssertionError("K=1 has no carried state")


def check_conv_reformulations(mutant=0):
    """The conv equals concat + im2col + matmul and multiply + row sums
    (the two reformulations discussed on the llama.cpp page), including a
    carried state and a bias."""
    rng = np.random.default_rng(82)
    T, Cn, K = 9, 6, 4
    x = rng.standard_normal((1, T, Cn))
    w = rng.standard_normal((Cn, K))
    b = rng.standard_normal(Cn)
    st = rng.standard_normal((1, Cn, K - 1))
    out, so = oracle.conv1d_fwd(x, w, b=b, state_in=st, activation=True, mutant=mutant)
    ref, ref_state = conv_im2col(x[0], w, b, st[0])
    _close(out[0], ref, rtol=1e-13, what="im2col")
    _close(out[0], conv_mul_sumrows(x[0], w, b, st[0]), rtol=1e-13, what="mul+sum_rows")
    _close(so[0], ref_state, rtol=0, atol=0, what="conv state out")


def check_fused_conv_matches_standalone(mutant=0):
    """The scan's fused conv front-end equals the standalone conv op feeding an
    unfused scan."""
    d = W.mamba1_inputs(83, 2, 10, 4, 3, dtype="f32", conv_bias=True, conv_state=True)
    y, hf, cs = _m1_scan(d, mutant)
    xc, so = oracle.conv1d_fwd(d["x"], d["conv_w"], b=d["conv_b"], state_in=d["conv_state_in"], mutant=mutant)
    e = dict(d)
    e["x"], e["conv_w"], e["conv_b"], e["conv_state_in"] = xc, None, None, None
    y2, h2, _ = _m1_scan(e, mutant)
    _close(y, y2, rtol=1e-13, what="fused vs standalone conv y")
    _close(hf, h2, rtol=1e-13, what="fused vs standalone conv h")
    _close(cs, so, rtol=0, atol=0, what="fused vs standalone conv state")


ALL_CHECKS = [
    check_A_zero_is_cumsum, check_zero_delta_keeps_h0, check_geometric_fixed_point, check_bruteforce_m1,
    check_bruteforce_m2, check_split_invariance, check_m2_reduces_to_m1, check_prefill_equals_decode,
    check_decode_wide_conv_state, check_varlen_equals_per_sequence, check_conv_impulse, check_conv_width_one,
    check_conv_reformulations, check_fused_conv_matches_standalone, check_intermediate_states_are_prefix_states,
    check_backward_matches_finite_differences,
]
