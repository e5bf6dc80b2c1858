"""A CPU stand-in, in fp64, for the calls a split scan makes.

``SegmentScan`` takes a ``backend`` with the package's entry points; this one
lets the split protocol (the two exchanges, the rank bookkeeping, the
packing of the pairs) run on CPU ranks.  ``scan_fwd`` is the oracle's
unsplit scan of one segment.  The four split steps are written out here from
their definitions, with numpy:

- the conv tail: the last K-1 entries of concat(carried state, raw inputs);
- cum_delta: the running sum of delta = softplus(dt + dt_bias) over the
  segment's tokens;
- combine: H_0 = h_loc_0, H_k = exp(A * sum_delta_k) * H_{k-1} + h_loc_k;
- fix-up: y_t += silu(z_t) * sum_n C_t[n] * exp(A cs_t) * h_in[..., n].

The scan element (exp(delta*A), h) and its seed (1, h0) come from "Adding
Initial Value Support to Selective Scan Forward Kernel" (state-spaces/mamba
issue 285).  Test infrastructure only.
"""
import numpy as np
import torch

import oracle

M1 = oracle.MAMBA1
PACK_DTYPE = torch.float64     # the exchanged pairs keep the oracle's precision


def _np(t):
    return None if t is None else t.detach().cpu().numpy().astype(np.float64)


def _t(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _silu(v):
    return v / (1.0 + np.exp(-v))


def scan_fwd(mode, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None, h0=None, conv_w=None, conv_b=None,
             conv_state_in=None, delta_softplus=True, h_final=None, stream=None):
    y, hf, cs = oracle.scan_fwd(mode, _np(x), _np(dt), _np(A), _np(B), _np(C_), D=_np(D), z=_np(z),
                                dt_bias=_np(dt_bias), h0=_np(h0), conv_w=_np(conv_w), conv_b=_np(conv_b),
                                conv_state_in=_np(conv_state_in), delta_softplus=delta_softplus)
    hf = _t(hf)
    if h_final is not None:
        h_final.copy_(hf)
        hf = h_final
    return _t(y), hf, _t(cs)


def _conv_inputs(mode, x, B, C_):
    """Raw conv channels ``[b, T, conv_dim]`` (x, or x | B | C)."""
    b, T = x.shape[0], x.shape[1]
    if mode == M1:
        return _np(x)
    return np.concatenate([_np(x).reshape(b, T, -1), _np(B).reshape(b, T, -1), _np(C_).reshape(b, T, -1)], axis=2)


def split_conv_tail(mode, x, dt, A, B, C_, *, conv_w, conv_state_in=None, stream=None, **_):
    u = _conv_inputs(mode, x, B, C_)
    b, T, cdim = u.shape
    K = conv_w.shape[1]
    hist = np.zeros((b, cdim, K - 1)) if conv_state_in is None else _np(conv_state_in)
    full = np.concatenate([hist, u.transpose(0, 2, 1)], axis=2)
    return _t(full[:, :, full.shape[2] - (K - 1):])


def split_cum_delta(mode, x, dt, A, B, C_, *, dt_bias=None, delta_softplus=True, cum=True, sum_delta=None,
                    stream=None, **_):
    r = _np(dt) + (0.0 if dt_bias is None else _np(dt_bias))
    d = np.log1p(np.exp(r)) if delta_softplus else r
    cs = np.cumsum(d, axis=1)
    sd = _t(d.sum(axis=1))
    if sum_delta is not None:
        sum_delta.copy_(sd)
        sd = sum_delta
    return (_t(cs) if cum else None), sd


def split_combine(mode, A, sum_delta_all, h_local_all, rank, *, stream=None):
    sd, hl, a = _np(sum_delta_all), _np(h_local_all), _np(A)
    H = hl[0]
    before = np.zeros_like(H)
    for k in range(1, rank + 1):
        before = H
        if mode == M1:
            dec = np.exp(a[None] * sd[k][:, :, None])
        else:
            dec = np.exp(a[None, :, None, None] * sd[k][:, :, None, None])
        H = dec * H + hl[k]
    return _t(before), _t(H)


def split_fixup(mode, x, dt, A, B, C_, y, cum_delta, h_in, *, z=None, conv_w=None, conv_b=None,
                conv_state_in=None, stream=None, **_):
    cs, h, a = _np(cum_delta), _np(h_in), _np(A)
    gate = 1.0 if z is None else _silu(_np(z))
    if mode == M1:
        corr = np.einsum("btn,btdn,bdn->btd", _np(C_), np.exp(a[None, None] * cs[..., None]), h)
    else:
        b, T, Hh, P = x.shape
        G, N = C_.shape[2], C_.shape[3]
        Craw = _np(C_).reshape(b, T, G * N)
        if conv_w is not None:
            off = Hh * P + G * N
            si = None if conv_state_in is None else _np(conv_state_in)[:, off:, :]
            Cc, _ = oracle.conv1d_fwd(Craw, _np(conv_w)[off:], b=None if conv_b is None else _np(conv_b)[off:],
                                      state_in=si, activation=True)
        else:
            Cc = Craw
        Cg = np.repeat(Cc.reshape(b, T, G, N), Hh // G, axis=2)
        corr = np.einsum("bthn,bhpn->bthp", Cg, h) * np.exp(a[None, None, :] * cs)[..., None]
    y.copy_(_t(_np(y) + gate * corr))
    return y
