"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
CUDA path through the C ABI, run the oracle on the same values, compare.

Tolerances (max|err| / max|ref| per output tensor): 1e-4 for fp32 inputs and
2e-2 for bf16 inputs, for y, the final state and the conv state.  The bf16
bound covers the one rounding of y to bf16 (2^-9 relative) with margin for
the fp32 accumulation order; fp32 runs additionally meet NMSE <= 1e-7, the
threshold test-backend-ops uses for these ops.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import state_space_model_conv1d_b200 as ssm

TOL = {"f32": 1e-4, "bf16": 2e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}
ACT_KEYS = ("x", "z", "dt", "B", "C", "conv_state_in", "conv_state")


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if ref.size == 0:
        return 0.0
    den = np.max(np.abs(ref))
    err = np.max(np.abs(got - ref))
    return float(err / den) if den > 0 else float(err)


def nmse(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.sum(ref * ref)
    return float(np.sum((got - ref) ** 2) / den) if den > 0 else 0.0


def assert_close(got, ref, dtype, what):
    e = rel_err(got, ref)
    assert e <= TOL[dtype], f"{what}: max|err|/max|ref| = {e:.3e} > {TOL[dtype]}"
    if dtype == "f32":
        assert nmse(got, ref) <= 1e-7, f"{what}: NMSE {nmse(got, ref):.3e}"


def to_dev(d: dict, dtype: str) -> dict:
    out = {}
    for k, v in d.items():
        if v is None or k == "cu_seqlens":
            out[k] = None if v is None else torch.from_numpy(np.asarray(v, np.int32)).cuda()
            continue
        t = torch.from_numpy(np.ascontiguousarray(v))
        out[k] = t.to(device="cuda", dtype=TDT[dtype] if k in ACT_KEYS else torch.float32)
    return out


def as_views(t: dict, mode: int) -> dict:
    """Re-home x and z as views of one wider projection row (x | z), and for
    Mamba-2 x, B and C as views of one x | B | C row, like an in_proj output."""
    t = dict(t)
    x, z = t["x"], t["z"]
    b, T = x.shape[0], x.shape[1]
    if mode == oracle.MAMBA1:
        Dn = x.shape[2]
        buf = torch.empty((b, T, 2 * Dn + 8), dtype=x.dtype, device=x.device)
        buf[..., :Dn] = x
        t["x"] = buf[..., :Dn]
        if z is not None:
            buf[..., Dn:2 * Dn] = z
            t["z"] = buf[..., Dn:2 * Dn]
    else:
        H, P = x.shape[2], x.shape[3]
        G, N = t["B"].shape[2], t["B"].shape[3]
        w = H * P + 2 * G * N
        buf = torch.empty((b, T, w + 16), dtype=x.dtype, device=x.device)
        buf[..., :H * P] = x.reshape(b, T, H * P)
        buf[..., H * P:H * P + G * N] = t["B"].reshape(b, T, G * N)
        buf[..., H * P + G * N:w] = t["C"].reshape(b, T, G * N)
        t["x"] = buf[..., :H * P].unflatten(2, (H, P))
        t["B"] = buf[..., H * P:H * P + G * N].unflatten(2, (G, N))
        t["C"] = buf[..., H * P + G * N:w].unflatten(2, (G, N))
        if z is not None:
            zb = torch.empty((b, T, H * P + 24), dtype=x.dtype, device=x.device)
            zb[..., 8:8 + H * P] = z.reshape(b, T, H * P)
            t["z"] = zb[..., 8:8 + H * P].unflatten(2, (H, P))
    return t


def gpu_scan(mode, t: dict, chunk=0, delta_softplus=True, segments=0):
    y, hf, cs = ssm.scan_fwd(mode, t["x"], t["dt"], t["A"], t["B"], t["C"], D=t.get("D"), z=t.get("z"),
                             dt_bias=t.get("dt_bias"), h0=t.get("h0"), cu_seqlens=t.get("cu_seqlens"),
                             conv_w=t.get("conv_w"), conv_b=t.get("conv_b"), conv_state_in=t.get("conv_state_in"),
                             delta_softplus=delta_softplus, chunk=chunk, segments=segments)
    torch.cuda.synchronize()
    f = lambda a: None if a is None else a.float().cpu().numpy().astype(np.float64)
    return f(y), f(hf), f(cs)


def oracle_scan(mode, d: dict, delta_softplus=True):
    return oracle.scan_fwd(mode, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d.get("D"), z=d.get("z"),
                           dt_bias=d.get("dt_bias"), h0=d.get("h0"), cu_seqlens=d.get("cu_seqlens"),
                           conv_w=d.get("conv_w"), conv_b=d.get("conv_b"), conv_state_in=d.get("conv_state_in"),
                           delta_softplus=delta_softplus, nthreads=8)


def check_scan(mode, d: dict, dtype: str, views=False, chunk=0, what="", segments=0):
    t = to_dev(d, dtype)
    if views:
        t = as_views(t, mode)
    y, hf, cs = gpu_scan(mode, t, chunk=chunk, segments=segments)
    ry, rh, rc = oracle_scan(mode, d)
    assert_close(y, ry, dtype, f"{what} y")
    assert_close(hf, rh, dtype, f"{what} h_final")
    if rc is not None:
        assert cs is not None
        assert_close(cs, rc, dtype, f"{what} conv_state_out")
    return y, hf, cs
