"""Thin PyTorch-facing binding of the C ABI (same entry-point names).

Argument marshalling only: shapes and strides are read from the tensors,
outputs are allocated with PyTorch's allocator when the caller does not pass
them, and the call is enqueued on the current CUDA stream.  Every step of the
computation runs inside ``libssm.so``.

Tensor conventions (channel dimension contiguous; batch / token strides free):

Mamba-1: x, z, dt, y ``[b, T, D]``; B, C ``[b, T, N]``; A ``[D, N]``; D,
dt_bias ``[D]``; h0 / h_final ``[nseq, D, N]``; conv_w ``[D, K]``; conv states
``[nseq, D, K-1]``.

Mamba-2: x, z, y ``[b, T, H, P]``; dt ``[b, T, H]``; B, C ``[b, T, G, N]``;
A, D, dt_bias ``[H]``; h0 / h_final ``[nseq, H, P, N]``; conv_w
``[H*P + 2*G*N, K]`` (x | B | C); conv states ``[nseq, H*P + 2*G*N, K-1]``.

Packed varlen: b = 1 and ``cu_seqlens`` int32 ``[nseq + 1]`` on the device.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _abi
from ._abi import SSM_BF16, SSM_F32, SSM_MAMBA1, SSM_MAMBA2

MAMBA1, MAMBA2 = SSM_MAMBA1, SSM_MAMBA2


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    if t.dtype == torch.float32:
        return SSM_F32
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _need(t, name, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _rows(t, inner_dims: int, name: str):
    """(batch stride, token stride) of a [b, T, *inner] tensor whose inner dims are contiguous."""
    if t is None:
        return 0, 0
    exp = 1
    for d in range(t.dim() - 1, t.dim() - 1 - inner_dims, -1):
        if t.shape[d] != 1 and t.stride(d) != exp:
            raise ValueError(f"{name}: the channel dimensions must be contiguous")
        exp *= t.shape[d]
    return t.stride(0), t.stride(1)


def _c32(t, name):
    if t is None:
        return None
    _need(t, name, torch.float32)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous float32")
    return t


def conv1d_fwd(x, weight, bias=None, *, state_in=None, state_out=None, cu_seqlens=None, activation=True,
               out=None, stream=None):
    """Causal depthwise conv over ``x [b, T, C]`` with weight ``[C, K]``."""
    _need(x, "x")
    b, T, Cn = x.shape
    K = weight.shape[1]
    if out is None:
        out = torch.empty((b, T, Cn), dtype=x.dtype, device=x.device)
    a = _abi.ConvArgs()
    a.batch, a.seqlen, a.channels, a.width = b, T, Cn, K
    a.dtype, a.activation = _dtype_code(x), int(bool(activation))
    a.nseqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    a.x = _p(x)
    a.x_batch_stride, a.x_token_stride = _rows(x, 1, "x")
    a.weight, a.bias = _p(_c32(weight, "weight")), _p(_c32(bias, "bias"))
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None and (not t.is_contiguous() or t.dtype != x.dtype):
            raise ValueError(f"{n} must be contiguous with x's dtype")
    a.state_in, a.state_out = _p(state_in), _p(state_out)
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32)
    a.cu_seqlens = _p(cu_seqlens)
    a.out = _p(out)
    a.out_batch_stride, a.out_token_stride = _rows(out, 1, "out")
    _abi.check(_abi.lib().ssm_conv1d_fwd(C.byref(a), _stream(stream)), "ssm_conv1d_fwd")
    return out


def _scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, h0, h_final, cu_seqlens, conv_w, conv_b, conv_state_in,
               conv_state_out, y, delta_softplus, chunk):
    a = _abi.ScanArgs()
    a.mode, a.dtype, a.delta_softplus = mode, _dtype_code(x), int(bool(delta_softplus))
    b, T = x.shape[0], x.shape[1]
    if mode == MAMBA1:
        Dn, N = x.shape[2], B.shape[2]
        H, P, G = 0, 0, 1
        inner_x, inner_dt, inner_bc = 1, 1, 1
    else:
        H, P = x.shape[2], x.shape[3]
        G, N = B.shape[2], B.shape[3]
        Dn = H * P
        inner_x, inner_dt, inner_bc = 2, 1, 2
    a.batch, a.seqlen, a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate = b, T, Dn, H, P, G, N
    a.d_conv = 0 if conv_w is None else conv_w.shape[1]
    a.nseqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    for t, n in ((x, "x"), (dt, "dt"), (B, "B"), (C_, "C"), (z, "z"), (y, "y")):
        _need(t, n, x.dtype)
    a.x = _p(x); a.x_batch_stride, a.x_token_stride = _rows(x, inner_x, "x")
    a.z = _p(z); a.z_batch_stride, a.z_token_stride = _rows(z, inner_x, "z")
    a.dt = _p(dt); a.dt_batch_stride, a.dt_token_stride = _rows(dt, inner_dt, "dt")
    a.B = _p(B); a.B_batch_stride, a.B_token_stride = _rows(B, inner_bc, "B")
    a.C = _p(C_); a.C_batch_stride, a.C_token_stride = _rows(C_, inner_bc, "C")
    a.y = _p(y); a.y_batch_stride, a.y_token_stride = _rows(y, inner_x, "y")
    a.A, a.D, a.dt_bias = _p(_c32(A, "A")), _p(_c32(D, "D")), _p(_c32(dt_bias, "dt_bias"))
    a.h0, a.h_final = _p(_c32(h0, "h0")), _p(_c32(h_final, "h_final"))
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", torch.int32)
    a.cu_seqlens = _p(cu_seqlens)
    a.conv_w, a.conv_b = _p(_c32(conv_w, "conv_w")), _p(_c32(conv_b, "conv_b"))
    for t, n in ((conv_state_in, "conv_state_in"), (conv_state_out, "conv_state_out")):
        if t is not None and (not t.is_contiguous() or t.dtype != x.dtype):
            raise ValueError(f"{n} must be contiguous with x's dtype")
    a.conv_state_in, a.conv_state_out = _p(conv_state_in), _p(conv_state_out)
    a.chunk = int(chunk)
    return a


def scan_workspace_size(mode, x, dt, A, B, C_, *, cu_seqlens=None, conv_w=None, segments=0, **_):
    """Bytes of device workspace ssm_scan_fwd needs for these shapes (0 = none)."""
    a = _abi.ScanArgs()
    a.mode, a.dtype = mode, _dtype_code(x)
    a.batch, a.seqlen = x.shape[0], x.shape[1]
    if mode == MAMBA1:
        a.d_inner, a.ngroups, a.dstate = x.shape[2], 1, B.shape[2]
    else:
        a.nheads, a.headdim = x.shape[2], x.shape[3]
        a.d_inner = a.nheads * a.headdim
        a.ngroups, a.dstate = B.shape[2], B.shape[3]
    a.d_conv = 0 if conv_w is None else conv_w.shape[1]
    a.cu_seqlens = _p(cu_seqlens)
    a.nseqs = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    a.segments = int(segments)
    return int(_abi.lib().ssm_scan_workspace_size(C.byref(a)))


def scan_segments(mode, x, dt, A, B, C_, *, z=None, cu_seqlens=None, conv_w=None, segments=0, **_):
    """Token segments ``scan_fwd`` cuts each row into for these tensors (1 = rows stay whole)."""
    a = _scan_args(mode, x, dt, A, B, C_, None, z, None, None, None, cu_seqlens, conv_w, None, None, None, x, True, 0)
    a.segments = int(segments)
    return int(_abi.lib().ssm_scan_segments(C.byref(a)))


def scan_fwd(mode, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None, h0=None, cu_seqlens=None, conv_w=None,
             conv_b=None, conv_state_in=None, delta_softplus=True, y=None, h_final=None, conv_state_out=None,
             return_final_state=True, return_conv_state=None, workspace=None, chunk=0, stream=None,
             state_interval=0, inter_slots=None, inter_states=None, inter_conv=None, segments=0):
    """Forward selective scan (conv fused in front when ``conv_w`` is given).

    Returns ``(y, h_final, conv_state_out)``; the last two are None when not
    requested.  ``workspace`` (uint8 CUDA tensor) is allocated when needed and
    not given.

    Intermediate states (prefix caching): with ``state_interval`` (a positive
    multiple of 64) and ``inter_slots`` (int32 ``[nseq, stride]``), the state
    after every ``state_interval`` tokens of each sequence is written to row
    ``inter_slots[s, k]`` of ``inter_states`` (fp32 ``[nslots, ...state]``) and
    its conv history to ``inter_conv`` (``[nslots, conv_dim, K-1]``, x's
    dtype); negative or out-of-range slots write nothing.

    ``segments`` (Mamba-2 tensor-core path, rows without ``cu_seqlens``): 0 lets
    the library choose, 1 keeps one CTA per (row, head), n >= 2 scans about n
    runs of every row at the same time (see ``ssm_scan_args.segments``).
    """
    _need(x, "x")
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    nseq = x.shape[0] if cu_seqlens is None else cu_seqlens.numel() - 1
    if mode == MAMBA1:
        hshape = (nseq, x.shape[2], B.shape[2])
        cdim = x.shape[2]
    else:
        hshape = (nseq, x.shape[2], x.shape[3], B.shape[3])
        cdim = x.shape[2] * x.shape[3] + 2 * B.shape[2] * B.shape[3]
    if h_final is None and return_final_state:
        h_final = torch.empty(hshape, dtype=torch.float32, device=x.device)
    if return_conv_state is None:
        return_conv_state = conv_w is not None and conv_w.shape[1] > 1
    if conv_state_out is None and return_conv_state and conv_w is not None and conv_w.shape[1] > 1:
        conv_state_out = torch.empty((nseq, cdim, conv_w.shape[1] - 1), dtype=x.dtype, device=x.device)
    a = _scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, h0, h_final, cu_seqlens, conv_w, conv_b, conv_state_in,
                   conv_state_out, y, delta_softplus, chunk)
    a.segments = int(segments)
    if state_interval:
        if inter_slots is None or (inter_states is None and inter_conv is None):
            raise ValueError("state_interval needs inter_slots and a pool")
        _need(inter_slots, "inter_slots", torch.int32)
        if not inter_slots.is_contiguous():
            raise ValueError("inter_slots must be contiguous")
        if inter_states is not None and (inter_states.dtype != torch.float32 or not inter_states.is_contiguous()):
            raise ValueError("inter_states must be contiguous fp32")
        if inter_conv is not None and (inter_conv.dtype != x.dtype or not inter_conv.is_contiguous()):
            raise ValueError("inter_conv must be contiguous with x's dtype")
        a.state_interval = int(state_interval)
        a.inter_slots = _p(inter_slots)
        a.inter_stride = inter_slots.shape[1] if inter_slots.dim() == 2 else inter_slots.numel()
        pool = inter_states if inter_states is not None else inter_conv
        a.inter_nslots = pool.shape[0]
        a.inter_states, a.inter_conv = _p(inter_states), _p(inter_conv)
    l = _abi.lib()
    need = int(l.ssm_scan_workspace_size(C.byref(a)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_ptr = _p(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel()
    _abi.check(l.ssm_scan_fwd(C.byref(a), ws_ptr, ws_bytes, _stream(stream)), "ssm_scan_fwd")
    return y, h_final, conv_state_out


def workspace_error(workspace, stream=None):
    """Synchronizes and returns the device error code held in a scan workspace (0 = none)."""
    code = _abi._i32(0)
    st = _abi.lib().ssm_workspace_error(_p(workspace), C.byref(code), _stream(stream))
    if st not in (_abi.SSM_OK, _abi.SSM_ERR_DEVICE):
        _abi.check(st, "ssm_workspace_error")
    return int(code.value)


def state_update(mode, state, conv_state, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None, conv_w=None,
                 conv_b=None, delta_softplus=True, state_batch_indices=None, y=None, stream=None):
    """One decode token per row, state and conv_state updated in place; returns y.

    Mamba-1: x, z, dt ``[b, D]``; B, C ``[b, N]``; state ``[slots, D, N]``.
    Mamba-2: x, z ``[b, H, P]``; dt ``[b, H]``; B, C ``[b, G, N]``; state
    ``[slots, H, P, N]``.  conv_state ``[slots, conv_dim, L]`` with L >= K-1.
    """
    _need(x, "x")
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, device=x.device)
    a = _abi.UpdateArgs()
    a.mode, a.dtype, a.delta_softplus = mode, _dtype_code(x), int(bool(delta_softplus))
    b = x.shape[0]
    if mode == MAMBA1:
        Dn, N = x.shape[1], B.shape[1]
        H, P, G = 0, 0, 1
    else:
        H, P = x.shape[1], x.shape[2]
        G, N = B.shape[1], B.shape[2]
        Dn = H * P
    a.batch, a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate = b, Dn, H, P, G, N
    a.d_conv = 0 if conv_w is None else conv_w.shape[1]
    a.conv_state_len = 0 if conv_state is None else conv_state.shape[-1]
    if not state.is_contiguous() or state.dtype != torch.float32:
        raise ValueError("state must be contiguous float32")
    if conv_state is not None and (not conv_state.is_contiguous() or conv_state.dtype != x.dtype):
        raise ValueError("conv_state must be contiguous with x's dtype")
    a.state, a.conv_state = _p(state), _p(conv_state)
    a.conv_w, a.conv_b = _p(_c32(conv_w, "conv_w")), _p(_c32(conv_b, "conv_b"))

    def bs(t, name, inner):
        if t is None:
            return 0
        _need(t, name, x.dtype)
        exp = 1
        for d in range(t.dim() - 1, t.dim() - 1 - inner, -1):
            if t.shape[d] != 1 and t.stride(d) != exp:
                raise ValueError(f"{name}: the channel dimensions must be contiguous")
            exp *= t.shape[d]
        return t.stride(0)

    inner = 1 if mode == MAMBA1 else 2
    a.x, a.x_batch_stride = _p(x), bs(x, "x", inner)
    a.z, a.z_batch_stride = _p(z), bs(z, "z", inner)
    a.dt, a.dt_batch_stride = _p(dt), bs(dt, "dt", 1)
    a.B, a.B_batch_stride = _p(B), bs(B, "B", inner)
    a.C, a.C_batch_stride = _p(C_), bs(C_, "C", inner)
    a.y, a.y_batch_stride = _p(y), bs(y, "y", inner)
    a.A, a.D, a.dt_bias = _p(_c32(A, "A")), _p(_c32(D, "D")), _p(_c32(dt_bias, "dt_bias"))
    if state_batch_indices is not None:
        _need(state_batch_indices, "state_batch_indices", torch.int32)
    a.state_batch_indices = _p(state_batch_indices)
    a.nslots = state.shape[0]
    _abi.check(_abi.lib().ssm_state_update(C.byref(a), _stream(stream)), "ssm_state_update")
    return y


def kernel_timing(enable: bool) -> None:
    """Turn on / off device timing of each call's dominant kernel (process-wide)."""
    _abi.check(_abi.lib().ssm_kernel_timing(int(bool(enable))), "ssm_kernel_timing")


def kernel_time_ms():
    """(summed milliseconds, launches) of the timed kernels since the last read; synchronizes."""
    ms, n = C.c_float(0.0), _abi._i32(0)
    _abi.check(_abi.lib().ssm_kernel_time_ms(C.byref(ms), C.byref(n)), "ssm_kernel_time_ms")
    return float(ms.value), int(n.value)



def scan_bwd(mode, x, dt, A, B, C_, dy, *, D=None, z=None, dt_bias=None, h0=None, cu_seqlens=None, conv_w=None,
             conv_b=None, conv_state_in=None, delta_softplus=True, dh_final=None, dconv_state_out=None,
             workspace=None, out=None, stream=None):
    """Backward of :func:`scan_fwd`: gradients of sum(dy*y) + sum(dh_final*h_final)
    + sum(dconv_state_out*conv_state_out) with respect to every input.

    Returns a dict of fp32 CUDA tensors shaped like the inputs: ``dx, dz, ddt,
    dB, dC`` (raw, before the conv), ``dA, dD, ddt_bias, dh0, dconv_w, dconv_b,
    dconv_state_in`` (None where the input is None).  ``out`` (such a dict from
    an earlier call with the same shapes) is filled instead of allocating.
    """
    _need(dy, "dy", x.dtype)
    nseq = x.shape[0] if cu_seqlens is None else cu_seqlens.numel() - 1
    if mode == MAMBA1:
        hshape = (nseq, x.shape[2], B.shape[2])
        cdim = x.shape[2]
    else:
        hshape = (nseq, x.shape[2], x.shape[3], B.shape[3])
        cdim = x.shape[2] * x.shape[3] + 2 * B.shape[2] * B.shape[3]
    dev = x.device
    f32 = lambda shape: torch.empty(shape, dtype=torch.float32, device=dev)
    K = 0 if conv_w is None else conv_w.shape[1]
    if out is None:
        out = dict(dx=f32(x.shape), dz=None if z is None else f32(z.shape), ddt=f32(dt.shape), dB=f32(B.shape),
                   dC=f32(C_.shape), dA=f32(A.shape), dD=None if D is None else f32(D.shape),
                   ddt_bias=None if dt_bias is None else f32(dt_bias.shape), dh0=f32(hshape),
                   dconv_w=None if conv_w is None else f32(conv_w.shape),
                   dconv_b=None if conv_b is None or conv_w is None else f32(conv_b.shape),
                   dconv_state_in=f32((nseq, cdim, K - 1)) if K > 1 else None)
    b = _abi.ScanBwdArgs()
    b.fwd = _scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, h0, None, cu_seqlens, conv_w, conv_b, conv_state_in,
                       None, dy, delta_softplus, 0)
    b.dy = _p(dy)
    b.dy_batch_stride, b.dy_token_stride = b.fwd.y_batch_stride, b.fwd.y_token_stride
    b.dh_final = _p(_c32(dh_final, "dh_final"))
    if dconv_state_out is not None and (not dconv_state_out.is_contiguous() or dconv_state_out.dtype != x.dtype):
        raise ValueError("dconv_state_out must be contiguous with x's dtype")
    b.dconv_state_out = _p(dconv_state_out)
    for k, v in out.items():
        setattr(b, k, _p(v))
    l = _abi.lib()
    need = int(l.ssm_scan_bwd_workspace_size(C.byref(b)))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _abi.check(l.ssm_scan_bwd(C.byref(b), _p(workspace), workspace.numel(), _stream(stream)), "ssm_scan_bwd")
    return out


def scan_bwd_workspace_size(mode, x, dt, A, B, C_, dy, *, cu_seqlens=None, conv_w=None, **_):
    """Bytes of device workspace ssm_scan_bwd needs for these shapes."""
    b = _abi.ScanBwdArgs()
    b.fwd = _scan_args(mode, x, dt, A, B, C_, None, None, None, None, None, cu_seqlens, conv_w, None, None, None, dy,
                       True, 0)
    b.dy = _p(dy)
    return int(_abi.lib().ssm_scan_bwd_workspace_size(C.byref(b)))


# ---------------------------------------------------------------- sequence split
# One batch of sequences split along its tokens across ranks (see
# seq_split.py for the whole protocol).  Each call below takes the segment's
# tensors as scan_fwd does; y stands in for the output layout and is only
# written by split_fixup.

def _split_scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, conv_w, conv_b, conv_state_in, y, delta_softplus):
    return _scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, None, None, None, conv_w, conv_b, conv_state_in, None,
                      x if y is None else y, delta_softplus, 0)


def _conv_dim(mode, x, B):
    return x.shape[2] if mode == MAMBA1 else x.shape[2] * x.shape[3] + 2 * B.shape[2] * B.shape[3]


def split_conv_tail(mode, x, dt, A, B, C_, *, conv_w, D=None, z=None, dt_bias=None, conv_b=None,
                    conv_state_in=None, delta_softplus=True, tail=None, stream=None):
    """The segment's last K-1 raw conv inputs, ``[b, conv_dim, K-1]`` in x's dtype (conv_state_out layout)."""
    K = conv_w.shape[1]
    if tail is None:
        tail = torch.empty((x.shape[0], _conv_dim(mode, x, B), K - 1), dtype=x.dtype, device=x.device)
    a = _split_scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, conv_w, conv_b, conv_state_in, None, delta_softplus)
    _abi.check(_abi.lib().ssm_split_conv_tail(C.byref(a), _p(tail), _stream(stream)), "ssm_split_conv_tail")
    return tail


def split_cum_delta(mode, x, dt, A, B, C_, *, dt_bias=None, delta_softplus=True, cum=True, sum_delta=None, D=None,
                    z=None, conv_w=None, conv_b=None, conv_state_in=None, stream=None):
    """``(cum_delta [b, T, U] or None, sum_delta [b, U])`` of the segment, fp32 (U = channels or heads);
    ``sum_delta`` (contiguous fp32 ``[b, U]``) receives the totals when given."""
    U = x.shape[2]
    b, T = x.shape[0], x.shape[1]
    cd = torch.empty((b, T, U), dtype=torch.float32, device=x.device) if cum else None
    if sum_delta is None:
        sd = torch.empty((b, U), dtype=torch.float32, device=x.device)
    else:
        sd = _c32(sum_delta, "sum_delta")
        if tuple(sd.shape) != (b, U):
            raise ValueError(f"sum_delta must be [{b}, {U}]")
    a = _split_scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, conv_w, conv_b, conv_state_in, None, delta_softplus)
    _abi.check(_abi.lib().ssm_split_cum_delta(C.byref(a), _p(cd), _p(sd), _stream(stream)), "ssm_split_cum_delta")
    return cd, sd


def _rank_blocks(t, name):
    """``(t, rank stride)`` for a ``[R, ...]`` fp32 tensor whose rank blocks are each
    contiguous: stride 0 (dense) or the view's own, else a contiguous copy."""
    _need(t, name, torch.float32)
    if t.is_contiguous():
        return t, 0
    blk = 1
    for v in t.shape[1:]:
        blk *= v
    inner = t[0] if t.shape[0] > 0 else t
    if t.shape[0] > 0 and inner.is_contiguous() and t.stride(0) >= blk and t.stride(0) % 4 == 0:
        return t, int(t.stride(0))
    return t.contiguous(), 0


def split_combine(mode, A, sum_delta_all, h_local_all, rank, *, h_in=None, h_out=None, stream=None):
    """Fold the gathered ``(sum_delta, h_loc)`` of ranks 0..rank: ``(h_in, h_out)`` of this rank's segment.

    ``sum_delta_all`` is ``[R, b, U]`` and ``h_local_all`` ``[R, b, *state]``, fp32.  Each rank's block
    must be contiguous; the rank dimension may be strided (views of one gathered buffer of packed pairs),
    which the library reads in place when the stride is a multiple of 4 elements.
    """
    R, b = h_local_all.shape[0], h_local_all.shape[1]
    state = tuple(h_local_all.shape[2:])
    sum_delta_all, sd_rs = _rank_blocks(sum_delta_all, "sum_delta_all")
    h_local_all, hl_rs = _rank_blocks(h_local_all, "h_local_all")
    if h_in is None:
        h_in = torch.empty((b,) + state, dtype=torch.float32, device=h_local_all.device)
    if h_out is None:
        h_out = torch.empty((b,) + state, dtype=torch.float32, device=h_local_all.device)
    a = _abi.SplitArgs()
    a.mode, a.rank, a.nranks = mode, int(rank), R
    a.batch = b
    if mode == MAMBA1:
        a.d_inner, a.dstate = state[0], state[1]
    else:
        a.nheads, a.headdim, a.dstate = state
        a.d_inner = state[0] * state[1]
    a.A, a.sum_delta, a.h_local = _p(_c32(A, "A")), _p(sum_delta_all), _p(h_local_all)
    a.sum_delta_rank_stride, a.h_local_rank_stride = sd_rs, hl_rs
    a.h_in, a.h_out = _p(_c32(h_in, "h_in")), _p(_c32(h_out, "h_out"))
    _abi.check(_abi.lib().ssm_split_combine(C.byref(a), _stream(stream)), "ssm_split_combine")
    return h_in, h_out


def split_fixup(mode, x, dt, A, B, C_, y, cum_delta, h_in, *, D=None, z=None, dt_bias=None, conv_w=None,
                conv_b=None, conv_state_in=None, delta_softplus=True, stream=None):
    """Add the entering state's contribution to the segment's y, in place."""
    a = _split_scan_args(mode, x, dt, A, B, C_, D, z, dt_bias, conv_w, conv_b, conv_state_in, y, delta_softplus)
    _abi.check(_abi.lib().ssm_split_fixup(C.byref(a), _p(_c32(cum_delta, "cum_delta")), _p(_c32(h_in, "h_in")),
                                          _stream(stream)), "ssm_split_fixup")
    return y
