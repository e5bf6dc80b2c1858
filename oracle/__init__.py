"""fp64 CPU oracle for the Mamba conv1d + selective-scan hot path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the package smoke
check and by the benchmark's CPU-baseline leg, never by the product path.  It
shares no code with the CUDA library; the only thing both sides use is the
seeded input generator module, which holds no arithmetic of the method.

The arithmetic lives in ``ssm_oracle.c`` (plain sequential loops over tokens
in C doubles).  This module only marshals numpy arrays into that library and
returns float64 numpy arrays.

Array conventions (numpy, any float dtype; widened exactly to float64):

Mamba-1 (``mode=1``): x, z, dt ``[b, T, D]``; B, C ``[b, T, N]``; A ``[D, N]``;
D, dt_bias ``[D]``; h0 / h_final ``[nseq, D, N]``; conv channels = D.

Mamba-2 (``mode=2``): x, z ``[b, T, H, P]``; dt ``[b, T, H]``; B, C
``[b, T, G, N]``; A, D, dt_bias ``[H]``; h0 / h_final ``[nseq, H, P, N]``;
conv channels = H*P + 2*G*N in the order x | B | C.

Packed variable-length input: ``b == 1`` and ``cu_seqlens`` (``nseq + 1``
non-decreasing offsets starting at 0) splits the token axis into sequences.
Without it every batch row is one sequence of length T.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build_oracle

MAMBA1 = 1
MAMBA2 = 2

_dp = C.POINTER(C.c_double)
_lp = C.POINTER(C.c_int64)


class _ScanArgs(C.Structure):
    _fields_ = [
        ("mode", C.c_int32), ("delta_softplus", C.c_int32), ("nthreads", C.c_int32), ("pad_", C.c_int32),
        ("nseqs", C.c_int64), ("seq_start", _lp),
        ("d_inner", C.c_int64), ("nheads", C.c_int64), ("headdim", C.c_int64),
        ("ngroups", C.c_int64), ("dstate", C.c_int64), ("d_conv", C.c_int64),
        ("x", _dp), ("z", _dp), ("dt", _dp), ("B", _dp), ("C", _dp),
        ("A", _dp), ("D", _dp), ("dt_bias", _dp),
        ("h0", _dp),
        ("conv_w", _dp), ("conv_b", _dp), ("conv_state_in", _dp),
        ("y", _dp), ("h_final", _dp), ("conv_state_out", _dp),
        ("state_interval", C.c_int64), ("inter_slots", C.POINTER(C.c_int32)),
        ("inter_stride", C.c_int64), ("inter_nslots", C.c_int64),
        ("inter_states", _dp), ("inter_conv", _dp),
    ]


class _ScanBwdArgs(C.Structure):
    _fields_ = [
        ("fwd", _ScanArgs),
        ("dy", _dp), ("dh_final", _dp), ("dconv_state_out", _dp),
        ("dx", _dp), ("dz", _dp), ("ddt", _dp), ("dB", _dp), ("dC", _dp),
        ("dA", _dp), ("dD", _dp), ("ddt_bias", _dp),
        ("dh0", _dp),
        ("dconv_w", _dp), ("dconv_b", _dp),
        ("dconv_state_in", _dp),
    ]


class _ConvArgs(C.Structure):
    _fields_ = [
        ("activation", C.c_int32), ("pad_", C.c_int32),
        ("nseqs", C.c_int64), ("seq_start", _lp),
        ("channels", C.c_int64), ("width", C.c_int64),
        ("x", _dp), ("w", _dp), ("b", _dp), ("state_in", _dp),
        ("out", _dp), ("state_out", _dp),
    ]


class _UpdateArgs(C.Structure):
    _fields_ = [
        ("mode", C.c_int32), ("delta_softplus", C.c_int32),
        ("batch", C.c_int64), ("d_inner", C.c_int64), ("nheads", C.c_int64), ("headdim", C.c_int64),
        ("ngroups", C.c_int64), ("dstate", C.c_int64),
        ("d_conv", C.c_int64), ("conv_state_len", C.c_int64),
        ("state", _dp), ("conv_state", _dp),
        ("conv_w", _dp), ("conv_b", _dp),
        ("x", _dp), ("z", _dp), ("dt", _dp), ("B", _dp), ("C", _dp),
        ("A", _dp), ("D", _dp), ("dt_bias", _dp),
        ("y", _dp),
    ]


_LIBS: dict[int, C.CDLL] = {}


def _lib(mutant: int = 0) -> C.CDLL:
    if mutant not in _LIBS:
        path = build_oracle.build(mutant)
        lib = C.CDLL(path)
        lib.oracle_scan_fwd.argtypes = [C.POINTER(_ScanArgs)]
        lib.oracle_scan_fwd.restype = C.c_int
        lib.oracle_conv1d_fwd.argtypes = [C.POINTER(_ConvArgs)]
        lib.oracle_conv1d_fwd.restype = C.c_int
        lib.oracle_state_update.argtypes = [C.POINTER(_UpdateArgs)]
        lib.oracle_state_update.restype = C.c_int
        lib.oracle_scan_bwd.argtypes = [C.POINTER(_ScanBwdArgs)]
        lib.oracle_scan_bwd.restype = C.c_int
        lib.oracle_mutant_id.restype = C.c_int
        _LIBS[mutant] = lib
    return _LIBS[mutant]


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _seq_start(batch, seqlen, cu_seqlens):
    if cu_seqlens is None:
        return np.arange(batch + 1, dtype=np.int64) * seqlen
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if batch != 1 or cu[0] != 0 or np.any(np.diff(cu) < 0) or cu[-1] != seqlen:
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at the token count (batch 1)")
    return np.ascontiguousarray(cu)


def scan_fwd(mode, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None, h0=None, cu_seqlens=None,
             conv_w=None, conv_b=None, conv_state_in=None, delta_softplus=True, nthreads=1, mutant=0,
             state_interval=0, inter_slots=None, inter_states=None, inter_conv=None):
    """Forward scan (optionally with the causal conv + SiLU in front).

    Returns ``(y, h_final, conv_state_out)`` as float64 arrays
    (``conv_state_out`` is None without a conv).

    Intermediate states: with ``state_interval > 0`` and ``inter_slots``
    (int ``[nseq, stride]``), the state and conv history after every
    ``state_interval`` tokens of each sequence are written into the float64
    pools ``inter_states [nslots, ...state]`` / ``inter_conv [nslots, conv_dim,
    K-1]`` (modified in place) at the rows the slot table names; negative or
    out-of-range slots write nothing.
    """
    x = _f64(x)
    b, T = x.shape[0], x.shape[1]
    if mode == MAMBA1:
        Dn = x.shape[2]
        N = np.asarray(B).shape[2]
        H, P, G = Dn, 1, 1
    else:
        H, P = x.shape[2], x.shape[3]
        G, N = np.asarray(B).shape[2], np.asarray(B).shape[3]
        Dn = H * P
    seq = _seq_start(b, T, cu_seqlens)
    nseq = len(seq) - 1
    K = 0 if conv_w is None else np.asarray(conv_w).shape[1]
    cdim = Dn if mode == MAMBA1 else Dn + 2 * G * N
    arrs = dict(x=x, dt=_f64(dt), A=_f64(A), B=_f64(B), C=_f64(C_), D=_f64(D), z=_f64(z),
                dt_bias=_f64(dt_bias), h0=_f64(h0), conv_w=_f64(conv_w), conv_b=_f64(conv_b),
                conv_state_in=_f64(conv_state_in))
    y = np.zeros(x.shape, dtype=np.float64)
    hshape = (nseq, Dn, N) if mode == MAMBA1 else (nseq, H, P, N)
    hf = np.zeros(hshape, dtype=np.float64)
    cso = np.zeros((nseq, cdim, K - 1), dtype=np.float64) if K > 1 else None
    a = _ScanArgs()
    a.mode, a.delta_softplus, a.nthreads = mode, int(bool(delta_softplus)), int(nthreads)
    a.nseqs, a.seq_start = nseq, seq.ctypes.data_as(_lp)
    a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate, a.d_conv = Dn, H, P, G, N, K
    for k, v in arrs.items():
        setattr(a, k, _ptr(v))
    a.y, a.h_final, a.conv_state_out = _ptr(y), _ptr(hf), _ptr(cso)
    slots_keep = None
    if state_interval and inter_slots is not None:
        slots_keep = np.ascontiguousarray(inter_slots, dtype=np.int32)
        for pool in (inter_states, inter_conv):
            if pool is not None and (pool.dtype != np.float64 or not pool.flags.c_contiguous):
                raise ValueError("intermediate pools must be C-contiguous float64 arrays")
        a.state_interval = int(state_interval)
        a.inter_slots = slots_keep.ctypes.data_as(C.POINTER(C.c_int32))
        a.inter_stride = slots_keep.shape[1] if slots_keep.ndim == 2 else slots_keep.size
        a.inter_nslots = inter_states.shape[0] if inter_states is not None else inter_conv.shape[0]
        a.inter_states, a.inter_conv = _ptr(inter_states), _ptr(inter_conv)
    rc = _lib(mutant).oracle_scan_fwd(C.byref(a))
    if rc != 0:
        raise ValueError(f"oracle_scan_fwd rejected its arguments ({rc})")
    return y, hf, cso


def scan_bwd(mode, x, dt, A, B, C_, dy, *, D=None, z=None, dt_bias=None, h0=None, cu_seqlens=None,
             conv_w=None, conv_b=None, conv_state_in=None, delta_softplus=True, dh_final=None,
             dconv_state_out=None, mutant=0):
    """Gradients of ``sum(dy*y) + sum(dh_final*h_final) + sum(dconv_state_out*conv_state_out)``
    with respect to every input of :func:`scan_fwd` (same arguments).

    Returns a dict of float64 arrays shaped like the inputs: ``dx, dz, ddt, dB,
    dC`` (raw inputs, before the conv), ``dA, dD, ddt_bias, dh0, dconv_w,
    dconv_b, dconv_state_in`` (None where the input is None).
    """
    x = _f64(x)
    b, T = x.shape[0], x.shape[1]
    if mode == MAMBA1:
        Dn = x.shape[2]
        N = np.asarray(B).shape[2]
        H, P, G = Dn, 1, 1
    else:
        H, P = x.shape[2], x.shape[3]
        G, N = np.asarray(B).shape[2], np.asarray(B).shape[3]
        Dn = H * P
    seq = _seq_start(b, T, cu_seqlens)
    nseq = len(seq) - 1
    K = 0 if conv_w is None else np.asarray(conv_w).shape[1]
    cdim = Dn if mode == MAMBA1 else Dn + 2 * G * N
    ins = dict(x=x, dt=_f64(dt), A=_f64(A), B=_f64(B), C=_f64(C_), D=_f64(D), z=_f64(z),
               dt_bias=_f64(dt_bias), h0=_f64(h0), conv_w=_f64(conv_w), conv_b=_f64(conv_b),
               conv_state_in=_f64(conv_state_in))
    hshape = (nseq, Dn, N) if mode == MAMBA1 else (nseq, H, P, N)
    z0 = lambda k: None if ins[k] is None else np.zeros(ins[k].shape, dtype=np.float64)
    out = dict(dx=z0("x"), dz=z0("z"), ddt=z0("dt"), dB=z0("B"), dC=z0("C"), dA=z0("A"), dD=z0("D"),
               ddt_bias=z0("dt_bias"), dh0=np.zeros(hshape, dtype=np.float64), dconv_w=z0("conv_w"),
               dconv_b=z0("conv_b"),
               dconv_state_in=np.zeros((nseq, cdim, K - 1), dtype=np.float64) if K > 1 else None)
    a = _ScanBwdArgs()
    f = a.fwd
    f.mode, f.delta_softplus, f.nthreads = mode, int(bool(delta_softplus)), 1
    f.nseqs, f.seq_start = nseq, seq.ctypes.data_as(_lp)
    f.d_inner, f.nheads, f.headdim, f.ngroups, f.dstate, f.d_conv = Dn, H, P, G, N, K
    for k, v in ins.items():
        setattr(f, k, _ptr(v))
    dyv, dhf, dcs = _f64(dy), _f64(dh_final), _f64(dconv_state_out)
    a.dy, a.dh_final, a.dconv_state_out = _ptr(dyv), _ptr(dhf), _ptr(dcs)
    for k, v in out.items():
        setattr(a, k, _ptr(v))
    rc = _lib(mutant).oracle_scan_bwd(C.byref(a))
    if rc != 0:
        raise ValueError(f"oracle_scan_bwd rejected its arguments ({rc})")
    return out


def conv1d_fwd(x, w, *, b=None, state_in=None, cu_seqlens=None, activation=True, mutant=0):
    """Causal depthwise conv over ``x [batch, T, channels]``; returns ``(out, state_out)``."""
    x = _f64(x)
    bsz, T, Cn = x.shape
    w = _f64(w)
    K = w.shape[1]
    seq = _seq_start(bsz, T, cu_seqlens)
    nseq = len(seq) - 1
    out = np.zeros_like(x)
    so = np.zeros((nseq, Cn, K - 1), dtype=np.float64) if K > 1 else None
    bb, si = _f64(b), _f64(state_in)
    a = _ConvArgs()
    a.activation = int(bool(activation))
    a.nseqs, a.seq_start = nseq, seq.ctypes.data_as(_lp)
    a.channels, a.width = Cn, K
    a.x, a.w, a.b, a.state_in, a.out, a.state_out = _ptr(x), _ptr(w), _ptr(bb), _ptr(si), _ptr(out), _ptr(so)
    rc = _lib(mutant).oracle_conv1d_fwd(C.byref(a))
    if rc != 0:
        raise ValueError(f"oracle_conv1d_fwd rejected its arguments ({rc})")
    return out, so


def state_update(mode, state, conv_state, x, dt, A, B, C_, *, D=None, z=None, dt_bias=None,
                 conv_w=None, conv_b=None, delta_softplus=True, mutant=0):
    """One decode token per batch row.  ``state`` and ``conv_state`` are
    updated in place (float64 arrays are required so the update is visible);
    returns ``y``.  Shapes: as the scan with the token axis removed; conv_state
    ``[batch, conv_dim, conv_state_len]``."""
    if state.dtype != np.float64 or not state.flags.c_contiguous:
        raise TypeError("state must be a C-contiguous float64 array (updated in place)")
    x = _f64(x)
    bsz = x.shape[0]
    if mode == MAMBA1:
        Dn = x.shape[1]
        N = np.asarray(B).shape[1]
        H, P, G = Dn, 1, 1
    else:
        H, P = x.shape[1], x.shape[2]
        G, N = np.asarray(B).shape[1], np.asarray(B).shape[2]
        Dn = H * P
    K = 0 if conv_w is None else np.asarray(conv_w).shape[1]
    if K > 0 and (conv_state is None or conv_state.dtype != np.float64 or not conv_state.flags.c_contiguous):
        raise TypeError("conv_state must be a C-contiguous float64 array (updated in place)")
    Ls = conv_state.shape[2] if conv_state is not None else 0
    y = np.zeros(x.shape, dtype=np.float64)
    arrs = dict(x=x, dt=_f64(dt), A=_f64(A), B=_f64(B), C=_f64(C_), D=_f64(D), z=_f64(z),
                dt_bias=_f64(dt_bias), conv_w=_f64(conv_w), conv_b=_f64(conv_b))
    a = _UpdateArgs()
    a.mode, a.delta_softplus = mode, int(bool(delta_softplus))
    a.batch, a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate = bsz, Dn, H, P, G, N
    a.d_conv, a.conv_state_len = K, Ls
    a.state, a.conv_state = _ptr(state), _ptr(conv_state)
    for k, v in arrs.items():
        setattr(a, k, _ptr(v))
    a.y = _ptr(y)
    rc = _lib(mutant).oracle_state_update(C.byref(a))
    if rc != 0:
        raise ValueError(f"oracle_state_update rejected its arguments ({rc})")
    return y


def mutant_id(mutant: int) -> int:
    return _lib(mutant).oracle_mutant_id()


def library_path() -> str:
    return build_oracle.lib_path(0)


__all__ = ["MAMBA1", "MAMBA2", "scan_fwd", "conv1d_fwd", "state_update", "mutant_id", "library_path"]
os.environ.setdefault("OMP_WAIT_POLICY", "PASSIVE")
