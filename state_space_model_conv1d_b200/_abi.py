"""ctypes mirror of ``include/ssm.h`` and the loader of ``libssm.so``.

Argument marshalling only.  The library is loaded on first use; when it is
missing (not built) the call raises immediately -- there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm.so")

SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_ALIGNMENT = 0, -1, -2, -3
SSM_ERR_WORKSPACE, SSM_ERR_CUDA, SSM_ERR_DEVICE = -4, -5, -6
SSM_F32, SSM_BF16 = 0, 1
ABI_VERSION = 3                # SSM_ABI_VERSION of the header this mirror follows
SSM_MAMBA1, SSM_MAMBA2 = 1, 2
SSM_DEVERR_NONE, SSM_DEVERR_CU_SEQLENS, SSM_DEVERR_TIMEOUT, SSM_DEVERR_BOUNDS = 0, 1, 2, 3

_vp = C.c_void_p
_i64 = C.c_int64
_i32 = C.c_int32


class ConvArgs(C.Structure):
    _fields_ = [
        ("batch", _i64), ("seqlen", _i64), ("channels", _i64), ("width", _i64),
        ("dtype", _i32), ("activation", _i32), ("nseqs", _i32), ("reserved0", _i32),
        ("x", _vp), ("x_batch_stride", _i64), ("x_token_stride", _i64),
        ("weight", _vp), ("bias", _vp), ("state_in", _vp), ("state_out", _vp),
        ("cu_seqlens", _vp),
        ("out", _vp), ("out_batch_stride", _i64), ("out_token_stride", _i64),
    ]


class ScanArgs(C.Structure):
    _fields_ = [
        ("mode", _i32), ("dtype", _i32), ("delta_softplus", _i32), ("nseqs", _i32),
        ("batch", _i64), ("seqlen", _i64), ("d_inner", _i64), ("nheads", _i64), ("headdim", _i64),
        ("ngroups", _i64), ("dstate", _i64), ("d_conv", _i64),
        ("x", _vp), ("x_batch_stride", _i64), ("x_token_stride", _i64),
        ("z", _vp), ("z_batch_stride", _i64), ("z_token_stride", _i64),
        ("dt", _vp), ("dt_batch_stride", _i64), ("dt_token_stride", _i64),
        ("B", _vp), ("B_batch_stride", _i64), ("B_token_stride", _i64),
        ("C", _vp), ("C_batch_stride", _i64), ("C_token_stride", _i64),
        ("y", _vp), ("y_batch_stride", _i64), ("y_token_stride", _i64),
        ("A", _vp), ("D", _vp), ("dt_bias", _vp),
        ("h0", _vp), ("h_final", _vp),
        ("cu_seqlens", _vp),
        ("conv_w", _vp), ("conv_b", _vp), ("conv_state_in", _vp), ("conv_state_out", _vp),
        ("chunk", _i64),
        ("state_interval", _i64), ("inter_slots", _vp), ("inter_stride", _i64), ("inter_nslots", _i64),
        ("inter_states", _vp), ("inter_conv", _vp),
        ("segments", _i64),
    ]


class UpdateArgs(C.Structure):
    _fields_ = [
        ("mode", _i32), ("dtype", _i32), ("delta_softplus", _i32), ("reserved0", _i32),
        ("batch", _i64), ("d_inner", _i64), ("nheads", _i64), ("headdim", _i64), ("ngroups", _i64),
        ("dstate", _i64), ("d_conv", _i64), ("conv_state_len", _i64),
        ("state", _vp), ("conv_state", _vp), ("conv_w", _vp), ("conv_b", _vp),
        ("x", _vp), ("x_batch_stride", _i64),
        ("z", _vp), ("z_batch_stride", _i64),
        ("dt", _vp), ("dt_batch_stride", _i64),
        ("B", _vp), ("B_batch_stride", _i64),
        ("C", _vp), ("C_batch_stride", _i64),
        ("y", _vp), ("y_batch_stride", _i64),
        ("A", _vp), ("D", _vp), ("dt_bias", _vp),
        ("state_batch_indices", _vp), ("nslots", _i64),
    ]


class ScanBwdArgs(C.Structure):
    _fields_ = [
        ("fwd", ScanArgs),
        ("dy", _vp), ("dy_batch_stride", _i64), ("dy_token_stride", _i64),
        ("dh_final", _vp), ("dconv_state_out", _vp),
        ("dx", _vp), ("dz", _vp), ("ddt", _vp), ("dB", _vp), ("dC", _vp),
        ("dA", _vp), ("dD", _vp), ("ddt_bias", _vp),
        ("dh0", _vp),
        ("dconv_w", _vp), ("dconv_b", _vp),
        ("dconv_state_in", _vp),
    ]


class SplitArgs(C.Structure):
    _fields_ = [
        ("mode", _i32), ("rank", _i32), ("nranks", _i32), ("reserved0", _i32),
        ("batch", _i64), ("d_inner", _i64), ("nheads", _i64), ("headdim", _i64), ("dstate", _i64),
        ("A", _vp), ("sum_delta", _vp), ("h_local", _vp), ("h_in", _vp), ("h_out", _vp),
        ("sum_delta_rank_stride", _i64), ("h_local_rank_stride", _i64),
    ]


# Every symbol the header declares, with its ctypes signature.
SIGNATURES = {
    "ssm_abi_version": ([], _i32),
    "ssm_status_string": ([_i32], C.c_char_p),
    "ssm_last_cuda_error": ([], _i32),
    "ssm_conv1d_fwd": ([C.POINTER(ConvArgs), _vp], _i32),
    "ssm_scan_workspace_size": ([C.POINTER(ScanArgs)], C.c_size_t),
    "ssm_scan_segments": ([C.POINTER(ScanArgs)], _i64),
    "ssm_scan_fwd": ([C.POINTER(ScanArgs), _vp, C.c_size_t, _vp], _i32),
    "ssm_state_update": ([C.POINTER(UpdateArgs), _vp], _i32),
    "ssm_workspace_error": ([_vp, C.POINTER(_i32), _vp], _i32),
    "ssm_scan_fwd_noalloc": ([C.POINTER(ScanArgs), _vp], _i32),
    "ssm_scan_bwd_workspace_size": ([C.POINTER(ScanBwdArgs)], C.c_size_t),
    "ssm_scan_bwd": ([C.POINTER(ScanBwdArgs), _vp, C.c_size_t, _vp], _i32),
    "ssm_kernel_timing": ([_i32], _i32),
    "ssm_kernel_time_ms": ([C.POINTER(C.c_float), C.POINTER(_i32)], _i32),
    "ssm_split_conv_tail": ([C.POINTER(ScanArgs), _vp, _vp], _i32),
    "ssm_split_cum_delta": ([C.POINTER(ScanArgs), _vp, _vp, _vp], _i32),
    "ssm_split_combine": ([C.POINTER(SplitArgs), _vp], _i32),
    "ssm_split_fixup": ([C.POINTER(ScanArgs), _vp, _vp, _vp], _i32),
    "ssm_check_bounds_enabled": ([], _i32),
    "ssm_bounds_record": ([C.POINTER(_i32), C.POINTER(_i32), C.POINTER(_i64), C.POINTER(_i64), _i32], _i32),
}

_lock = threading.Lock()
_lib = None


def lib() -> C.CDLL:
    """The loaded ``libssm.so``; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"libssm.so not found at {LIB_PATH}: build it with "
                                       "`python -m state_space_model_conv1d_b200.build` (no CPU fallback exists)")
                handle = C.CDLL(LIB_PATH)
                for name, (argtypes, restype) in SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.argtypes = argtypes
                    fn.restype = restype
                if handle.ssm_abi_version() != ABI_VERSION:
                    raise RuntimeError("libssm.so ABI version mismatch")
                _lib = handle
    return _lib


_checked = None


def checked_lib() -> C.CDLL:
    """The bounds-checked build ``libssm_checked.so`` (same symbols and
    signatures); raises if it has not been built (``build --check-bounds``)."""
    global _checked
    if _checked is None:
        with _lock:
            if _checked is None:
                path = os.path.join(_HERE, "libssm_checked.so")
                if not os.path.exists(path):
                    raise RuntimeError(f"libssm_checked.so not found at {path}: build it with "
                                       "`python -m state_space_model_conv1d_b200.build --check-bounds`")
                handle = C.CDLL(path)
                for name, (argtypes, restype) in SIGNATURES.items():
                    fn = getattr(handle, name)
                    fn.argtypes = argtypes
                    fn.restype = restype
                _checked = handle
    return _checked


class SSMError(RuntimeError):
    def __init__(self, status: int, what: str):
        l = lib()
        msg = l.ssm_status_string(status).decode()
        if status == SSM_ERR_CUDA:
            msg += f" (cudaError {l.ssm_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]")
        self.status = status


def check(status: int, what: str) -> None:
    if status != SSM_OK:
        raise SSMError(status, what)
