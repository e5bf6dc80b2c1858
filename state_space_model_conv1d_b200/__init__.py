"""Mamba conv1d + selective-scan hot path for B200 (sm_100a), behind a C ABI.

The compute lives in ``libssm.so`` (hand-written CUDA for sm_100a); this
package is a thin ctypes binding with the same entry-point names.  The
library is loaded on first use and a missing library raises immediately:
there is no CPU fallback.
"""
from .ops import (MAMBA1, MAMBA2, conv1d_fwd, kernel_time_ms, kernel_timing, scan_bwd, scan_fwd,  # noqa: F401
                  scan_segments, scan_workspace_size, state_update, workspace_error)
from ._abi import LIB_PATH, SSMError  # noqa: F401
from .seq_split import SegmentScan, scan_fwd_seq_split  # noqa: F401
