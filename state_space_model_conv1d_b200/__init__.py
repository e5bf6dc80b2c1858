"""Mamba conv1d + selective-scan hot path for B200 (sm_100a), behind a C ABI.

The compute lives in ``libssm.so`` (hand-written CUDA for sm_100a); this
package is a thin ctypes binding with the same entry-point names.  The
library is loaded on first use and a missing library raises immediately:
there is no CPU fallback.
"""
