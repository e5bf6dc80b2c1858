"""The C-ABI library on the host: it loads, exports every symbol the header
declares, and rejects bad arguments before anything reaches a GPU.

Every call here is one the library must refuse during host-side validation,
so nothing is launched (no GPU is needed, and none is touched when one is present).
"""
import ctypes as C
import os
import re
import subprocess

import pytest

from state_space_model_conv1d_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_symbols():
    names = set()
    for h in HEADERS:
        with open(h) as fh:
            src = fh.read()
        names |= set(re.findall(r"SSM_API\s+[\w\s\*]+?\b(ssm_\w+)\s*\(", src))
    return names


def test_library_exists_and_loads():
    assert os.path.exists(_abi.LIB_PATH), "build libssm.so first"
    lib = _abi.lib()
    assert lib.ssm_abi_version() == _abi.ABI_VERSION == 3


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert {"ssm_conv1d_fwd", "ssm_scan_fwd", "ssm_state_update", "ssm_scan_workspace_size"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert names <= exported, f"missing: {names - exported}"
    assert set(_abi.SIGNATURES) == names, "ctypes signatures must mirror the header"
    # nothing beyond the ABI leaks out of the library
    assert {e for e in exported if e.startswith("ssm")} == names


STRUCTS = (("ssm_conv_args", _abi.ConvArgs), ("ssm_scan_args", _abi.ScanArgs), ("ssm_update_args", _abi.UpdateArgs),
           ("ssm_scan_bwd_args", _abi.ScanBwdArgs), ("ssm_split_args", _abi.SplitArgs))


def test_struct_layouts_match_header(tmp_path):
    """Compile a probe against the real header and compare every field offset
    with the ctypes mirror."""
    probes = []
    for cname, py in STRUCTS:
        probes.append(f'printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            probes.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    src = tmp_path / "probe.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "ssm.h"\nint main(void){' + "".join(probes) +
                   "return 0;}\n")
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        c, f, v = line.split()
        got[(c, f)] = int(v)
    for cname, py in STRUCTS:
        assert got[(cname, "sizeof")] == C.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_status_strings():
    lib = _abi.lib()
    for s in range(0, -7, -1):
        assert lib.ssm_status_string(s)
    assert lib.ssm_status_string(-99) == b"unknown status"


FAKE = 0x10000000  # never dereferenced: every call below is rejected on the host


def _scan(**kw):
    a = _abi.ScanArgs()
    a.mode, a.dtype, a.delta_softplus = 2, _abi.SSM_BF16, 1
    a.batch, a.seqlen, a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate = 2, 16, 8, 4, 2, 2, 16
    for k in ("x", "dt", "B", "C", "y", "A"):
        setattr(a, k, FAKE)
    a.x_token_stride, a.x_batch_stride = 8, 128
    a.y_token_stride, a.y_batch_stride = 8, 128
    a.dt_token_stride, a.dt_batch_stride = 4, 64
    a.B_token_stride, a.B_batch_stride = 32, 512
    a.C_token_stride, a.C_batch_stride = 32, 512
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(mode=3), _abi.SSM_ERR_INVALID_ARG),
    (dict(dtype=7), _abi.SSM_ERR_INVALID_ARG),
    (dict(ngroups=3), _abi.SSM_ERR_INVALID_ARG),                 # heads not divisible into groups
    (dict(nheads=3), _abi.SSM_ERR_INVALID_ARG),                  # nheads * headdim != d_inner
    (dict(dstate=1024), _abi.SSM_ERR_UNSUPPORTED),
    (dict(x=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(A=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(x=FAKE + 1), _abi.SSM_ERR_ALIGNMENT),                  # bf16 needs 2-byte alignment
    (dict(h0=FAKE + 2), _abi.SSM_ERR_ALIGNMENT),
    (dict(x_token_stride=4), _abi.SSM_ERR_INVALID_ARG),          # rows overlap
    (dict(d_conv=2), _abi.SSM_ERR_INVALID_ARG),                  # conv width without weights
    (dict(d_conv=9, conv_w=FAKE), _abi.SSM_ERR_UNSUPPORTED),
    (dict(cu_seqlens=FAKE, nseqs=2), _abi.SSM_ERR_INVALID_ARG),  # varlen needs batch == 1
    (dict(cu_seqlens=FAKE, nseqs=2, batch=1), _abi.SSM_ERR_WORKSPACE),
    (dict(mode=1, ngroups=2, d_inner=8), _abi.SSM_ERR_UNSUPPORTED),
    (dict(mode=1, ngroups=1, dstate=128), _abi.SSM_ERR_UNSUPPORTED),
    (dict(delta_softplus=2), _abi.SSM_ERR_INVALID_ARG),
    # intermediate-state extraction
    (dict(state_interval=32, inter_slots=FAKE, inter_states=FAKE), _abi.SSM_ERR_INVALID_ARG),   # not a multiple of 64
    (dict(state_interval=-64, inter_slots=FAKE, inter_states=FAKE), _abi.SSM_ERR_INVALID_ARG),
    (dict(state_interval=64, inter_states=FAKE), _abi.SSM_ERR_INVALID_ARG),                     # no slot table
    (dict(state_interval=64, inter_slots=FAKE), _abi.SSM_ERR_INVALID_ARG),                      # no pool
    (dict(state_interval=64, inter_slots=FAKE, inter_states=FAKE, inter_nslots=-1), _abi.SSM_ERR_INVALID_ARG),
    (dict(state_interval=64, inter_slots=FAKE + 2, inter_states=FAKE), _abi.SSM_ERR_ALIGNMENT),
    (dict(state_interval=64, inter_slots=FAKE, inter_conv=FAKE + 1), _abi.SSM_ERR_ALIGNMENT),
])
def test_scan_rejects(kw, status):
    a = _scan(**kw)
    assert _abi.lib().ssm_scan_fwd(C.byref(a), None, 0, None) == status


def test_scan_rejects_null_args():
    assert _abi.lib().ssm_scan_fwd(None, None, 0, None) == _abi.SSM_ERR_INVALID_ARG
    assert _abi.lib().ssm_conv1d_fwd(None, None) == _abi.SSM_ERR_INVALID_ARG
    assert _abi.lib().ssm_state_update(None, None) == _abi.SSM_ERR_INVALID_ARG


def test_workspace_size_is_host_only():
    a = _scan()                                         # Mamba-2 shapes off the tensor-core path
    assert _abi.lib().ssm_scan_workspace_size(C.byref(a)) == 0
    a = _scan(cu_seqlens=FAKE, nseqs=1000, batch=1)
    n = _abi.lib().ssm_scan_workspace_size(C.byref(a))
    assert n >= 256 + 4 * 1000 and n % 256 == 0
    # headdim 64 / dstate 128 / bf16 / conv: error word + conv'd B and C (2 bytes each)
    a = _scan(nheads=4, headdim=64, d_inner=256, ngroups=2, dstate=128, d_conv=4, conv_w=FAKE)
    n = _abi.lib().ssm_scan_workspace_size(C.byref(a))
    assert n == 256 + 2 * (2 * 16 * 2 * 128 * 2)
    a = _scan(mode=1, d_inner=8, ngroups=1)             # Mamba-1 needs none
    assert _abi.lib().ssm_scan_workspace_size(C.byref(a)) == 0


def test_segment_plan_is_host_only():
    lib = _abi.lib()
    big = dict(batch=4, seqlen=4096, nheads=80, headdim=64, d_inner=5120, ngroups=8, dstate=128, d_conv=4,
               conv_w=FAKE, x_token_stride=5120, x_batch_stride=5120 * 4096, y_token_stride=5120,
               y_batch_stride=5120 * 4096, dt_token_stride=80, dt_batch_stride=80 * 4096, B_token_stride=1024,
               B_batch_stride=1024 * 4096, C_token_stride=1024, C_batch_stride=1024 * 4096)
    # 320 (row, head) chains of 64 chunks: cut when the library chooses
    assert lib.ssm_scan_segments(C.byref(_scan(**big))) >= 2
    assert lib.ssm_scan_segments(C.byref(_scan(segments=1, **big))) == 1
    assert lib.ssm_scan_segments(C.byref(_scan(segments=4, **big))) == 4
    assert lib.ssm_scan_segments(C.byref(_scan(segments=3, **big))) == 3          # runs of 22, 22, 20 chunks
    # many chains already fill the GPU: rows stay whole
    assert lib.ssm_scan_segments(C.byref(_scan(**dict(big, batch=64, x_batch_stride=5120 * 4096)))) == 1
    # packed sequences: one run length for all, chosen from the total (64
    # chunks); the count is the bound nseqs + ceil(total / run) on their runs
    packed = dict(big, batch=1, cu_seqlens=FAKE, nseqs=3)
    assert lib.ssm_scan_segments(C.byref(_scan(segments=4, **packed))) == 3 + 11    # runs of 6 chunks
    assert lib.ssm_scan_segments(C.byref(_scan(segments=1, **packed))) == 1
    # chosen: the fixed-length choice for nseqs rows of the mean length; one
    # sequence of 4096 tokens is cut like a row of 4096 (3 runs of 22 chunks)
    one = dict(packed, nseqs=1)
    assert lib.ssm_scan_segments(C.byref(_scan(**dict(big, batch=1)))) == 3
    assert lib.ssm_scan_segments(C.byref(_scan(**one))) == 1 + 3
    # three means of 22 chunks (240 chains) stay whole, as do many sequences
    assert lib.ssm_scan_segments(C.byref(_scan(**packed))) == 1
    assert lib.ssm_scan_segments(C.byref(_scan(**dict(packed, nseqs=1000)))) == 1
    assert lib.ssm_scan_segments(C.byref(_scan(**dict(packed, nseqs=9)))) == 1
    assert lib.ssm_scan_segments(C.byref(_scan(segments=2, **dict(packed, nseqs=9)))) == 9 + 16
    # more runs than a grid's second dimension holds (65535): the sequences stay whole
    many = dict(packed, nseqs=60000, seqlen=6000000, x_batch_stride=5120 * 6000000)
    assert lib.ssm_scan_segments(C.byref(_scan(segments=2, **many))) == 1
    # Mamba-1 is never cut; bad arguments give 0
    assert lib.ssm_scan_segments(C.byref(_scan(mode=1, d_inner=8, ngroups=1, dt_token_stride=8, dt_batch_stride=128))) == 1
    assert lib.ssm_scan_segments(C.byref(_scan(segments=-1, **big))) == 0
    assert lib.ssm_scan_fwd(C.byref(_scan(segments=-1, **big)), None, 0, None) == _abi.SSM_ERR_INVALID_ARG


def test_workspace_holds_segment_states():
    # 640 tokens = 10 chunks asked in 4 segments: runs of 3 chunks, 4 segments;
    # the three with a successor keep an fp32 P x N state and a log-decay per
    # (row, head) after the conv'd B and C
    kw = dict(nheads=4, headdim=64, d_inner=256, ngroups=2, dstate=128, d_conv=4, conv_w=FAKE, seqlen=640,
              x_token_stride=256, x_batch_stride=256 * 640, y_token_stride=256, y_batch_stride=256 * 640,
              dt_token_stride=4, dt_batch_stride=4 * 640, B_token_stride=256, B_batch_stride=256 * 640,
              C_token_stride=256, C_batch_stride=256 * 640)
    lib = _abi.lib()
    one = lib.ssm_scan_workspace_size(C.byref(_scan(segments=1, **kw)))
    four = lib.ssm_scan_workspace_size(C.byref(_scan(segments=4, **kw)))
    rows = 2 * 3 * 4
    assert four - one == rows * 64 * 128 * 4 + 256
    # packed sequences, 10 chunks asked in about 4 runs each: runs of 2 chunks,
    # at most 2 + 5 table entries, each with a state row per head, plus the
    # table itself and its count
    packed = dict(kw, batch=1, cu_seqlens=FAKE, nseqs=2)
    entries = 2 + 5
    extra = entries * 4 * 64 * 128 * 4 + 256 + 256
    assert lib.ssm_scan_workspace_size(C.byref(_scan(segments=4, **packed))) - \
        lib.ssm_scan_workspace_size(C.byref(_scan(segments=1, **packed))) == extra


def _conv(**kw):
    a = _abi.ConvArgs()
    a.batch, a.seqlen, a.channels, a.width, a.dtype, a.activation = 2, 8, 16, 4, _abi.SSM_F32, 1
    a.x, a.out, a.weight = FAKE, FAKE, FAKE
    a.x_token_stride, a.x_batch_stride, a.out_token_stride, a.out_batch_stride = 16, 128, 16, 128
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(width=0), _abi.SSM_ERR_UNSUPPORTED),
    (dict(width=9), _abi.SSM_ERR_UNSUPPORTED),
    (dict(weight=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(activation=2), _abi.SSM_ERR_INVALID_ARG),
    (dict(x=FAKE + 2), _abi.SSM_ERR_ALIGNMENT),
    (dict(out_token_stride=8), _abi.SSM_ERR_INVALID_ARG),
    (dict(channels=0), _abi.SSM_ERR_INVALID_ARG),
    (dict(cu_seqlens=FAKE, nseqs=3), _abi.SSM_ERR_INVALID_ARG),
])
def test_conv_rejects(kw, status):
    a = _conv(**kw)
    assert _abi.lib().ssm_conv1d_fwd(C.byref(a), None) == status


def _upd(**kw):
    a = _abi.UpdateArgs()
    a.mode, a.dtype, a.delta_softplus = 2, _abi.SSM_BF16, 1
    a.batch, a.d_inner, a.nheads, a.headdim, a.ngroups, a.dstate = 4, 8, 4, 2, 2, 16
    a.d_conv, a.conv_state_len = 4, 4
    for k in ("state", "conv_state", "conv_w", "x", "dt", "B", "C", "y", "A"):
        setattr(a, k, FAKE)
    a.x_batch_stride, a.y_batch_stride, a.dt_batch_stride = 8, 8, 4
    a.B_batch_stride = a.C_batch_stride = 32
    a.nslots = 4
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(conv_state_len=2), _abi.SSM_ERR_INVALID_ARG),
    (dict(conv_state=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(state=FAKE + 4), _abi.SSM_ERR_ALIGNMENT),              # float4 state rows need 16 bytes
    (dict(nslots=2), _abi.SSM_ERR_INVALID_ARG),                  # fewer slots than rows, no indices
    (dict(ngroups=3), _abi.SSM_ERR_INVALID_ARG),
    (dict(x_batch_stride=4), _abi.SSM_ERR_INVALID_ARG),
    (dict(mode=0), _abi.SSM_ERR_INVALID_ARG),
])
def test_update_rejects(kw, status):
    a = _upd(**kw)
    assert _abi.lib().ssm_state_update(C.byref(a), None) == status


def test_workspace_error_needs_a_workspace():
    assert _abi.lib().ssm_workspace_error(None, None, None) == _abi.SSM_ERR_INVALID_ARG


# ---------------------------------------------------------------- sequence split
@pytest.mark.parametrize("kw,status", [
    (dict(cu_seqlens=FAKE, nseqs=2, batch=1), _abi.SSM_ERR_UNSUPPORTED),   # batch mode only
    (dict(seqlen=65535 * 16 + 1, batch=1), _abi.SSM_ERR_UNSUPPORTED),     # longer than the fix-up grid tiles
    (dict(dstate=1024), _abi.SSM_ERR_UNSUPPORTED),                         # the scan's own checks apply
    (dict(x=None), _abi.SSM_ERR_INVALID_ARG),
])
def test_split_scan_calls_reject(kw, status):
    lib = _abi.lib()
    a = _scan(d_conv=4, conv_w=FAKE, **kw)
    assert lib.ssm_split_conv_tail(C.byref(a), FAKE, None) == status
    assert lib.ssm_split_cum_delta(C.byref(a), FAKE, FAKE, None) == status
    assert lib.ssm_split_fixup(C.byref(a), FAKE, FAKE, None) == status


def test_split_own_arguments_rejected():
    lib = _abi.lib()
    a = _scan(d_conv=4, conv_w=FAKE)
    assert lib.ssm_split_conv_tail(C.byref(a), None, None) == _abi.SSM_ERR_INVALID_ARG        # no tail buffer
    assert lib.ssm_split_conv_tail(C.byref(a), FAKE + 1, None) == _abi.SSM_ERR_ALIGNMENT
    a1 = _scan(d_conv=1, conv_w=FAKE)
    assert lib.ssm_split_conv_tail(C.byref(a1), FAKE, None) == _abi.SSM_ERR_INVALID_ARG       # no history to hand on
    assert lib.ssm_split_cum_delta(C.byref(a), FAKE, None, None) == _abi.SSM_ERR_INVALID_ARG  # sum_delta required
    assert lib.ssm_split_cum_delta(C.byref(a), FAKE + 2, FAKE, None) == _abi.SSM_ERR_ALIGNMENT
    assert lib.ssm_split_fixup(C.byref(a), None, FAKE, None) == _abi.SSM_ERR_INVALID_ARG
    assert lib.ssm_split_fixup(C.byref(a), FAKE, None, None) == _abi.SSM_ERR_INVALID_ARG


def test_split_fixup_of_an_empty_segment_is_a_no_op():
    # A rank whose segment holds no tokens has no y to fix; its cum_delta and
    # h_in are empty, so their pointers may be NULL.
    lib = _abi.lib()
    a = _scan(seqlen=0)
    assert lib.ssm_split_fixup(C.byref(a), None, None, None) == _abi.SSM_OK


def _split(**kw):
    a = _abi.SplitArgs()
    a.mode, a.rank, a.nranks = 2, 1, 2
    a.batch, a.d_inner, a.nheads, a.headdim, a.dstate = 2, 8, 4, 2, 16
    a.A, a.sum_delta, a.h_local, a.h_in, a.h_out = FAKE, FAKE, FAKE, FAKE, FAKE
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(rank=2), _abi.SSM_ERR_INVALID_ARG),
    (dict(rank=-1), _abi.SSM_ERR_INVALID_ARG),
    (dict(nranks=0, rank=0), _abi.SSM_ERR_INVALID_ARG),
    (dict(mode=0), _abi.SSM_ERR_INVALID_ARG),
    (dict(nheads=3), _abi.SSM_ERR_INVALID_ARG),
    (dict(h_local=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(sum_delta=None), _abi.SSM_ERR_INVALID_ARG),
    (dict(A=FAKE + 2), _abi.SSM_ERR_ALIGNMENT),
    (dict(h_out=FAKE + 1), _abi.SSM_ERR_ALIGNMENT),
    # rank strides: at least one rank's block (batch x U = 8, batch x state = 256), multiples of 4
    (dict(sum_delta_rank_stride=4), _abi.SSM_ERR_INVALID_ARG),
    (dict(sum_delta_rank_stride=10), _abi.SSM_ERR_INVALID_ARG),
    (dict(sum_delta_rank_stride=-8), _abi.SSM_ERR_INVALID_ARG),
    (dict(h_local_rank_stride=252), _abi.SSM_ERR_INVALID_ARG),
    (dict(h_local_rank_stride=258), _abi.SSM_ERR_INVALID_ARG),
    # a state of more than 2^31 elements per row
    (dict(mode=1, d_inner=1 << 20, dstate=1 << 12), _abi.SSM_ERR_UNSUPPORTED),
])
def test_split_combine_rejects(kw, status):
    a = _split(**kw)
    assert _abi.lib().ssm_split_combine(C.byref(a), None) == status
    assert _abi.lib().ssm_split_combine(None, None) == _abi.SSM_ERR_INVALID_ARG


def test_plain_c_consumer(tmp_path):
    """A C program built against include/ssm.h and linked to libssm.so (no Python in the call path)."""
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(_abi.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_consumer.c"), "-o", str(exe), "-L", libdir, "-lssm",
                    f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr


def test_bounds_checked_build_plumbing():
    """The bounds-checked build exports the same ABI and reports itself as
    checked; the normal build reports that it is not and has no record to read."""
    lib = _abi.lib()
    assert lib.ssm_check_bounds_enabled() == 0
    assert lib.ssm_bounds_record(None, None, None, None, 0) == _abi.SSM_ERR_UNSUPPORTED
    path = os.path.join(os.path.dirname(_abi.LIB_PATH), "libssm_checked.so")
    assert os.path.exists(path), "build the checked library: python -m state_space_model_conv1d_b200.build --check-bounds"
    chk = _abi.checked_lib()
    assert chk.ssm_check_bounds_enabled() == 1
    assert chk.ssm_abi_version() == _abi.ABI_VERSION
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert declared_symbols() <= exported
    # host-side validation is the same code in both builds
    assert chk.ssm_scan_fwd(None, None, 0, None) == _abi.SSM_ERR_INVALID_ARG
