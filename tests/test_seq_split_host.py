"""The sequence split on CPU: its protocol and algebra against the unsplit oracle.

Every rank scans its own segment of each batch row from a zero state; the
conv tails and the (sum of delta, end state) pairs are exchanged; each rank
folds the pairs of the segments before it into its entering state and adds
that state's contribution to y.  With the fp64 stand-in backend
(tests/split_double.py, the oracle for the segment scans) the joined outputs
equal the oracle's scan of the whole sequence to rounding.

Mutants of the stand-in show that the comparison sees the mistakes a split
can make: a dropped segment decay, an exclusive instead of an inclusive
prefix of delta in the fix-up, and a lost conv tail.  The protocol also runs
on two gloo ranks through torch.distributed, and with a rank that holds no
tokens.
"""
import os
import socket
import types

import numpy as np
import pytest
import torch

import oracle
import split_double
from state_space_model_conv1d_b200 import seq_split
from state_space_model_conv1d_b200 import workloads as W

M1, M2 = oracle.MAMBA1, oracle.MAMBA2
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _inputs(mode, seed, T, dtype="f32"):
    if mode == M1:
        return W.mamba1_inputs(seed, 2, T, 12, 6, dtype=dtype, conv_bias=True, conv_state=True)
    return W.mamba2_inputs(seed, 2, T, 4, 3, 2, 5, dtype=dtype, conv_bias=True, conv_state=True)


def _segment(d, lo, hi):
    """Torch views of tokens [lo, hi) of every batch row (parameters whole)."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
        elif k in ("x", "z", "dt", "B", "C"):
            out[k] = torch.from_numpy(np.asarray(v, np.float64))[:, lo:hi]
        else:
            out[k] = torch.from_numpy(np.asarray(v, np.float64))
    return out


def _kw(s):
    return dict(D=s["D"], z=s["z"], dt_bias=s["dt_bias"], h0=s["h0"], conv_w=s["conv_w"], conv_b=s["conv_b"],
                conv_state_in=s["conv_state_in"])


def run_split(mode, d, bounds, backend):
    """Every rank's SegmentScan with the exchanges done by stacking: (y, h_outs, conv_out of the last)."""
    R = len(bounds) - 1
    segs = []
    for r in range(R):
        s = _segment(d, bounds[r], bounds[r + 1])
        segs.append(seq_split.SegmentScan(mode, r, R, s["x"], s["dt"], s["A"], s["B"], s["C"], backend=backend,
                                          **_kw(s)))
    tails = [s.tail() for s in segs]
    tails = torch.stack(tails) if tails[0] is not None else None
    pairs = torch.stack([s.scan(tails) for s in segs])
    outs = [s.join(pairs) for s in segs]
    y = torch.cat([o[0] for o in outs], dim=1).numpy()
    return y, [o[1].numpy() for o in outs], outs[-1][2]


def _ref(mode, d, upto=None):
    T = d["x"].shape[1] if upto is None else upto
    cut = {k: (None if v is None else (v[:, :T] if k in ("x", "z", "dt", "B", "C") else v)) for k, v in d.items()}
    return oracle.scan_fwd(mode, cut["x"], cut["dt"], cut["A"], cut["B"], cut["C"], D=cut["D"], z=cut["z"],
                           dt_bias=cut["dt_bias"], h0=cut["h0"], conv_w=cut["conv_w"], conv_b=cut["conv_b"],
                           conv_state_in=cut["conv_state_in"])


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


CASES = [(M1, [0, 9, 20, 31]), (M1, [0, 16, 40]), (M2, [0, 3, 19, 27, 40]), (M2, [0, 25, 33])]


@pytest.mark.parametrize("mode,bounds", CASES)
def test_split_equals_unsplit_scan(mode, bounds):
    d = _inputs(mode, 700 + len(bounds), bounds[-1])
    y, houts, conv_out = run_split(mode, d, bounds, split_double)
    ry, rh, rc = _ref(mode, d)
    assert _rel(y, ry) < 1e-11
    assert _rel(houts[-1], rh) < 1e-11
    np.testing.assert_array_equal(conv_out.numpy(), rc)
    for r in range(len(bounds) - 1):            # every rank's h_out is the state at its segment's end
        _, rhr, _ = _ref(mode, d, upto=bounds[r + 1])
        assert _rel(houts[r], rhr) < 1e-11, r


def _mutant(**over):
    m = types.SimpleNamespace(**{k: getattr(split_double, k) for k in
                                 ("scan_fwd", "split_conv_tail", "split_cum_delta", "split_combine", "split_fixup")})
    for k, v in over.items():
        setattr(m, k, v)
    return m


def _no_decay_combine(mode, A, sd, hl, rank, stream=None):
    return split_double.split_combine(mode, A, torch.zeros_like(sd), hl, rank)


def _exclusive_cum(*a, **k):
    cs, sd = split_double.split_cum_delta(*a, **k)
    if cs is not None:
        cs = torch.cat([torch.zeros_like(cs[:, :1]), cs[:, :-1]], dim=1)
    return cs, sd


def _zero_tail(*a, **k):
    return torch.zeros_like(split_double.split_conv_tail(*a, **k))


@pytest.mark.parametrize("mode", [M1, M2])
@pytest.mark.parametrize("name,backend", [("dropped decay", _mutant(split_combine=_no_decay_combine)),
                                          ("exclusive prefix", _mutant(split_cum_delta=_exclusive_cum)),
                                          ("lost conv tail", _mutant(split_conv_tail=_zero_tail))])
def test_split_mutants_are_caught(mode, name, backend):
    bounds = [0, 14, 30]
    d = _inputs(mode, 731, bounds[-1])
    y, houts, _ = run_split(mode, d, bounds, backend)
    ry, rh, _ = _ref(mode, d)
    assert max(_rel(y, ry), _rel(houts[-1], rh)) > 1e-6, name


def test_segment_shorter_than_conv_history_is_rejected():
    d = _inputs(M1, 740, 2)
    s = _segment(d, 0, 2)
    with pytest.raises(ValueError):
        seq_split.SegmentScan(M1, 1, 2, s["x"], s["dt"], s["A"], s["B"], s["C"], conv_w=s["conv_w"],
                              backend=split_double)


# ---------------------------------------------------------------- two gloo ranks
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _gloo_rank(rank, world, port, mode, bounds, out):
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import split_double as sd_backend
        from state_space_model_conv1d_b200 import seq_split as ss
        d = _inputs(mode, 750, bounds[-1])
        s = _segment(d, bounds[rank], bounds[rank + 1])
        y, h_out, conv_out = ss.scan_fwd_seq_split(mode, s["x"], s["dt"], s["A"], s["B"], s["C"], rank=rank,
                                                   nranks=world, backend=sd_backend, **_kw(s))
        out[rank] = (y.numpy(), h_out.numpy(), conv_out.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [M1, M2])
def test_two_gloo_ranks_join_to_the_unsplit_scan(mode):
    import torch.multiprocessing as mp
    world, bounds = 2, [0, 17, 35]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, world, port, mode, bounds, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    d = _inputs(mode, 750, bounds[-1])
    ry, rh, rc = _ref(mode, d)
    y = np.concatenate([out[0][0], out[1][0]], axis=1)
    assert _rel(y, ry) < 1e-11
    assert _rel(out[1][1], rh) < 1e-11
    np.testing.assert_array_equal(out[1][2], rc)


@pytest.mark.parametrize("mode", [M1, M2])
def test_empty_segment_without_conv(mode):
    """A rank holding no tokens passes the state through unchanged (decay exp(0) = 1, no input)."""
    bounds = [0, 13, 13, 30]
    if mode == M1:
        d = W.mamba1_inputs(760, 2, bounds[-1], 12, 6, d_conv=0, dtype="f32")
    else:
        d = W.mamba2_inputs(761, 2, bounds[-1], 4, 3, 2, 5, d_conv=0, dtype="f32")
    y, houts, _ = run_split(mode, d, bounds, split_double)
    ry, rh, _ = _ref(mode, d)
    assert _rel(y, ry) < 1e-11
    assert _rel(houts[-1], rh) < 1e-11
    np.testing.assert_array_equal(houts[1], houts[0])
