"""Intermediate-state extraction (prefix caching) on the GPU against the oracle.

After every ``state_interval`` tokens of each sequence the scan writes its
state and conv history into pool rows named by a slot table; negative and
out-of-range slots write nothing ("Clean up SSM ops directory structure",
Megatron-LM PR 6444: intermediate_extraction, scatter_intermediate_ssm /
scatter_intermediate_conv).  Each case covers the three kernels that serve a
scan: the Mamba-1 kernel, the tensor-core Mamba-2 kernel (bf16, headdim 64,
dstate 128) and the SIMT Mamba-2 kernel (every other shape).
"""
import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu
M1, M2 = oracle.MAMBA1, oracle.MAMBA2


def _slots(nseq, stride, nslots, seed):
    """A slot table with permuted rows, some -1 and some past the pool's end."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(nslots).astype(np.int32)
    tab = np.full((nseq, stride), -1, dtype=np.int32)
    flat = tab.reshape(-1)
    take = min(flat.size, nslots)
    flat[:take] = perm[:take]
    flat[rng.random(flat.size) < 0.2] = -1
    flat[rng.random(flat.size) < 0.1] = nslots + 3
    return tab


def _run(mode, d, dtype, interval, stride, nslots, seed, segments=0):
    cu = d.get("cu_seqlens")
    nseq = d["h0"].shape[0]
    tab = _slots(nseq, stride, nslots, seed)
    K = d["conv_w"].shape[1]
    cdim = d["conv_w"].shape[0]
    rng = np.random.default_rng(seed + 1)
    pool_h = rng.standard_normal((nslots,) + d["h0"].shape[1:]).astype(np.float32)
    pool_c = W.round_bf16(rng.standard_normal((nslots, cdim, K - 1))) if dtype == "bf16" else \
        rng.standard_normal((nslots, cdim, K - 1)).astype(np.float32)
    # GPU
    t = to_dev(d, dtype)
    gh = torch.from_numpy(pool_h.copy()).cuda()
    gc = torch.from_numpy(np.asarray(pool_c, np.float32)).to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)
    ssm.scan_fwd(mode, t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"], dt_bias=t["dt_bias"], h0=t["h0"],
                 cu_seqlens=t.get("cu_seqlens"), conv_w=t["conv_w"], conv_b=t.get("conv_b"),
                 conv_state_in=t.get("conv_state_in"), state_interval=interval,
                 inter_slots=torch.from_numpy(tab).cuda(), inter_states=gh, inter_conv=gc, segments=segments)
    torch.cuda.synchronize()
    # oracle on the same values
    rh = pool_h.astype(np.float64)
    rc = np.asarray(pool_c, np.float64).copy()
    oracle.scan_fwd(mode, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"], dt_bias=d["dt_bias"],
                    h0=d["h0"], cu_seqlens=cu, conv_w=d["conv_w"], conv_b=d.get("conv_b"),
                    conv_state_in=d.get("conv_state_in"), nthreads=8, state_interval=interval, inter_slots=tab,
                    inter_states=rh, inter_conv=rc)
    gh = gh.cpu().numpy().astype(np.float64)
    gc = gc.float().cpu().numpy().astype(np.float64)
    # which rows were written, from the slot table and the sequence lengths
    lens = np.diff(cu) if cu is not None else np.full(nseq, d["x"].shape[1])
    written = set()
    for s in range(nseq):
        for k in range(stride):
            if (k + 1) * interval <= lens[s] and 0 <= tab[s, k] < nslots:
                written.add(int(tab[s, k]))
    assert written, "the case writes no pool row"
    for r in range(nslots):
        if r in written:
            e = rel_err(gh[r], rh[r])
            assert e <= TOL[dtype], f"slot {r} state: {e:.3e}"
            np.testing.assert_array_equal(gc[r], rc[r], err_msg=f"slot {r} conv history")
        else:
            np.testing.assert_array_equal(gh[r], pool_h[r].astype(np.float64), err_msg=f"slot {r} state touched")
            np.testing.assert_array_equal(gc[r], np.asarray(pool_c[r], np.float64), err_msg=f"slot {r} conv touched")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("interval", [64, 128])
def test_mamba1_batch(dtype, interval):
    d = W.mamba1_inputs(801, 2, 300, 96, 16, dtype=dtype, conv_bias=True, conv_state=True)
    _run(M1, d, dtype, interval, stride=5, nslots=9, seed=11)


def test_mamba1_varlen():
    lengths = [130, 0, 64, 257, 63]
    d = W.mamba1_inputs(802, 1, sum(lengths), 64, 16, dtype="bf16", conv_bias=True, conv_state=True,
                        nseqs=len(lengths))
    d["cu_seqlens"] = W.cu_from_lengths(lengths)
    _run(M1, d, "bf16", 64, stride=4, nslots=8, seed=12)


@pytest.mark.parametrize("segments", [1, 3])
@pytest.mark.parametrize("interval", [64, 128])
def test_mamba2_tensor_core_batch(interval, segments):
    d = W.mamba2_inputs(803, 2, 320, 4, 64, 2, 128, dtype="bf16", conv_bias=True, conv_state=True)
    _run(M2, d, "bf16", interval, stride=5, nslots=7, seed=13, segments=segments)


@pytest.mark.parametrize("segments", [0, 2])       # whole sequences; runs of one chunk
def test_mamba2_tensor_core_varlen(segments):
    lengths = [130, 0, 64, 257, 63, 192]
    d = W.mamba2_inputs(804, 1, sum(lengths), 4, 64, 2, 128, dtype="bf16", conv_bias=True, conv_state=True,
                        nseqs=len(lengths))
    d["cu_seqlens"] = W.cu_from_lengths(lengths)
    _run(M2, d, "bf16", 64, stride=4, nslots=10, seed=14, segments=segments)


@pytest.mark.parametrize("dtype,P,N", [("f32", 64, 128), ("bf16", 48, 64), ("f32", 16, 32)])
def test_mamba2_simt(dtype, P, N):
    lengths = [200, 64, 0, 129]
    d = W.mamba2_inputs(805, 1, sum(lengths), 4, P, 2, N, dtype=dtype, conv_bias=True, conv_state=True,
                        nseqs=len(lengths))
    d["cu_seqlens"] = W.cu_from_lengths(lengths)
    _run(M2, d, dtype, 64, stride=3, nslots=6, seed=15)
