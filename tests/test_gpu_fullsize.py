"""Parity at the full benchmark sizes, in the launch configuration bench.py times.

The whole workload runs on the GPU; the fp64 oracle then recomputes a sample
of independent units one by one (Mamba-1 channels, Mamba-2 heads with their
group's B / C, decode batch rows) and the sampled outputs are compared.
"""
import numpy as np
import pytest
import torch

import oracle
import state_space_model_conv1d_b200 as ssm
from state_space_model_conv1d_b200 import workloads as W

from gpu_util import TOL, assert_close, gpu_scan, to_dev

pytestmark = pytest.mark.gpu
M1, M2 = oracle.MAMBA1, oracle.MAMBA2


def test_mamba1_layer_fullsize_sampled_channels():
    w = W.WORKLOADS["mamba1_layer_b8_l2048_d1536_n16"]
    d = W.workload_inputs(w)
    y, hf, cs = gpu_scan(M1, to_dev(d, "bf16"))
    sel = np.array([0, 1, 31, 32, 33, 511, 777, 1023, 1024, 1500, 1535])
    sub = dict(x=d["x"][:, :, sel], z=d["z"][:, :, sel], dt=d["dt"][:, :, sel], B=d["B"], C=d["C"], A=d["A"][sel],
               D=d["D"][sel], dt_bias=d["dt_bias"][sel], h0=d["h0"][:, sel], conv_w=d["conv_w"][sel])
    ry, rh, rc = oracle.scan_fwd(M1, sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"], D=sub["D"], z=sub["z"],
                                 dt_bias=sub["dt_bias"], h0=sub["h0"], conv_w=sub["conv_w"], nthreads=8)
    assert_close(y[:, :, sel], ry, "bf16", "M1 full-size y")
    assert_close(hf[:, sel], rh, "bf16", "M1 full-size h_final")
    assert_close(cs[:, sel], rc, "bf16", "M1 full-size conv state")


def _m2_head_problem(d, h, H, P, G, N):
    """The independent sub-problem of one Mamba-2 head: its x channels, its
    group's B / C, and the matching conv weights and states."""
    g = h // (H // G)
    Dn = H * P
    xch = np.arange(h * P, (h + 1) * P)
    bch = Dn + g * N + np.arange(N)
    cch = Dn + G * N + g * N + np.arange(N)
    rows = np.concatenate([xch, bch, cch])
    sub = dict(x=d["x"][:, :, h:h + 1], z=d["z"][:, :, h:h + 1], dt=d["dt"][:, :, h:h + 1],
               B=d["B"][:, :, g:g + 1], C=d["C"][:, :, g:g + 1], A=d["A"][h:h + 1], D=d["D"][h:h + 1],
               dt_bias=d["dt_bias"][h:h + 1], h0=d["h0"][:, h:h + 1], conv_w=d["conv_w"][rows],
               conv_state_in=None if d.get("conv_state_in") is None else d["conv_state_in"][:, rows], rows=rows)
    return sub


# The library's choice for these shapes: the fixed-length workloads and the
# two long packed sequences run cut into token segments, the 16 packed
# sequences (1024 chains) whole.
@pytest.mark.parametrize("name,cut", [("mamba2_ssd_b4_l4096_h80_p64_g8_n128", True),
                                      ("mamba2_varlen_16seq_h64_p64_g1_n128", False),
                                      ("mamba2_seq_b1_l16384_h80_p64_g8_n128", True),
                                      ("mamba2_varlen_2seq_h80_p64_g8_n128", True)])
def test_mamba2_fullsize_sampled_heads(name, cut):
    w = W.WORKLOADS[name]
    d = W.workload_inputs(w)
    t = to_dev(d, "bf16")
    nseg = ssm.scan_segments(M2, t["x"], t["dt"], t["A"], t["B"], t["C"], z=t["z"], cu_seqlens=t.get("cu_seqlens"),
                             conv_w=t["conv_w"])
    assert (nseg > 1) == cut, nseg
    y, hf, cs = gpu_scan(M2, t)
    H, P, G, N = w.nheads, w.headdim, w.ngroups, w.dstate
    for h in (0, H // 2 - 1, H // 2, H - 1):
        sub = _m2_head_problem(d, h, H, P, G, N)
        ry, rh, rc = oracle.scan_fwd(M2, sub["x"], sub["dt"], sub["A"], sub["B"], sub["C"], D=sub["D"], z=sub["z"],
                                     dt_bias=sub["dt_bias"], h0=sub["h0"], conv_w=sub["conv_w"],
                                     conv_state_in=sub["conv_state_in"], cu_seqlens=d.get("cu_seqlens"), nthreads=8)
        assert_close(y[:, :, h:h + 1], ry, "bf16", f"{name} head {h} y")
        assert_close(hf[:, h:h + 1], rh, "bf16", f"{name} head {h} h_final")
        # the head's x channels and its group's B / C channels of the carried conv state
        assert_close(cs[:, sub["rows"]], rc, "bf16", f"{name} head {h} conv_state_out")


def test_decode_fullsize_sampled_rows():
    w = W.WORKLOADS["mamba2_decode_b256_h128_p64_g8_n128"]
    d = W.workload_inputs(w)
    t = to_dev({k: v for k, v in d.items() if k not in ("state", "conv_state")}, "bf16")
    state = torch.from_numpy(d["state"]).cuda()
    cstate = torch.from_numpy(d["conv_state"]).to(torch.bfloat16).cuda()
    import state_space_model_conv1d_b200 as ssm
    y = ssm.state_update(M2, state, cstate, t["x"][0], t["dt"][0], t["A"], t["B"][0], t["C"][0], D=t["D"],
                         z=t["z"][0], dt_bias=t["dt_bias"], conv_w=t["conv_w"])
    torch.cuda.synchronize()
    for r in (0, 1, 127, 255):
        st = d["state"][r:r + 1].astype(np.float64).copy()
        cst = d["conv_state"][r:r + 1].astype(np.float64).copy()
        ry = oracle.state_update(M2, st, cst, d["x"][0][r:r + 1], d["dt"][0][r:r + 1], d["A"], d["B"][0][r:r + 1],
                                 d["C"][0][r:r + 1], D=d["D"], z=d["z"][0][r:r + 1], dt_bias=d["dt_bias"],
                                 conv_w=d["conv_w"])
        assert_close(y[r:r + 1].float().cpu().numpy(), ry, "bf16", f"decode row {r} y")
        assert_close(state[r:r + 1].cpu().numpy(), st, "bf16", f"decode row {r} state")
        assert_close(cstate[r:r + 1].float().cpu().numpy(), cst, "bf16", f"decode row {r} conv state")


def test_mamba1_layer_backward_fullsize():
    """The backward at the Mamba-1 layer's full size: per-channel gradients on
    sampled channels of every row, and the channel-summed dB / dC of row 0
    from a full-width oracle run of that row."""
    w = W.WORKLOADS["mamba1_layer_b8_l2048_d1536_n16_bwd"]
    d = W.workload_inputs(w)
    rng = np.random.default_rng(w.seed + 7)
    dy = W.round_bf16(rng.standard_normal(d["x"].shape))
    dhf = rng.standard_normal(d["h0"].shape).astype(np.float32).astype(np.float64)
    t = to_dev(d, "bf16")
    import state_space_model_conv1d_b200 as ssm
    g = ssm.scan_bwd(M1, t["x"], t["dt"], t["A"], t["B"], t["C"], torch.from_numpy(dy).to("cuda", torch.bfloat16),
                     D=t["D"], z=t["z"], dt_bias=t["dt_bias"], h0=t["h0"], conv_w=t["conv_w"],
                     dh_final=torch.from_numpy(dhf).float().cuda())
    torch.cuda.synchronize()
    g = {k: (None if v is None else v.cpu().numpy()) for k, v in g.items()}
    sel = np.array([0, 1, 31, 32, 777, 1535])
    r = oracle.scan_bwd(M1, d["x"][:, :, sel], d["dt"][:, :, sel], d["A"][sel], d["B"], d["C"], dy[:, :, sel],
                        D=d["D"][sel], z=d["z"][:, :, sel], dt_bias=d["dt_bias"][sel], h0=d["h0"][:, sel],
                        conv_w=d["conv_w"][sel], dh_final=dhf[:, sel])
    assert_close(g["dx"][:, :, sel], r["dx"], "bf16", "bwd dx")
    assert_close(g["dz"][:, :, sel], r["dz"], "bf16", "bwd dz")
    assert_close(g["ddt"][:, :, sel], r["ddt"], "bf16", "bwd ddt")
    assert_close(g["dA"][sel], r["dA"], "bf16", "bwd dA")
    assert_close(g["dD"][sel], r["dD"], "bf16", "bwd dD")
    assert_close(g["ddt_bias"][sel], r["ddt_bias"], "bf16", "bwd ddt_bias")
    assert_close(g["dh0"][:, sel], r["dh0"], "bf16", "bwd dh0")
    assert_close(g["dconv_w"][sel], r["dconv_w"], "bf16", "bwd dconv_w")
    row = oracle.scan_bwd(M1, d["x"][:1], d["dt"][:1], d["A"], d["B"][:1], d["C"][:1], dy[:1], D=d["D"], z=d["z"][:1],
                          dt_bias=d["dt_bias"], h0=d["h0"][:1], conv_w=d["conv_w"], dh_final=dhf[:1])
    assert_close(g["dB"][:1], row["dB"], "bf16", "bwd dB row 0")
    assert_close(g["dC"][:1], row["dC"], "bf16", "bwd dC row 0")
