#!/usr/bin/env python
"""Throughput benchmark of the conv1d + selective-scan hot path on B200.

Default workload: the packed variable-length Mamba-2 batch (16 sequences of
128..8192 tokens given by cu_seqlens, 56 501 tokens in all, 64 heads of
headdim 64, one group, dstate 128, conv width 4 over x|B|C, bf16
activations, fp32 state); one step is one forward pass of the fused conv +
chunked scan over that batch.  Other workloads can be picked with
``--workload`` (the Mamba-1 layer, fixed-length Mamba-2, decode, the
backward, the sequence split).

Prints ONE JSON line (rank 0).  Device time comes from CUDA events on the
launching stream around each step; L2 is flushed (a 256 MiB write) between
timed steps, outside the events.  With torchrun, each rank runs its own copy
of the workload (independent batches: weak scaling, no data-path
collective) and the reported time is the max over ranks.

``--impl reference`` times the fp64 CPU oracle instead, on a bounded sample
of the same workload, on this machine's host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from state_space_model_conv1d_b200 import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "mamba2_varlen_16seq_h64_p64_g1_n128"
METRIC = "scan tokens/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "dram_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
MUFU_PER_CLK_PER_SM = 16       # ex2 lanes per SM per clock (4 per SM sub-partition)
NUM_SMS = 148


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--segments", type=int, default=0,
                   help="token segments asked of the Mamba-2 tensor-core scan (0: the library's choice, 1: whole rows)")
    return p.parse_args()


def load_peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "state_space_model_conv1d_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------ clocks
def _nvml_poll(uuid, index, phase, done, ready, out):
    """Sampling process: NVML's SM clock and clock-event reasons of one GPU,
    as fast as the queries return (a few ms each), tagged with the phase the
    launching process has set (0: none, 1: timed region, 2: end-to-end leg);
    read-only queries."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByUUID(uuid) if uuid else pynvml.nvmlDeviceGetHandleByIndex(index)
        names = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                 "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        mx = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
    except Exception as exc:
        print(f"clock sampler: NVML unavailable ({exc!r})", file=sys.stderr, flush=True)
        ready.set()
        out.put(None)
        return
    ready.set()
    samples = []
    errors = 0
    while not done.is_set():
        ph = phase.value
        if ph:
            try:
                sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                errors += 1
                time.sleep(0.001)
                continue
            samples.append((ph, sm, sorted(n for n, bit in names.items() if r & bit)))   # phase at the query's start
            time.sleep(0.0002)
        else:
            time.sleep(0.0005)
    out.put((mx, samples, errors))


class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU during the timed
    region: a spawned process polls NVML back to back (no GIL shared with the
    launching thread) and keeps only samples between mark_start() and
    mark_stop(); without NVML, nvidia-smi samples every 200 ms.  The GPU is
    found by its UUID, so the index CUDA sees needs no translation."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.child = None
        self.lines = []
        self.source = None
        try:
            import torch
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.uuid = None

    def start(self):
        try:
            import multiprocessing as mp
            ctx = mp.get_context("spawn")
            self.phase, self.done, ready = ctx.Value("i", 0), ctx.Event(), ctx.Event()
            self.q = ctx.Queue()
            self.child = ctx.Process(target=_nvml_poll, args=(self.uuid, self.idx, self.phase, self.done, ready, self.q),
                                     daemon=True)
            self.child.start()
            if ready.wait(timeout=60):
                self.source = "nvml, every ~0.2 ms"
            else:
                print("clock sampler: NVML process did not start", file=sys.stderr, flush=True)
                self.child.terminate()
                self.child = None
        except Exception as exc:
            print(f"clock sampler: {exc!r}", file=sys.stderr, flush=True)
            self.child = None
        # nvidia-smi alongside: the fallback when NVML gives no sample of the timed region
        try:
            dev = self.uuid if self.uuid else str(self.idx)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", dev, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except FileNotFoundError:
            self.proc = None

    def mark_start(self, phase=1):
        if self.child is not None:
            self.phase.value = phase

    def mark_stop(self):
        if self.child is not None:
            self.phase.value = 0

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _stop_child(self):
        self.done.set()
        try:
            res = self.q.get(timeout=30)
        except Exception:
            res = None
        self.child.join(timeout=5)
        if not res:
            print("clock sampler: the NVML process returned nothing", file=sys.stderr, flush=True)
            return None
        mx, samples, errors = res
        if not any(x[0] == 1 for x in samples):
            print(f"clock sampler: {len(samples)} NVML samples, none in the timed region ({errors} query errors)",
                  file=sys.stderr, flush=True)
        out = {}
        for ph, key in ((1, "timed"), (2, "e2e")):
            sm = [x[1] for x in samples if x[0] == ph]
            if sm:
                out[key] = {"sm_mhz": float(np.median(sm)), "sm_min_mhz": float(min(sm)), "sm_max_mhz": mx,
                            "reasons": sorted({n for x in samples if x[0] == ph for n in x[2]}), "samples": len(sm)}
        if "timed" not in out:
            return None
        clk = dict(out["timed"], source=self.source, query_errors=errors)
        if "e2e" in out:
            clk["during_e2e_leg"] = out["e2e"]
        return clk

    def stop(self):
        clk = self._stop_child() if self.child is not None else None
        smi = self._stop_smi()
        if clk is not None:
            return clk
        if smi is not None:
            print("clock sampler: no NVML sample of the timed region; nvidia-smi's window is reported",
                  file=sys.stderr, flush=True)
        return smi

    def _stop_smi(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 200 ms, from 0.3 s before the timed region to its end"}


# --------------------------------------------------------------- workloads
class Job:
    """One workload on the device: step(), bytes and units per step, e2e step."""

    def __init__(self, w: W.Workload, rank: int, torch, ssm, segments: int = 0):
        self.w, self.torch, self.ssm = w, torch, ssm
        self.seg_request = segments    # passed to every scan call (0: the library's choice)
        dev = torch.device("cuda", torch.cuda.current_device())
        seed_shift = rank_seed(0, rank)
        bf = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.launches_per_step = 1
        self.split = None          # set by the sequence-split workloads
        self.bwd = None            # set by the backward workloads
        self.timing_on = False     # kernel timing enabled (the timed region)
        self.segments = 1          # token segments per row (tensor-core Mamba-2 path)
        self.varlen = False
        if w.kind in ("mamba1", "mamba2", "mamba2_varlen"):
            mode = ssm.MAMBA1 if w.kind == "mamba1" else ssm.MAMBA2
            ww = W.Workload(**{**w.__dict__, "seed": w.seed + seed_shift})
            d = W.workload_inputs(ww)
            self.host = {}
            t = {}
            act = ("x", "z", "dt", "B", "C")
            for k, v in d.items():
                if v is None:
                    t[k] = None
                    continue
                if k == "cu_seqlens":
                    t[k] = torch.from_numpy(v).to(dev)
                    continue
                src = torch.from_numpy(np.ascontiguousarray(v)).to(bf if k in act else torch.float32)
                self.host[k] = src.pin_memory()
                t[k] = self.host[k].to(dev)
            self.t = t
            self.mode = mode
            x = t["x"]
            nseq = x.shape[0] if t.get("cu_seqlens") is None else t["cu_seqlens"].numel() - 1
            self.tokens = x.shape[0] * x.shape[1]
            self.y = torch.empty_like(x)
            if mode == ssm.MAMBA1:
                hshape, cdim = (nseq, x.shape[2], t["B"].shape[2]), x.shape[2]
            else:
                hshape = (nseq, x.shape[2], x.shape[3], t["B"].shape[3])
                cdim = x.shape[2] * x.shape[3] + 2 * t["B"].shape[2] * t["B"].shape[3]
            self.hf = torch.empty(hshape, dtype=torch.float32, device=dev)
            self.cso = torch.empty((nseq, cdim, t["conv_w"].shape[1] - 1), dtype=bf, device=dev)
            need = ssm.scan_workspace_size(mode, x, t["dt"], t["A"], t["B"], t["C"], cu_seqlens=t.get("cu_seqlens"),
                                           conv_w=t["conv_w"], segments=segments)
            self.ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev) if need else None
            self.ssd = mode == ssm.MAMBA2 and w.dtype == "bf16" and w.headdim == 64 and w.dstate == 128 and w.d_conv <= 4
            varlen = self.varlen = t.get("cu_seqlens") is not None
            if self.ssd:
                # the B / C conv pre-pass, then the chunked tensor-core scan (+ the varlen plan)
                self.launches_per_step = 2 + (1 if varlen else 0)
            else:
                self.launches_per_step = 1 + (1 if varlen else 0)
            read = sum(v.numel() * v.element_size() for k, v in t.items() if v is not None)
            wrote = sum(v.numel() * v.element_size() for v in (self.y, self.hf, self.cso))
            self.inter = {}
            if w.state_interval:
                # every boundary of every sequence gets its own pool row, in order
                lens = np.diff(d["cu_seqlens"]) if d.get("cu_seqlens") is not None else np.full(nseq, x.shape[1])
                stride = max(1, int(lens.max()) // w.state_interval)
                tab = np.full((nseq, stride), -1, dtype=np.int32)
                nslots = 0
                for si, L in enumerate(lens):
                    for k in range(int(L) // w.state_interval):
                        tab[si, k] = nslots
                        nslots += 1
                self.inter = dict(state_interval=w.state_interval, inter_slots=torch.from_numpy(tab).to(dev),
                                  inter_states=torch.zeros((nslots,) + tuple(self.hf.shape[1:]), dtype=torch.float32,
                                                           device=dev),
                                  inter_conv=torch.zeros((nslots,) + tuple(self.cso.shape[1:]), dtype=bf, device=dev))
                read += tab.nbytes
                wrote += sum(self.inter[k].numel() * self.inter[k].element_size() for k in ("inter_states", "inter_conv"))
            self.bytes_per_step = read + wrote
            self.units = self.tokens
            self.bwd = None
            self.split = None
            if w.split_ranks:
                self._split_setup(w, mode, t, dev, bf)
            if w.backward:
                # upstream gradients of y and h_final; the step is ssm_scan_bwd, whose fp32
                # gradients of every input are what it writes
                rng = np.random.default_rng(w.seed + 7)
                dy = torch.from_numpy(rng.standard_normal(tuple(x.shape)).astype(np.float32)).to(bf)
                self.host["dy"] = dy.pin_memory()
                self.t["dy"] = self.host["dy"].to(dev)
                self.t["dh_final"] = torch.from_numpy(rng.standard_normal(tuple(self.hf.shape)).astype(np.float32)).to(dev)
                self.bwd = ssm.scan_bwd(mode, x, t["dt"], t["A"], t["B"], t["C"], self.t["dy"], D=t["D"], z=t["z"],
                                        dt_bias=t["dt_bias"], h0=t["h0"], cu_seqlens=t.get("cu_seqlens"),
                                        conv_w=t["conv_w"], conv_b=t["conv_b"], conv_state_in=t["conv_state_in"],
                                        dh_final=self.t["dh_final"])
                self.bwd_ws = torch.empty(max(1, ssm.ops.scan_bwd_workspace_size(
                    mode, x, t["dt"], t["A"], t["B"], t["C"], self.t["dy"], cu_seqlens=t.get("cu_seqlens"),
                    conv_w=t["conv_w"])), dtype=torch.uint8, device=dev)
                read = sum(v.numel() * v.element_size() for k, v in self.t.items() if v is not None and k != "cu_seqlens")
                wrote = sum(v.numel() * v.element_size() for v in self.bwd.values() if v is not None)
                self.bytes_per_step = read + wrote
                self.y = self.bwd["dx"]                       # what the end-to-end leg copies back
            if self.split is not None:
                x = self.t["x"]
            if w.backward:
                # executed exps: the checkpoint pass, the per-chunk recompute and the reverse step
                self.kernel, self.sources = "scan_bwd_kernel", ("scan_bwd.cu",)
                self.mufu = 3 * x.shape[0] * x.shape[1] * x.shape[2] * t["B"].shape[2]
                self.flops = None
                self.launches_per_step = 1 + (1 if mode == ssm.MAMBA2 else 0)
            elif mode == ssm.MAMBA1:
                # the library runs the time-parallel form when the sequential one would
                # leave the SMs short of warps (fewer than 7 per SM, dstate 16 / 32)
                nsm = torch.cuda.get_device_properties(dev).multi_processor_count
                tp = w.dstate in (16, 32) and w.d_conv <= 4 and nseq * ((w.d_inner + 31) // 32) * 4 < 7 * nsm
                self.kernel = "scan_m1_tp_kernel" if tp else "scan_m1_kernel"
                self.sources = ("scan_m1.cu",)
                self.mufu = x.shape[0] * x.shape[1] * x.shape[2] * t["B"].shape[2]
                self.flops = None
            elif self.ssd:
                self.kernel, self.sources = "ssd_kernel", ("ssd_m2.cu",)
                # rows the library cuts into token segments add the state-only pass, which
                # the kernel timing brackets together with the scan
                self.segments = ssm.scan_segments(mode, x, t["dt"], t["A"], t["B"], t["C"], z=t["z"],
                                                  cu_seqlens=t.get("cu_seqlens"), conv_w=t["conv_w"],
                                                  segments=segments)
                if self.segments > 1:
                    self.kernel = "ssd_state_kernel+ssd_kernel"
                    # packed sequences: also the segment-table pre-pass
                    self.launches_per_step += 2 if varlen else 1
                self.mufu = None
                # tensor-core work of the 64-token chunked form: per (sequence, head, chunk)
                # C.B^T (2 Q^2 N) + M.X (2 Q^2 P) + C'.S^T (2 Q N P) + B'^T.X (2 Q N P)
                Q, P, N = 64, w.headdim, w.dstate
                nchunks = int(sum((int(L) + Q - 1) // Q for L in np.diff(d["cu_seqlens"]))) if varlen else \
                    x.shape[0] * ((x.shape[1] + Q - 1) // Q)
                self.flops = nchunks * w.nheads * (2 * Q * Q * N + 2 * Q * Q * P + 4 * Q * N * P)
            else:
                self.kernel, self.sources = "scan_m2_simt_kernel", ("scan_m2_simt.cu",)
                self.mufu = None
                self.flops = None
            if self.split is not None:
                # a rank's step of the split: its largest kernel is the fix-up
                if mode == ssm.MAMBA1:
                    self.kernel = "split_fixup_m1_kernel"
                elif w.dtype == "bf16" and w.headdim == 64 and w.dstate == 128:
                    self.kernel = "split_fixup_tc_kernel"      # C'.h_in^T on the tensor cores
                else:
                    self.kernel = "split_fixup_m2_kernel"
                self.sources = ("seq_split.cu",)
        elif w.kind == "decode":
            ww = W.Workload(**{**w.__dict__, "seed": w.seed + seed_shift})
            d = W.workload_inputs(ww)
            act = ("x", "z", "dt", "B", "C", "conv_state")
            t = {}
            self.host = {}
            for k, v in d.items():
                if v is None:
                    t[k] = None
                    continue
                src = torch.from_numpy(np.ascontiguousarray(v)).to(bf if k in act else torch.float32)
                self.host[k] = src.pin_memory() if k not in ("state", "conv_state") else src
                t[k] = src.to(dev)
            self.t = t
            self.mode = ssm.MAMBA2
            self.nsets = w.nsets
            self.step_i = 0
            self.tokens = w.batch
            self.y = torch.empty_like(t["x"][0])
            per_set = sum(t[k][0].numel() * t[k][0].element_size() for k in ("x", "z", "dt", "B", "C"))
            params = sum(t[k].numel() * t[k].element_size() for k in ("A", "D", "dt_bias", "conv_w"))
            self.bytes_per_step = (2 * t["state"].numel() * 4 + 2 * t["conv_state"].numel() * t["conv_state"].element_size()
                                   + per_set + self.y.numel() * self.y.element_size() + params)
            self.units = w.batch
            self.kernel = "decode_kernel"
            self.sources = ("decode.cu",)
            self.mufu = None
            self.flops = None
        else:
            raise ValueError(w.kind)

    def _split_setup(self, w, mode, t, dev, bf):
        """One rank's part of an equal token split: the other ranks' conv tails and
        (sum of delta, end state) pairs are computed once here and staged in HBM, so
        the step runs exactly this rank's kernels and reads what the exchanges
        would have delivered."""
        from state_space_model_conv1d_b200 import seq_split
        torch, R, r = self.torch, w.split_ranks, w.split_rank
        seq = ("x", "z", "dt", "B", "C")
        bounds = [w.seqlen * k // R for k in range(R + 1)]
        kw = dict(D=t["D"], dt_bias=t["dt_bias"], h0=t["h0"], conv_w=t["conv_w"], conv_b=t["conv_b"],
                  conv_state_in=t["conv_state_in"])
        segs = []
        for k in range(R):
            s = {n: t[n][:, bounds[k]:bounds[k + 1]] for n in seq}
            segs.append(seq_split.SegmentScan(mode, k, R, s["x"], s["dt"], t["A"], s["B"], s["C"], z=s["z"], **kw))
        tails = torch.stack([s_.tail() for s_ in segs])
        pairs = torch.stack([s_.scan(tails) for s_ in segs])
        torch.cuda.synchronize()
        del segs
        # this rank's segment becomes the job's input (contiguous, pinned on the host for e2e)
        for n in seq:
            seg = self.host[n][:, bounds[r]:bounds[r + 1]].contiguous()
            self.host[n] = seg.pin_memory()
            t[n] = self.host[n].to(dev)
        self.host["h0"] = None
        self.split = dict(R=R, r=r, tails=tails, pairs=pairs, kw=dict(kw, h0=t["h0"] if r == 0 else None,
                                                                      conv_state_in=t["conv_state_in"] if r == 0 else None),
                          mod=seq_split)
        self.tokens = self.units = t["x"].shape[0] * t["x"].shape[1]
        self.y = torch.empty_like(t["x"])
        # algorithmic bytes: the segment's inputs and parameters, what the exchanges
        # deliver (the previous rank's tail, every rank's pair) and what the rank
        # writes (y, its outgoing state, its tail and its pair)
        read = sum(t[n].numel() * t[n].element_size() for n in seq if t[n] is not None)
        read += sum(t[n].numel() * t[n].element_size() for n in ("A", "D", "dt_bias", "conv_w", "conv_b")
                    if t[n] is not None)
        read += tails[0].numel() * tails.element_size() + pairs.numel() * pairs.element_size()
        wrote = self.y.numel() * self.y.element_size() + self.hf.numel() * 4 + tails[0].numel() * tails.element_size() \
            + pairs[0].numel() * pairs.element_size()
        self.bytes_per_step = read + wrote
        # tail, the scan's launches, cum_delta, combine, fix-up (the scan and cum_delta
        # write the pair into the exchange buffer; the combine reads it in place)
        self.launches_per_step = 1 + self.launches_per_step + 3
        # The fix-up is the step's largest kernel: the roofline names it, with its own
        # algorithmic bytes (y read and written, z, the raw C rows and their conv taps,
        # the prefix sums of delta and the entering state) and, for Mamba-2, the
        # fp32 FMAs of C_t . h_in (2 N P per token and head).  Its launches alone
        # are bracketed by the kernel-timing events (see _split_step).
        cum_units = w.d_inner if mode == self.ssm.MAMBA1 else w.nheads
        b_, T_ = t["x"].shape[0], t["x"].shape[1]
        self.fix_bytes = (3 * self.y.numel() * self.y.element_size() + t["C"].numel() * t["C"].element_size()
                          + b_ * T_ * cum_units * 4 + self.hf.numel() * 4)
        if mode == self.ssm.MAMBA1:
            self.fix_mufu = b_ * T_ * w.d_inner * w.dstate          # exp(A cs_t) per (token, channel, state)
            self.fix_flops = None
        else:
            self.fix_mufu = None
            self.fix_flops = 2 * b_ * T_ * w.nheads * w.headdim * w.dstate

    def _split_step(self):
        sp, t = self.split, self.t
        seg = sp["mod"].SegmentScan(self.mode, sp["r"], sp["R"], t["x"], t["dt"], t["A"], t["B"], t["C"], z=t["z"],
                                    **sp["kw"])
        timed = self.timing_on
        if timed:
            self.ssm.kernel_timing(False)         # only the fix-up is bracketed
        seg.tail()
        # this rank's pair goes straight into its block of the exchange buffer, as an
        # in-place all-gather (all_gather_into_tensor with the rank's own slice as input) has it
        seg.scan(sp["tails"], out=sp["pairs"][sp["r"]])
        if timed:
            self.ssm.kernel_timing(True)
        self.y, self.hf, _ = seg.join(sp["pairs"])

    def step(self):
        ssm, t = self.ssm, self.t
        if self.split is not None:
            self._split_step()
            return
        if self.w.kind == "decode":
            i = self.step_i % self.nsets
            self.step_i += 1
            self._decode(i, self.y)
            return
        if self.bwd is not None:
            ssm.scan_bwd(self.mode, t["x"], t["dt"], t["A"], t["B"], t["C"], t["dy"], D=t["D"], z=t["z"],
                         dt_bias=t["dt_bias"], h0=t["h0"], cu_seqlens=t.get("cu_seqlens"), conv_w=t["conv_w"],
                         conv_b=t["conv_b"], conv_state_in=t["conv_state_in"], dh_final=t["dh_final"],
                         workspace=self.bwd_ws, out=self.bwd)
            return
        self._scan(t, self.y)

    def _decode(self, i, y):
        t = self.t
        self.ssm.state_update(self.mode, t["state"], t["conv_state"], t["x"][i], t["dt"][i], t["A"], t["B"][i],
                              t["C"][i], D=t["D"], z=t["z"][i], dt_bias=t["dt_bias"], conv_w=t["conv_w"],
                              conv_b=t["conv_b"], y=y)

    def _scan(self, t, y):
        self.ssm.scan_fwd(self.mode, t["x"], t["dt"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"], dt_bias=t["dt_bias"],
                          h0=t["h0"], cu_seqlens=t.get("cu_seqlens"), conv_w=t["conv_w"], conv_b=t["conv_b"],
                          conv_state_in=t["conv_state_in"], y=y, h_final=self.hf, conv_state_out=self.cso,
                          workspace=self.ws, segments=self.seg_request, **self.inter)

    def e2e_pipelined(self):
        """Whether the end-to-end leg overlaps copies with compute (forward scans and decode)."""
        return self.split is None and self.bwd is None

    def e2e_run(self, n, out_hosts, stream):
        """n end-to-end steps of a forward scan, pipelined across steps: step i's
        inputs go host->device on one stream while step i-1 computes on `stream`
        and step i-2's y goes device->host on a third (both PCIe directions at
        once); device inputs and y are double-buffered.  Every step copies all of
        its inputs in and its y out.  Returns (h2d, d2h) bytes per step."""
        torch = self.torch
        if self.w.kind == "decode":
            return self._e2e_decode(n, out_hosts, stream)
        keys = [k for k in ("x", "z", "dt", "B", "C", "h0") if self.host.get(k) is not None]
        if not hasattr(self, "_t2"):
            self._t2 = dict(self.t)
            for k in keys:
                self._t2[k] = torch.empty_like(self.t[k])
            self._y2 = torch.empty_like(self.y)
        sets = [(self.t, self.y), (self._t2, self._y2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {name: [torch.cuda.Event(), torch.cuda.Event()] for name in ("in", "comp", "out")}
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            b = i % 2
            tb, yb = sets[b]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev["comp"][b])          # step i-2 has finished reading these inputs
                for k in keys:
                    tb[k].copy_(self.host[k], non_blocking=True)
                ev["in"][b].record(s_in)
            stream.wait_event(ev["in"][b])
            if i >= 2:
                stream.wait_event(ev["out"][b])             # step i-2's y has reached the host
            self._scan(tb, yb)
            ev["comp"][b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["comp"][b])
                out_hosts[b].copy_(yb, non_blocking=True)
                ev["out"][b].record(s_out)
        for b in range(min(n, 2)):
            stream.wait_event(ev["out"][b])
        h2d = sum(self.host[k].numel() * self.host[k].element_size() for k in keys)
        return h2d, out_hosts[0].numel() * out_hosts[0].element_size()

    def _e2e_decode(self, n, out_hosts, stream):
        """Decode steps with the copies overlapped: the token inputs of step i go
        into its input set (sets cycle, so a set is rewritten only after the
        step that last read it) while earlier steps compute; y alternates
        between two buffers.  The state update itself stays in order on
        `stream`, one step after the other."""
        torch, t = self.torch, self.t
        keys = [k for k in ("x", "z", "dt", "B", "C") if self.host.get(k) is not None]
        if not hasattr(self, "_y2"):
            self._y2 = torch.empty_like(self.y)
        ys = [self.y, self._y2]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(self.nsets)]
        ev_comp = [torch.cuda.Event() for _ in range(self.nsets)]
        ev_out = [torch.cuda.Event(), torch.cuda.Event()]
        start = torch.cuda.Event()
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for j in range(n):
            i = self.step_i % self.nsets
            self.step_i += 1
            b = j % 2
            with torch.cuda.stream(s_in):
                if j >= self.nsets:
                    s_in.wait_event(ev_comp[i])
                for k in keys:
                    t[k][i].copy_(self.host[k][i], non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if j >= 2:
                stream.wait_event(ev_out[b])
            self._decode(i, ys[b])
            ev_comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                out_hosts[b].copy_(ys[b], non_blocking=True)
                ev_out[b].record(s_out)
        for b in range(min(n, 2)):
            stream.wait_event(ev_out[b])
        h2d = sum(self.host[k][0].numel() * self.host[k][0].element_size() for k in keys)
        return h2d, out_hosts[0].numel() * out_hosts[0].element_size()

    def e2e_step(self, out_host):
        """Host-resident inputs: pinned H2D copies, the step, then y back to the host."""
        torch, t = self.torch, self.t
        h2d = 0
        if self.w.kind == "decode":
            i = self.step_i % self.nsets
            for k in ("x", "z", "dt", "B", "C"):
                t[k][i].copy_(self.host[k][i], non_blocking=True)
                h2d += self.host[k][i].numel() * self.host[k][i].element_size()
        else:
            for k in ("x", "z", "dt", "B", "C", "h0", "dy"):
                if self.host.get(k) is not None:
                    t[k].copy_(self.host[k], non_blocking=True)
                    h2d += self.host[k].numel() * self.host[k].element_size()
        self.step()
        out_host.copy_(self.y, non_blocking=True)
        return h2d, out_host.numel() * out_host.element_size()


def flush_l2(buf):
    buf.add_(1)       # 256 MiB read + write, twice the 126 MB L2


def reduce_max_ms(ms: float, world: int, device) -> float:
    """Max over ranks of a device-measured time (the slowest rank sets the pace)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch (weak scaling)."""
    return units_per_rank * steps * world / (max_ms / 1e3)


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own synthetic batch."""
    return base + 7919 * rank


def gpu_local_cpus(device_index: int):
    """The host CPUs NVML names as closest to this process's GPU (read-only
    query; found by UUID), or None."""
    try:
        import torch
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(torch.cuda.get_device_properties(device_index).uuid))
        words = pynvml.nvmlDeviceGetCpuAffinity(h, 64)
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (int(w) >> b) & 1}
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


def run_cuda(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import state_space_model_conv1d_b200 as ssm

    # Keep this process (and so its pinned host buffers) on the GPU's own CPU
    # socket while the GPU runs: host<->device copies then cross no socket link.
    # The full CPU set comes back for the CPU baseline.
    all_cpus = os.sched_getaffinity(0)
    near = gpu_local_cpus(local)
    if near:
        os.sched_setaffinity(0, near)
    w = W.WORKLOADS[args.workload]
    job = Job(w, rank, torch, ssm, segments=args.segments)
    flush = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 0)):
        job.step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
        time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ssm.kernel_time_ms()                       # drop any earlier tally
    ssm.kernel_timing(True)                    # events around the dominant kernel of each call, on its stream
    job.timing_on = True
    clocks.mark_start()
    for i in range(args.steps):
        flush_l2(flush)
        evs[i][0].record(stream)
        job.step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clocks.mark_stop()
    ssm.kernel_timing(False)
    job.timing_on = False
    kern_ms_total, kern_launches = ssm.kernel_time_ms()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = reduce_max_ms(float(sum(step_ms)), world, "cuda")
    # the dominant kernel's own average launch duration (max over ranks), for the roofline
    kern_ms = reduce_max_ms(kern_ms_total / max(kern_launches, 1), world, "cuda")
    ms_per_step = total_ms / max(args.steps, 1)
    value = weak_scaling_value(job.units, args.steps, world, total_ms)

    # end to end through the public API with host-resident inputs
    e2e = None
    if not args.no_e2e:
        out_host = torch.empty(job.y.shape, dtype=job.y.dtype).pin_memory()
        ne = max(1, min(args.steps, 10))
        pipelined = job.e2e_pipelined()
        if pipelined:
            out_hosts = [out_host, torch.empty(job.y.shape, dtype=job.y.dtype).pin_memory()]
            job.e2e_run(2, out_hosts, stream)                  # warm-up (allocates the second buffer set)
        else:
            job.e2e_step(out_host)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.mark_start(2)
        e0.record(stream)
        h2d = d2h = 0
        if pipelined:
            h2d, d2h = job.e2e_run(ne, out_hosts, stream)
        else:
            for _ in range(ne):
                h2d, d2h = job.e2e_step(out_host)
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_stop()
        ems = reduce_max_ms(e0.elapsed_time(e1), world, "cuda")
        e2e = {"value": weak_scaling_value(job.units, ne, world, ems), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": ne,
               "copies": ("overlapped across steps: inputs in on one stream, y out on another, compute on a third; "
                          "device buffers double-buffered" if pipelined else "in order within each step"),
               "host_cpus": (f"{len(near)} CPUs local to the GPU (NVML affinity), pinned buffers allocated there"
                             if near else "unrestricted")}

    clk = clocks.stop() if rank == 0 else None
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    src = lambda key: f"measured (MEASURED_PEAKS.json {key})" if peak_src == "measured" else f"fallback ({key})"
    gbs = job.bytes_per_step / (ms_per_step / 1e3) / 1e9
    kbytes = job.fix_bytes if job.split is not None else job.bytes_per_step   # the timed kernel's own bytes
    kgbs = kbytes / (kern_ms / 1e3) / 1e9 if kern_ms > 0 else gbs
    if job.split is not None:
        job.mufu, job.flops = job.fix_mufu, None
    traffic = None
    if os.path.exists(TRAFFIC_PATH):
        with open(TRAFFIC_PATH) as f:
            tr = json.load(f).get(args.workload)
        if tr and tr.get("source_sha") == source_sha(*job.sources):
            traffic = tr.get("dram_bytes_per_launch")
    if job.mufu is not None:
        clock_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        peak_g = NUM_SMS * MUFU_PER_CLK_PER_SM * clock_mhz * 1e6 / 1e9
        achieved = job.mufu / (kern_ms / 1e3) / 1e9
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak_g, "unit": "Gexp/s",
                    "frac": achieved / peak_g, "traffic": traffic, "kernel": job.kernel,
                    "peak_source": f"derived: {NUM_SMS} SMs x {MUFU_PER_CLK_PER_SM} MUFU ex2/clk x {clock_mhz:.0f} MHz",
                    "hbm": {"achieved": kgbs, "peak": hbm_peak, "unit": "GB/s", "frac": kgbs / hbm_peak,
                            "peak_source": src("hbm_gbs")}}
    else:
        roofline = {"bound": "hbm", "achieved": kgbs, "peak": hbm_peak, "unit": "GB/s", "frac": kgbs / hbm_peak,
                    "traffic": traffic, "kernel": job.kernel,
                    "peak_source": src("hbm_gbs")}
        if job.flops:
            tf = job.flops / (kern_ms / 1e3) / 1e12
            tpk = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1400.0)))
            roofline["tensor"] = {"achieved": tf, "peak": tpk, "unit": "TFLOP/s", "frac": tf / tpk,
                                  "flops_per_step": int(job.flops), "peak_source": src("bf16_tflops_sustained")}
    if job.split is not None and job.fix_flops and job.kernel == "split_fixup_tc_kernel":
        tpk = float(peaks.get("bf16_tflops", 1590.0))
        ftf = job.fix_flops / (kern_ms / 1e3) / 1e12
        roofline["tensor"] = {"achieved": ftf, "peak": tpk, "unit": "TFLOP/s", "frac": ftf / tpk,
                              "flops_per_launch": int(job.fix_flops), "peak_source": src("bf16_tflops")}
    elif job.split is not None and job.fix_flops:
        fma_peak = NUM_SMS * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12
        ftf = job.fix_flops / (kern_ms / 1e3) / 1e12
        roofline["fma"] = {"achieved": ftf, "peak": fma_peak, "unit": "TFLOP/s", "frac": ftf / fma_peak,
                           "flops_per_launch": int(job.fix_flops),
                           "peak_source": f"derived: {NUM_SMS} SMs x 128 fp32 FMA/clk x 2 x clock"}
    roofline["algorithmic_bytes_per_launch"] = int(kbytes)
    roofline["kernel_ms"] = kern_ms
    roofline["kernel_launches_timed"] = kern_launches
    roofline["timing"] = ("CUDA events around every launch of the kernel, on its stream, inside the timed region "
                          "(ssm_kernel_timing); achieved = algorithmic bytes (or exps, flops) of the step / kernel_ms")

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        os.sched_setaffinity(0, all_cpus)
        cpu = cpu_baseline(w, args)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "global_batch": (w.batch or 1) * world, "seq_len": w.seqlen or None,
                   "parallelism": (f"seqsplit{w.split_ranks}: rank {w.split_rank}'s step, exchanges staged in HBM"
                                   if w.split_ranks else (f"replicas{world}" if world > 1 else "single")),
                   "l2": "flushed between timed steps (256 MiB write, outside the events)",
                   "tokens_per_step": job.units,
                   ("token_segment_rows_launched" if job.varlen else "token_segments_per_row"): job.segments,
                   "token_segments_requested": args.segments or "library choice"},
        "hbm_gbs": gbs, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
        "gpu_launches": job.launches_per_step * args.steps, "impl": "cuda",
        "step_ms": {"min": min(step_ms), "median": float(np.median(step_ms)), "max": max(step_ms)},
    }
    print(json.dumps(out), flush=True)


# --------------------------------------------------------------- oracle side
def oracle_sample(w: W.Workload, target_s: float):
    """A bounded sample of the workload for the fp64 oracle: whole sequences
    (all channels / heads), as many as fit the time budget."""
    import oracle
    cores = os.cpu_count() or 1
    if w.kind == "mamba1" and w.backward:
        # the backward keeps every step's state: one batch row (all channels)
        nch = w.d_inner
        ww = W.Workload(**{**w.__dict__, "batch": 1, "d_inner": nch})
        d = W.workload_inputs(ww)
        dy = np.random.default_rng(w.seed + 7).standard_normal(d["x"].shape)
        run = lambda: oracle.scan_bwd(oracle.MAMBA1, d["x"], d["dt"], d["A"], d["B"], d["C"], dy, D=d["D"], z=d["z"],
                                      dt_bias=d["dt_bias"], h0=d["h0"], conv_w=d["conv_w"])
        return (run, w.seqlen * nch / w.d_inner, 1,
                f"1 of {w.batch} batch rows x {w.seqlen} tokens, all {w.d_inner} channels")
    if w.kind == "mamba1":
        nrows = min(w.batch, max(1, cores))
        ww = W.Workload(**{**w.__dict__, "batch": nrows})
        d = W.workload_inputs(ww)
        run = lambda: oracle.scan_fwd(oracle.MAMBA1, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                                      dt_bias=d["dt_bias"], h0=d["h0"], conv_w=d["conv_w"], nthreads=nrows)
        return run, nrows * w.seqlen, nrows, f"{nrows} of {w.batch} batch rows x {w.seqlen} tokens, all {w.d_inner} channels"
    if w.kind in ("mamba2", "mamba2_varlen"):
        # nrows sequences of T tokens (all heads): T grows in steps of 256 tokens, up
        # to the workload's sequence length, until one run takes about target_s
        # (timed once at 256 tokens)
        nrows = min(8, max(1, cores), w.batch if w.kind == "mamba2" else w.nseqs)
        t_max = max(256, (w.seqlen if w.kind == "mamba2" else w.len_hi) // 256 * 256)

        def make(T):
            ww = W.Workload(**{**w.__dict__, "kind": "mamba2", "batch": nrows, "seqlen": T})
            d = W.workload_inputs(ww)
            return lambda: oracle.scan_fwd(oracle.MAMBA2, d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"],
                                           z=d["z"], dt_bias=d["dt_bias"], h0=d["h0"], conv_w=d["conv_w"],
                                           nthreads=nrows)
        T, run = 256, make(256)
        t0 = time.perf_counter()
        run()
        per256 = time.perf_counter() - t0
        steps = int(min(t_max // 256, max(1, target_s // max(per256, 1e-3))))
        if steps > 1:
            T, run = 256 * steps, make(256 * steps)
        return run, nrows * T, nrows, f"{nrows} sequences x {T} tokens, all {w.nheads} heads"
    if w.kind == "decode":
        nb = 16
        ww = W.Workload(**{**w.__dict__, "batch": nb, "nsets": 1})
        d = W.workload_inputs(ww)
        state = d["state"].astype(np.float64)
        cs = d["conv_state"].astype(np.float64)
        run = lambda: oracle.state_update(oracle.MAMBA2, state, cs, d["x"][0], d["dt"][0], d["A"], d["B"][0], d["C"][0],
                                          D=d["D"], z=d["z"][0], dt_bias=d["dt_bias"], conv_w=d["conv_w"])
        return run, nb, 1, f"one decode step of {nb} of {w.batch} rows"
    raise ValueError(w.kind)


def cpu_baseline(w: W.Workload, args):
    run, units, cores, what = oracle_sample(w, 10.0)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    return {"value": units / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": what,
            "seconds": dt}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    # every step a sample sized so the whole run takes about two minutes
    run, units, cores, what = oracle_sample(w, 120.0 / max(1, args.steps + max(args.warmup, 0)))
    for _ in range(max(args.warmup, 0)):
        run()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run()
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = units * args.steps / total
    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": total / max(args.steps, 1) * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": w.name, "global_batch": w.batch or 1, "seq_len": w.seqlen or None,
                      "parallelism": "host cores", "sample": what},
           "impl": "reference",
           "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": what},
           "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_cuda(args)


if __name__ == "__main__":
    main()
