#!/usr/bin/env python3
"""Gated DSA layer benchmark on B200.

Headline (one JSON line): decode tokens/s of one Gated DSA layer at a 128K
context, batch 8 -- 32x128 e4m3 indexer without RoPE, top-K = 2048, 128
query heads over the 576-wide paged latent cache (512 value dims), sigmoid
gate -- measured through the C ABI (dsa_layer_forward) on synthetic inputs
already resident in HBM.  Also reported: the dominant kernel (the decode
indexer's key stream) against the measured HBM copy bandwidth, the per-stage
split, the prefill indexer (T = 32768, 16x128) against a measured FP8 GEMM
peak, an end-to-end figure through host buffers, the CPU oracle on the
host's cores, and the SM clocks seen during the timed region.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Under torchrun (N > 1) every rank serves its own batch of 8 sequences (the
path shards by sequence; no collective on the data path): weak scaling,
value = tokens of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "DSA-layer decode tokens/s @128K ctx; prefill indexer TFLOPS & % HBM/FP8 roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20   # > 126 MB L2


class L2Flush:
    """Evicts the step's data from L2 between timed steps: writes a buffer
    larger than L2, then reads another one, so the dirty lines of the write
    are written back here and not inside the next timed step."""

    def __init__(self):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")

    def zero_(self):
        self.w.zero_()
        self.r.sum()
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "indexer_decode_B8_L131072.md")


# ---------------------------------------------------------------- helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--context", type=int, default=131072)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the prefill-indexer, e2e, CPU-baseline and parity legs (profiling runs)")
    ap.add_argument("--ref-budget-s", type=float, default=120.0,
                    help="wall-clock budget of the --impl reference run")
    ap.add_argument("--prefill-only", type=int, default=0, metavar="T",
                    help="time only the prefill indexer at T queries (small cases for profiling)")
    ap.add_argument("--with-topk", action="store_true",
                    help="with --prefill-only: also time dsa_topk over the indexer's causal rows")
    ap.add_argument("--attn-only", type=int, default=0, metavar="T",
                    help="time only the prefill attention on T queries (small cases for profiling)")
    ap.add_argument("--hybrid-only", action="store_true",
                    help="time only the hybrid serving step (one DSA and five sliding-window layers), for profiling")
    ap.add_argument("--append-only", action="store_true",
                    help="time only the append step (dsa_append_kv), for profiling")
    ap.add_argument("--workload", choices=["decode", "cp_decode_1m"], default="decode",
                    help="cp_decode_1m: one 1,048,576-token sequence's history split over the N ranks "
                         "(context-parallel decode, two NCCL all-gathers per step)")
    return ap.parse_args(argv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def aggregate(local_ms: float, local_tokens: int, world: int):
    """Max-over-ranks time and summed tokens (collective only when world > 1)."""
    if world == 1:
        return local_ms, local_tokens
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    n = torch.tensor([float(local_tokens)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), int(n.item())


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
    BAD = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}

    def __init__(self, torch_device: int, period_s: float = 0.0005):
        self.samples = []  # (sm MHz, reason bits, host time)
        self.period = period_s
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def sample_now(self):
        """One reading from the calling thread.  The timed loop calls this while
        the GPU still runs the steps it has queued, so even a short timed region
        (a few milliseconds) holds readings taken under load."""
        if not self.ok:
            return
        try:
            self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM), self._reasons(),
                                 time.perf_counter()))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample_now()
            time.sleep(self.period)

    def __enter__(self):
        # the timed loop is a tight Python loop: let the sampler thread get the
        # interpreter often enough to sample during it
        self._switch = sys.getswitchinterval()
        sys.setswitchinterval(0.0002)
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
        sys.setswitchinterval(self._switch)
        return False

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "no NVML")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r, _ in self.samples:
            bits |= r
        names = [n for b, n in self.REASONS.items() if bits & b]
        t = sorted(s[2] for s in self.samples)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples), "span_ms": round((t[-1] - t[0]) * 1e3, 3)}

    # reasons that explain clocks below the maximum (a power cap is kept and noted)
    EXPLAINED = {"sw_power_cap", "hw_power_brake_slowdown", "sync_boost", "applications_clocks_setting"}
    LOW_FRACTION = 0.85

    def rejected(self):
        """A thermal or hardware slowdown, or SM clocks well below the maximum
        with no reason that explains them (a leftover clock lock)."""
        s = self.summary()
        reasons = set(s.get("reasons", []))
        if reasons & self.BAD:
            return True
        mhz, top = s.get("sm_mhz"), s.get("sm_max_mhz")
        return bool(mhz and top and mhz < self.LOW_FRACTION * top and not reasons & self.EXPLAINED)


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "long_context_sparse_02_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


# the files that define the decode indexer kernel (the grouped few-query kernel lives apart)
INDEXER_SOURCES = ("indexer.cu", "indexer_common.cuh", "dsa_device.cuh")


def profiled_traffic():
    """dram read+write bytes per launch of the decode indexer from the committed
    ncu summary, or None when the kernel source changed since that capture."""
    if not os.path.exists(PROFILE_SUMMARY):
        return None, "no ncu summary"
    txt = open(PROFILE_SUMMARY).read()
    m = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", txt)
    t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m or not t:
        return None, "summary lacks traffic/source hash"
    if m.group(1) != source_hash(*INDEXER_SOURCES):
        return None, "indexer source changed since the ncu capture"
    return float(t.group(1)), "ncu capture (profiles/)"


# ---------------------------------------------------------------- algorithmic work

def decode_bytes(case):
    """Bytes the decode layer must move (no score round trip), and the decode
    indexer's algorithmic bytes (its key stream, queries and weights: the score
    round trip is not part of the method)."""
    L = case.seq_lens.astype(float)
    kI = float((L * case.DI).sum())
    qI = case.T * case.HI * case.DI + case.T * case.HI * 4
    rows = float(sum(min(case.K, int(x)) for x in case.seq_lens))
    gather = rows * case.Dqk * 2
    q = case.T * case.H * case.Dqk * 2
    gate = case.T * case.H * 2
    out = case.T * case.H * case.Dv * 2
    layer = kI + qI + gather + q + gate + out
    indexer = kI + qI
    return layer, indexer


def score_write_bytes(case):
    """The fp32 scores the decode indexer writes (one per key): the score
    round trip, reported beside the algorithmic figure."""
    return float(case.seq_lens.astype(float).sum()) * 4


# nominal B200 peaks, reported beside the measured ones: HBM3e 7.7 TB/s (HGX), dense FP8 4.5 PFLOP/s
SPEC_HBM_GBS = 7700.0
SPEC_FP8_TFLOPS = 4500.0


def swa_bytes(B, H, D, window, min_len):
    """Bytes one sliding-window decode layer must move: each sequence's K and
    V rings over the window (all of it once the sequence is that long), the
    query row and the output row, bf16."""
    return float(B * H * D * 2 * (2 * min(window, int(min_len)) + 2))


def prefill_topk_bytes(T, K):
    """The top-K over T causal score rows (row t holds t + 1 fp32 scores):
    the scores read plus the T x K int32 indices written."""
    return 4.0 * T * (T + 1) / 2 + 4.0 * T * K


def prefill_indexer_flops(T, HI, DI):
    """2 * HI * DI multiply-adds per (query, causal key) pair, T(T+1)/2 pairs."""
    return 2.0 * HI * DI * T * (T + 1) / 2


# ---------------------------------------------------------------- native arm

def run_native(args):
    import numpy as np
    import torch

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    from long_context_sparse_02_b200 import build, synth
    build.build()
    from long_context_sparse_02_b200 import _lib
    from long_context_sparse_02_b200.runtime import LayerOnDevice, to_dev

    B, Lctx = args.batch, args.context
    case = synth.decode_case(args.seed + 1000 * rank, [Lctx] * B, HI=32, name=f"decode_B{B}_L{Lctx}")
    lay = LayerOnDevice(case, decode=True, want_idx=True)
    launches = _lib.layer_kernel_launches(lay.args)
    flush = L2Flush()
    stream = torch.cuda.current_stream()
    _lib.device_error(reset=True)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        flush.zero_()
        lay.forward()
    barrier()

    # ---- timed region: K steps of the layer through the C ABI, L2 flushed
    # between steps (outside the step's events).  The layer's kernels run as
    # programmatic dependents of one another, so nothing is recorded between
    # them here; the stage split comes from separate steps through
    # dsa_layer_forward_profiled, which records an event between stages (and
    # so serialises them).
    def make_events(K, n):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n)] for _ in range(K)]
        for es in ev:
            for e in es:
                e.record(stream)  # creates the handle
        torch.cuda.synchronize()
        return ev

    def timed(K, clk):
        ev = make_events(K, 2)
        barrier()
        for i, (e0, e1) in enumerate(ev):
            flush.zero_()
            e0.record(stream)
            lay.forward()
            e1.record(stream)
            if i == 0:
                clk.sample_now()  # the first step is running
        clk.sample_now()  # the queued steps are still running
        barrier()
        return ev

    def staged(K):
        ev = make_events(K, 4)
        for e4 in ev:
            flush.zero_()
            lay.forward_profiled(e4)
        torch.cuda.synchronize()
        return ev

    for attempt in range(2):
        clk = ClockSampler(local)
        with clk:
            ev = timed(args.steps, clk)
        if not clk.rejected():
            break
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    total_ms = sum(step_ms)
    err = _lib.device_error(reset=True)
    if err:
        raise RuntimeError(f"device error word {err:#x} after the timed region")
    max_ms, tokens = aggregate(total_ms, B * args.steps, world)
    value = tokens / (max_ms / 1e3)
    evs = staged(max(20, min(args.steps, 200)))
    st = {k: statistics.mean(e4[i].elapsed_time(e4[i + 1]) for e4 in evs) * 1e3
          for i, k in enumerate(["indexer", "topk", "attention"])}
    st_total = statistics.mean(e4[0].elapsed_time(e4[3]) for e4 in evs) * 1e3

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    layer_bytes, idx_bytes = decode_bytes(case)
    idx_gbs = idx_bytes / (st["indexer"] * 1e-6) / 1e9
    io_gbs = (idx_bytes + score_write_bytes(case)) / (st["indexer"] * 1e-6) / 1e9
    traffic, traffic_src = profiled_traffic()
    roofline = {"bound": "hbm", "kernel": "indexer_decode_kernel<128,32> (stage 1 of dsa_layer_forward)",
                "achieved": round(idx_gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(idx_gbs / hbm, 4),
                "peak_spec": SPEC_HBM_GBS, "frac_spec": round(idx_gbs / SPEC_HBM_GBS, 4),
                "traffic": traffic, "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": idx_bytes, "launch_us": round(st["indexer"], 2),
                "with_score_writes": {"bytes_per_launch": idx_bytes + score_write_bytes(case),
                                      "achieved": round(io_gbs, 1), "frac": round(io_gbs / hbm, 4)},
                "peak_source": f"hbm_gbs, {peak_src}"}
    step_mean_ms = total_ms / args.steps
    layer_gbs = layer_bytes / (step_mean_ms * 1e-3) / 1e9

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5),
        "ms_per_step_median": round(statistics.median(step_ms), 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 indexer / bf16 attention, fp32 accumulate",
        "data": "synthetic (seeded; dyadic FP8 indexer operands, N(0,1) bf16 latent/q/gate)",
        "config": {"workload": case.name, "batch_per_gpu": B, "context": Lctx, "indexer_heads": case.HI,
                   "indexer_dim": case.DI, "top_k": case.K, "q_heads": case.H, "latent_dim": case.Dqk,
                   "value_dim": case.Dv, "page_size": case.page_size,
                   "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
                   "l2": "flushed between timed steps, outside the step events (256 MiB write, then a "
                         "256 MiB read so no dirty lines remain)"},
        "roofline": roofline,
        "layer_roofline": {"bound": "hbm", "algorithmic_bytes_per_step": layer_bytes,
                           "achieved": round(layer_gbs, 1), "peak": hbm, "unit": "GB/s",
                           "frac": round(layer_gbs / hbm, 4), "peak_spec": SPEC_HBM_GBS,
                           "frac_spec": round(layer_gbs / SPEC_HBM_GBS, 4)},
        "stages_us": {k: round(v, 2) for k, v in st.items()},
        "stages_note": f"separate steps with an event between stages (no overlap of kernel boundaries; "
                       f"{st_total:.2f} us per step there)",
        "gpu_launches": launches * args.steps,
        "gpu_launches_per_step": launches,
        "clocks": clk.summary(),
    }

    if not args.no_extras:
        res["e2e"] = e2e_leg(args, lay, flush, stream, _lib)
        if world == 1 and rank == 0:
            res["prefill_indexer"] = prefill_indexer_leg(args, flush, with_topk=True)
            res["append_kv"] = append_leg(args, flush, peaks)
            res["mtp_decode"] = mtp_leg(args, flush, case)
            res["cpu_baseline"], orc_idx, orc_out = cpu_baseline_leg(case)
            got_idx = lay.idx.cpu().numpy()
            got = lay.out.float().cpu().numpy().astype(np.float64)
            res["parity"] = {"idx_bit_exact": bool(np.array_equal(got_idx, orc_idx)),
                             "out_max_abs_err": float(np.abs(got - orc_out).max()),
                             "out_rel_fro_err": float(np.linalg.norm(got - orc_out) / np.linalg.norm(orc_out))}
            res.update(long_context_leg(args, flush, peaks))
            res["prefill_layer"] = prefill_layer_leg(args, flush, peaks)
            res["tiny_prefill"] = tiny_layer_leg(args, flush)
            res["mxfp8_decode"] = mx_leg(args, flush, peaks)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def e2e_leg(args, lay, flush, stream, _lib):
    """The decode step end to end through dsa_layer_forward: each step's inputs
    (qI, w, q, gate, seq_lens, in one pinned host buffer) go over in one copy
    and its output comes back to pinned host memory.  Pipelined as a serving
    loop runs it: two input and two output buffers; step i+1's upload (one
    copy stream) and step i-1's download (another) overlap step i's layer on
    the compute stream, ordered by events.  One event pair spans all K steps
    (on the download stream, after the last copy); every step streams its
    134 MB of keys and its gathered rows, more than the 126 MB L2, so nothing
    stays cached from step to step.  The unpipelined form (copy in, layer,
    copy out; L2 flushed between steps) is reported beside it."""
    import torch
    K = max(20, args.steps // 2)
    c = lay.case
    srcs = [lay.q_idx, lay.w, lay.q, lay.gate, lay.seq_lens]
    offs, off = [], 0
    for t in srcs:
        offs.append(off)
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    host_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    for t, o in zip(srcs, offs):
        nb = t.numel() * t.element_size()
        host_in[o:o + nb].copy_(t.reshape(-1).view(torch.uint8).cpu())
    bufs = []
    for _ in range(2):
        dev_in = torch.empty(off, dtype=torch.uint8, device="cuda")
        views = [dev_in[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(srcs, offs)]
        pg = _lib.paged(views[4], lay.block_table, c.num_pages, c.page_size)
        out = torch.empty_like(lay.out)
        a = _lib.layer_args(_lib.MODE_DECODE, views[0], views[1], lay.k_cache, views[2], lay.kv_cache, views[3], pg,
                            None, None, c.K, c.Dv, c.sm_scale, lay.max_len, out, lay.idx, None)
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        bufs.append((dev_in, a, out, host_out))
    d2h = bufs[0][3].numel() * bufs[0][3].element_size()

    # unpipelined: one step at a time, L2 flushed between steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K + 3)]
    dev_in, a, out, host_out = bufs[0]
    for s, e in ev:
        flush.zero_()
        s.record(stream)
        dev_in.copy_(host_in, non_blocking=True)
        _lib.layer_forward(a, lay.ws)
        host_out.copy_(out, non_blocking=True)
        e.record(stream)
    torch.cuda.synchronize()
    serial_ms = sum(s.elapsed_time(e) for s, e in ev[3:]) / K
    if not torch.equal(host_out, lay.out.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident run")

    # pipelined
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    copied_out = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run(n, timed):
        torch.cuda.synchronize()
        if timed:
            t0.record(up)
        for i in range(n + 1):
            if i < n:  # upload step i (its buffer is free once step i-2's layer is done)
                b = i & 1
                with torch.cuda.stream(up):
                    if i >= 2:
                        up.wait_event(done[b])
                    bufs[b][0].copy_(host_in, non_blocking=True)
                    in_ready[b].record(up)
                stream.wait_event(in_ready[b])
                if i >= 2:
                    stream.wait_event(copied_out[b])  # its output buffer has been read back
                _lib.layer_forward(bufs[b][1], lay.ws)
                done[b].record(stream)
            if i >= 1:  # download step i-1
                b = (i - 1) & 1
                with torch.cuda.stream(down):
                    down.wait_event(done[b])
                    bufs[b][3].copy_(bufs[b][2], non_blocking=True)
                    copied_out[b].record(down)
        if timed:
            up.wait_stream(down)
            t1.record(up)
        torch.cuda.synchronize()

    run(4, False)
    run(K, True)
    piped_ms = t0.elapsed_time(t1) / K
    if not torch.equal(bufs[(K - 1) & 1][3], lay.out.cpu()):
        raise RuntimeError("pipelined end-to-end output differs from the device-resident run")
    return {"value": round(c.T / (piped_ms / 1e3), 1), "unit": UNIT, "h2d_bytes_per_step": int(off),
            "d2h_bytes_per_step": d2h, "ms_per_step": round(piped_ms, 5),
            "note": "dsa_layer_forward in a pipelined loop: each step's inputs (qI, w, q, gate, seq_lens) one "
                    "pinned-host->device copy, its output device->pinned-host, uploads and downloads on their own "
                    "streams overlapping the neighbouring steps' layers; one event pair over all steps; caches "
                    "stay resident; per-step working set > L2",
            "serial": {"value": round(c.T / (serial_ms / 1e3), 1), "ms_per_step": round(serial_ms, 5),
                       "note": "copy in, layer, copy out, one step at a time, L2 flushed between steps"}}


def fp8_peak_tflops():
    """Dense e4m3 GEMM peak measured with torch._scaled_mm (8192^3, best of 10):
    a library measuring stick for the prefill indexer's roofline."""
    import torch
    n = 8192
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()
    one = torch.ones((), device="cuda")
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    best = float("inf")
    for _ in range(10):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e))
    return 2 * n ** 3 / (best * 1e-3) / 1e12


def mtp_leg(args, flush, case, n=4, steps=200):
    """Several query tokens per sequence (draft tokens of speculative
    decoding): the decode workload's caches, 4 queries per sequence at its
    last 4 positions, as explicit (sequence, position) queries through
    dsa_layer_forward.  Same timing rules as the headline."""
    import numpy as np
    import torch
    from long_context_sparse_02_b200 import synth
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    B = case.T
    q_seq = np.repeat(np.arange(B, dtype=np.int32), n)
    q_pos = case.seq_lens[q_seq] - n + np.tile(np.arange(n, dtype=np.int32), B)
    mc = synth.with_queries(case, args.seed + 13, q_seq, q_pos, f"mtp_B{B}x{n}_L{int(case.seq_lens.max())}")
    lay = LayerOnDevice(mc, decode=False)
    for _ in range(5):
        flush.zero_()
        lay.forward()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        flush.zero_()
        e0.record()
        lay.forward()
        e1.record()
    torch.cuda.synchronize()
    ms = sum(e0.elapsed_time(e1) for e0, e1 in ev)
    from long_context_sparse_02_b200 import _lib
    assert _lib.device_error(reset=True) == 0
    res = {"workload": mc.name, "queries_per_step": mc.T, "us_per_step": round(ms / steps * 1e3, 2),
           "tokens_per_s": round(mc.T * steps / (ms / 1e3), 1)}
    del lay
    torch.cuda.empty_cache()
    return res


def long_context_leg(args, flush, peaks, steps=100, which=("decode_1m", "hybrid")):
    """The layer's other decode workloads, timed like the headline (L2 flushed
    between steps, outside the events): one sequence of 1,048,576 tokens, and
    the hybrid serving step -- 64 sequences with lengths uniform in [4096,
    65536] through one DSA layer (16x128 indexer) and five sliding-window
    layers (64 heads x 128, window 128, each with its own K/V ring).  Each
    workload's failure is recorded in its own entry."""
    import torch
    from long_context_sparse_02_b200 import _lib, synth
    from long_context_sparse_02_b200.runtime import LayerOnDevice, to_dev
    hbm = float(peaks["hbm_gbs"])

    def ms_per_step(fn):
        for _ in range(5):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            flush.zero_()
            e0.record()
            fn()
            e1.record()
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps

    def hbm_roofline(nbytes, ms):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "algorithmic_bytes_per_step": nbytes, "achieved": round(gbs, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(gbs / hbm, 4), "peak_spec": SPEC_HBM_GBS,
                "frac_spec": round(gbs / SPEC_HBM_GBS, 4)}

    def stages(lay, K=50):
        """Stage split of the layer (separate steps, an event between stages)."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        for e4 in ev:
            for e in e4:
                e.record()  # creates the handle
        torch.cuda.synchronize()
        for e4 in ev:
            flush.zero_()
            lay.forward_profiled(e4)
        torch.cuda.synchronize()
        return {k: round(sum(e4[i].elapsed_time(e4[i + 1]) for e4 in ev) / K * 1e3, 2)
                for i, k in enumerate(["indexer", "topk", "attention"])}

    def device_ok(entry):
        err = _lib.device_error(reset=True)
        if err:
            entry["device_error"] = hex(err)
        return entry

    res = {}
    try:
        if "decode_1m" not in which:
            raise LookupError
        c1 = synth.decode_1m(args.seed)
        lay = LayerOnDevice(c1, decode=True)
        ms = ms_per_step(lay.forward)
        res["decode_1m"] = device_ok({"workload": c1.name, "us_per_step": round(ms * 1e3, 2),
                                      "tokens_per_s": round(c1.T / (ms * 1e-3), 1),
                                      "roofline": hbm_roofline(decode_bytes(c1)[0], ms),
                                      "stages_us": stages(lay)})
        del lay, c1
    except LookupError:
        pass
    except Exception as e:  # recorded, not raised: the headline line must still print
        res["decode_1m"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    torch.cuda.empty_cache()
    try:
        if "hybrid" not in which:
            raise LookupError
        hc = synth.hybrid_dsa(args.seed)
        lay = LayerOnDevice(hc, decode=True)
        sw = synth.swa_case(args.seed + 3, hc.seq_lens)
        q, seq_lens = to_dev(sw.q), to_dev(sw.seq_lens)
        k0, v0 = to_dev(sw.k_ring), to_dev(sw.v_ring)
        rings = [(k0, v0)] + [(k0.clone(), v0.clone()) for _ in range(4)]
        o = torch.empty_like(q)

        def swa(i=0):
            _lib.swa_decode(q, rings[i][0], rings[i][1], seq_lens, sw.window, sw.sm_scale, out=o)

        def group():
            lay.forward()
            for i in range(5):
                swa(i)

        B, H, D = sw.q.shape
        nbytes_swa = swa_bytes(B, H, D, sw.window, sw.seq_lens.min())
        dsa_ms, swa_ms, group_ms = ms_per_step(lay.forward), ms_per_step(swa), ms_per_step(group)
        res["hybrid"] = device_ok({
            "workload": f"{hc.name} + 5 x swa_B{B}_H{H}_D{D}_W{sw.window}",
            "dsa_layer": {"us_per_step": round(dsa_ms * 1e3, 2),
                          "roofline": hbm_roofline(decode_bytes(hc)[0], dsa_ms), "stages_us": stages(lay)},
            "swa_layer": {"us_per_step": round(swa_ms * 1e3, 2), "roofline": hbm_roofline(nbytes_swa, swa_ms)},
            "group_1_dsa_5_swa": {"us_per_step": round(group_ms * 1e3, 2),
                                  "tokens_per_s": round(B / (group_ms * 1e-3), 1)}})
        del lay, rings, k0, v0
    except LookupError:
        pass
    except Exception as e:
        res["hybrid"] = {"error": f"{type(e).__name__}: {e}"[:300]}
    torch.cuda.empty_cache()
    return res


def append_leg(args, flush, peaks):
    """The step before the layer: dsa_append_kv for a 32768-token prefill chunk
    (HBM-bound: per token 2*128 + 2*576 bytes read, 128 + 2*576 written) and for
    one decode step's 8 tokens (latency), into 128K-token paged caches."""
    import numpy as np
    import torch
    from long_context_sparse_02_b200 import _lib, synth
    from long_context_sparse_02_b200.runtime import to_dev
    DI, Dqk, L = 128, 576, 131072
    ss = np.random.SeedSequence(args.seed + 9).spawn(3)
    bt, npg = synth.paged_layout(np.random.default_rng(ss[0]), [L])
    pg = _lib.paged(to_dev(np.array([L], np.int32)), to_dev(bt), npg)
    k_cache = torch.zeros((npg, 64, DI), dtype=torch.uint8, device="cuda")
    kv_cache = torch.zeros((npg, 64, Dqk), dtype=torch.bfloat16, device="cuda")
    out = {}
    for name, n in (("prefill_chunk", 32768), ("decode_step", 8)):
        k_new = torch.randn((n, DI), device="cuda").to(torch.bfloat16)
        lat = torch.randn((n, Dqk), device="cuda").to(torch.bfloat16)
        tok_seq = torch.zeros(n, dtype=torch.int32, device="cuda")
        tok_pos = torch.arange(L - n, L, dtype=torch.int32, device="cuda")
        call = lambda: _lib.append_kv(k_new, 1.0, lat, tok_seq, tok_pos, pg, k_cache, kv_cache)  # noqa: E731
        for _ in range(3):
            call()
        us = []
        for _ in range(20):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            us.append(e0.elapsed_time(e1) * 1e3)
        t = statistics.median(us)
        nbytes = n * (2 * DI + 2 * Dqk + DI + 2 * Dqk)
        gbs = nbytes / (t * 1e-6) / 1e9
        out[name] = {"tokens": n, "us": round(t, 2), "bytes": nbytes, "GB/s": round(gbs, 1),
                     "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4)}
    assert _lib.device_error(reset=True) == 0
    del k_cache, kv_cache
    torch.cuda.empty_cache()
    return out


def prefill_indexer_leg(args, flush, T=32768, with_peak=True, with_topk=False):
    import numpy as np
    import torch
    from long_context_sparse_02_b200 import _lib, synth
    from long_context_sparse_02_b200.runtime import to_dev
    rng = np.random.default_rng(args.seed + 7)
    HI, DI = 16, 128
    ss = np.random.SeedSequence(args.seed + 7).spawn(3)
    bt, npg = synth.paged_layout(np.random.default_rng(ss[0]), [T])
    q_idx = to_dev(synth.dyadic_e4m3(np.random.default_rng(ss[1]), (T, HI, DI)))
    k_cache = to_dev(synth.dyadic_e4m3(np.random.default_rng(ss[2]), (npg, 64, DI)))
    w = to_dev(synth.dyadic_weights(rng, (T, HI)))
    seq_lens = to_dev(np.array([T], np.int32))
    pg = _lib.paged(seq_lens, to_dev(bt), npg)
    q_seq = torch.zeros(T, dtype=torch.int32, device="cuda")
    q_pos = torch.arange(T, dtype=torch.int32, device="cuda")
    scores = torch.empty((T, T), dtype=torch.float32, device="cuda")
    call = lambda: _lib.indexer_scores(q_idx, w, k_cache, pg, q_seq, q_pos, T, scores)  # noqa: E731
    for _ in range(3):
        call()
    ms = []
    for _ in range(10):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        call()
        e.record()
        torch.cuda.synchronize()
        ms.append(s.elapsed_time(e))
    t = statistics.median(ms)
    flops = prefill_indexer_flops(T, HI, DI)
    peak = fp8_peak_tflops() if with_peak else float("nan")
    tf = flops / (t * 1e-3) / 1e12
    res = {"workload": f"prefill_T{T}_indexer_{HI}x{DI}", "ms": round(t, 4), "tflops": round(tf, 1),
           "fp8_peak_tflops": round(peak, 1), "frac": round(tf / peak, 4), "bound": "tensor",
           "fp8_spec_tflops": SPEC_FP8_TFLOPS, "frac_spec": round(tf / SPEC_FP8_TFLOPS, 4),
           "peak_source": "measured in this run: torch._scaled_mm e4m3 8192^3, best of 10",
           "algorithmic_flops": flops}
    if with_topk:
        res["topk"] = prefill_topk_timing(flush, scores, q_pos, T)
    del scores
    torch.cuda.empty_cache()
    return res


def prefill_attn_flops(T, H, K, Dqk, Dv):
    """Attention over the selected rows, causal prefill: query t attends to
    min(K, t + 1) rows; 2*H*(Dqk + Dv) FLOP per (query, row)."""
    rows = sum(min(K, t + 1) for t in range(T))
    return 2.0 * H * (Dqk + Dv) * rows


def prefill_layer_leg(args, flush, peaks, T=32768, reps=3):
    """The whole prefill layer at T = 32768 (one sequence, 16x128 indexer,
    K = 2048, 128 heads over the 576-wide latent, gated) through
    dsa_layer_forward: layer time, its stage split, the attention alone
    (TFLOPS against the sustained bf16 peak), and the oracle's time for the
    same work extrapolated from timed rows.  Indexer operands are dyadic
    (numpy, seeded); q, the latent cache and the gate logits are N(0,1) bf16
    drawn on the device (seeded) to keep the run short.  A failure is
    recorded, not raised."""
    import numpy as np
    import torch
    from long_context_sparse_02_b200 import _lib, synth
    from long_context_sparse_02_b200.runtime import to_dev
    try:
        HI, DI, K, H, Dqk, Dv = 16, 128, 2048, 128, 576, 512
        ss = np.random.SeedSequence(args.seed + 21).spawn(4)
        bt, npg = synth.paged_layout(np.random.default_rng(ss[0]), [T])
        q_idx_np = synth.dyadic_e4m3(np.random.default_rng(ss[1]), (T, HI, DI))
        k_cache_np = synth.dyadic_e4m3(np.random.default_rng(ss[2]), (npg, 64, DI))
        w_np = synth.dyadic_weights(np.random.default_rng(ss[3]), (T, HI))
        gen = torch.Generator(device="cuda")
        gen.manual_seed(args.seed + 22)

        def randn(shape):
            t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
            flat = t.view(-1)
            for i in range(0, flat.numel(), 1 << 27):
                n = min(1 << 27, flat.numel() - i)
                flat[i:i + n] = torch.randn(n, dtype=torch.bfloat16, device="cuda", generator=gen)
            return t

        q, kv, gate = randn((T, H, Dqk)), randn((npg, 64, Dqk)), randn((T, H))
        q_idx, k_cache, w = to_dev(q_idx_np), to_dev(k_cache_np), to_dev(w_np)
        seq_lens = to_dev(np.array([T], np.int32))
        pg = _lib.paged(seq_lens, to_dev(bt), npg)
        q_seq = torch.zeros(T, dtype=torch.int32, device="cuda")
        q_pos = torch.arange(T, dtype=torch.int32, device="cuda")
        out = torch.empty((T, H, Dv), dtype=torch.bfloat16, device="cuda")
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        sm_scale = 1.0 / math.sqrt(Dqk)
        la = _lib.layer_args(_lib.MODE_PREFILL, q_idx.view(torch.uint8), w, k_cache.view(torch.uint8), q,
                             kv.view(torch.bfloat16), gate, pg, q_seq, q_pos, K, Dv, sm_scale, T, out, idx)
        ws = torch.zeros(_lib.layer_workspace_bytes(la), dtype=torch.uint8, device="cuda")

        def timed(fn, n):
            ms = []
            for _ in range(n):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                ms.append(e0.elapsed_time(e1))
            return statistics.median(ms)

        _lib.layer_forward(la, ws)
        layer_ms = timed(lambda: _lib.layer_forward(la, ws), reps)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for e in ev:
            e.record()
        flush.zero_()
        _lib.layer_forward_profiled(la, ws, ev)
        torch.cuda.synchronize()
        stages = {k: round(ev[i].elapsed_time(ev[i + 1]), 4) for i, k in enumerate(["indexer", "topk", "attention"])}
        attn_ms = timed(lambda: _lib.sparse_attn(q, kv, pg, q_seq, idx, gate, sm_scale, Dv, out=out), reps)
        flops = prefill_attn_flops(T, H, K, Dqk, Dv)
        tf = flops / (attn_ms * 1e-3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1400.0)))
        res = {"workload": f"prefill_T{T}_layer_{HI}x{DI}_K{K}_H{H}", "layer_ms": round(layer_ms, 3),
               "stages_ms": stages,
               "attention": {"ms": round(attn_ms, 3), "algorithmic_flops": flops, "tflops": round(tf, 1),
                             "peak": peak, "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                             "peak_source": "bf16_tflops_sustained, measured (MEASURED_PEAKS.json)"}}
        err = _lib.device_error(reset=True)
        if err:
            res["device_error"] = hex(err)
        # the oracle on a few rows, extrapolated by each stage's work
        from oracle import oracle
        rows = np.array([511, 4095, 16383, T - 1], np.int64)
        q_h = q[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
        g_h = gate[torch.from_numpy(rows).cuda()].view(torch.int16).cpu().numpy().view(np.uint16)
        kv_h = kv.view(torch.int16).cpu().numpy().view(np.uint16)
        opg = oracle.Paged(np.array([T], np.int32), bt, 64, npg)
        t0 = time.perf_counter()
        sc = oracle.indexer_scores(q_idx_np[rows], w_np[rows], k_cache_np, opg, np.zeros(len(rows), np.int32),
                                   rows.astype(np.int32), ld=T)
        t1 = time.perf_counter()
        sel = oracle.topk(sc, (rows + 1).astype(np.int32), K)
        t2 = time.perf_counter()
        oracle.sparse_attn(q_h, kv_h, opg, np.zeros(len(rows), np.int32), sel, g_h, sm_scale, Dv)
        t3 = time.perf_counter()
        keys_s, keys_all = float((rows + 1).sum()), T * (T + 1) / 2.0
        att_s, att_all = float(np.minimum(K, rows + 1).sum()), float(sum(min(K, t + 1) for t in range(T)))
        est = (t1 - t0) * keys_all / keys_s + (t2 - t1) * keys_all / keys_s + (t3 - t2) * att_all / att_s
        cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
        res["cpu_oracle_extrapolated"] = {"seconds": round(est, 1), "cores": cores, "kind": "oracle",
                                          "sample": f"rows {rows.tolist()} timed per stage, scaled by keys scored "
                                                    f"and rows attended", **host_cpu()}
        del q, kv, gate, out, idx, ws
        torch.cuda.empty_cache()
        return res
    except Exception as e:
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def mx_leg(args, flush, peaks, steps=100):
    """MXFP8 indexer operands at the headline's shape (8 x 131072, 32x128):
    the indexer alone against HBM (keys 128 B + 4 scale bytes per key read,
    4 B of score written, plus the queries and their scales) and the decode
    layer with them.  A failure is recorded, not raised."""
    import numpy as np
    import torch
    from long_context_sparse_02_b200 import _lib, synth
    from long_context_sparse_02_b200.runtime import LayerOnDevice, to_dev
    try:
        c = synth.decode_128k(args.seed + 31)
        r1, r2 = [np.random.default_rng(s) for s in np.random.SeedSequence(args.seed + 32).spawn(2)]
        c.q_idx, q_sc = synth.mx_dyadic(r1, c.q_idx.shape)
        c.k_cache, k_sc = synth.mx_dyadic(r2, c.k_cache.shape)
        lay = LayerOnDevice(c, decode=True)
        qs, ks = to_dev(q_sc), to_dev(k_sc)
        la = _lib.layer_args(_lib.MODE_DECODE, lay.q_idx, lay.w, lay.k_cache, lay.q, lay.kv_cache, lay.gate, lay.pg,
                             None, None, c.K, c.Dv, c.sm_scale, lay.max_len, lay.out, lay.idx, None, qs, ks)
        ws = torch.zeros(_lib.layer_workspace_bytes(la), dtype=torch.uint8, device="cuda")
        scores = torch.empty((c.T, lay.max_len), dtype=torch.float32, device="cuda")

        def timed(fn):
            for _ in range(5):
                flush.zero_()
                fn()
            tot = 0.0
            for _ in range(steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                tot += e0.elapsed_time(e1)
            return tot / steps

        idx_ms = timed(lambda: _lib.indexer_scores_mx(lay.q_idx, qs, lay.w, lay.k_cache, ks, lay.pg, None, None,
                                                      lay.max_len, scores))
        layer_ms = timed(lambda: _lib.layer_forward(la, ws))
        L, B, HI, DI = int(c.seq_lens[0]), c.T, c.HI, c.DI
        nbytes = B * L * (DI + DI // 32 + 4) + B * HI * (DI + DI // 32 + 4)
        gbs = nbytes / (idx_ms * 1e-3) / 1e9
        hbm = float(peaks["hbm_gbs"])
        res = {"workload": f"{c.name}_mxfp8",
               "indexer": {"us": round(idx_ms * 1e3, 2), "algorithmic_bytes": nbytes, "achieved_gbs": round(gbs, 1),
                           "peak": hbm, "frac_of_hbm": round(gbs / hbm, 4)},
               "layer": {"us_per_step": round(layer_ms * 1e3, 2), "tokens_per_s": round(B / (layer_ms * 1e-3), 1)}}
        err = _lib.device_error(reset=True)
        if err:
            res["device_error"] = hex(err)
        del lay, ws, scores
        torch.cuda.empty_cache()
        return res
    except Exception as e:
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def attn_only_leg(args, flush, T, L=32768, K=2048, H=128, Dqk=576, Dv=512, reps=5):
    """dsa_sparse_attn alone on the last T prefill queries of an L-token
    sequence, K selected causal rows each (seeded, uniform over the causal
    prefix), 128 heads over the 576-wide latent: TFLOPS over the algorithmic
    2 H (Dqk + Dv) K T.  For profiling the prefill attention kernel on a
    small case."""
    import torch
    from long_context_sparse_02_b200 import _lib
    g = torch.Generator(device="cuda")
    g.manual_seed(args.seed + 3)
    npg = L // 64
    bt = torch.randperm(npg, generator=g, device="cuda").to(torch.int32).view(1, -1)
    pg = _lib.paged(torch.tensor([L], dtype=torch.int32, device="cuda"), bt, npg)
    q = (torch.randn((T, H, Dqk), device="cuda", generator=g) * 0.1).to(torch.bfloat16)
    kv = torch.randn((npg, 64, Dqk), device="cuda", generator=g).to(torch.bfloat16)
    gate = torch.randn((T, H), device="cuda", generator=g).to(torch.bfloat16)
    pos = torch.arange(L - T, L, device="cuda")
    idx = torch.sort((torch.rand((T, K), device="cuda", generator=g) * (pos[:, None] + 1).float()).long(),
                     dim=1).values.to(torch.int32)
    q_seq = torch.zeros(T, dtype=torch.int32, device="cuda")
    out = torch.empty((T, H, Dv), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(_lib.sparse_attn_workspace_bytes(T, H, K, Dv), 1), dtype=torch.uint8, device="cuda")
    call = lambda: _lib.sparse_attn(q, kv, pg, q_seq, idx, gate, Dqk ** -0.5, Dv, out=out, ws=ws)  # noqa: E731
    for _ in range(2):
        call()
    ms = []
    for _ in range(reps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        call()
        e.record()
        torch.cuda.synchronize()
        ms.append(s.elapsed_time(e))
    t = statistics.median(ms)
    flops = 2.0 * H * (Dqk + Dv) * K * T  # every query has K >= 2048 causal rows to choose from
    res = {"workload": f"prefill_attn_T{T}_of_{L}_K{K}_H{H}", "ms": round(t, 4), "algorithmic_flops": flops,
           "tflops": round(flops / (t * 1e-3) / 1e12, 1)}
    err = _lib.device_error(reset=True)
    if err:
        res["device_error"] = hex(err)
    return res


def tiny_layer_leg(args, flush, reps=200):
    """The tiny prefill workload (T = 1024, 4x64 indexer, K = 128, 8 heads over
    a 64-wide latent): layer latency, L2 flushed between calls."""
    import torch
    from long_context_sparse_02_b200 import synth
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    c = synth.tiny_prefill(args.seed)
    lay = LayerOnDevice(c, decode=False)
    for _ in range(5):
        lay.forward()
    ms = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lay.forward()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    return {"workload": c.name, "us_per_call_median": round(statistics.median(ms) * 1e3, 2),
            "us_per_call_min": round(min(ms) * 1e3, 2)}


def prefill_topk_timing(flush, scores, q_pos, T, K=2048, reps=5):
    """dsa_topk over the T causal rows the prefill indexer just wrote (row t
    holds t + 1 scores): HBM-bound on the 4 * T(T+1)/2 bytes of scores read
    plus the T * K * 4 bytes of indices written.  A failure is recorded, not
    raised."""
    import torch
    from long_context_sparse_02_b200 import _lib
    try:
        row_len = q_pos + 1
        idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
        need = _lib.topk_workspace_bytes(T, K, T)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
        call = lambda: _lib.topk(scores, row_len, K, T, idx=idx, ws=ws)  # noqa: E731
        for _ in range(2):
            call()
        ms = []
        for _ in range(reps):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            call()
            e.record()
            torch.cuda.synchronize()
            ms.append(s.elapsed_time(e))
        t = statistics.median(ms)
        nbytes = prefill_topk_bytes(T, K)
        peaks, _ = load_peaks()
        gbs = nbytes / (t * 1e-3) / 1e9
        out = {"ms": round(t, 4), "algorithmic_bytes": nbytes, "achieved_gbs": round(gbs, 1),
               "frac_of_hbm": round(gbs / float(peaks["hbm_gbs"]), 4)}
        err = _lib.device_error(reset=True)
        if err:
            out["device_error"] = hex(err)
        return out
    except Exception as e:
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def host_cpu():
    """The host's CPU model and logical CPU count, recorded beside a CPU timing."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    if not model:
        import platform
        model = platform.processor() or platform.machine()
    return {"cpu_model": model, "host_cpus": os.cpu_count()}


def cpu_baseline_leg(case, min_seconds=10.0, max_steps=8):
    """The oracle as it stands on this host: whole decode steps of the workload
    (every sequence, full context, all heads), repeated until about
    min_seconds of CPU work have run (at most max_steps)."""
    import numpy as np
    from oracle import oracle
    pg = oracle.Paged(case.seq_lens, case.block_table, case.page_size, case.num_pages)
    steps, dt = 0, 0.0
    while steps < max_steps and (steps == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        _, idx, out = oracle.layer_forward(case.q_idx, case.w, case.k_cache, case.q, case.kv_cache, case.gate, pg,
                                           np.arange(case.T, dtype=np.int32), case.seq_lens - 1, case.K, case.Dv,
                                           case.sm_scale)
        dt += time.perf_counter() - t0
        steps += 1
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = int(os.environ.get("OMP_NUM_THREADS", cores))
    return ({"value": round(steps * case.T / dt, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
             "seconds": round(dt, 2), **host_cpu(),
             "sample": f"{steps} full decode steps of {case.name} ({case.T} sequences x {case.max_len} tokens, "
                       f"all heads) through oracle.c (fp64, OpenMP)"}, idx, out)


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    """--impl reference: the CPU oracle, as it stands, on this host's cores.
    Each step is a bounded sample of one decode token: 1/F of its keys and
    1/F of its heads (F a power of two sized so the run fits the budget);
    throughput is scaled back by F."""
    import numpy as np
    from long_context_sparse_02_b200 import synth
    from oracle import oracle
    rank, world, _ = dist_env()
    if rank != 0:
        return
    oracle.build()
    B, Lctx = args.batch, args.context

    def sample(F, seed):
        L = max(Lctx // F, 64)
        H = max(128 // F, 1)
        return synth.decode_case(seed, [L], HI=32, H=H, name=f"decode_1of{F}")

    def step(c):
        pg = oracle.Paged(c.seq_lens, c.block_table, c.page_size, c.num_pages)
        t0 = time.perf_counter()
        oracle.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, np.zeros(1, np.int32),
                             c.seq_lens - 1, c.K, c.Dv, c.sm_scale)
        return time.perf_counter() - t0

    probe = sample(16, args.seed)
    t16 = step(probe)
    per_step = args.ref_budget_s / max(1, args.steps + args.warmup)
    F = 1
    while F < 128 and t16 * 16 / F > per_step:
        F *= 2
    c = sample(F, args.seed)
    for _ in range(args.warmup):
        step(c)
    times = [step(c) for _ in range(args.steps)]
    total = sum(times)
    value = (args.steps / F) / total
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    sample_desc = (f"per step: one decode token with 1/{F} of its work -- {c.max_len} of {Lctx} keys through "
                   f"the 32x128 indexer and top-2048, {c.H} of 128 heads of attention; tokens/s scaled by 1/{F}")
    res = {"metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {"workload": f"decode_B{B}_L{Lctx}", "batch_per_gpu": B, "context": Lctx},
           "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                            "sample": sample_desc, **host_cpu()},
           "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def run_cp(args):
    """Context-parallel decode of one 1,048,576-token sequence over the N
    ranks: every rank holds the caches (it reads only its own pages), runs
    its local indexer and top-K, all-gathers the candidates, attends over the
    kept rows it holds, all-gathers (output, log-sum-exp) and merges.  The
    step time is the max over ranks of the CUDA-event time of K steps
    (the exchanges included); one token per step."""
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    from long_context_sparse_02_b200 import build, synth
    build.build()
    from long_context_sparse_02_b200 import _lib, cp
    from long_context_sparse_02_b200.runtime import to_dev
    c = synth.decode_1m(args.seed)
    k_cache, kv_cache = to_dev(c.k_cache), to_dev(c.kv_cache)
    q_idx, w, q, gate = to_dev(c.q_idx), to_dev(c.w), to_dev(c.q), to_dev(c.gate)
    rk = cp.CpRank(rank, world, c.seq_lens, c.block_table, c.num_pages, k_cache, kv_cache, c.K, c.Dv, c.sm_scale)
    if world > 1:
        ag = cp.torch_all_gather()
        step = lambda: cp.decode_step(rk, q_idx, w, q, gate, ag)  # noqa: E731
    else:
        step = lambda: cp.emulate([rk], q_idx, w, q, gate)  # noqa: E731
    flush = L2Flush()
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    total = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    if world > 1:
        torch.distributed.barrier()
    max_ms, _ = aggregate(total, args.steps, world)
    err = _lib.device_error(reset=True)
    res = {"metric": "context-parallel decode tokens/s, one 1,048,576-token sequence", "value":
           round(args.steps / (max_ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5), "higher_is_better": True,
           "scaling": "strong", "vs_baseline": None, "dtype": "e4m3 indexer / bf16 attention, fp32 accumulate",
           "data": "synthetic (seeded)", "config": {"workload": c.name, "parallelism": f"cp{world}",
                                                    "l2": "flushed between timed steps"},
           "device_error": err}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    a = parse_args()
    if a.impl == "reference":
        run_reference(a)
    elif a.workload == "cp_decode_1m":
        run_cp(a)
    elif a.prefill_only:
        import torch
        from long_context_sparse_02_b200 import build
        build.build()
        fl = L2Flush()
        print(json.dumps(prefill_indexer_leg(a, fl, T=a.prefill_only, with_peak=False, with_topk=a.with_topk)))
    elif a.attn_only:
        from long_context_sparse_02_b200 import build
        build.build()
        print(json.dumps(attn_only_leg(a, L2Flush(), a.attn_only)))
    elif a.hybrid_only:
        from long_context_sparse_02_b200 import build
        build.build()
        fl = L2Flush()
        print(json.dumps(long_context_leg(a, fl, load_peaks()[0], steps=a.steps, which=("hybrid",))))
    elif a.append_only:
        from long_context_sparse_02_b200 import build
        build.build()
        fl = L2Flush()
        print(json.dumps(append_leg(a, fl, load_peaks()[0])))
    else:
        run_native(a)
