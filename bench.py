#!/usr/bin/env python
"""Throughput of the FlashMemory DS-V4 retriever hot path on B200.

One step = the whole path for one batch of decode rows: query prep for all
three CSA layers, the fused scoring pass (3 layers + ensemble), and the top-K
keep-mask.  Default workload: B=64 rows x N=262144 chunks per layer (6.6 GB of
fp8 keys, larger than L2), max ensemble, top-4096, query prep timed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I]
    python bench.py --impl reference ...   # the CPU oracle on host cores

Multi-GPU (torchrun): every rank scores its own batch (weak scaling, no
collective on the data path); the time is the max over ranks.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gen import synthetic as G  # noqa: E402

METRIC = "retriever chunks scored/sec (3-layer ensemble + top-K)"
UNIT = "chunks/s"
NOMINAL_HBM_GBS = 8000.0  # the nominal HBM3e figure the target is stated against


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="4",
                    help="index of the synthetic workload (0-4), or 'all': one JSON line per workload")
    ap.add_argument("--q-pieces", type=int, default=2)
    ap.add_argument("--cta-pairs", type=int, default=0, choices=[0, 1],
                    help="scoring pass on CTA pairs (tcgen05 cta_group::2); 0 is the default form")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--shared-keys", action="store_true",
                    help="one compressed_k tensor scored by all three layers' queries (the README "
                         "Usage signature taken literally); reports against the fp8 tensor peak")
    ap.add_argument("--decode-rows", type=int, default=64,
                    help="--path decode: rows of the 262144-chunk workload (64 is the bench line; fewer "
                         "give a small case for profiling)")
    ap.add_argument("--path", default="retrieve", choices=["retrieve", "recall", "level2", "decode"],
                    help="retrieve: the scoring path (default); recall: keep mask -> index lists -> "
                         "gather of the kept chunks' records into a resident buffer; level2: the "
                         "per-step top-512 over a resident set of 4096 chunks per row, one CUDA graph; "
                         "decode: the toy sparse decode loop (retrieval every 64 steps, attention over the "
                         "kept chunks every step)")
    return ap.parse_args()


def scoring_kernel_sha1() -> str:
    """sha1 of the scoring kernel's device source: score_tc.cu followed by the
    device part of fm_internal.cuh (from its `#if defined(__CUDACC__)` line)."""
    import hashlib
    src = os.path.join(ROOT, "learned_kv_chunk_b200", "csrc")
    m = hashlib.sha1()
    m.update(open(os.path.join(src, "score_tc.cu"), "rb").read())
    header = open(os.path.join(src, "fm_internal.cuh"), "rb").read()
    m.update(header[header.index(b"#if defined(__CUDACC__)"):])
    return m.hexdigest()


def recorded_traffic(decisions: int):
    """DRAM bytes per scoring launch from the committed ncu counters
    (profiles/score_kernel_B8xN65536.json), scaled to this launch's decisions;
    None once the kernel source differs from the one they were taken on."""
    try:
        with open(os.path.join(ROOT, "profiles", "score_kernel_B8xN65536.json")) as f:
            rec = json.load(f)
        if rec["kernel_source_sha1"] != scoring_kernel_sha1():
            return None
        return int(float(rec["traffic_bytes_per_decision"]) * decisions)
    except Exception:
        return None


def fp8_tensor_peak():
    """Dense fp8 tensor peak: the measured cuBLAS bf16 burst figure times the
    nominal fp8/bf16 ratio (2)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 x 2 (nominal fp8/bf16 ratio)"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


def bf16_tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s): the measured cuBLAS burst figure."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while running."""

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[device_index]) if vis else device_index
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((mhz, reasons, util))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        nv = self.nv
        names = {
            "gpu_idle": nv.nvmlClocksEventReasonGpuIdle,
            "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap,
            "hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
            "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
            "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
            "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
            "applications_clocks_setting": nv.nvmlClocksEventReasonApplicationsClocksSetting,
        }
        loaded = [s for s in self.samples if s[2] > 0] or self.samples
        seen = set()
        for _, r, _ in loaded:
            for n, bit in names.items():
                if r & bit and n != "gpu_idle":
                    seen.add(n)
        return {"sm_mhz": float(statistics.median(s[0] for s in loaded)),
                "sm_max_mhz": float(self.max_mhz), "reasons": sorted(seen),
                "samples": len(loaded)}


# ------------------------------------------------------- multi-rank helpers
# Weak scaling: every rank scores its own batch of the workload (its own keys,
# drawn from a rank-specific seed); the only collectives are the timing
# reductions below, outside the timed region's data path.
def rank_key_seed(base_seed: int, rank: int) -> int:
    return base_seed + 7919 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest `value` over all ranks (every rank gets it)."""
    t = torch.tensor([value], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(decisions_per_rank: int, world: int, steps: int, elapsed_max_ms: float) -> float:
    """Whole-job decisions per second: all ranks' work over the slowest rank's time."""
    return decisions_per_rank * world * steps / (elapsed_max_ms / 1e3)


# -------------------------------------------------------------- our arm
def run_ours(args, wl, rank, world, local_rank):
    from learned_kv_chunk_b200 import fm

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp = G.make_query_inputs(wl)
    B, N, L = wl.B, wl.N, G.N_LAYERS
    r = fm.Retriever(inp.weights, device=local_rank, max_batch=max(64, B), q_pieces=args.q_pieces,
                     cta_pairs=args.cta_pairs)
    hidden = inp.hidden.to(dev)
    positions = inp.positions.to(dev)
    n_valid = inp.n_valid.to(dev)
    q, w = r.fm_query_prep(hidden, positions)
    plant = q[:, :, 0, :].permute(1, 0, 2).contiguous().cpu()
    if args.shared_keys:
        keys = G.make_keys(rank_key_seed(wl.seed(G.SEED_KEYS), rank), [int(x) for x in inp.n_valid], N, 1,
                           plant[:1], device=dev) * L
    else:
        keys = G.make_keys(rank_key_seed(wl.seed(G.SEED_KEYS), rank), [int(x) for x in inp.n_valid], N, L,
                           plant, device=dev)
    torch.cuda.synchronize()
    decisions = int(inp.n_valid.sum())          # valid (row, chunk) pairs per step
    key_layers = 1 if args.shared_keys else L
    key_bytes = key_layers * decisions * G.RECORD_BYTES  # valid records only

    ens = torch.empty(B, N, device=dev, dtype=torch.float32)
    keep = torch.empty(B, N, device=dev, dtype=torch.bool)
    keep_thr = torch.empty(B, N, device=dev, dtype=torch.bool) if wl.threshold is not None else None
    ws = torch.empty(fm.fm_topk_workspace_bytes_fast(B, N), device=dev, dtype=torch.uint8)
    qb = torch.empty(B, L, 64, 128, device=dev)
    wb = torch.empty(B, L, 64, device=dev)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = key_bytes < 4 * l2
    flush_buf = torch.empty(max(2 * l2, 1 << 28) // 4, device=dev, dtype=torch.float32) if flush else None

    ev_sc = []  # per timed step: events before prep, before scoring, after scoring, after top-K

    def step(timed=False):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if timed else None
        if timed:
            ev[0].record(stream)
        r.fm_query_prep(hidden, positions, q=qb, fused_w=wb)
        if timed:
            ev[1].record(stream)
        r.fm_score_fused(keys, qb, wb, mode=wl.mode, threshold=wl.threshold, n_valid=n_valid, N=N,
                         ens=ens, keep_thr=keep_thr)
        if timed:
            ev[2].record(stream)
        fm.fm_select_topk(ens, wl.top_k, n_valid, out=keep, workspace=ws)
        if timed:
            ev[3].record(stream)
            ev_sc.append(ev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    r.fm_sync_status()

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    launches0 = fm.fm_launch_count()
    with sampler:
        barrier()
        if not flush:
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                step(timed=True)
            t1.record(stream)
            torch.cuda.synchronize()
            elapsed_ms = t0.elapsed_time(t1)
        else:
            elapsed_ms = 0.0
            for _ in range(args.steps):
                flush_l2(flush_buf)
                t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                t0.record(stream)
                step(timed=True)
                t1.record(stream)
                torch.cuda.synchronize()
                elapsed_ms += t0.elapsed_time(t1)
        barrier()
    launches = fm.fm_launch_count() - launches0
    r.fm_sync_status()
    score_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in ev_sc]))
    stages_ms = {"query_prep": round(float(np.mean([e[0].elapsed_time(e[1]) for e in ev_sc])), 4),
                 "scoring_pass": round(score_ms, 4),
                 "topk": round(float(np.mean([e[2].elapsed_time(e[3]) for e in ev_sc])), 4)}

    elapsed_max = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = elapsed_max / args.steps
    value = job_throughput(decisions, world, args.steps, elapsed_max)

    hbm_peak, peak_kind = peaks()
    alg_bytes = decisions * (key_layers * G.RECORD_BYTES + 4)  # keys + ensembled score per decision
    achieved = alg_bytes / (score_ms / 1e3) / 1e9
    if not args.shared_keys:
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(achieved / hbm_peak, 4), "traffic": recorded_traffic(decisions),
                    "frac_of_nominal_8000": round(achieved / NOMINAL_HBM_GBS, 4),
                    "kernel": "score_kernel (fused scoring pass, via fm_score_fused)",
                    "kernel_ms": round(score_ms, 4), "peak_kind": peak_kind,
                    "alg_bytes_per_launch": alg_bytes}
    else:
        # one key read feeds three layers' products: 16384 MMA FLOP per record and layer
        flops = decisions * L * 2 * 128 * 64
        fp8_peak, fp8_kind = fp8_tensor_peak()
        ach_tf = flops / (score_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(ach_tf, 1), "peak": fp8_peak, "unit": "TFLOP/s",
                    "frac": round(ach_tf / fp8_peak, 4), "traffic": None,
                    "kernel": "score_kernel (fused scoring pass, one key tensor for all layers)",
                    "kernel_ms": round(score_ms, 4), "peak_kind": fp8_kind,
                    "alg_flops_per_launch": flops, "hbm_alg_bytes_per_launch": alg_bytes,
                    "hbm_achieved_gbs": round(achieved, 1), "hbm_frac": round(achieved / hbm_peak, 4)}

    # end to end through the C ABI's host-buffer call: H2D of the step's inputs, D2H of the masks
    e2e = None
    if not args.no_e2e and not args.shared_keys:
        hk = [k.cpu().pin_memory() for k in keys]
        hh, hp, hn = hidden.cpu().pin_memory(), positions.cpu().pin_memory(), inp.n_valid.pin_memory()
        bufs = {}
        r.retrieve_from_host(hh, hp, hk, hn, wl.mode, wl.top_k, wl.threshold, N, bufs)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            kt, kh = r.retrieve_from_host(hh, hp, hk, hn, wl.mode, wl.top_k, wl.threshold, N, bufs)
        e1.record(stream)
        torch.cuda.synchronize()
        et_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
        h2d = sum(k.numel() for k in hk) + hh.numel() * 4 + hp.numel() * 8 + hn.numel() * 4
        d2h = B * N * (2 if wl.threshold is not None else 1)
        e2e = {"value": job_throughput(decisions, world, args.e2e_steps, et_max), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps,
               "call": "fm_retrieve_host (C ABI): pinned host inputs in, host masks out, one step per call"}
        del hk
        # the serving reading: the compressed keys stay resident on the GPU (the
        # model card keeps the indexer keys there), so a step's host inputs are
        # the hidden states, positions and valid lengths, and its output the masks
        dh, dp, dn = torch.empty_like(hidden), torch.empty_like(positions), torch.empty_like(n_valid)
        hm = torch.empty(B, N, dtype=torch.bool).pin_memory()
        hmt = torch.empty(B, N, dtype=torch.bool).pin_memory() if wl.threshold is not None else None

        def resident_step():
            dh.copy_(hh, non_blocking=True)
            dp.copy_(hp, non_blocking=True)
            dn.copy_(hn.to(torch.int32), non_blocking=True)
            _, kt2, kthr2 = r.retrieve(dh, keys, dp, dn, wl.mode, wl.top_k, wl.threshold, N)
            hm.copy_(kt2, non_blocking=True)
            if hmt is not None:
                hmt.copy_(kthr2, non_blocking=True)

        for _ in range(3):
            resident_step()
        barrier()
        steps_r = max(args.e2e_steps, 20)
        e0.record(stream)
        for _ in range(steps_r):
            resident_step()
        e1.record(stream)
        torch.cuda.synchronize()
        rt_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e["resident_keys"] = {
            "value": job_throughput(decisions, world, steps_r, rt_max), "unit": UNIT,
            "h2d_bytes_per_step": int(hh.numel() * 4 + hp.numel() * 8 + hn.numel() * 4),
            "d2h_bytes_per_step": int(d2h), "steps": steps_r,
            "call": "Retriever.retrieve with device-resident keys: pinned host hidden states, positions and "
                    "valid lengths in, host masks out, every step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_sample(inp, keys, wl, q_row=0)
        if wl.index == 0:  # the small workload's oracle is also timed on one core
            try:
                import threadpoolctl
                with threadpoolctl.threadpool_limits(1):
                    one = cpu_baseline_sample(inp, keys, wl, q_row=0)
                cpu["single_thread"] = {"value": one["value"], "unit": UNIT, "cores": 1,
                                        "sample": one["sample"]}
            except Exception as e:  # noqa: BLE001
                cpu["single_thread"] = {"unavailable": str(e)}

    r.close()
    return dict(value=value, ms_per_step=ms_per_step, roofline=roofline, e2e=e2e, cpu=cpu,
                clocks=sampler.summary(), launches=launches, decisions=decisions, flush=flush,
                key_bytes=key_bytes, stages_ms=stages_ms)


# ------------------------------------------------------------ recall path
def flush_l2(flush_buf):
    """Flushes L2: writes a buffer of at least twice its size, then reads it back, so the
    timed work starts with a cold L2 that holds no dirty lines (the write-back
    of the flush's own lines is not charged to the timed kernels)."""
    flush_buf.fill_(1.0)
    flush_buf.sum()


def _timed_flushed(fn, steps, flush_buf, stream):
    """Mean CUDA-event time (ms) of fn() over `steps` calls, L2 flushed before each."""
    total = 0.0
    for _ in range(steps):
        flush_l2(flush_buf)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    return total / steps


def run_recall(args):
    """Keep mask -> index lists -> the kept chunks' records gathered into a
    resident buffer, on the top-4096 masks of 64 rows x 262144 chunks.  The
    records are 132 bytes (the compressed_k record, the one chunk record size
    the pages define); the source is device memory or pinned host memory."""
    from learned_kv_chunk_b200 import fm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, N, K, rec = 64, 262144, 4096, 132
    g = torch.Generator(device=dev).manual_seed(2024)
    ens = torch.rand(B, N, device=dev, generator=g)
    keep = fm.fm_select_topk(ens, K)
    src_dev = torch.randint(0, 256, (B, N, rec), device=dev, dtype=torch.uint8, generator=g)
    src_host = src_dev.cpu().pin_memory()
    idx = torch.empty(B, K, device=dev, dtype=torch.int32)
    count = torch.empty(B, device=dev, dtype=torch.int32)
    ws = torch.empty(int(fm.lib().fm_compact_workspace_bytes(B, N)), device=dev, dtype=torch.uint8)
    dst = torch.empty(B, K, rec, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 1 << 28) // 4, device=dev, dtype=torch.float32)

    def compact():
        fm.fm_compact_mask(keep, K, idx=idx, count=count, workspace=ws)

    def step_dev():
        compact()
        fm.fm_gather_records(src_dev, idx, count, dst)

    def gather_host():
        fm.fm_gather_records(src_host, idx, count, dst)

    for _ in range(max(3, args.warmup)):
        step_dev()
        gather_host()
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    launches0 = fm.fm_launch_count()
    with sampler:
        t_step = _timed_flushed(step_dev, args.steps, flush_buf, stream)
        t_compact = _timed_flushed(compact, args.steps, flush_buf, stream)
        t_host = _timed_flushed(gather_host, max(3, args.steps // 10), flush_buf, stream)
    launches = fm.fm_launch_count() - launches0
    # the same gather by torch's own indexing kernel (records as 33 int32 words),
    # for the rate a library gather reaches on this access pattern
    flat = (idx.to(torch.int64) + torch.arange(B, device=dev, dtype=torch.int64)[:, None] * N).view(-1)
    words = src_dev.view(B * N, rec).view(torch.int32)
    t_torch = _timed_flushed(lambda: torch.index_select(words, 0, flat), args.steps, flush_buf, stream)
    # the bus: one pinned host -> device copy of 256 MB with the copy engine, same run
    hbuf = torch.empty(1 << 28, dtype=torch.uint8).pin_memory()
    dbuf = torch.empty(1 << 28, dtype=torch.uint8, device=dev)
    dbuf.copy_(hbuf, non_blocking=True)
    t_h2d = _timed_flushed(lambda: dbuf.copy_(hbuf, non_blocking=True), 5, flush_buf, stream)
    h2d_gbs = (1 << 28) / (t_h2d / 1e3) / 1e9

    torch.cuda.synchronize()
    assert int(count.min()) == K
    sel = B * K
    alg_dev = B * N + sel * 4 + B * 4 + 2 * sel * rec  # mask once, index list, count, records in + out
    hbm_peak, peak_kind = peaks()
    ach = alg_dev / (t_step / 1e3) / 1e9
    host_gbs = sel * rec / (t_host / 1e3) / 1e9
    out = {"metric": "resident-set records recalled/sec (mask -> index list -> gather)",
           "value": sel / (t_step / 1e3), "unit": "records/s", "n_gpus": 1, "steps": args.steps,
           "warmup": max(3, args.warmup), "ms_per_step": t_step, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic (seeded)",
           "config": {"workload": "recall_B64_N262144_top4096_rec132", "rows": B, "chunks_per_row": N,
                      "kept_per_row": K, "record_bytes": rec, "source": "device memory",
                      "l2": "flushed between steps (256 MB written, then read back)"},
           "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                        "frac": round(ach / hbm_peak, 4), "traffic": None, "peak_kind": peak_kind,
                        "kernel": "compaction (2 kernels) + gather, one step",
                        "alg_bytes_per_step": alg_dev},
           "compact_ms": round(t_compact, 4),
           "gather_ms": round(t_step - t_compact, 4),
           "torch_index_select_ms": round(t_torch, 4),
           "host_source": {"value": sel / (t_host / 1e3), "unit": "records/s", "gather_ms": round(t_host, 4),
                           "achieved_gbs": round(host_gbs, 2),
                           "h2d_copy_gbs": round(h2d_gbs, 2),
                           "frac_of_h2d_copy": round(host_gbs / h2d_gbs, 4),
                           "note": "records read from pinned host memory by the kernel over the bus; "
                                   "denominator: a 256 MB pinned host-to-device copy in the same run"},
           "gpu_launches": launches, "clocks": sampler.summary(),
           "cpu_baseline": recall_oracle_sample(keep, src_dev, K)}
    return out


def run_recall_reference(args):
    """--path recall --impl reference: the recall oracle on host cores, one
    row of the workload per step."""
    g = torch.Generator().manual_seed(2024)
    B, N, K, rec = 64, 262144, 4096, 132
    keep = torch.zeros(1, N, dtype=torch.bool)
    keep[0, torch.randperm(N, generator=g)[:K]] = True
    src = torch.randint(0, 256, (1, N, rec), generator=g, dtype=torch.uint8)
    for _ in range(args.warmup):
        recall_oracle_sample(keep, src, K)
    vals = [recall_oracle_sample(keep, src, K) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    return {"impl": "reference", "metric": "resident-set records recalled/sec (mask -> index list -> gather)",
            "value": v, "unit": "records/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": K / v * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u8", "data": "synthetic (seeded)",
            "config": {"workload": "recall_B64_N262144_top4096_rec132", "rows": B, "chunks_per_row": N,
                       "kept_per_row": K, "record_bytes": rec},
            "cpu_baseline": dict(vals[0], value=v),
            "e2e": {"value": v, "unit": "records/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------ level-2 path
def run_level2(args):
    """The per-step selection over the resident set (one CUDA graph launch per
    decode step): 64 rows, 4096 resident chunks per row (the recalled top-4096
    of 262144), top-512.  Resident records come from the seeded key generator;
    each step reads the 154 MB of query weights and the 104 MB of resident
    keys, and L2 is flushed before each step (the rest of a decode step would
    evict it)."""
    from learned_kv_chunk_b200 import fm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B, R, k, N1 = 64, 4096, 512, 262144
    weights = G.make_weights(5000, G.N_LAYERS)
    r = fm.Retriever(weights, device=0, max_batch=B, q_pieces=args.q_pieces)
    g = torch.Generator().manual_seed(5001)
    ids = torch.stack([torch.randperm(N1, generator=g)[:R].sort().values for _ in range(B)]).to(torch.int32)
    res_keys = G.make_keys(5002, [R] * B, R, G.N_LAYERS, None, device=dev)
    res_ids = ids.to(dev)
    count = torch.full((B,), R, dtype=torch.int32, device=dev)
    step = fm.Level2Step(r, res_keys, res_ids, count, k=k, mode="max")
    step.hidden.copy_(G.make_hidden(5003, B).to(dev))
    step.positions.copy_(torch.full((B,), 4 * N1, dtype=torch.int64).to(dev))
    stream = torch.cuda.current_stream()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 1 << 28) // 4, device=dev, dtype=torch.float32)
    for _ in range(max(3, args.warmup)):
        step.launch()
    torch.cuda.synchronize()
    r.fm_sync_status()
    sampler = ClockSampler(0)
    with sampler:
        t_step = _timed_flushed(step.launch, args.steps, flush_buf, stream)
    r.fm_sync_status()
    assert int(step.out_count.min()) == k
    cfg = r.cfg
    L, HID, RK, H, D = G.N_LAYERS, cfg.hidden, cfg.q_lora_rank, cfg.n_heads, cfg.head_dim
    w_bytes = 4 * L * ((RK + H) * HID + H * D * RK)
    alg = w_bytes + B * HID * 4 + B * R * (L * G.RECORD_BYTES + 4) + B * R * 4 * 3 + B * R + B * k * 8
    hbm_peak, peak_kind = peaks()
    ach = alg / (t_step / 1e3) / 1e9
    step.close()
    r.close()
    return {"metric": "level-2 resident chunks scored/sec (per-step top-512, CUDA graph)",
            "value": B * R / (t_step / 1e3), "unit": "chunks/s", "n_gpus": 1, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3", "data": "synthetic (seeded generator, random-init weights)",
            "config": {"workload": "level2_B64_R4096_top512", "rows": B, "resident_per_row": R, "top_k": k,
                       "layers": L, "ensemble": "max", "query_prep_in_step": True,
                       "l2": "flushed between steps (256 MB written, then read back)"},
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(ach / hbm_peak, 4), "traffic": None, "peak_kind": peak_kind,
                         "kernel": "the whole step (one graph: query prep, scoring, top-k, compaction, id map)",
                         "alg_bytes_per_step": int(alg)},
            "gpu_launches_per_step": "one graph launch", "clocks": sampler.summary()}


# -------------------------------------------------------------- decode path
def run_decode(args):
    """The README's toy decode loop on the 64-row workload (64 rows x 262144
    chunks per layer, top-4096): one timed unit is a retrieval cycle, i.e. 64
    decode steps of which the first runs the retriever over all chunks; every
    step runs the sparse attention over the 4096 kept chunks and the state
    update.  The attention kernel is also timed alone (L2 flushed first)."""
    from learned_kv_chunk_b200 import fm

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = G.WORKLOADS[4]
    if args.decode_rows != wl.B:
        import dataclasses
        wl = dataclasses.replace(wl, B=int(args.decode_rows))
    inp = G.make_query_inputs(wl)
    B, N, L, K = wl.B, wl.N, G.N_LAYERS, wl.top_k
    r = fm.Retriever(inp.weights, device=0, max_batch=B, q_pieces=args.q_pieces)
    hidden = inp.hidden.to(dev)
    q, _ = r.fm_query_prep(hidden, inp.positions.to(dev))
    plant = q[:, :, 0, :].permute(1, 0, 2).contiguous().cpu()
    keys = G.make_keys(wl.seed(G.SEED_KEYS), [int(x) for x in inp.n_valid], N, L, plant, device=dev)
    n_valid = inp.n_valid.to(dev)
    dec = fm.ToySparseDecoder(r, keys, n_valid, hidden, inp.positions, top_k=K, mode=wl.mode)
    stream = torch.cuda.current_stream()
    interval = dec.interval
    for _ in range(max(3, args.warmup)):
        dec.step()
    while dec.t % interval:
        dec.step()
    torch.cuda.synchronize()
    r.fm_sync_status()
    cycles = max(1, args.steps // interval) if args.steps >= interval else 1
    sampler = ClockSampler(0)
    launches0 = fm.fm_launch_count()
    with sampler:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(cycles * interval):
            dec.step()
        b.record(stream)
        torch.cuda.synchronize()
        t_cycle = a.elapsed_time(b) / cycles
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        flush_buf = torch.empty(max(2 * l2, 1 << 28) // 4, device=dev, dtype=torch.float32)
        ws = torch.empty(int(fm.lib().fm_decode_attention_workspace_bytes(B, K)), device=dev, dtype=torch.uint8)
        out = torch.empty(B, 32, 128, device=dev)
        t_attn = _timed_flushed(dec.attend, 20, flush_buf, stream)
    launches = fm.fm_launch_count() - launches0
    r.fm_sync_status()
    kept = int(dec.count.clamp(max=K).sum())
    flops = kept * 32 * 128 * 4  # q.x and p.x: one multiply-add each per (chunk, head, dim)
    # the kept records once (the resident buffer), the query in, the output out
    attn_bytes = kept * G.RECORD_BYTES + 2 * B * 32 * 128 * 4
    hbm_peak, peak_kind = peaks()
    ach = attn_bytes / (t_attn / 1e3) / 1e9
    tc_frac = flops / (t_attn / 1e3) / 1e12 / bf16_tensor_peak()
    r.close()
    return {"metric": "toy sparse decode tokens/sec (retrieval every 64 steps, attention over kept chunks)",
            "value": B * interval / (t_cycle / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": cycles * interval,
            "warmup": max(3, args.warmup), "ms_per_step": t_cycle / interval, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16 pieces, f32 accumulate (attention), e4m3 (retrieval)",
            "data": "synthetic (seeded generator, random-init weights)",
            "config": {"workload": f"decode_B{B}_N262144_top4096_interval64", "rows": B, "chunks_per_row": N,
                       "kept_per_row": K, "retrieval_interval": interval, "attention_heads": 32,
                       "l2": "cycle inputs larger than L2 (6.64 GB of keys per retrieval); attention timed "
                             "alone after a 256 MB L2 flush"},
            "cycle_ms": round(t_cycle, 4),
            "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(ach / hbm_peak, 4), "traffic": None, "peak_kind": peak_kind,
                         "kernel": "sparse attention over the resident kept records (segments on tcgen05 + "
                                   "combine), L2 flushed before each launch",
                         "kernel_ms": round(t_attn, 4), "alg_bytes_per_launch": attn_bytes,
                         "alg_flops_per_launch": flops,
                         "tensor_frac_of_bf16_peak": round(tc_frac, 4)},
            "gpu_launches": launches, "clocks": sampler.summary()}


def recall_oracle_sample(keep, src, K, rows=1):
    """The recall oracle (compaction + gather, plain loops) on the first rows."""
    import oracle.recall as OR
    km = keep[:rows].cpu().numpy()
    sm = src[:rows].cpu().numpy()
    t0 = time.perf_counter()
    idx, cnt = OR.compact_mask(km, K)
    OR.gather_records(sm, idx, cnt, np.zeros((rows, K, sm.shape[2]), np.uint8))
    dt = time.perf_counter() - t0
    return {"value": rows * K / dt, "unit": "records/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows} row(s) of the workload: compaction of {km.shape[1]} mask bytes and "
                      f"gather of {K} records ({dt:.2f} s)"}


def _oracle_threads():
    try:
        import threadpoolctl
        return max(i["num_threads"] for i in threadpoolctl.threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


def cpu_baseline_sample(inp, keys, wl, q_row=0):
    """The CPU oracle, as it stands, on one row of the workload (all chunks,
    3 layers, query prep, ensemble, top-K)."""
    import oracle.retriever as O
    b = q_row
    n = int(inp.n_valid[b])
    layers = [{k: v.numpy().astype(np.float64) for k, v in w_.items()} for w_ in inp.weights]
    host = [k[b, :n].cpu().numpy() for k in keys]
    h = inp.hidden[b:b + 1].numpy().astype(np.float64)
    pos = inp.positions[b:b + 1].numpy()
    t0 = time.perf_counter()
    qw = [O.query_prep(l, h, pos) for l in layers]
    s = np.stack([O.score_chunks(host[l], qw[l][0][0], qw[l][1][0]) for l in range(len(layers))])
    e = O.ensemble(s, wl.mode)[None]
    O.select_topk(e, np.array([n]), wl.top_k)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
            "cpu_model": _cpu_model(), "host_cpus": len(os.sched_getaffinity(0)),
            "sample": f"row {b} of the workload: {n} chunks x 3 layers, query prep, ensemble, "
                      f"top-{wl.top_k} ({dt:.1f} s)"}


# ---------------------------------------------------------- reference arm
def run_reference(args, wl):
    """The CPU oracle on the host cores: each step scores a bounded sample
    (one row's query prep + 8192 chunks x 3 layers + ensemble + top-K)."""
    import oracle.retriever as O
    inp = G.make_query_inputs(wl)
    layers = [{k: v.numpy().astype(np.float64) for k, v in w_.items()} for w_ in inp.weights]
    M = min(8192, wl.N)
    samples = []
    for s in range(2):
        b = s % wl.B
        h = inp.hidden[b:b + 1].numpy().astype(np.float64)
        pos = inp.positions[b:b + 1].numpy()
        keys = [G.make_key_slab(wl.seed(G.SEED_KEYS), l, b, M, None).numpy() for l in range(3)]
        samples.append((h, pos, keys))

    def step(i):
        h, pos, keys = samples[i % len(samples)]
        qw = [O.query_prep(l, h, pos) for l in layers]
        sc = np.stack([O.score_chunks(keys[l], qw[l][0][0], qw[l][1][0]) for l in range(3)])
        e = O.ensemble(sc, wl.mode)[None]
        O.select_topk(e, np.array([M]), min(wl.top_k, M))

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = M * args.steps / dt
    cores = _oracle_threads()
    sample = f"per step: one row's query prep + {M} chunks x 3 layers + ensemble + top-{min(wl.top_k, M)}"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, args.gpus),
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample, "value": value,
                             "unit": UNIT},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_of(wl, gpus, flush=None, key_bytes=None, shared_keys=False, cta_pairs=0):
    c = {"workload": wl.name + ("_shared_keys" if shared_keys else ""), "global_batch": wl.B * gpus, "chunks_per_row": wl.N, "layers": 3,
         "ensemble": wl.mode, "top_k": wl.top_k, "threshold": wl.threshold,
         "query_prep_in_step": True, "parallelism": f"rows sharded over {gpus} GPU(s), no collective"}
    if cta_pairs:
        c["scoring_form"] = "CTA pairs (tcgen05 cta_group::2)"
    if flush is not None:
        c["l2"] = ("flushed between steps (256 MB written, then read back)" if flush
                   else f"inputs larger than L2 ({key_bytes / 1e9:.2f} GB of keys per step)")
    return c


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.path == "decode":
        if rank == 0:
            print(json.dumps(run_decode(args)), flush=True)
        return
    if args.path == "level2":
        if rank == 0:
            print(json.dumps(run_level2(args)), flush=True)
        return
    if args.path == "recall":
        if rank == 0:
            print(json.dumps(run_recall_reference(args) if args.impl == "reference" else run_recall(args)),
                  flush=True)
        return
    wls = G.WORKLOADS if args.workload == "all" else [G.WORKLOADS[int(args.workload)]]
    if args.impl == "reference":
        if rank == 0:
            for wl in wls:
                print(json.dumps(run_reference(args, wl)), flush=True)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        for wl in wls:
            res = run_ours(args, wl, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(result_line(args, wl, world, res)), flush=True)
            torch.cuda.empty_cache()
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


def result_line(args, wl, world, res):
    out = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "e4m3",
           "data": "synthetic (seeded generator, random-init weights)",
           "config": config_of(wl, world, res["flush"], res["key_bytes"], args.shared_keys, args.cta_pairs),
           "roofline": res["roofline"], "stages_ms": res["stages_ms"], "e2e": res["e2e"],
           "gpu_launches": res["launches"],
           "clocks": res["clocks"], "cpu_baseline": res["cpu"]}
    return out


if __name__ == "__main__":
    main()
