#!/usr/bin/env python3
"""Benchmark of the PN-Mix quantized-KV decode path on B200.

Workload (synthetic, seeded): 16 sequences, 32 query / 8 KV heads, head_dim 128,
a 4096-token prefill whose last 64 queries pick 8 of 64 RoPE pairs per KV head
(2.25 key code bits), then one token appended and attended per step.  The timed
steps are the last ones before the context reaches 32768 tokens.  A step is
pnmix_append + pnmix_decode_attention for every sequence; the metric is decode
tokens/s (sequences x steps / time) and the decode kernel's achieved HBM GB/s.

The cache state before the timed steps is built by quantizing tokens [0, T0) in
bulk with the prefill's salient pairs, which gives the same bytes as appending
them one at a time (checked by the tests).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pnmix|reference]

Under torchrun (N > 1) each rank runs its own 16 sequences (weak scaling, no
data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn GB/s (% of B200 HBM peak) + tokens/s at 32K ctx, 2.25-bit keys"
B, HQ, HKV, D = 16, 32, 8, 128
PREFILL, CONTEXT, WINDOW = 4096, 32768, 64
K_SALIENT, BHI, BLO = 8, 4, 2
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of one decode launch from the committed ncu capture (profiles/
# decode_mma_stream32k.md): read + write bytes, the launch's algorithmic bytes, and a hash
# of the decode sources it was taken on.  Reported only while the sources still match.
DECODE_CAPTURE = {"sources_sha256_16": "f2df43601d39f9be", "traffic_bytes": 426606336,
                  "algorithmic_bytes": 420855808}
DECODE_SOURCES = ["decode_attention_prefill_b200/csrc/decode_mma.cu",
                  "decode_attention_prefill_b200/csrc/decode_common.cuh",
                  "decode_attention_prefill_b200/csrc/common.cuh",
                  "decode_attention_prefill_b200/csrc/decode_frag.cuh",
                  "decode_attention_prefill_b200/csrc/decode_group.cuh",
                  "decode_attention_prefill_b200/csrc/quantize_group.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="pnmix", choices=["pnmix", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="stream_32k",
                    choices=["stream_32k", "llama3_8b", "sweep_128k", "pipeline_32l", "verify_32k",
                             "stream_full"],
                    help="stream_32k is the benchmark line; the others print per-workload "
                         "measurements (decode GB/s and tokens/s; for the sweep the relative L2 "
                         "error against unquantized bf16 attention; for the 32-layer pipeline the "
                         "prefill latencies and the extrapolated end-to-end tokens/s; verify_32k: "
                         "two new tokens per sequence attended at once at 32K; stream_full: the "
                         "whole 4096 -> 32768 stream, measured)")
    ap.add_argument("--pipeline-sampled", action="store_true",
                    help="pipeline_32l: time the decode phase at 8 contexts and integrate, instead of "
                         "running all 28672 steps")
    ap.add_argument("--pipeline-layers-generated", type=int, default=4,
                    help="pipeline_32l: layers whose prefill inputs are generated (seed + layer); "
                         "the others reuse them cyclically")
    ap.add_argument("--shrunk-only", action="store_true",
                    help="sweep_128k: run only the points whose cache was shrunk (pnmix_shrink_keys)")
    ap.add_argument("--profile-decode", action="store_true",
                    help="build the 32K state, then run only --warmup + --steps decode launches "
                         "(small device footprint, for profiler captures); prints no bench line")
    ap.add_argument("--decode-kernel", default="auto", choices=["auto", "simt", "mma", "ws", "tc"],
                    help="with --profile-decode: the decode kernel those launches run (default: the "
                         "automatic choice, the one the bench times)")
    return ap.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def captured_traffic(alg_bytes_per_launch: float):
    """Per-launch DRAM traffic scaled from the recorded capture, or None if the decode
    sources changed since it was taken."""
    import hashlib
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != DECODE_CAPTURE["sources_sha256_16"]:
        return None
    return DECODE_CAPTURE["traffic_bytes"] * alg_bytes_per_launch / DECODE_CAPTURE["algorithmic_bytes"]


def decode_bytes(n_tokens: int, units: int, G: int, record_bytes: int) -> int:
    """Algorithmic bytes of one decode launch: packed records, residual rows,
    queries and outputs of every (sequence, KV head) unit."""
    ng, r = divmod(n_tokens, 32)
    return units * (ng * record_bytes + r * 2 * D * 2 + G * D * 2 + G * D * 4)


class ClockSampler:
    """NVML samples of the SM clock and the clock-event (throttle) reasons, polled every
    few milliseconds from a thread during the timed region.  Read-only."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int):
        self.dev = torch_device
        self.samples = []
        self.max_mhz = None
        self.h = None
        self._stop = threading.Event()

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(cvd.split(",")[self.dev]) if cvd else self.dev
            return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def _sample(self):
        import pynvml
        mhz = pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        try:
            reasons = pynvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            reasons = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((mhz, reasons))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        try:
            import pynvml
            self.h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        except Exception:
            self.h = None
        return self

    def __exit__(self, *exc):
        if self.h is not None:
            self._stop.set()
            self.t.join(timeout=2)
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return None
        active = set()
        for _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    active.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(active), "samples": len(self.samples), "source": "nvml"}


def max_over_ranks(ms: float, pg, dev) -> float:
    """The slowest rank's time (every rank takes part; pg is torch.distributed or None)."""
    if not pg:
        return ms
    import torch
    t = torch.tensor([ms], device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, steps: int, ms: float) -> float:
    """Tokens of all ranks (B sequences each, one token per sequence per step) over the
    slowest rank's time."""
    return world * B * steps / (ms / 1e3)


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def gen_inputs(seed: int, T_total: int, q_positions: list[int]):
    import workload
    kin = workload.rows(seed, workload.K, B, HKV, 0, T_total)
    vin = workload.rows(seed, workload.V, B, HKV, 0, T_total)
    qwin = workload.rows(seed, workload.Q, B, HQ, PREFILL - WINDOW, WINDOW, group=HQ // HKV)
    qs = np.stack([workload.rows(seed, workload.Q, B, HQ, p, 1, group=HQ // HKV)[:, :, 0]
                   for p in q_positions]) if q_positions else None
    return kin, vin, qwin, qs


def _oracle_unit_seconds(args):
    """Worker of the all-cores CPU baseline: build one (sequence, KV head) unit in the
    oracle at n_tokens context and time its decode attention (seconds)."""
    seed, b, h, n_tokens = args
    import oracle
    import workload
    G = HQ // HKV
    kin = workload.unit_rows(seed, workload.K, b, h, 1, 0, n_tokens, threads=1)[None]
    vin = workload.unit_rows(seed, workload.V, b, h, 1, 0, n_tokens, threads=1)[None]
    qwin = workload.unit_rows(seed, workload.Q, b, h * G, G, PREFILL - WINDOW, WINDOW, group=G, threads=1)
    q = workload.unit_rows(seed, workload.Q, b, h * G, G, n_tokens, 1, group=G, threads=1)[:, 0]
    oc = oracle.Cache(1, 1, (n_tokens + 32) // 32 * 32, K_SALIENT, BHI, BLO)
    oc.select(qwin[None], kin, PREFILL)
    oc.prefill(kin, vin, n_tokens)
    t0 = time.perf_counter()
    oc.attend_unit(np.ascontiguousarray(q), 0, 0)
    return time.perf_counter() - t0


def cpu_baseline_all_cores(seed: int, n_tokens: int):
    """The same oracle unit decode spread over every host core (one process per core,
    started with spawn), on min(128, 2 x cores) units; the step time is the wall time of
    the attention calls scaled to 128 units."""
    import concurrent.futures
    import multiprocessing
    cores = os.cpu_count() or 1
    units = [(seed, b, h, n_tokens) for b in range(B) for h in range(HKV)][:min(B * HKV, 2 * cores)]
    with concurrent.futures.ProcessPoolExecutor(max_workers=cores,
                                                mp_context=multiprocessing.get_context("spawn")) as ex:
        secs = list(ex.map(_oracle_unit_seconds, units))
    # the attention calls of `cores` workers overlap: per-unit cost / cores
    step_s = (sum(secs) / len(secs)) * (B * HKV) / min(cores, len(units))
    return {"value": B / step_s, "unit": "tokens/s", "cores": min(cores, len(units)), "kind": "oracle",
            "sample": f"oracle decode attention of {len(units)} (sequence, KV head) units at {n_tokens} "
                      f"tokens on {min(cores, len(units))} processes, scaled to a full {B}-sequence step"}


def cpu_baseline(seed: int, budget_s: float, n_tokens: int):
    """The oracle, as it stands, on a bounded sample of the timed step: decode
    attention of whole (sequence, KV head) units at n_tokens context, scaled to a
    full 16-sequence step.  Single-threaded."""
    import oracle
    import workload
    G = HQ // HKV
    units_done, elapsed = 0, 0.0
    t_start = time.time()
    for (b, h) in [(b, h) for b in range(B) for h in range(HKV)]:
        if elapsed >= budget_s or time.time() - t_start > 6 * budget_s:
            break
        kin = workload.unit_rows(seed, workload.K, b, h, 1, 0, n_tokens)[None]
        vin = workload.unit_rows(seed, workload.V, b, h, 1, 0, n_tokens)[None]
        qwin = workload.unit_rows(seed, workload.Q, b, h * G, G, PREFILL - WINDOW, WINDOW, group=G)
        q = workload.unit_rows(seed, workload.Q, b, h * G, G, n_tokens, 1, group=G)[:, 0]
        oc = oracle.Cache(1, 1, (n_tokens + 32) // 32 * 32, K_SALIENT, BHI, BLO)
        oc.select(qwin[None], kin, PREFILL)
        oc.prefill(kin, vin, n_tokens)
        t0 = time.perf_counter()
        oc.attend_unit(np.ascontiguousarray(q), 0, 0)
        elapsed += time.perf_counter() - t0
        units_done += 1
    step_s = elapsed / units_done * (B * HKV)
    return {"value": B / step_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"oracle decode attention of {units_done} of {B * HKV} (sequence, KV head) "
                      f"units at {n_tokens}-token context ({elapsed:.1f} s), scaled to a full "
                      f"{B}-sequence step"}


def stream_config(world: int) -> dict:
    """`config` of the stream_32k line (both arms)."""
    return {"workload": "stream_32k", "batch_per_gpu": B, "n_q_heads": HQ, "n_kv_heads": HKV,
            "head_dim": D, "context": CONTEXT, "prefill": PREFILL, "salient_pairs": K_SALIENT,
            "key_bits": [BHI, BLO], "value_bits": 2, "key_code_bits": 2.25,
            "parallelism": f"dp{world}", "l2": "inputs larger than L2 (419 MB cache read per step)"}


def run_reference(args, world, rank):
    """Reference arm: the oracle on the host cores, same metric and workload."""
    if rank != 0:
        return 0
    import oracle
    import workload
    G = HQ // HKV
    n_tokens = CONTEXT - 1
    h, b = 0, 0
    kin = np.ascontiguousarray(workload.rows(args.seed, workload.K, 1, HKV, 0, n_tokens + args.steps + args.warmup)[:, :1])
    vin = np.ascontiguousarray(workload.rows(args.seed, workload.V, 1, HKV, 0, n_tokens + args.steps + args.warmup)[:, :1])
    qwin = workload.rows(args.seed, workload.Q, 1, HQ, PREFILL - WINDOW, WINDOW, group=G)[:, :G]
    oc = oracle.Cache(1, 1, CONTEXT + 2 * 32 + args.steps + args.warmup, K_SALIENT, BHI, BLO)
    oc.select(np.ascontiguousarray(qwin), kin, PREFILL)
    start = n_tokens - args.steps - args.warmup
    oc.prefill(kin, vin, start)
    times = []
    for i in range(args.warmup + args.steps):
        t = start + i
        q = workload.rows(args.seed, workload.Q, 1, HQ, t, 1, group=G)[:, :G, 0]
        t0 = time.perf_counter()
        oc.append(kin[:, :, t], vin[:, :, t])
        oc.attend(np.ascontiguousarray(q))
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt * B * HKV)      # one unit -> a full 16-sequence step
    units = B * HKV
    sampled_s = sum(times) / units          # wall time the sampled steps actually took
    value = B * len(times) / sum(times)     # whole-step throughput: each step scaled by `units`
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sampled_s / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": stream_config(world),
        "sampled": {"units_per_step": 1, "units_per_full_step": units,
                    "value_scale": f"each timed step is 1 of {units} (sequence, KV head) units; value "
                                   f"divides {B} tokens per step by {units} x the sampled time",
                    "ms_per_step": "wall time of the sampled step (one unit)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"oracle append + decode attention of 1 of {units} (sequence, KV head) "
                                   f"units per step, scaled to a full {B}-sequence step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def exact_bf16_attention(q: np.ndarray, kin: np.ndarray, vin: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(128)) v over the unquantized bf16 rows, in fp64: the quality
    yardstick of the bit sweep (q [G][128], kin / vin [n][128], all bf16 bits)."""
    import workload
    qf = workload.bf16_to_float(q).astype(np.float64)
    kf = workload.bf16_to_float(kin).astype(np.float64)
    vf = workload.bf16_to_float(vin).astype(np.float64)
    logits = qf @ kf.T / np.sqrt(128.0)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    return (p @ vf) / p.sum(axis=1, keepdims=True)


def timed_rotation(fns, reps: int, warmup: int) -> float:
    """Average device time (s) of one launch over `reps` back-to-back launches that cycle
    through `fns` (one per cache replica; the replicas together exceed L2, so every
    launch reads its cache from HBM).  CUDA events bracket the whole run."""
    import torch
    for i in range(warmup):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(reps):
        fns[i % len(fns)]()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / reps


def two_part_point(args, pm, wl, k_dev, v_dev, qwin_dev, q_dev, exact, peak, l2_bytes,
                   k_hi=16, k_lo=8, percent=50):
    """The mixed-precision point of the bit sweep: the prefill's 32-token groups ranked by
    the saliency window's mean-query logit (pnmix_split_groups), the best `percent` kept with
    k_hi salient pairs and the rest with k_lo, and decode attention over both parts
    (pnmix_decode_attention_two).  Reports the split's time, the decode's, and the
    relative L2 error against unquantized bf16 attention."""
    import torch
    Bw, Hq, Hkv, ctx = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.context
    G = Hq // Hkv
    cfg_hi = pm.Config.make(Hq, Hkv, 4, 2, k_hi, WINDOW)
    cfg_lo = pm.Config.make(Hq, Hkv, 4, 2, k_lo, WINDOW)
    L_hi, L_lo = pm.split_sizes(ctx, percent)
    split = lambda: pm.pnmix_split_groups(cfg_hi, qwin_dev, k_dev, v_dev, ctx, percent)  # noqa: E731
    for _ in range(2):
        parts = split()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        parts = split()
    e1.record()
    torch.cuda.synchronize()
    split_ms = e0.elapsed_time(e1) / 3

    def build():
        pair = []
        for cfg, kp, vp, Lp in ((cfg_hi, parts["k_hi"], parts["v_hi"], L_hi), (cfg_lo, parts["k_lo"], parts["v_lo"], L_lo)):
            c = pm.PNMixCache(cfg, Bw, ctx + 32, max_context=ctx)
            pm.pnmix_select_pairs(cfg, qwin_dev, k_dev, ctx, c)
            if Lp:
                pm.pnmix_quantize_keys(cfg, kp, Lp, c)
                pm.pnmix_quantize_values(cfg, vp, Lp, c)
            pair.append(c)
        return pair
    first = build()
    per_rep = sum(pm.cache_bytes(c.cfg, Bw, ctx + 32) for c in first)
    n_rep = max(3, -(-3 * l2_bytes // per_rep))
    reps = [first] + [build() for _ in range(n_rep - 1)]
    out = torch.empty(Bw, Hq, D, dtype=torch.float32, device=q_dev.device)
    fns = [(lambda a_=a_, b_=b_: pm.pnmix_decode_attention_two(a_, b_, q_dev, out)) for a_, b_ in reps]
    t = timed_rotation(fns, max(args.steps, 3 * n_rep), args.warmup)
    pm.pnmix_decode_attention_two(first[0], first[1], q_dev, out)
    assert all(c.read_error() == 0 for pair in reps for c in pair)
    units = Bw * Hkv
    R_hi, R_lo = first[0].c.record_bytes, first[1].c.record_bytes
    alg = decode_bytes(L_hi, units, G, R_hi) + decode_bytes(L_lo, units, G, R_lo) - units * G * D * (2 + 4)
    bits = (L_hi * (2 + 0.5 * k_hi / 16) + L_lo * (2 + 0.5 * k_lo / 16)) / ctx
    r = {"key_bits": [4, 2], "salient_pairs": [k_hi, k_lo], "two_precision_percent_high": percent,
         "saliency_score": "pair-norm product", "pruned_query_pairs": 0, "shrunk_to_low_bits": False,
         "key_code_bits": bits, "bytes_per_token_head": (L_hi * R_hi + L_lo * R_lo) / 32 / ctx,
         "split_ms": split_ms, "decode_us": t * 1e6, "decode_gbs": alg / t / 1e9, "frac": alg / t / 1e9 / peak,
         "frac_of_8tbs": alg / t / 8e12, "tokens_per_s": Bw / t, "replicas": n_rep}
    if exact is not None:
        got = out.cpu().numpy().astype(np.float64)
        num = sum(float(np.sum((got[b, h * G:(h + 1) * G] - e) ** 2)) for (b, h), e in exact.items())
        den = sum(float(np.sum(e ** 2)) for e in exact.values())
        r["rel_l2_vs_bf16_attention"] = (num / den) ** 0.5
    del reps, first, parts
    return r


def run_decode_workload(args):
    """Decode-only measurements: llama3_8b (batch 8, 32/8 heads, one step at 8192) and
    sweep_128k (batch 2, 28/4 heads, 131072 tokens, six bit points and the statistic,
    pruning and shrinking variants, each with the relative L2 error against unquantized
    bf16 attention over every (sequence, KV head) unit).
    These caches fit in L2, so the timed launches rotate over enough identical cache
    replicas to exceed it three times over."""
    import torch

    import decode_attention_prefill_b200 as pm
    import workload
    wl = workload.WORKLOADS[args.workload]
    Bw, Hq, Hkv, ctx = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.context
    G = Hq // Hkv
    # (bit point, saliency statistic, pruned query pairs, shrunk, pruned key slices): the
    # sweep adds the key-only (1) and key-range x query (2) statistics at two bit points,
    # 40 % dynamic query-channel pruning (26 of 64 pairs) at 2.25 bits, key-slice pruning
    # (3 of the 7 low-precision slices, 48 of 128 channels), and two caches whose salient
    # keys were shrunk to the low bit width after quantization (pnmix_shrink_keys); the
    # llama3_8b shape adds key-slice pruning of 2, 3 and 4 slices (the cost of the decision)
    p42 = workload.BitPoint(4, 2, 8)
    points = [(bp, 0, 0, False, 0) for bp in (wl.sweep if wl.sweep else (wl.bits,))]
    if wl.sweep:
        points += [(p42, 1, 0, False, 0), (p42, 2, 0, False, 0),
                   (workload.BitPoint(2, 1, 16), 1, 0, False, 0), (workload.BitPoint(2, 1, 16), 2, 0, False, 0),
                   (p42, 0, 26, False, 0), (p42, 0, 0, False, 3),
                   (p42, 0, 0, True, 0), (workload.BitPoint(2, 1, 16), 0, 0, True, 0)]
        if args.shrunk_only:
            points = [p_ for p_ in points if p_[3]]
    elif wl.bits.key_bits_lo == 2:
        points += [(wl.bits, 0, 0, False, n) for n in (2, 3, 4)]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kin = workload.rows(args.seed, workload.K, Bw, Hkv, 0, ctx)
    vin = workload.rows(args.seed, workload.V, Bw, Hkv, 0, ctx)
    qwin = workload.rows(args.seed, workload.Q, Bw, Hq, ctx - WINDOW, WINDOW, group=G)
    q = np.ascontiguousarray(workload.rows(args.seed, workload.Q, Bw, Hq, ctx, 1, group=G)[:, :, 0])
    k_dev = torch.from_numpy(kin).view(torch.bfloat16).to(dev)
    v_dev = torch.from_numpy(vin).view(torch.bfloat16).to(dev)
    qwin_dev = torch.from_numpy(qwin).view(torch.bfloat16).to(dev)
    q_dev = torch.from_numpy(q).view(torch.bfloat16).to(dev)
    peak, peak_kind = measured_peaks()
    l2_bytes = 126 << 20
    exact = None
    if wl.sweep:
        exact = {(b, h): exact_bf16_attention(q[b, h * G:(h + 1) * G], kin[b, h], vin[b, h])
                 for b in range(Bw) for h in range(Hkv)}
    results = []
    with ClockSampler(0) as clocks:
        for bp, score, prune, shrink, slices in points:
            qcfg = pm.Config.make(Hq, Hkv, bp.key_bits_hi, bp.key_bits_lo, bp.n_salient_pairs, WINDOW,
                                  saliency_score=score, n_pruned_pairs=prune, n_pruned_slices=slices)
            cfg = qcfg.without_salient() if shrink else qcfg
            src = pm.PNMixCache(qcfg, Bw, ctx + 32, max_context=ctx)
            src.prefill(qwin_dev, k_dev, v_dev, ctx)
            n_rep = max(3, -(-3 * l2_bytes // pm.cache_bytes(cfg, Bw, ctx + 32)))
            shrink_us = shrink_gbs = None
            if shrink:
                replicas = [src.shrunk() for _ in range(n_rep)]
                # one shrink reads every source record and writes every destination record,
                # and copies both residual windows
                ng = ctx // 32
                shrink_bytes = Bw * Hkv * (ng * (src.c.record_bytes + replicas[0].c.record_bytes)
                                           + 2 * 2 * 32 * D * 2)
                # two sources alternate and the destinations rotate, so each launch finds
                # neither its source nor its destination in L2
                src2 = pm.PNMixCache(qcfg, Bw, ctx + 32, max_context=ctx)
                src2.prefill(qwin_dev, k_dev, v_dev, ctx)
                sfns = [(lambda s_=(src, src2)[i % 2], d_=r_: pm.pnmix_shrink_keys(qcfg, s_, d_))
                        for i, r_ in enumerate(replicas + replicas[:1] if n_rep % 2 else replicas)]
                t_s = timed_rotation(sfns, max(args.steps, 2 * len(sfns)), args.warmup)
                del src2
                shrink_us, shrink_gbs = t_s * 1e6, shrink_bytes / t_s / 1e9
                pm.pnmix_shrink_keys(qcfg, src, replicas[0])
                del src
            else:
                replicas = [src]
                for _ in range(n_rep - 1):
                    r = pm.PNMixCache(cfg, Bw, ctx + 32, max_context=ctx)
                    r.prefill(qwin_dev, k_dev, v_dev, ctx)
                    replicas.append(r)
            cache = replicas[0]
            out = torch.empty(Bw, Hq, D, dtype=torch.float32, device=dev)
            fns = [(lambda c_=c_: pm.pnmix_decode_attention(cfg, q_dev, c_, out)) for c_ in replicas]
            t = timed_rotation(fns, max(args.steps, 3 * n_rep), args.warmup)
            pm.pnmix_decode_attention(cfg, q_dev, cache, out)
            assert all(c_.read_error() == 0 for c_ in replicas)
            alg = decode_bytes(ctx, Bw * Hkv, G, cache.c.record_bytes)   # records are read whole
            r = {"key_bits": [bp.key_bits_hi, bp.key_bits_lo], "salient_pairs": bp.n_salient_pairs,
                 "saliency_score": ["pair-norm product", "key only", "key range x query"][score],
                 "pruned_query_pairs": prune, "pruned_key_slices": slices, "shrunk_to_low_bits": shrink,
                 "shrink_us": shrink_us, "shrink_gbs": shrink_gbs,
                 "key_code_bits": bp.key_bits_lo if shrink else bp.key_code_bits,
                 "bytes_per_token_head": cache.c.record_bytes / 32,
                 "decode_us": t * 1e6, "decode_gbs": alg / t / 1e9, "frac": alg / t / 1e9 / peak,
                 "frac_of_8tbs": alg / t / 8e12, "tokens_per_s": Bw / t, "replicas": n_rep}
            if exact is not None:
                got = out.cpu().numpy().astype(np.float64)
                num = sum(float(np.sum((got[b, h * G:(h + 1) * G] - e) ** 2)) for (b, h), e in exact.items())
                den = sum(float(np.sum(e ** 2)) for e in exact.values())
                r["rel_l2_vs_bf16_attention"] = (num / den) ** 0.5
            results.append(r)
            del cache, replicas
        if wl.sweep and not args.shrunk_only:
            results.append(two_part_point(args, pm, wl, k_dev, v_dev, qwin_dev, q_dev, exact, peak, l2_bytes))
    line = {"workload": args.workload, "metric": "decode-attn GB/s (% of B200 HBM peak) + tokens/s",
            "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "data": "synthetic", "dtype": "f32",
            "config": {"batch": Bw, "n_q_heads": Hq, "n_kv_heads": Hkv, "head_dim": D,
                       "context": ctx, "l2": "back-to-back launches rotating over cache replicas "
                                             "that together exceed L2 three times"},
            "peak": peak, "peak_source": peak_kind, "points": results, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_verify(args):
    """verify_32k: the stream_32k shape (16 x 32/8 heads, 32768 tokens) with T new tokens
    per sequence attended at once (pnmix_decode_attention_multi after T appends), for
    T = 1, 2, 4, 8, 16 and 32 (4 to 128 query rows per KV head), each against the roofline of
    the bytes it must read.  The 419 MB cache exceeds L2.  Besides the algorithmic bytes,
    each point reports the tensor-core work per launch (the key- and value-side products
    of every row with every cached token)."""
    import torch

    import decode_attention_prefill_b200 as pm
    Ts = [1, 2, 4, 8, 16, 32]
    Tmax = max(Ts)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n0 = CONTEXT - Tmax
    kin, vin, qwin, _ = gen_inputs(args.seed, CONTEXT, [])
    qm = workload_rows_q(args.seed, CONTEXT - Tmax, Tmax)                # [B][Tmax][Hq][128]
    cfg = pm.Config.make(HQ, HKV, BHI, BLO, K_SALIENT, WINDOW)
    cache = pm.PNMixCache(cfg, B, CONTEXT + 32, max_context=CONTEXT, max_queries=Tmax)
    k_dev = torch.from_numpy(kin).view(torch.bfloat16).to(dev)
    v_dev = torch.from_numpy(vin).view(torch.bfloat16).to(dev)
    pm.pnmix_select_pairs(cfg, torch.from_numpy(qwin).view(torch.bfloat16).to(dev), k_dev, PREFILL, cache)
    pm.pnmix_quantize_keys(cfg, k_dev, n0, cache)
    pm.pnmix_quantize_values(cfg, v_dev, n0, cache)
    for t in range(n0, CONTEXT):
        pm.pnmix_append(cfg, k_dev[:, :, t].contiguous(), v_dev[:, :, t].contiguous(), cache)
    del k_dev, v_dev
    torch.cuda.empty_cache()
    q_all = torch.from_numpy(qm).view(torch.bfloat16).to(dev)
    G = HQ // HKV
    rec = cache.c.record_bytes
    peak, peak_kind = measured_peaks()
    points = []
    with ClockSampler(0) as clocks:
        for T in Ts:
            q_dev = q_all[:, Tmax - T:].contiguous()   # the last T queries: the newest T tokens
            out = torch.empty(B, T, HQ, D, dtype=torch.float32, device=dev)
            if T == 1:
                q1 = q_dev[:, 0].contiguous()
                o1 = out[:, 0]
                fn = lambda: pm.pnmix_decode_attention(cfg, q1, cache, o1)   # noqa: E731
            else:
                fn = lambda q_=q_dev, o_=out: pm.pnmix_decode_attention_multi(cfg, q_, cache, o_)   # noqa: E731
            t = timed_rotation([fn], args.steps, args.warmup)
            alg = decode_bytes(CONTEXT, B * HKV, G * T, rec)
            flops = 2 * 2 * B * HQ * T * CONTEXT * D     # q.k and p.v per row and token
            points.append({"queries_per_sequence": T, "rows_per_kv_head": G * T, "decode_us": t * 1e6,
                           "tokens_per_s": B * T / t, "decode_gbs": alg / t / 1e9, "frac": alg / t / 1e9 / peak,
                           "tensor_tflops": flops / t / 1e12})
    assert cache.read_error() == 0
    line = {"workload": "verify_32k", "metric": "multi-token decode attention at 32K", "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "data": "synthetic", "dtype": "f32",
            "config": {"batch": B, "n_q_heads": HQ, "n_kv_heads": HKV, "context": CONTEXT,
                       "key_code_bits": 2.25, "l2": "inputs larger than L2 (419 MB cache per launch)"},
            "points": points, "peak": peak, "peak_source": peak_kind, "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_stream_full(args):
    """stream_full: the whole stream_32k stream, measured rather than sampled: a 4096-token
    prefill (saliency + quantize), then all 28672 append + decode steps to 32768 tokens,
    one token per sequence per step.  K/V rows are the generator's at their true
    positions; the queries of 1024 consecutive positions are reused cyclically (the decode
    cost does not depend on the query values).  Reports the whole-stream time and the
    average decode tokens/s."""
    import torch

    import decode_attention_prefill_b200 as pm
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kin, vin, qwin, _ = gen_inputs(args.seed, CONTEXT, [])
    n_q = 1024
    q_dev = torch.from_numpy(workload_rows_q(args.seed, PREFILL, n_q)).view(torch.bfloat16).to(dev) \
        .permute(1, 0, 2, 3).contiguous()           # [n_q][B][Hq][128]
    cfg = pm.Config.make(HQ, HKV, BHI, BLO, K_SALIENT, WINDOW)
    cache = pm.PNMixCache(cfg, B, CONTEXT + 32, max_context=CONTEXT)
    k_dev = torch.from_numpy(kin).view(torch.bfloat16).to(dev)
    v_dev = torch.from_numpy(vin).view(torch.bfloat16).to(dev)
    kn = k_dev.permute(2, 0, 1, 3).contiguous()     # [T][B][Hkv][128]
    vn = v_dev.permute(2, 0, 1, 3).contiguous()
    qwin_dev = torch.from_numpy(qwin).view(torch.bfloat16).to(dev)
    out = torch.empty(B, HQ, D, dtype=torch.float32, device=dev)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clocks:
        e[0].record()
        cache.prefill(qwin_dev, k_dev, v_dev, PREFILL)
        e[1].record()
        for t in range(PREFILL, CONTEXT):
            pm.pnmix_append_decode(cfg, kn[t], vn[t], q_dev[(t - PREFILL) % n_q], cache, out)
        e[2].record()
        torch.cuda.synchronize()
    assert cache.read_error() == 0 and int(cache.lengths().min().item()) == CONTEXT
    prefill_s = e[0].elapsed_time(e[1]) / 1e3
    stream_s = e[1].elapsed_time(e[2]) / 1e3
    steps = CONTEXT - PREFILL
    line = {"workload": "stream_full", "metric": "whole-stream time, 4096 -> 32768 tokens",
            "unit": "s", "n_gpus": 1, "data": "synthetic", "dtype": "f32",
            "config": {"batch": B, "n_q_heads": HQ, "n_kv_heads": HKV, "prefill": PREFILL,
                       "context": CONTEXT, "key_code_bits": 2.25,
                       "queries": f"{n_q} consecutive positions reused cyclically"},
            "prefill_s": prefill_s, "stream_s": stream_s, "steps": steps,
            "decode_tokens_per_s": B * steps / stream_s, "mean_step_us": stream_s / steps * 1e6,
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def workload_rows_q(seed: int, pos0: int, n: int) -> np.ndarray:
    """Queries of positions pos0 .. pos0+n-1 of the bench workload: bf16 [B][n][Hq][128]."""
    import workload
    q = workload.rows(seed, workload.Q, B, HQ, pos0, n, group=HQ // HKV)
    return np.ascontiguousarray(q.transpose(0, 2, 1, 3))


def run_pipeline(args):
    """pipeline_32l: 32 layers, batch 32, 32/8 heads.  Per layer a 4096-token prefill
    (saliency + quantize), then decode steps (append + attend in every layer) to 32768.
    Prefill is timed on all 32 layers; the decode phase is timed at sampled contexts and
    integrated over the 28672 steps (decode time is linear in the context), which the
    output labels as extrapolated.  Layer l's inputs are those of seed + l for the
    prefill; the decode-time caches past the prefill are filled by quantizing the
    generated rows of layer 0 repeated along time (the decode cost does not depend on the
    values), which keeps host generation to one layer."""
    import torch

    import decode_attention_prefill_b200 as pm
    import workload
    wl = workload.WORKLOADS["pipeline_32l"]
    Bw, Hq, Hkv, L, C, NL = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.prefill, wl.context, wl.layers
    G = Hq // Hkv
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n_gen = min(NL, max(1, args.pipeline_layers_generated))
    cfg = pm.Config.make(Hq, Hkv, BHI, BLO, K_SALIENT, WINDOW)
    caches = [pm.PNMixCache(cfg, Bw, C + 32, max_context=C) for _ in range(NL)]
    inputs = []
    for l in range(n_gen):
        s = args.seed + l
        inputs.append((torch.from_numpy(workload.rows(s, workload.Q, Bw, Hq, L - WINDOW, WINDOW, group=G))
                       .view(torch.bfloat16).to(dev),
                       torch.from_numpy(workload.rows(s, workload.K, Bw, Hkv, 0, L)).view(torch.bfloat16).to(dev),
                       torch.from_numpy(workload.rows(s, workload.V, Bw, Hkv, 0, L)).view(torch.bfloat16).to(dev)))
    # ---- prefill of all layers: saliency, then quantize, each layer in turn
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * NL)]
    for rep in range(2):
        for l in range(NL):
            qw, kk, vv = inputs[l % n_gen]
            caches[l].reset()
            ev[3 * l].record()
            pm.pnmix_select_pairs(cfg, qw, kk, L, caches[l])
            ev[3 * l + 1].record()
            pm.pnmix_quantize_keys(cfg, kk, L, caches[l])
            pm.pnmix_quantize_values(cfg, vv, L, caches[l])
            ev[3 * l + 2].record()
        torch.cuda.synchronize()
    sal_ms = sum(ev[3 * l].elapsed_time(ev[3 * l + 1]) for l in range(NL))
    qnt_ms = sum(ev[3 * l + 1].elapsed_time(ev[3 * l + 2]) for l in range(NL))
    prefill_ms = ev[0].elapsed_time(ev[3 * NL - 1])
    if not args.pipeline_sampled:
        return run_pipeline_full(args, pm, wl, cfg, caches, sal_ms, qnt_ms, prefill_ms, n_gen)
    # ---- decode phase at sampled contexts
    reps = 8
    k_rep = inputs[0][1].repeat(1, 1, C // L, 1)           # [B][Hkv][C][128]
    v_rep = inputs[0][2].repeat(1, 1, C // L, 1)
    steps_in = workload.rows(args.seed, workload.K, Bw, Hkv, L, reps)
    kn = torch.from_numpy(np.ascontiguousarray(steps_in.transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)
    vn = torch.from_numpy(np.ascontiguousarray(
        workload.rows(args.seed, workload.V, Bw, Hkv, L, reps).transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)
    qn = torch.from_numpy(np.ascontiguousarray(
        workload.rows(args.seed, workload.Q, Bw, Hq, L, reps, group=G).transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)
    out = torch.empty(Bw, Hq, D, dtype=torch.float32, device=dev)
    samples = []
    contexts = [L + 1 + reps, 8192, 12288, 16384, 20480, 24576, 28672, C]
    with ClockSampler(0) as clocks:
        for ctx in contexts:
            start = ctx - reps           # cache length before the first sampled step
            for l in range(NL):
                pm.pnmix_quantize_keys(cfg, k_rep, start, caches[l])
                pm.pnmix_quantize_values(cfg, v_rep, start, caches[l])
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            for i in range(reps):
                if i == 2:
                    e0.record()
                for l in range(NL):
                    pm.pnmix_append_decode(cfg, kn[i], vn[i], qn[i], caches[l], out)
            e1.record()
            torch.cuda.synchronize()
            step_ms = e0.elapsed_time(e1) / (reps - 2)
            samples.append({"context": start + 1 + (2 + reps - 1) / 2, "step_ms": step_ms})
    assert all(c.read_error() == 0 for c in caches)
    # integrate the step time over the decode steps (contexts L+1 .. C), trapezoid rule
    xs = [s["context"] for s in samples]
    ys = [s["step_ms"] for s in samples]
    steps = C - L
    grid = np.arange(L + 1, C + 1, dtype=np.float64)
    total_ms = float(np.sum(np.interp(grid, xs, ys)))
    line = {"workload": "pipeline_32l", "metric": "end-to-end attention-path tokens/s",
            "unit": "tokens/s", "n_gpus": 1, "data": "synthetic", "dtype": "f32",
            "config": {"layers": NL, "batch": Bw, "n_q_heads": Hq, "n_kv_heads": Hkv,
                       "prefill": L, "context": C, "salient_pairs": K_SALIENT, "key_bits": [BHI, BLO],
                       "prefill_inputs": f"seed + layer for {n_gen} generated layer(s), reused cyclically",
                       "l2": "32 layers of cache between re-reads of a layer (>= 3 GB)"},
            "prefill": {"saliency_ms_all_layers": sal_ms, "quantize_ms_all_layers": qnt_ms,
                        "prefill_ms_all_layers": prefill_ms,
                        "quantize_tokens_per_s": NL * Bw * L / (qnt_ms / 1e3)},
            "decode_samples": samples,
            "decode": {"steps": steps, "total_s_extrapolated": total_ms / 1e3,
                       "tokens_per_s_extrapolated": Bw * steps / (total_ms / 1e3)},
            "end_to_end": {"total_s_extrapolated": (total_ms + prefill_ms) / 1e3,
                           "tokens_per_s_extrapolated": Bw * steps / ((total_ms + prefill_ms) / 1e3)},
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_pipeline_full(args, pm, wl, cfg, caches, sal_ms, qnt_ms, prefill_ms, n_gen):
    """pipeline_32l decode phase measured whole: after the prefill of every layer, all
    C - L decode steps, each one pnmix_append_decode per layer, timed between two events.
    The appended K / V rows and the queries of 1024 consecutive positions are reused
    cyclically (the cost does not depend on their values)."""
    import torch

    import workload
    Bw, Hq, Hkv, L, C, NL = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.prefill, wl.context, wl.layers
    G = Hq // Hkv
    dev = torch.device("cuda", 0)
    pool = 1024
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a.transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)  # noqa: E731
    kn = to(workload.rows(args.seed, workload.K, Bw, Hkv, L, pool))
    vn = to(workload.rows(args.seed, workload.V, Bw, Hkv, L, pool))
    qn = to(workload.rows(args.seed, workload.Q, Bw, Hq, L, pool, group=G))
    out = torch.empty(Bw, Hq, D, dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(0) as clocks:
        e0.record()
        for t in range(L, C):
            i = (t - L) % pool
            for l in range(NL):
                pm.pnmix_append_decode(cfg, kn[i], vn[i], qn[i], caches[l], out)
        e1.record()
        torch.cuda.synchronize()
    decode_s = e0.elapsed_time(e1) / 1e3
    assert all(c.read_error() == 0 and int(c.lengths().min().item()) == C for c in caches)
    steps = C - L
    line = {"workload": "pipeline_32l", "metric": "end-to-end attention-path tokens/s",
            "unit": "tokens/s", "n_gpus": 1, "data": "synthetic", "dtype": "f32",
            "value": Bw * steps / (decode_s + prefill_ms / 1e3),
            "config": {"layers": NL, "batch": Bw, "n_q_heads": Hq, "n_kv_heads": Hkv,
                       "prefill": L, "context": C, "salient_pairs": K_SALIENT, "key_bits": [BHI, BLO],
                       "prefill_inputs": f"seed + layer for {n_gen} generated layer(s), reused cyclically",
                       "decode_inputs": f"K / V rows and queries of {pool} positions reused cyclically",
                       "l2": "32 layers of cache between re-reads of a layer (>= 3 GB)"},
            "prefill": {"saliency_ms_all_layers": sal_ms, "quantize_ms_all_layers": qnt_ms,
                        "prefill_ms_all_layers": prefill_ms,
                        "quantize_tokens_per_s": NL * Bw * L / (qnt_ms / 1e3)},
            "decode": {"steps": steps, "launches": steps * NL, "total_s": decode_s,
                       "mean_step_ms": 1e3 * decode_s / steps, "tokens_per_s": Bw * steps / decode_s},
            "end_to_end": {"total_s": decode_s + prefill_ms / 1e3,
                           "tokens_per_s": Bw * steps / (decode_s + prefill_ms / 1e3)},
            "measured": "every step timed (not extrapolated)",
            "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.workload == "pipeline_32l":
        return run_pipeline(args)
    if args.workload == "verify_32k":
        return run_verify(args)
    if args.workload == "stream_full":
        return run_stream_full(args)
    if args.workload != "stream_32k":
        return run_decode_workload(args)

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        pg = dist
    import decode_attention_prefill_b200 as pm

    K, W = args.steps, args.warmup
    n_e2e = W + K
    if 3 * (W + K) >= CONTEXT - PREFILL:
        raise SystemExit("--steps/--warmup too large for the 32K stream")
    T0 = CONTEXT - 3 * (W + K)           # tokens already cached before the e2e steps
    seed = args.seed + 7919 * rank        # each rank: its own 16 sequences
    positions = list(range(T0, CONTEXT))  # one query per step
    kin, vin, qwin, qs = gen_inputs(seed, CONTEXT, positions)

    cfg = pm.Config.make(HQ, HKV, BHI, BLO, K_SALIENT, WINDOW)
    if args.profile_decode:
        cfg.decode_kernel = pm.DECODE_KERNELS[args.decode_kernel]
    cache = pm.PNMixCache(cfg, B, CONTEXT + 32, max_context=CONTEXT)
    dev = torch.device("cuda", local)
    out = torch.empty(B, HQ, D, dtype=torch.float32, device=dev)
    qwin_dev = torch.from_numpy(qwin).view(torch.bfloat16).to(dev)
    q_dev = torch.from_numpy(qs).view(torch.bfloat16).to(dev)            # [steps][B][HQ][D]
    # rows appended by the measured steps: [T][B][HKV][D]
    kn_dev = torch.from_numpy(np.ascontiguousarray(kin[:, :, T0:].transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)
    vn_dev = torch.from_numpy(np.ascontiguousarray(vin[:, :, T0:].transpose(2, 0, 1, 3))).view(torch.bfloat16).to(dev)

    # ---- prefill (saliency + quantize of the 4096-token prefill), timed separately
    k_dev = torch.from_numpy(kin[:, :, :T0].copy()).view(torch.bfloat16).to(dev)
    v_dev = torch.from_numpy(vin[:, :, :T0].copy()).view(torch.bfloat16).to(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for it in range(3):
        cache.reset()
        ev[0].record()
        pm.pnmix_select_pairs(cfg, qwin_dev, k_dev, PREFILL, cache)
        ev[1].record()
        pm.pnmix_quantize_keys(cfg, k_dev, PREFILL, cache)
        pm.pnmix_quantize_values(cfg, v_dev, PREFILL, cache)
        ev[2].record()
        torch.cuda.synchronize()
    saliency_ms = ev[0].elapsed_time(ev[1])
    quant_ms = ev[1].elapsed_time(ev[2])
    # ---- bulk state up to T0 with the prefill's salient pairs, then drop the bulk rows
    pm.pnmix_quantize_keys(cfg, k_dev, T0, cache)
    pm.pnmix_quantize_values(cfg, v_dev, T0, cache)
    torch.cuda.synchronize()
    del k_dev, v_dev, kin, vin
    torch.cuda.empty_cache()

    if args.profile_decode:
        # the bench's step (append + decode in one launch) from context T0, for profiler captures
        for i in range(W + K):
            pm.pnmix_append_decode(cfg, kn_dev[i], vn_dev[i], q_dev[i], cache, out)
        torch.cuda.synchronize()
        print(json.dumps({"profile_decode": True, "launches": W + K, "context": T0,
                          "error_word": cache.read_error()}), flush=True)
        return 0
    rec_bytes = cache.c.record_bytes

    # ---- end-to-end through host buffers (pinned), e2e steps T0 .. T0+n_e2e-1
    # Double-buffered: step i+1's inputs go host -> device on a copy stream while step i
    # appends and attends; step i's output goes device -> host on a third stream.
    q_host = torch.from_numpy(qs).view(torch.bfloat16).pin_memory()
    kn_host = kn_dev[:n_e2e].cpu().pin_memory()
    vn_host = vn_dev[:n_e2e].cpu().pin_memory()
    out_host = [torch.empty(B, HQ, D, dtype=torch.float32).pin_memory() for _ in range(2)]
    comp_s = torch.cuda.current_stream()
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = [{"q": torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev),
             "k": torch.empty(B, HKV, D, dtype=torch.bfloat16, device=dev),
             "v": torch.empty(B, HKV, D, dtype=torch.bfloat16, device=dev),
             "out": torch.empty(B, HQ, D, dtype=torch.float32, device=dev)} for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of a buffer landed
    ev_used = [torch.cuda.Event() for _ in range(2)]    # append + decode done with a buffer
    ev_out = [torch.cuda.Event() for _ in range(2)]     # its output copied to the host
    used = [False, False]

    def stage(i):
        j = i % 2
        if used[j]:
            h2d_s.wait_event(ev_used[j])
        with torch.cuda.stream(h2d_s):
            bufs[j]["q"].copy_(q_host[i], non_blocking=True)
            bufs[j]["k"].copy_(kn_host[i], non_blocking=True)
            bufs[j]["v"].copy_(vn_host[i], non_blocking=True)
            ev_in[j].record(h2d_s)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(n_e2e):
        j = i % 2
        if i == W:
            if pg:
                pg.barrier()
            torch.cuda.synchronize()
            e0.record()
        if i == 0 or i == W:
            stage(i)
        if i + 1 < n_e2e and i + 1 != W:
            stage(i + 1)
        comp_s.wait_event(ev_in[j])
        if used[j]:
            comp_s.wait_event(ev_out[j])     # the previous output of this buffer has left
        pm.pnmix_append_decode(cfg, bufs[j]["k"], bufs[j]["v"], bufs[j]["q"], cache, bufs[j]["out"])
        ev_used[j].record(comp_s)
        d2h_s.wait_event(ev_used[j])
        with torch.cuda.stream(d2h_s):
            out_host[j].copy_(bufs[j]["out"], non_blocking=True)
            ev_out[j].record(d2h_s)
        used[j] = True
    comp_s.wait_stream(d2h_s)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
    e2e_value = whole_job_tokens_per_s(world, K, e2e_ms)

    # ---- device-resident steps, two passes of W + K steps each.  Pass 1 (the bench value):
    # K whole steps between two events.  Pass 2 (the kernel roofline): the next steps with
    # an event around every launch (those records cost a little time between launches,
    # so they stay out of pass 1).  The last step brings the context to CONTEXT.  A step is
    # one pnmix_append_decode call: the append runs inside the decode launch.
    def run_steps(first, n, events=None):
        for i in range(n):
            t = first + i
            if events:
                events[0][i].record()
            pm.pnmix_append_decode(cfg, kn_dev[t - T0], vn_dev[t - T0], q_dev[t - T0], cache, out)
            if events:
                events[1][i].record()

    base = T0 + n_e2e
    run_steps(base, W)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record()
        run_steps(base + W, K)
        e1.record()
        torch.cuda.synchronize()
    total_ms = e0.elapsed_time(e1)
    base2 = base + W + K
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(K)] for _ in range(2)]
    run_steps(base2, W)
    torch.cuda.synchronize()
    run_steps(base2 + W, K, ev)
    torch.cuda.synchronize()
    dec_ms = [ev[0][i].elapsed_time(ev[1][i]) for i in range(K)]
    total_ms = max_over_ranks(total_ms, pg, dev)
    err = cache.read_error()
    lens = cache.lengths().cpu().numpy()
    assert err == 0 and int(lens.min()) == CONTEXT, (err, lens)

    # algorithmic bytes of the timed launches (context after each append): the decode's,
    # plus the append's new rows (read, and stored into the residual window)
    units, G = B * HKV, HQ // HKV
    alg = [decode_bytes(base2 + W + i + 1, units, G, rec_bytes) + units * 2 * 2 * D * 2 for i in range(K)]
    avg_dec_s = sum(dec_ms) / K / 1e3
    achieved = sum(alg) / K / avg_dec_s / 1e9
    peak, peak_kind = measured_peaks()
    value = whole_job_tokens_per_s(world, K, total_ms)
    out_line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": stream_config(world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": captured_traffic(sum(alg) / K),
                     "algorithmic_bytes": sum(alg) / K, "kernel": "pnmix append + decode attention (one launch)",
                     "peak_source": peak_kind, "frac_of_8tbs": achieved / 8000.0},
        "decode_kernel_us": 1e3 * sum(dec_ms) / K,
        "append_fused": True,
        "prefill": {"tokens": PREFILL, "saliency_ms": saliency_ms, "quantize_ms": quant_ms,
                    "quantize_tokens_per_s": B * PREFILL / (quant_ms / 1e3)},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_host[0].numel() * 2 + kn_host[0].numel() * 2 * 2),
                "d2h_bytes_per_step": int(out_host[0].numel() * 4),
                "overlap": "inputs of step i+1 and the output of step i-1 copy during step i"},
        "gpu_launches": K,
        "clocks": clocks.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        out_line["cpu_baseline"] = cpu_baseline(args.seed, args.cpu_seconds, CONTEXT)
        try:
            out_line["cpu_baseline"]["all_cores"] = cpu_baseline_all_cores(args.seed, CONTEXT)
        except Exception as e:   # the host may forbid process pools; the one-core figure stands
            out_line["cpu_baseline"]["all_cores"] = {"unavailable": str(e)[:200]}
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(out_line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
