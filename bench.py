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
DECODE_CAPTURE = {"sources_sha256_16": "9494d23a19085423", "traffic_bytes": 425101568,
                  "algorithmic_bytes": 420855808}
DECODE_SOURCES = ["decode_attention_prefill_b200/csrc/decode_mma.cu",
                  "decode_attention_prefill_b200/csrc/decode_common.cuh",
                  "decode_attention_prefill_b200/csrc/common.cuh"]


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
    ap.add_argument("--profile-decode", action="store_true",
                    help="build the 32K state, then run only --warmup + --steps decode launches "
                         "(small device footprint, for profiler captures); prints no bench line")
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
                   for p in q_positions])
    return kin, vin, qwin, qs


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
    total = sum(times)
    value = B * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "stream_32k", "batch": B, "n_q_heads": HQ, "n_kv_heads": HKV,
                   "context": CONTEXT, "key_code_bits": 2.25},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": "oracle append + decode attention of 1 of 128 (sequence, KV head) "
                                   "units per step, scaled to a full 16-sequence step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)

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
    if 2 * (W + K) >= CONTEXT - PREFILL:
        raise SystemExit("--steps/--warmup too large for the 32K stream")
    T0 = CONTEXT - 2 * (W + K)           # tokens already cached before the e2e steps
    seed = args.seed + 7919 * rank        # each rank: its own 16 sequences
    positions = list(range(T0, CONTEXT))  # one query per step
    kin, vin, qwin, qs = gen_inputs(seed, CONTEXT, positions)

    cfg = pm.Config.make(HQ, HKV, BHI, BLO, K_SALIENT, WINDOW)
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
        # decode-only launches at context T0 (for profiler captures)
        for i in range(W + K):
            pm.pnmix_decode_attention(cfg, q_dev[0], cache, out)
        torch.cuda.synchronize()
        print(json.dumps({"profile_decode": True, "launches": W + K, "context": T0,
                          "error_word": cache.read_error()}), flush=True)
        return 0
    rec_bytes = cache.c.record_bytes

    # ---- end-to-end through host buffers (pinned), e2e steps T0 .. T0+n_e2e-1
    q_host = torch.from_numpy(qs).view(torch.bfloat16).pin_memory()
    kn_host = kn_dev[:n_e2e].cpu().pin_memory()
    vn_host = vn_dev[:n_e2e].cpu().pin_memory()
    out_host = torch.empty(B, HQ, D, dtype=torch.float32).pin_memory()
    staging = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(n_e2e):
        if i == W:
            if pg:
                pg.barrier()
            torch.cuda.synchronize()
            e0.record()
        pm.decode_step_host(cache, q_host[i], kn_host[i], vn_host[i], out_host, staging)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if pg:
        t = torch.tensor([e2e_ms], device=dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * B * K / (e2e_ms / 1e3)

    # ---- device-resident timed steps: tokens T0+n_e2e .. CONTEXT-1
    base = T0 + n_e2e
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    app_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(W):
        t = base + i
        pm.pnmix_append(cfg, kn_dev[t - T0], vn_dev[t - T0], cache)
        pm.pnmix_decode_attention(cfg, q_dev[t - T0], cache, out)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record()
        for i in range(K):
            t = base + W + i
            app_ev[i][0].record()
            pm.pnmix_append(cfg, kn_dev[t - T0], vn_dev[t - T0], cache)
            app_ev[i][1].record()
            pm.pnmix_decode_attention(cfg, q_dev[t - T0], cache, out)
            dec_ev[i][1].record()
        e1.record()
        torch.cuda.synchronize()
    total_ms = e0.elapsed_time(e1)
    dec_ms = [app_ev[i][1].elapsed_time(dec_ev[i][1]) for i in range(K)]
    app_ms = [app_ev[i][0].elapsed_time(app_ev[i][1]) for i in range(K)]
    if pg:
        t = torch.tensor([total_ms], device=dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
        total_ms = float(t.item())
    err = cache.read_error()
    lens = cache.lengths().cpu().numpy()
    assert err == 0 and int(lens.min()) == CONTEXT, (err, lens)

    # algorithmic bytes of the timed decode launches (context after each append)
    units, G = B * HKV, HQ // HKV
    alg = [decode_bytes(base + W + i + 1, units, G, rec_bytes) for i in range(K)]
    avg_dec_s = sum(dec_ms) / K / 1e3
    achieved = sum(alg) / K / avg_dec_s / 1e9
    peak, peak_kind = measured_peaks()
    value = world * B * K / (total_ms / 1e3)
    out_line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "stream_32k", "batch_per_gpu": B, "n_q_heads": HQ, "n_kv_heads": HKV,
                   "head_dim": D, "context": CONTEXT, "prefill": PREFILL, "salient_pairs": K_SALIENT,
                   "key_bits": [BHI, BLO], "value_bits": 2, "key_code_bits": 2.25,
                   "parallelism": f"dp{world}", "l2": "inputs larger than L2 (419 MB cache read per step)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": captured_traffic(sum(alg) / K),
                     "algorithmic_bytes": sum(alg) / K, "kernel": "pnmix decode attention",
                     "peak_source": peak_kind, "frac_of_8tbs": achieved / 8000.0},
        "decode_kernel_us": 1e3 * sum(dec_ms) / K,
        "append_kernel_us": 1e3 * sum(app_ms) / K,
        "prefill": {"tokens": PREFILL, "saliency_ms": saliency_ms, "quantize_ms": quant_ms,
                    "quantize_tokens_per_s": B * PREFILL / (quant_ms / 1e3)},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(q_host[0].numel() * 2 + kn_host[0].numel() * 2 * 2),
                "d2h_bytes_per_step": int(out_host.numel() * 4)},
        "gpu_launches": 2 * K,
        "clocks": clocks.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        out_line["cpu_baseline"] = cpu_baseline(args.seed, args.cpu_seconds, CONTEXT)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank == 0:
        print(json.dumps(out_line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
