"""Multi-process host logic of the benchmark (gloo, world size 2, CPU).

The decode path shards into independent (sequence, KV head) units, so ranks share no
data; the only collectives are the barrier around the timed region and the max-over-ranks
reduction of the measured time.  These tests run that logic on CPU ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_setup(None)
    assert (w, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # each rank: its own sequences (seed offset), its own measured time; the bench's own
    # helpers reduce it to the slowest rank's and form the whole-job value
    seed = 0 + 7919 * rank
    dist.barrier()
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
    value = bench.whole_job_tokens_per_s(world, 4, ms)
    q.put((rank, seed, ms, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_shard_sequences_and_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    assert out[0][1] != out[1][1]                 # distinct sequences per rank
    assert out[0][2] == out[1][2] == 15.0         # the max over ranks
    assert out[0][3] == out[1][3] == pytest.approx(2 * 16 * 4 / 0.015)


def test_reference_arm_other_ranks_exit_quietly(capsys):
    import bench

    class A:
        steps, warmup, seed = 1, 0, 0
    assert bench.run_reference(A(), 2, 1) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_contract_line(capsys):
    """Rank 0 of the reference arm times the oracle and prints one JSON line with the
    contract's keys, its own cpu_baseline and an e2e block that moves no bytes."""
    import json

    import bench

    class A:
        steps, warmup, seed = 1, 0, 0
    assert bench.run_reference(A(), 1, 0) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "stream_32k"
    assert d["config"] == bench.stream_config(1)          # the GPU arm's config keys
    assert d["sampled"]["units_per_full_step"] == bench.B * bench.HKV
    # ms_per_step is the wall time actually spent per sampled step; value scales it to a step
    assert abs(d["value"] - bench.B / (d["ms_per_step"] / 1e3 * bench.B * bench.HKV)) <= 1e-6 * d["value"]
