"""The decode step (pnmix_append + pnmix_decode_attention) captured once into a CUDA graph
and replayed step after step gives the same cache bytes and outputs as the same calls
issued one by one on a second cache."""
import numpy as np
import pytest
import torch

import workload
from gpu_harness import to_dev

pytestmark = pytest.mark.gpu


def test_append_and_decode_replay_from_a_cuda_graph():
    import decode_attention_prefill_b200 as pm
    B, Hq, Hkv, L, steps = 2, 8, 2, 90, 40
    G = Hq // Hkv
    kin = workload.rows(21, workload.K, B, Hkv, 0, L + steps)
    vin = workload.rows(21, workload.V, B, Hkv, 0, L + steps)
    qwin = workload.rows(21, workload.Q, B, Hq, L - 64, 64, group=G)
    cfg = pm.Config.make(Hq, Hkv)
    eager = pm.PNMixCache(cfg, B, 160, max_context=160)
    graphed = pm.PNMixCache(cfg, B, 160, max_context=160)
    for c in (eager, graphed):
        c.prefill(to_dev(qwin), to_dev(kin), to_dev(vin), L)

    k_in = torch.empty(B, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    v_in = torch.empty_like(k_in)
    q_in = torch.empty(B, Hq, 128, dtype=torch.bfloat16, device="cuda")
    out_g = torch.empty(B, Hq, 128, dtype=torch.float32, device="cuda")
    out_e = torch.empty_like(out_g)

    def step_inputs(t):
        q = workload.rows(21, workload.Q, B, Hq, t, 1, group=G)[:, :, 0]
        return (to_dev(np.ascontiguousarray(kin[:, :, t])), to_dev(np.ascontiguousarray(vin[:, :, t])),
                to_dev(q))

    # the first step runs eagerly on both caches (it also caches the launch geometry)
    k0, v0, q0 = step_inputs(L)
    for c, o in ((eager, out_e), (graphed, out_g)):
        pm.pnmix_append(cfg, k0, v0, c)
        pm.pnmix_decode_attention(cfg, q0, c, o)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pm.pnmix_append(cfg, k_in, v_in, graphed, stream=stream)
        pm.pnmix_decode_attention(cfg, q_in, graphed, out_g, stream=stream)
    # capture recorded the work without running it; the graphed cache is still one step in

    for t in range(L + 1, L + steps):
        kt, vt, qt = step_inputs(t)
        k_in.copy_(kt)
        v_in.copy_(vt)
        q_in.copy_(qt)
        graph.replay()
        pm.pnmix_append(cfg, kt, vt, eager)
        pm.pnmix_decode_attention(cfg, qt, eager, out_e)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out_g.cpu().numpy(), out_e.cpu().numpy())
    assert eager.read_error() == 0 and graphed.read_error() == 0
    np.testing.assert_array_equal(graphed.lengths().cpu().numpy(), eager.lengths().cpu().numpy())
    np.testing.assert_array_equal(graphed.records().cpu().numpy(), eager.records().cpu().numpy())
    np.testing.assert_array_equal(graphed.resid("k").cpu().numpy(), eager.resid("k").cpu().numpy())


def test_multi_token_decode_replays_from_a_cuda_graph():
    """A verify step of 16 new tokens per sequence (64 query rows per KV head: the tcgen05
    kernel) captured once and replayed with fresh queries gives the eager call's output
    bit for bit."""
    import decode_attention_prefill_b200 as pm
    B, Hq, Hkv, L, T = 2, 32, 8, 700, 16
    G = Hq // Hkv
    kin = workload.rows(5, workload.K, B, Hkv, 0, L + T)
    vin = workload.rows(5, workload.V, B, Hkv, 0, L + T)
    qwin = workload.rows(5, workload.Q, B, Hq, L - 64, 64, group=G)
    cfg = pm.Config.make(Hq, Hkv)
    cache = pm.PNMixCache(cfg, B, (L + T + 31) // 32 * 32 + 32, max_queries=T)
    cache.prefill(to_dev(qwin), to_dev(kin), to_dev(vin), L)
    for t in range(L, L + T):
        cache.append(to_dev(np.ascontiguousarray(kin[:, :, t])), to_dev(np.ascontiguousarray(vin[:, :, t])))

    def queries(seed):
        q = workload.rows(seed, workload.Q, B, Hq, L, T, group=G)
        return to_dev(np.ascontiguousarray(q.transpose(0, 2, 1, 3)))

    q_in = torch.empty(B, T, Hq, 128, dtype=torch.bfloat16, device="cuda")
    out_g = torch.empty(B, T, Hq, 128, dtype=torch.float32, device="cuda")
    out_e = torch.empty_like(out_g)
    q_in.copy_(queries(0))
    cache.attend_multi(q_in, out_g)   # eager first call: caches the launch geometry
    torch.cuda.synchronize()

    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        cache.attend_multi(q_in, out_g, stream=stream)
    for seed in (1, 2, 3):
        q = queries(seed)
        q_in.copy_(q)
        graph.replay()
        cache.attend_multi(q, out_e)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(out_g.cpu().numpy(), out_e.cpu().numpy())
    assert cache.read_error() == 0
