"""Shared helpers of the GPU parity tests: the same seeded inputs go through the
CUDA library (via its C ABI) and through the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workload

# Attention tolerance of the path: fp32 accumulation against the fp64 oracle.
MAX_ABS = 2e-3
REL_L2 = 1e-3


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()


class Case:
    """One workload instance: inputs on host and device, a GPU cache and an oracle cache."""

    def __init__(self, B, Hq, Hkv, L, k=8, bhi=4, blo=2, capacity=None, seed=0, W=64,
                 max_context=None, extra_tokens=0, score=0, n_prune=0, kernel=None, max_queries=None,
                 n_prune_slices=0):
        import decode_attention_prefill_b200 as pm
        self.pm = pm
        self.B, self.Hq, self.Hkv, self.G, self.L = B, Hq, Hkv, Hq // Hkv, L
        self.k, self.bhi, self.blo, self.seed = k, bhi, blo, seed
        self.W = min(L, W)
        total = L + extra_tokens
        self.capacity = capacity or ((total + 31) // 32 * 32 + 32)
        self.cfg = pm.Config.make(Hq, Hkv, bhi, blo, k, W, saliency_score=score, n_pruned_pairs=n_prune,
                                  decode_kernel=pm.DECODE_KERNELS[kernel or "auto"],
                                  n_pruned_slices=n_prune_slices)
        self.kin = workload.rows(seed, workload.K, B, Hkv, 0, max(total, 1))
        self.vin = workload.rows(seed, workload.V, B, Hkv, 0, max(total, 1))
        self.qwin = workload.rows(seed, workload.Q, B, Hq, L - self.W, max(self.W, 1), group=self.G) \
            if L > 0 else None
        self.cache = pm.PNMixCache(self.cfg, B, self.capacity, max_context=max_context,
                                   max_queries=max_queries or max(1, 8 // self.G))
        self.ocache = oracle.Cache(B, Hkv, self.capacity, k, bhi, blo, score=score, n_prune=n_prune,
                                   n_prune_slices=n_prune_slices)
        self.k_dev = to_dev(self.kin)
        self.v_dev = to_dev(self.vin)

    def prefill(self, check=True):
        L = self.L
        q_dev = to_dev(self.qwin)
        self.cache.prefill(q_dev, self.k_dev, self.v_dev, L)
        self.ocache.select(self.qwin, self.kin, L)
        self.ocache.prefill(self.kin, self.vin, L)
        torch.cuda.synchronize()
        if check:
            self.check_state()

    def append(self, t: int):
        """Append token t (row t of the generated K/V) to every sequence."""
        kn = np.ascontiguousarray(self.kin[:, :, t])
        vn = np.ascontiguousarray(self.vin[:, :, t])
        self.cache.append(to_dev(kn), to_dev(vn))
        self.ocache.append(kn, vn)

    def query(self, pos: int) -> np.ndarray:
        return workload.rows(self.seed, workload.Q, self.B, self.Hq, pos, 1, group=self.G)[:, :, 0]

    def query_multi(self, pos0: int, T: int) -> np.ndarray:
        """Queries of positions pos0 .. pos0+T-1: bf16 [B][T][Hq][128]."""
        q = workload.rows(self.seed, workload.Q, self.B, self.Hq, pos0, T, group=self.G)
        return np.ascontiguousarray(q.transpose(0, 2, 1, 3))

    def attend_multi(self, q: np.ndarray):
        """GPU multi-query decode vs the oracle's causal rows: fp32 and fp64 [B][T][Hq][128]."""
        out = self.cache.attend_multi(to_dev(q)).cpu().numpy()
        want = self.ocache.attend_multi(q)
        return out, want

    def check_state(self, units=None):
        c, o = self.cache, self.ocache
        torch.cuda.synchronize()
        np.testing.assert_array_equal(c.lengths().cpu().numpy(), o.len)
        mask = c.pair_mask().cpu().numpy().view(np.uint64)
        np.testing.assert_array_equal(mask, o.mask)
        np.testing.assert_array_equal(c.pair_idx().cpu().numpy()[:, :, :self.k], o.idx[:, :, :self.k])
        np.testing.assert_array_equal(c.perm().cpu().numpy(), o.perm)
        np.testing.assert_array_equal(c.pair_scores().cpu().numpy().view(np.uint32),
                                      o.scores.view(np.uint32))
        n = int(o.len.min())
        ng = n // 32
        rec = c.records().cpu().numpy()
        if units is None:
            np.testing.assert_array_equal(rec[:, :, :ng], o.records[:, :, :ng])
        else:
            for b, h in units:
                np.testing.assert_array_equal(rec[b, h, :ng], o.records[b, h, :ng])
        r = n % 32
        if r:
            np.testing.assert_array_equal(c.resid("k").cpu().numpy().view(np.uint16)[:, :, :r],
                                          o.resid_k[:, :, :r])
            np.testing.assert_array_equal(c.resid("v").cpu().numpy().view(np.uint16)[:, :, :r],
                                          o.resid_v[:, :, :r])

    def attend(self, q: np.ndarray, units=None):
        """Run the GPU decode; return (gpu fp32 [B][Hq][128], oracle fp64 on the listed units)."""
        out = self.cache.attend(to_dev(q)).cpu().numpy()
        want = self.ocache.attend(q, units)
        return out, want


def assert_close(got: np.ndarray, want: np.ndarray, units=None, G=None):
    """Max-abs <= 2e-3 and relative L2 <= 1e-3 (over the compared rows)."""
    if units is not None:
        rows = [(b, h * G + j) for b, h in units for j in range(G)]
        got = np.stack([got[b, r] for b, r in rows])
        want = np.stack([want[b, r] for b, r in rows])
    assert np.all(np.isfinite(got))
    err = np.abs(got.astype(np.float64) - want)
    rel = np.linalg.norm(got.astype(np.float64) - want) / max(np.linalg.norm(want), 1e-30)
    assert err.max() <= MAX_ABS, f"max-abs {err.max():.3e}"
    assert rel <= REL_L2, f"rel-L2 {rel:.3e}"
    return float(err.max()), float(rel)
