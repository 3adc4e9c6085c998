"""Reference oracle of the PN-Mix KV-cache path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``decode_attention_prefill_b200``) never imports it and fails loudly when its
own extension is missing.

The arithmetic lives in ``pnmix_oracle.c`` (plain single-threaded C, compiled
here with gcc on first use); this module only marshals numpy arrays and loops
over (sequence, KV head) units.  It shares no code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pnmix_oracle.c")
_LIB = os.path.join(_HERE, "libpnmix_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-mno-fma"]

_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile pnmix_oracle.c into libpnmix_oracle.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags.c_contiguous, "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, i, d, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float
            sig = {
                "orc_f32_from_bf16": (f, [ctypes.c_uint16]),
                "orc_f32_from_f16": (f, [ctypes.c_uint16]),
                "orc_f16_from_f32": (ctypes.c_uint16, [f]),
                "orc_pair_scores": (None, [i, i, i, vp, vp, vp, vp, vp]),
                "orc_pair_scores_mode": (None, [i, i, i, i, vp, vp, vp]),
                "orc_attend_unit_rows": (i, [i, vp, d, i, i, i, vp, vp, i, vp, vp, i, vp, vp]),
                "orc_pruned_pairs": (ctypes.c_uint64, [vp, i]),
                "orc_ers": (ctypes.c_uint32, [ctypes.c_uint32, i]),
                "orc_shrink_record": (i, [i, i, i, vp, vp]),
                "orc_prune_queries": (None, [i, vp, i, vp]),
                "orc_pruned_slices": (ctypes.c_uint32, [i, vp, vp, i, i]),
                "orc_prune_query_slices": (None, [i, vp, vp, i, i, vp]),
                "orc_topk": (None, [vp, i, vp, vp]),
                "orc_position_order": (i, [ctypes.c_uint64, vp]),
                "orc_minmax_quant": (None, [vp, i, i, vp, vp, vp]),
                "orc_key_group": (None, [vp, vp, i, i, i, vp, vp, vp]),
                "orc_value_token": (None, [vp, i, vp, vp, vp]),
                "orc_record_bytes": (ctypes.c_long, [i, i, i]),
                "orc_pack_record": (i, [i, i, i, vp, vp, vp, vp, vp, vp, vp]),
                "orc_unpack_record": (i, [i, i, i, vp, vp, vp, vp, vp, vp, vp]),
                "orc_make_record": (i, [i, i, i, i, vp, vp, vp, vp]),
                "orc_prefill_unit": (i, [i, i, i, i, vp, i, vp, vp, vp, vp, vp]),
                "orc_append_unit": (i, [i, i, i, i, vp, i, vp, vp, vp, vp, vp]),
                "orc_attention_core": (None, [i, vp, vp, vp, ctypes.c_long, d, vp]),
                "orc_attend_unit": (i, [i, vp, d, i, i, i, vp, vp, i, vp, vp, i, vp, vp, vp]),
                "orc_exact_attention": (None, [i, vp, vp, vp, ctypes.c_long, d, vp]),
                "orc_key_code_bits": (d, [i, i, i]),
                "orc_mean_query": (None, [i, i, vp, vp]),
                "orc_group_scores": (None, [vp, i, vp, vp]),
                "orc_route_groups": (None, [i, vp, i, vp]),
                "orc_attend_two": (i, [i, vp, d, i, i, i, vp, vp, i, i, vp, vp, i, vp, vp, i, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


# ---------------------------------------------------------------- formats

def f16_from_f32(x: float) -> int:
    return int(lib().orc_f16_from_f32(float(np.float32(x))))


def f32_from_f16(h: int) -> float:
    return float(lib().orc_f32_from_f16(int(h)))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


# ---------------------------------------------------------------- step 1

def pair_scores(qwin: np.ndarray, k: np.ndarray):
    """qwin bf16 [G][W][128], k bf16 [L][128] -> (scores, key norms, query norms), fp32 [64]."""
    qwin = np.ascontiguousarray(qwin, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    G, W, _ = qwin.shape
    L = k.shape[0]
    s = np.zeros(64, np.float32)
    kn = np.zeros(64, np.float32)
    qn = np.zeros(64, np.float32)
    lib().orc_pair_scores(G, W, L, _p(qwin), _p(k), _p(s), _p(kn), _p(qn))
    return s, kn, qn


SCORE_PNMIX, SCORE_KEY_ONLY, SCORE_RANGE_QUERY = 0, 1, 2


def pruned_pairs(q_row: np.ndarray, n_prune: int) -> int:
    """Mask of the pairs one query row (bf16 [128]) prunes, see orc_pruned_pairs."""
    q_row = np.ascontiguousarray(q_row, dtype=np.uint16)
    return int(lib().orc_pruned_pairs(_p(q_row), n_prune))


def prune_queries(q: np.ndarray, n_prune: int) -> np.ndarray:
    """bf16 [..., 128] query rows with each row's pruned pairs zeroed."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    out = np.empty_like(q)
    if n_prune <= 0:
        out[...] = q
        return out
    lib().orc_prune_queries(q.size // 128, _p(q), n_prune, _p(out))
    return out


def pruned_slices(q_rows: np.ndarray, perm: np.ndarray, k: int, n_prune: int) -> int:
    """Mask of the position slices one unit's query rows (bf16 [rows][128]) prune, see
    orc_pruned_slices."""
    q_rows = np.ascontiguousarray(q_rows, dtype=np.uint16).reshape(-1, 128)
    perm = np.ascontiguousarray(perm, dtype=np.uint8)
    return int(lib().orc_pruned_slices(q_rows.shape[0], _p(q_rows), _p(perm), k, n_prune))


def prune_query_slices(q_rows: np.ndarray, perm: np.ndarray, k: int, n_prune: int) -> np.ndarray:
    """bf16 [rows][128] query rows of one unit with the channels of its pruned slices zeroed."""
    q_rows = np.ascontiguousarray(q_rows, dtype=np.uint16)
    out = np.empty_like(q_rows)
    if n_prune <= 0:
        out[...] = q_rows
        return out
    perm = np.ascontiguousarray(perm, dtype=np.uint8)
    lib().orc_prune_query_slices(q_rows.size // 128, _p(q_rows), _p(perm), k, n_prune, _p(out))
    return out


def pair_scores_mode(mode: int, qwin: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Scores fp32 [64] under statistic `mode` (SCORE_*), see orc_pair_scores_mode."""
    qwin = np.ascontiguousarray(qwin, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    G, W, _ = qwin.shape
    s = np.zeros(64, np.float32)
    lib().orc_pair_scores_mode(mode, G, W, k.shape[0], _p(qwin), _p(k), _p(s))
    return s


def ers(x: int, b: int) -> int:
    """Equivalent right shift of a 2b-bit code to b bits, see orc_ers."""
    return int(lib().orc_ers(x, b))


def topk(scores: np.ndarray, k: int):
    """-> (idx uint8 [k] ascending, mask int)."""
    scores = np.ascontiguousarray(scores, dtype=np.float32)
    idx = np.zeros(max(k, 1), np.uint8)
    mask = np.zeros(1, np.uint64)
    lib().orc_topk(_p(scores), k, _p(idx), _p(mask))
    return idx[:k].copy(), int(mask[0])


def position_order(mask: int):
    perm = np.zeros(128, np.uint8)
    nhi = lib().orc_position_order(ctypes.c_uint64(mask), _p(perm))
    return perm, nhi


def select_unit(qwin: np.ndarray, k: np.ndarray, n_salient: int, mode: int = SCORE_PNMIX):
    """Full step 1 of one (b, KV head): scores, idx, mask, perm."""
    s = pair_scores(qwin, k)[0] if mode == SCORE_PNMIX else pair_scores_mode(mode, qwin, k)
    idx, mask = topk(s, n_salient)
    perm, _ = position_order(mask)
    return s, idx, mask, perm


# ---------------------------------------------------------------- quantizer

def minmax_quant(x: np.ndarray, bits: int):
    """x fp32 [n] -> (codes uint8 [n], s16 bits, z16 bits)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    codes = np.zeros(x.shape[0], np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib().orc_minmax_quant(_p(x), x.shape[0], bits, _p(s), _p(z), _p(codes))
    return codes, int(s[0]), int(z[0])


def key_group(rows: np.ndarray, perm: np.ndarray, nhi: int, bhi: int, blo: int):
    rows = np.ascontiguousarray(rows, dtype=np.uint16)
    perm = np.ascontiguousarray(perm, dtype=np.uint8)
    codes = np.zeros((32, 128), np.uint8)
    s = np.zeros(128, np.uint16)
    z = np.zeros(128, np.uint16)
    lib().orc_key_group(_p(rows), _p(perm), nhi, bhi, blo, _p(codes), _p(s), _p(z))
    return codes, s, z


def value_token(row: np.ndarray, bits: int = 2):
    row = np.ascontiguousarray(row, dtype=np.uint16)
    codes = np.zeros(128, np.uint8)
    s = np.zeros(4, np.uint16)
    z = np.zeros(4, np.uint16)
    lib().orc_value_token(_p(row), bits, _p(codes), _p(s), _p(z))
    return codes, s, z


# ---------------------------------------------------------------- layout

def record_bytes(k: int, bhi: int, blo: int) -> int:
    return int(lib().orc_record_bytes(k, bhi, blo))


def key_code_bits(k: int, bhi: int, blo: int) -> float:
    return float(lib().orc_key_code_bits(k, bhi, blo))


def pack_record(k, bhi, blo, kcodes, ks, kz, vcodes, vs, vz) -> np.ndarray:
    R = record_bytes(k, bhi, blo)
    rec = np.zeros(R, np.uint8)
    arrs = [np.ascontiguousarray(a, dtype=t) for a, t in
            ((kcodes, np.uint8), (ks, np.uint16), (kz, np.uint16), (vcodes, np.uint8),
             (vs, np.uint16), (vz, np.uint16))]
    rc = lib().orc_pack_record(k, bhi, blo, *[_p(a) for a in arrs], _p(rec))
    if rc:
        raise ValueError("unsupported record parameters")
    return rec


def unpack_record(k, bhi, blo, rec):
    rec = np.ascontiguousarray(rec, dtype=np.uint8)
    kc = np.zeros((32, 128), np.uint8)
    ks = np.zeros(128, np.uint16)
    kz = np.zeros(128, np.uint16)
    vc = np.zeros((32, 128), np.uint8)
    vs = np.zeros((32, 4), np.uint16)
    vz = np.zeros((32, 4), np.uint16)
    rc = lib().orc_unpack_record(k, bhi, blo, _p(rec), _p(kc), _p(ks), _p(kz), _p(vc), _p(vs),
                                 _p(vz))
    if rc:
        raise ValueError("unsupported record parameters")
    return kc, ks, kz, vc, vs, vz


# ---------------------------------------------------------------- whole caches

class Cache:
    """Host image of the cache regions the tests compare with the device."""

    def __init__(self, batch, n_kv, capacity, k, bhi, blo, bv=2, score=SCORE_PNMIX, n_prune=0,
                 n_prune_slices=0):
        self.batch, self.n_kv, self.capacity = batch, n_kv, capacity
        self.k, self.bhi, self.blo, self.bv = k, bhi, blo, bv
        self.score = score
        self.n_prune = n_prune   # query pairs each decode row drops (0: none)
        self.n_prune_slices = n_prune_slices   # low-precision key slices each unit drops
        self.R = record_bytes(k, bhi, blo)
        if not self.R:
            raise ValueError("unsupported bit point")
        self.records = np.zeros((batch, n_kv, capacity // 32, self.R), np.uint8)
        self.resid_k = np.zeros((batch, n_kv, 32, 128), np.uint16)
        self.resid_v = np.zeros((batch, n_kv, 32, 128), np.uint16)
        self.len = np.zeros(batch, np.int32)
        self.idx = np.zeros((batch, n_kv, 64), np.uint8)
        self.mask = np.zeros((batch, n_kv), np.uint64)
        self.perm = np.zeros((batch, n_kv, 128), np.uint8)
        self.scores = np.zeros((batch, n_kv, 64), np.float32)

    def select(self, qwin: np.ndarray, kin: np.ndarray, L: int, units=None):
        """qwin bf16 [B][Hq][W][128]; kin bf16 [B][Hkv][>=L][128]."""
        G = qwin.shape[1] // self.n_kv
        for b, h in units or [(b, h) for b in range(self.batch) for h in range(self.n_kv)]:
            s, idx, mask, perm = select_unit(qwin[b, h * G:(h + 1) * G], kin[b, h, :L], self.k, self.score)
            self.scores[b, h] = s
            self.idx[b, h, :self.k] = idx
            self.mask[b, h] = mask
            self.perm[b, h] = perm

    def prefill(self, kin: np.ndarray, vin: np.ndarray, L: int, units=None):
        """Quantize tokens [0, L) of kin / vin (bf16 [B][Hkv][>=L][128])."""
        for b, h in units or [(b, h) for b in range(self.batch) for h in range(self.n_kv)]:
            kk = np.ascontiguousarray(kin[b, h, :L])
            vv = np.ascontiguousarray(vin[b, h, :L])
            rec = self.records[b, h]
            rk = self.resid_k[b, h]
            rv = self.resid_v[b, h]
            rc = lib().orc_prefill_unit(self.k, self.bhi, self.blo, self.bv,
                                        _p(self.perm[b, h]), L, _p(kk), _p(vv), _p(rec), _p(rk),
                                        _p(rv))
            assert rc == 0
        self.len[:] = L

    def append(self, knew: np.ndarray, vnew: np.ndarray):
        """knew, vnew bf16 [B][Hkv][128]."""
        for b in range(self.batch):
            n = int(self.len[b])
            if n >= self.capacity:
                continue
            for h in range(self.n_kv):
                lib().orc_append_unit(self.k, self.bhi, self.blo, self.bv, _p(self.perm[b, h]), n,
                                      _p(np.ascontiguousarray(knew[b, h])),
                                      _p(np.ascontiguousarray(vnew[b, h])), _p(self.records[b, h]),
                                      _p(self.resid_k[b, h]), _p(self.resid_v[b, h]))
            self.len[b] = n + 1

    def attend_unit(self, q: np.ndarray, b: int, h: int, scale: float | None = None) -> np.ndarray:
        """q bf16 [G][128] of KV head h of sequence b -> fp64 [G][128]."""
        q = prune_query_slices(prune_queries(q, self.n_prune), self.perm[b, h], self.k, self.n_prune_slices)
        G = q.shape[0]
        n = int(self.len[b])
        out = np.zeros((G, 128), np.float64)
        rc = lib().orc_attend_unit(G, _p(q), scale if scale else 1.0 / np.sqrt(128.0), self.k,
                                   self.bhi, self.blo, _p(self.perm[b, h]),
                                   _p(self.records[b, h]), n // 32, _p(self.resid_k[b, h]),
                                   _p(self.resid_v[b, h]), n % 32, None, None, _p(out))
        assert rc == 0
        return out

    def shrunk(self) -> "Cache":
        """The cache with its salient key positions shrunk from b_hi to b_lo = b_hi / 2 bits
        (orc_shrink_record on every full group): a k = 0 cache in the same position order."""
        out = Cache(self.batch, self.n_kv, self.capacity, 0, self.bhi, self.blo, self.bv,
                    self.score, self.n_prune, self.n_prune_slices)
        out.perm[:] = self.perm
        out.scores[:] = self.scores
        out.len[:] = self.len
        out.resid_k[:] = self.resid_k
        out.resid_v[:] = self.resid_v
        for b in range(self.batch):
            for h in range(self.n_kv):
                for g in range(int(self.len[b]) // 32):
                    rc = lib().orc_shrink_record(self.k, self.bhi, self.blo, _p(self.records[b, h, g]),
                                                 _p(out.records[b, h, g]))
                    assert rc == 0
        return out

    def attend_rows(self, q: np.ndarray, n_visible, b: int, h: int, scale: float | None = None) -> np.ndarray:
        """q bf16 [rows][128] of KV head h of sequence b, row r over the first n_visible[r]
        cached tokens -> fp64 [rows][128]."""
        q = prune_query_slices(prune_queries(q, self.n_prune), self.perm[b, h], self.k, self.n_prune_slices)
        nv = np.ascontiguousarray(n_visible, dtype=np.int32)
        n = int(self.len[b])
        out = np.zeros((q.shape[0], 128), np.float64)
        rc = lib().orc_attend_unit_rows(q.shape[0], _p(q), scale if scale else 1.0 / np.sqrt(128.0),
                                        self.k, self.bhi, self.blo, _p(self.perm[b, h]),
                                        _p(self.records[b, h]), n // 32, _p(self.resid_k[b, h]),
                                        _p(self.resid_v[b, h]), n % 32, _p(nv), _p(out))
        assert rc == 0
        return out

    def attend_multi(self, q: np.ndarray, heads=None) -> np.ndarray:
        """T new queries per sequence after their T tokens were appended: q bf16
        [B][T][Hq][128] -> fp64 [B][T][Hq][128], query j over the first len - T + 1 + j
        tokens (only the listed (b, kv head) units)."""
        B, T, Hq, _ = q.shape
        G = Hq // self.n_kv
        out = np.full((B, T, Hq, 128), np.nan)
        for b, h in heads or [(b, h) for b in range(B) for h in range(self.n_kv)]:
            rows = np.ascontiguousarray(q[b, :, h * G:(h + 1) * G].reshape(T * G, 128))
            nv = [int(self.len[b]) - T + 1 + j for j in range(T) for _ in range(G)]
            out[b, :, h * G:(h + 1) * G] = self.attend_rows(rows, nv, b, h).reshape(T, G, 128)
        return out

    def attend(self, q: np.ndarray, heads=None) -> np.ndarray:
        """q bf16 [B][Hq][128] -> fp64 [B][Hq][128] (only the listed (b, kv head) units)."""
        B, Hq, _ = q.shape
        G = Hq // self.n_kv
        out = np.full((B, Hq, 128), np.nan)
        for b, h in heads or [(b, h) for b in range(B) for h in range(self.n_kv)]:
            out[b, h * G:(h + 1) * G] = self.attend_unit(q[b, h * G:(h + 1) * G], b, h)
        return out


# ---------------------------------------------------------------- two-precision mixing
# SemKV abstract (token-level mixing of two adjacent precisions by a model-internal
# rank), with 32-token groups as the unit and two salient-pair counts as the precisions.

def mean_query(qwin_unit: np.ndarray) -> np.ndarray:
    """qwin_unit bf16 [G][W][128] -> fp32 [128] (orc_mean_query)."""
    q = np.ascontiguousarray(qwin_unit, dtype=np.uint16)
    out = np.zeros(128, np.float32)
    lib().orc_mean_query(q.shape[0], q.shape[1], _p(q), _p(out))
    return out


def group_scores(qbar: np.ndarray, k_unit: np.ndarray, L: int) -> np.ndarray:
    """Largest mean-query logit of each full 32-token group of k_unit (bf16 [>=L][128])."""
    kk = np.ascontiguousarray(k_unit[:L], dtype=np.uint16)
    qb = np.ascontiguousarray(qbar, dtype=np.float32)
    out = np.zeros(max(L // 32, 1), np.float32)
    lib().orc_group_scores(_p(qb), L, _p(kk), _p(out))
    return out[:L // 32]


def route_groups(scores: np.ndarray, n_hi: int) -> np.ndarray:
    """uint8 [ng]: 1 for the n_hi best-ranked groups (ties: lower index first)."""
    sc = np.ascontiguousarray(scores, dtype=np.float32)
    out = np.zeros(max(len(sc), 1), np.uint8)
    lib().orc_route_groups(len(sc), _p(sc), n_hi, _p(out))
    return out[:len(sc)]


def hi_groups(ng: int, percent: int) -> int:
    """Groups of a unit at the high precision: floor(ng * percent / 100)."""
    return ng * percent // 100


class TwoPrecision:
    """Host image of a two-precision cache: per (sequence, KV head) the full groups of the
    prefill are ranked by group_scores of the saliency window's mean query; the best
    hi_groups(ng, percent) of them are quantized with k_hi salient pairs into `hi`, the
    others with k_lo into `lo`, each part in ascending group order.  The residual tail
    and every appended token go to `lo`.  Both parts take their salient pairs from the
    same prefill statistic (top k_hi and top k_lo of one score vector)."""

    def __init__(self, batch, n_kv, capacity, k_hi, k_lo, bhi, blo, percent, score=SCORE_PNMIX):
        if not 0 <= percent <= 100:
            raise ValueError("percent outside [0, 100]")
        self.batch, self.n_kv, self.percent = batch, n_kv, percent
        self.hi = Cache(batch, n_kv, capacity, k_hi, bhi, blo, score=score)
        self.lo = Cache(batch, n_kv, capacity, k_lo, bhi, blo, score=score)
        self.route = np.zeros((batch, n_kv, capacity // 32), np.uint8)

    def prefill(self, qwin: np.ndarray, kin: np.ndarray, vin: np.ndarray, L: int):
        """qwin bf16 [B][Hq][W][128] (the saliency window); kin, vin bf16 [B][Hkv][>=L][128]."""
        self.hi.select(qwin, kin, L)
        self.lo.select(qwin, kin, L)
        G = qwin.shape[1] // self.n_kv
        ng = L // 32
        n_hi = hi_groups(ng, self.percent)
        for b in range(self.batch):
            for h in range(self.n_kv):
                qbar = mean_query(qwin[b, h * G:(h + 1) * G])
                route = route_groups(group_scores(qbar, kin[b, h], L), n_hi)
                self.route[b, h, :ng] = route
                for part, take in ((self.hi, 1), (self.lo, 0)):
                    rows = [np.arange(32 * g, 32 * g + 32) for g in range(ng) if route[g] == take]
                    if take == 0:
                        rows.append(np.arange(32 * ng, L))
                    idx = np.concatenate(rows) if rows else np.zeros(0, np.int64)
                    kk = np.ascontiguousarray(kin[b, h, idx], dtype=np.uint16)
                    vv = np.ascontiguousarray(vin[b, h, idx], dtype=np.uint16)
                    rc = lib().orc_prefill_unit(part.k, part.bhi, part.blo, part.bv, _p(part.perm[b, h]),
                                                len(idx), _p(kk), _p(vv), _p(part.records[b, h]),
                                                _p(part.resid_k[b, h]), _p(part.resid_v[b, h]))
                    assert rc == 0
            self.hi.len[b] = 32 * n_hi
            self.lo.len[b] = L - 32 * n_hi

    def append(self, knew: np.ndarray, vnew: np.ndarray):
        self.lo.append(knew, vnew)

    def attend(self, q: np.ndarray, heads=None) -> np.ndarray:
        """q bf16 [B][Hq][128] -> fp64 [B][Hq][128]: softmax over both parts' tokens."""
        B, Hq, _ = q.shape
        G = Hq // self.n_kv
        hi, lo = self.hi, self.lo
        out = np.full((B, Hq, 128), np.nan)
        for b, h in heads or [(b, h) for b in range(B) for h in range(self.n_kv)]:
            qq = np.ascontiguousarray(q[b, h * G:(h + 1) * G], dtype=np.uint16)
            o = np.zeros((G, 128), np.float64)
            n_lo = int(lo.len[b])
            rc = lib().orc_attend_two(G, _p(qq), 1.0 / np.sqrt(128.0), hi.bhi, hi.blo,
                                      hi.k, _p(hi.perm[b, h]), _p(hi.records[b, h]), int(hi.len[b]) // 32,
                                      lo.k, _p(lo.perm[b, h]), _p(lo.records[b, h]), n_lo // 32,
                                      _p(lo.resid_k[b, h]), _p(lo.resid_v[b, h]), n_lo % 32, _p(o))
            assert rc == 0
            out[b, h * G:(h + 1) * G] = o
        return out


def attend_passthrough(q: np.ndarray, kin: np.ndarray, vin: np.ndarray, n_groups: int,
                       resid_k: np.ndarray, resid_v: np.ndarray, n_resid: int,
                       scale: float | None = None) -> np.ndarray:
    """The 16-bit setting of orc_attend_unit: dequantized values are the bf16 inputs."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    G = q.shape[0]
    out = np.zeros((G, 128), np.float64)
    dummy = np.zeros(128, np.uint8)
    rc = lib().orc_attend_unit(G, _p(q), scale if scale else 1.0 / np.sqrt(128.0), 0, 16, 16,
                               _p(np.arange(128, dtype=np.uint8)), _p(dummy), n_groups,
                               _p(np.ascontiguousarray(resid_k, dtype=np.uint16)),
                               _p(np.ascontiguousarray(resid_v, dtype=np.uint16)), n_resid,
                               _p(np.ascontiguousarray(kin, dtype=np.uint16)),
                               _p(np.ascontiguousarray(vin, dtype=np.uint16)), _p(out))
    assert rc == 0
    return out


def exact_attention(q: np.ndarray, kin: np.ndarray, vin: np.ndarray,
                    scale: float | None = None) -> np.ndarray:
    """Plain softmax attention of q bf16 [G][128] over bf16 kin/vin [n][128], fp64."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    kin = np.ascontiguousarray(kin, dtype=np.uint16)
    vin = np.ascontiguousarray(vin, dtype=np.uint16)
    out = np.zeros((q.shape[0], 128), np.float64)
    lib().orc_exact_attention(q.shape[0], _p(q), _p(kin), _p(vin), kin.shape[0],
                              scale if scale else 1.0 / np.sqrt(128.0), _p(out))
    return out


def attention_core(q: np.ndarray, khat: np.ndarray, vhat: np.ndarray, scale: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float64)
    khat = np.ascontiguousarray(khat, dtype=np.float64)
    vhat = np.ascontiguousarray(vhat, dtype=np.float64)
    out = np.zeros((q.shape[0], 128), np.float64)
    lib().orc_attention_core(q.shape[0], _p(q), _p(khat), _p(vhat), khat.shape[0], scale, _p(out))
    return out
