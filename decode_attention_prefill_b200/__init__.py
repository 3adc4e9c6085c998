"""Python binding of libpnmix.so, the B200 PN-Mix KV-cache library (include/pnmix.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  Importing this package
raises if the compiled library is missing; there is no CPU fallback.

Entry points keep the C names:

    pnmix_select_pairs(cfg, q_window, k, L, cache)      prefill: salient pairs
    pnmix_quantize_keys(cfg, k, L, cache)               prefill: packed keys
    pnmix_quantize_values(cfg, v, L, cache)             prefill: packed values
    pnmix_append(cfg, k_new, v_new, cache)              decode: one token per sequence
    pnmix_decode_attention(cfg, q, cache, out, ws)      decode: attention, fp32 out

``PNMixCache`` owns the device buffers (cache + decode workspace) of one layer.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpnmix.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python decode_attention_prefill_b200/build.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_ALIGNMENT, ERR_DEVICE = range(7)
DEVERR_APPEND_FULL = 0x1
DEVERR_TIMEOUT = 0x2
# decode kernels (Config.decode_kernel)
DECODE_AUTO, DECODE_SIMT, DECODE_MMA, DECODE_PAIRS, DECODE_TC = range(5)
DECODE_KERNELS = {"auto": DECODE_AUTO, "simt": DECODE_SIMT, "mma": DECODE_MMA, "ws": DECODE_PAIRS, "tc": DECODE_TC}

EXPORTED = [
    "pnmix_record_bytes", "pnmix_cache_bytes", "pnmix_cache_init", "pnmix_cache_reset",
    "pnmix_select_pairs", "pnmix_quantize_keys", "pnmix_quantize_values", "pnmix_append",
    "pnmix_workspace_bytes", "pnmix_decode_attention", "pnmix_read_error",
    "pnmix_status_string", "pnmix_version", "pnmix_decode_attention_noalloc",
    "pnmix_workspace_bytes_multi", "pnmix_decode_attention_multi", "pnmix_shrink_keys",
    "pnmix_split_groups", "pnmix_debug_decode_stall", "pnmix_workspace_bytes_two",
    "pnmix_decode_attention_two", "pnmix_append_decode",
]


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "head_dim", "n_q_heads", "n_kv_heads", "group_tokens", "residual_tokens", "key_bits_hi",
        "key_bits_lo", "n_salient_pairs", "value_bits", "value_group", "saliency_window")] + [
        ("softmax_scale", ctypes.c_float), ("saliency_score", ctypes.c_int32),
        ("n_pruned_pairs", ctypes.c_int32), ("decode_kernel", ctypes.c_int32),
        ("n_pruned_slices", ctypes.c_int32)]

    @classmethod
    def make(cls, n_q_heads: int, n_kv_heads: int, key_bits_hi: int = 4, key_bits_lo: int = 2,
             n_salient_pairs: int = 8, saliency_window: int = 64, softmax_scale: float = 0.0,
             saliency_score: int = 0, n_pruned_pairs: int = 0, decode_kernel: int = 0,
             n_pruned_slices: int = 0):
        return cls(128, n_q_heads, n_kv_heads, 32, 32, key_bits_hi, key_bits_lo, n_salient_pairs,
                   2, 32, saliency_window, softmax_scale, saliency_score, n_pruned_pairs, decode_kernel,
                   n_pruned_slices)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def without_salient(self) -> "Config":
        """The same config with no salient pair (the layout pnmix_shrink_keys writes)."""
        c = Config.from_buffer_copy(self)
        c.n_salient_pairs = 0
        return c


class Cache(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("capacity_tokens", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32), ("record_bytes", ctypes.c_int32),
        ("records", ctypes.c_void_p), ("k_resid", ctypes.c_void_p), ("v_resid", ctypes.c_void_p),
        ("len", ctypes.c_void_p), ("pair_idx", ctypes.c_void_p), ("pair_mask", ctypes.c_void_p),
        ("perm", ctypes.c_void_p), ("pair_scores", ctypes.c_void_p), ("scratch", ctypes.c_void_p),
        ("error", ctypes.c_void_p), ("base", ctypes.c_void_p), ("total_bytes", ctypes.c_size_t),
    ]


_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_CP, _KP = ctypes.POINTER(Config), ctypes.POINTER(Cache)
_SIGS = {
    "pnmix_record_bytes": (_sz, [_CP]),
    "pnmix_cache_bytes": (_i, [_CP, _i, _i, ctypes.POINTER(_sz)]),
    "pnmix_cache_init": (_i, [_CP, _i, _i, _vp, _sz, _KP]),
    "pnmix_cache_reset": (_i, [_KP, _vp]),
    "pnmix_select_pairs": (_i, [_CP, _vp, _i, _vp, _i, _i, _KP, _vp]),
    "pnmix_quantize_keys": (_i, [_CP, _vp, _i, _i, _KP, _vp]),
    "pnmix_quantize_values": (_i, [_CP, _vp, _i, _i, _KP, _vp]),
    "pnmix_append": (_i, [_CP, _vp, _vp, _KP, _vp]),
    "pnmix_workspace_bytes": (_sz, [_CP, _i, _i]),
    "pnmix_decode_attention": (_i, [_CP, _vp, _KP, _i, _vp, _vp, _sz, _vp]),
    "pnmix_read_error": (_i, [_KP, _i, ctypes.POINTER(ctypes.c_uint32)]),
    "pnmix_status_string": (ctypes.c_char_p, [_i]),
    "pnmix_version": (ctypes.c_char_p, []),
    "pnmix_decode_attention_noalloc": (_i, [_CP, _vp, _KP, _i, _vp, _vp]),
    "pnmix_workspace_bytes_multi": (_sz, [_CP, _i, _i, _i]),
    "pnmix_decode_attention_multi": (_i, [_CP, _vp, _i, _KP, _i, _vp, _vp, _sz, _vp]),
    "pnmix_shrink_keys": (_i, [_CP, _KP, _KP, _vp]),
    "pnmix_split_groups": (_i, [_CP, _i, _vp, _i, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp]),
    "pnmix_debug_decode_stall": (_i, [_CP, _vp, _KP, _i, _vp, _vp, _sz, _i, ctypes.c_uint32, _vp]),
    "pnmix_workspace_bytes_two": (_sz, [_CP, _CP, _i, _i, _i]),
    "pnmix_decode_attention_two": (_i, [_CP, _KP, _i, _CP, _KP, _i, _vp, _vp, _vp, _sz, _vp]),
    "pnmix_append_decode": (_i, [_CP, _vp, _vp, _vp, _KP, _i, _vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class PNMixError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.pnmix_status_string(status).decode()} (status {status})")


def _check(status: int, where: str):
    if status != OK:
        raise PNMixError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def version() -> str:
    return _lib.pnmix_version().decode()


def record_bytes(cfg: Config) -> int:
    return int(_lib.pnmix_record_bytes(ctypes.byref(cfg)))


def cache_bytes(cfg: Config, batch: int, capacity_tokens: int) -> int:
    out = _sz(0)
    _check(_lib.pnmix_cache_bytes(ctypes.byref(cfg), batch, capacity_tokens, ctypes.byref(out)),
           "pnmix_cache_bytes")
    return int(out.value)


def workspace_bytes(cfg: Config, batch: int, max_context: int) -> int:
    return int(_lib.pnmix_workspace_bytes(ctypes.byref(cfg), batch, max_context))


# ---------------------------------------------------------------- the five calls

def pnmix_select_pairs(cfg: Config, q_window: torch.Tensor, k: torch.Tensor, L: int, cache: "PNMixCache",
                       stream=None):
    """q_window bf16 [B][Hq][W'][128] (W' = min(L, W)), k bf16 [B][Hkv][ld][128]."""
    _check(_lib.pnmix_select_pairs(ctypes.byref(cfg), _dev(q_window, torch.bfloat16, "q_window"),
                                   q_window.shape[2], _dev(k, torch.bfloat16, "k"), L, k.shape[2],
                                   ctypes.byref(cache.c), _stream(stream)), "pnmix_select_pairs")


def pnmix_quantize_keys(cfg: Config, k: torch.Tensor, L: int, cache: "PNMixCache", stream=None):
    _check(_lib.pnmix_quantize_keys(ctypes.byref(cfg), _dev(k, torch.bfloat16, "k"), L, k.shape[2],
                                    ctypes.byref(cache.c), _stream(stream)), "pnmix_quantize_keys")


def pnmix_quantize_values(cfg: Config, v: torch.Tensor, L: int, cache: "PNMixCache", stream=None):
    _check(_lib.pnmix_quantize_values(ctypes.byref(cfg), _dev(v, torch.bfloat16, "v"), L, v.shape[2],
                                      ctypes.byref(cache.c), _stream(stream)), "pnmix_quantize_values")


def pnmix_append(cfg: Config, k_new: torch.Tensor, v_new: torch.Tensor, cache: "PNMixCache", stream=None):
    """k_new, v_new bf16 [B][Hkv][128]."""
    _check(_lib.pnmix_append(ctypes.byref(cfg), _dev(k_new, torch.bfloat16, "k_new"),
                             _dev(v_new, torch.bfloat16, "v_new"), ctypes.byref(cache.c),
                             _stream(stream)), "pnmix_append")


def pnmix_decode_attention(cfg: Config, q: torch.Tensor, cache: "PNMixCache", out: torch.Tensor,
                           workspace: torch.Tensor | None = None, max_context: int | None = None,
                           stream=None):
    """q bf16 [B][Hq][128] -> out fp32 [B][Hq][128]."""
    ws = cache.workspace if workspace is None else workspace
    mc = cache.max_context if max_context is None else max_context
    _check(_lib.pnmix_decode_attention(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q"),
                                       ctypes.byref(cache.c), mc, _dev(out, torch.float32, "out"),
                                       _dev(ws, torch.uint8, "workspace"), ws.numel(),
                                       _stream(stream)), "pnmix_decode_attention")


def pnmix_append_decode(cfg: Config, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                        cache: "PNMixCache", out: torch.Tensor, workspace: torch.Tensor | None = None,
                        max_context: int | None = None, stream=None):
    """One decode step: append k_new, v_new bf16 [B][Hkv][128], then attend q bf16 [B][Hq][128]
    over the cache including the new token -> out fp32 [B][Hq][128]."""
    ws = cache.workspace if workspace is None else workspace
    mc = cache.max_context if max_context is None else max_context
    _check(_lib.pnmix_append_decode(ctypes.byref(cfg), _dev(k_new, torch.bfloat16, "k_new"),
                                    _dev(v_new, torch.bfloat16, "v_new"), _dev(q, torch.bfloat16, "q"),
                                    ctypes.byref(cache.c), mc, _dev(out, torch.float32, "out"),
                                    _dev(ws, torch.uint8, "workspace"), ws.numel(), _stream(stream)),
           "pnmix_append_decode")


def workspace_bytes_multi(cfg: Config, batch: int, max_context: int, n_queries: int) -> int:
    return int(_lib.pnmix_workspace_bytes_multi(ctypes.byref(cfg), batch, max_context, n_queries))


def pnmix_decode_attention_multi(cfg: Config, q: torch.Tensor, cache: "PNMixCache", out: torch.Tensor,
                                 workspace: torch.Tensor | None = None, max_context: int | None = None,
                                 stream=None):
    """q bf16 [B][T][Hq][128] -> out fp32 [B][T][Hq][128]; query j over the first len - T + 1 + j tokens."""
    ws = cache.workspace if workspace is None else workspace
    mc = cache.max_context if max_context is None else max_context
    _check(_lib.pnmix_decode_attention_multi(ctypes.byref(cfg), _dev(q, torch.bfloat16, "q"), q.shape[1],
                                             ctypes.byref(cache.c), mc, _dev(out, torch.float32, "out"),
                                             _dev(ws, torch.uint8, "workspace"), ws.numel(),
                                             _stream(stream)), "pnmix_decode_attention_multi")


def pnmix_shrink_keys(cfg: Config, src: "PNMixCache", dst: "PNMixCache", stream=None):
    """src: a cache of cfg (b_hi = 2 b_lo, k > 0); dst: a cache of cfg with n_salient_pairs = 0."""
    _check(_lib.pnmix_shrink_keys(ctypes.byref(cfg), ctypes.byref(src.c), ctypes.byref(dst.c), _stream(stream)),
           "pnmix_shrink_keys")


def workspace_bytes_two(cfg_a: Config, cfg_b: Config, batch: int, max_context_a: int, max_context_b: int) -> int:
    return int(_lib.pnmix_workspace_bytes_two(ctypes.byref(cfg_a), ctypes.byref(cfg_b), batch, max_context_a,
                                              max_context_b))


def pnmix_decode_attention_two(cache_a: "PNMixCache", cache_b: "PNMixCache", q: torch.Tensor, out: torch.Tensor,
                               workspace: torch.Tensor | None = None, stream=None):
    """Attention of q bf16 [B][Hq][128] over the union of two caches' tokens -> out fp32 [B][Hq][128]."""
    if workspace is None:
        n = workspace_bytes_two(cache_a.cfg, cache_b.cfg, cache_a.batch, cache_a.max_context, cache_b.max_context)
        workspace = getattr(cache_b, "_two_ws", None)
        if workspace is None or workspace.numel() < n:
            ws = torch.zeros(n + 256, dtype=torch.uint8, device=q.device)
            off = (-ws.data_ptr()) % 256
            workspace = cache_b._two_ws = ws[off:off + n]
    _check(_lib.pnmix_decode_attention_two(ctypes.byref(cache_a.cfg), ctypes.byref(cache_a.c), cache_a.max_context,
                                           ctypes.byref(cache_b.cfg), ctypes.byref(cache_b.c), cache_b.max_context,
                                           _dev(q, torch.bfloat16, "q"), _dev(out, torch.float32, "out"),
                                           _dev(workspace, torch.uint8, "workspace"), workspace.numel(),
                                           _stream(stream)), "pnmix_decode_attention_two")


def split_sizes(L: int, hi_percent: int) -> tuple[int, int]:
    """(L_hi, L_lo): tokens of the high and low parts of a two-precision prefill."""
    n_hi = (L // 32) * hi_percent // 100
    return 32 * n_hi, L - 32 * n_hi


def pnmix_split_groups(cfg: Config, q_window: torch.Tensor, k: torch.Tensor, v: torch.Tensor, L: int,
                       hi_percent: int, stream=None) -> dict:
    """Rank the 32-token groups of a prefill and split K / V into a high and a low part.
    q_window bf16 [B][Hq][W'][128]; k, v bf16 [B][Hkv][ld][128].  Returns the device tensors
    scores fp32 / route uint8 / dest int32 [B][Hkv][L/32] and k_hi, v_hi [B][Hkv][L_hi][128],
    k_lo, v_lo [B][Hkv][L_lo][128]."""
    B, Hkv = k.shape[0], k.shape[1]
    ng = L // 32
    L_hi, L_lo = split_sizes(L, hi_percent)
    dev = k.device
    r = {"scores": torch.empty(B, Hkv, ng, dtype=torch.float32, device=dev),
         "route": torch.empty(B, Hkv, ng, dtype=torch.uint8, device=dev),
         "dest": torch.empty(B, Hkv, ng, dtype=torch.int32, device=dev),
         "k_hi": torch.empty(B, Hkv, L_hi, 128, dtype=torch.bfloat16, device=dev),
         "v_hi": torch.empty(B, Hkv, L_hi, 128, dtype=torch.bfloat16, device=dev),
         "k_lo": torch.empty(B, Hkv, L_lo, 128, dtype=torch.bfloat16, device=dev),
         "v_lo": torch.empty(B, Hkv, L_lo, 128, dtype=torch.bfloat16, device=dev)}

    def ptr(t):
        return t.data_ptr() if t.numel() else None
    _check(_lib.pnmix_split_groups(ctypes.byref(cfg), B, _dev(q_window, torch.bfloat16, "q_window"),
                                   q_window.shape[2], _dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                                   L, k.shape[2], hi_percent, ptr(r["scores"]), ptr(r["route"]), ptr(r["dest"]),
                                   ptr(r["k_hi"]), ptr(r["v_hi"]), ptr(r["k_lo"]), ptr(r["v_lo"]),
                                   _stream(stream)), "pnmix_split_groups")
    return r


# ---------------------------------------------------------------- owner of device buffers

class PNMixCache:
    """Cache + decode workspace of one layer, allocated with torch on `device`."""

    def __init__(self, cfg: Config, batch: int, capacity_tokens: int, device="cuda",
                 max_context: int | None = None, stream=None, max_queries: int = 1):
        self.cfg = cfg
        self.batch = batch
        self.capacity = capacity_tokens
        self.max_context = capacity_tokens if max_context is None else max_context
        nbytes = cache_bytes(cfg, batch, capacity_tokens)
        self.buffer = torch.zeros(nbytes + 256, dtype=torch.uint8, device=device)
        base = (self.buffer.data_ptr() + 255) & ~255
        self.c = Cache()
        _check(_lib.pnmix_cache_init(ctypes.byref(cfg), batch, capacity_tokens, ctypes.c_void_p(base),
                                     nbytes, ctypes.byref(self.c)), "pnmix_cache_init")
        self._base_off = base - self.buffer.data_ptr()
        ws = max(workspace_bytes(cfg, batch, self.max_context),
                 workspace_bytes_multi(cfg, batch, self.max_context, max_queries) if max_queries > 1 else 0)
        self.workspace = torch.zeros(ws + 256, dtype=torch.uint8, device=device)
        # 256-byte aligned view
        off = (-self.workspace.data_ptr()) % 256
        self.workspace = self.workspace[off:off + ws]
        self.reset(stream)

    def reset(self, stream=None):
        _check(_lib.pnmix_cache_reset(ctypes.byref(self.c), _stream(stream)), "pnmix_cache_reset")

    def _region(self, ptr: int, nbytes: int) -> torch.Tensor:
        off = ptr - self.buffer.data_ptr()
        return self.buffer[off:off + nbytes]

    # Views of the device regions (for tests and inspection).
    def records(self) -> torch.Tensor:
        R = self.c.record_bytes
        return self._region(self.c.records, self.batch * self.cfg.n_kv_heads * (self.capacity // 32) * R) \
            .view(self.batch, self.cfg.n_kv_heads, self.capacity // 32, R)

    def resid(self, which: str) -> torch.Tensor:
        ptr = self.c.k_resid if which == "k" else self.c.v_resid
        return self._region(ptr, self.batch * self.cfg.n_kv_heads * 32 * 128 * 2).view(torch.int16) \
            .view(self.batch, self.cfg.n_kv_heads, 32, 128)

    def lengths(self) -> torch.Tensor:
        return self._region(self.c.len, 4 * self.batch).view(torch.int32)

    def pair_idx(self) -> torch.Tensor:
        return self._region(self.c.pair_idx, self.batch * self.cfg.n_kv_heads * 64) \
            .view(self.batch, self.cfg.n_kv_heads, 64)

    def pair_mask(self) -> torch.Tensor:
        return self._region(self.c.pair_mask, self.batch * self.cfg.n_kv_heads * 8).view(torch.int64) \
            .view(self.batch, self.cfg.n_kv_heads)

    def perm(self) -> torch.Tensor:
        return self._region(self.c.perm, self.batch * self.cfg.n_kv_heads * 128) \
            .view(self.batch, self.cfg.n_kv_heads, 128)

    def pair_scores(self) -> torch.Tensor:
        return self._region(self.c.pair_scores, self.batch * self.cfg.n_kv_heads * 256).view(torch.float32) \
            .view(self.batch, self.cfg.n_kv_heads, 64)

    def read_error(self, clear: bool = True) -> int:
        val = ctypes.c_uint32(0)
        st = _lib.pnmix_read_error(ctypes.byref(self.c), 1 if clear else 0, ctypes.byref(val))
        if st not in (OK, ERR_DEVICE):
            raise PNMixError(st, "pnmix_read_error")
        return int(val.value)

    # Convenience wrappers of the five calls.
    def prefill(self, q_window, k, v, L: int, stream=None):
        pnmix_select_pairs(self.cfg, q_window, k, L, self, stream)
        pnmix_quantize_keys(self.cfg, k, L, self, stream)
        pnmix_quantize_values(self.cfg, v, L, self, stream)

    def append(self, k_new, v_new, stream=None):
        pnmix_append(self.cfg, k_new, v_new, self, stream)

    def shrunk(self, stream=None, max_queries: int = 1) -> "PNMixCache":
        """A new cache holding this one with its salient keys shrunk to key_bits_lo bits."""
        dst = PNMixCache(self.cfg.without_salient(), self.batch, self.capacity, device=self.buffer.device,
                         max_context=self.max_context, stream=stream, max_queries=max_queries)
        pnmix_shrink_keys(self.cfg, self, dst, stream)
        return dst

    def attend_multi(self, q, out=None, stream=None) -> torch.Tensor:
        """q bf16 [B][T][Hq][128] of T tokens already appended -> fp32 [B][T][Hq][128]."""
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        pnmix_decode_attention_multi(self.cfg, q, self, out, stream=stream)
        return out

    def attend(self, q, out=None, stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        pnmix_decode_attention(self.cfg, q, self, out, stream=stream)
        return out


def decode_step_host(cache: PNMixCache, q_host: torch.Tensor, k_host: torch.Tensor, v_host: torch.Tensor,
                     out_host: torch.Tensor, staging: dict, stream=None):
    """One decode step from pinned HOST buffers: copy q, k_new, v_new to the device,
    append + attend, copy the fp32 output back into out_host (asynchronously on `stream`)."""
    s = torch.cuda.current_stream() if stream is None else stream
    with torch.cuda.stream(s):
        for name, src in (("q", q_host), ("k", k_host), ("v", v_host)):
            dst = staging.get(name)
            if dst is None or dst.shape != src.shape:
                dst = staging[name] = torch.empty(src.shape, dtype=src.dtype, device="cuda")
            dst.copy_(src, non_blocking=True)
        out = staging.get("out")
        if out is None or out.shape != out_host.shape:
            out = staging["out"] = torch.empty(out_host.shape, dtype=torch.float32, device="cuda")
        pnmix_append(cache.cfg, staging["k"], staging["v"], cache, s)
        pnmix_decode_attention(cache.cfg, staging["q"], cache, out, stream=s)
        out_host.copy_(out, non_blocking=True)
