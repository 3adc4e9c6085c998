"""Seeded synthetic inputs for the PN-Mix KV-cache path.

This package makes Q/K/V rows and nothing else: the CUDA library and the CPU
oracle both consume the bytes it writes, and neither shares any other code.
The rows are produced by ``workload.c`` (compiled here with gcc on first use);
see that file for the recipe.

Workloads (all head_dim 128, 32-token groups, 32-token residual, 2-bit values):

``tiny``            1 sequence, 1/1 heads, prefill 512, one decode query, k = 8.
``llama3_8b``       batch 8, 32/8 heads (GQA 4), context 8192, one decode step, k = 8.
``stream_32k``      batch 16, 32/8 heads, prefill 4096, then appends one token at a
                    time to 32768 total context, k = 8 (2.25 key code bits).
``sweep_128k``      batch 2, 28/4 heads (GQA 7), context 131072, bit points below.
``pipeline_32l``    32 layers, batch 32, 32/8 heads, prefill 4096 -> 32768.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "workload.c")
_LIB = os.path.join(_HERE, "libpnmix_workload.so")
_lock = threading.Lock()
_lib = None

Q, K, V = 0, 1, 2
THETA = 500000.0
KEY_OUTLIER_SCALE = 8.0
QUERY_OUTLIER_SCALE = 4.0


def build(force: bool = False) -> str:
    """Compile workload.c into libpnmix_workload.so next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.wl_fill.restype = ctypes.c_int
            lib.wl_fill.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                    ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                    ctypes.c_void_p, ctypes.c_int]
            lib.wl_fill_block.restype = ctypes.c_int
            lib.wl_fill_block.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                          ctypes.c_int, ctypes.c_int64, ctypes.c_double,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_void_p,
                                          ctypes.c_int]
            lib.wl_outlier_pairs.restype = None
            lib.wl_outlier_pairs.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_void_p]
            lib.wl_row_double.restype = None
            lib.wl_row_double.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                          ctypes.c_void_p]
            lib.wl_row_unrotated.restype = None
            lib.wl_row_unrotated.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int64, ctypes.c_void_p]
            lib.wl_bf16_from_double.restype = ctypes.c_uint16
            lib.wl_bf16_from_double.argtypes = [ctypes.c_double]
            _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def rows(seed: int, tensor: int, batch: int, heads: int, t0: int, n: int, *, group: int = 1,
         out: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """bf16 bits uint16 [batch][heads][n][128] for positions t0 .. t0+n-1.

    ``tensor`` is ``Q`` (heads are query heads, ``group`` = query heads per KV
    head), ``K`` or ``V``.  ``out`` may be a larger [batch][heads][ld][128]
    array whose first n rows per head are written.
    """
    lib = _load()
    if out is None:
        out = np.empty((batch, heads, n, 128), dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous
    assert out.shape[0] == batch and out.shape[1] == heads and out.shape[3] == 128
    ld = out.shape[2]
    rc = lib.wl_fill(seed, tensor, batch, heads, group, t0, n, ld, THETA, KEY_OUTLIER_SCALE,
                     QUERY_OUTLIER_SCALE, out.ctypes.data, threads or default_threads())
    if rc != 0:
        raise ValueError("wl_fill rejected its arguments")
    return out


def unit_rows(seed: int, tensor: int, b: int, head0: int, heads: int, t0: int, n: int, *,
              group: int = 1, threads: int | None = None) -> np.ndarray:
    """Rows of batch row b, heads head0 .. head0+heads-1: uint16 [heads][n][128]."""
    lib = _load()
    out = np.empty((1, heads, n, 128), dtype=np.uint16)
    rc = lib.wl_fill_block(seed, tensor, b, 1, head0, heads, group, t0, n, n, THETA,
                           KEY_OUTLIER_SCALE, QUERY_OUTLIER_SCALE, out.ctypes.data,
                           threads or default_threads())
    if rc != 0:
        raise ValueError("wl_fill_block rejected its arguments")
    return out[0]


def outlier_pairs(seed: int, query: bool, b: int, kv_head: int) -> list[int]:
    lib = _load()
    buf = (ctypes.c_int32 * 4)()
    lib.wl_outlier_pairs(seed, 1 if query else 0, b, kv_head, buf)
    return list(buf)


def row_double(seed: int, tensor: int, b: int, head: int, pos: int, group: int = 1,
               rotated: bool = True) -> np.ndarray:
    lib = _load()
    out = np.empty(128, dtype=np.float64)
    if rotated:
        lib.wl_row_double(seed, tensor, group, THETA, KEY_OUTLIER_SCALE, QUERY_OUTLIER_SCALE,
                          b, head, pos, out.ctypes.data)
    else:
        lib.wl_row_unrotated(seed, tensor, group, KEY_OUTLIER_SCALE, QUERY_OUTLIER_SCALE,
                             b, head, pos, out.ctypes.data)
    return out


def bf16_from_double(x: float) -> int:
    return int(_load().wl_bf16_from_double(float(x)))


def bf16_to_float(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bits to float32 exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class BitPoint:
    key_bits_hi: int
    key_bits_lo: int
    n_salient_pairs: int

    @property
    def key_code_bits(self) -> float:
        f = self.n_salient_pairs / 64.0
        return self.key_bits_lo + f * (self.key_bits_hi - self.key_bits_lo)


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    prefill: int            # prefill length L
    context: int            # context at the measured decode step
    bits: BitPoint = BitPoint(4, 2, 8)
    layers: int = 1
    window: int = 64
    seed: int = 0
    streaming: bool = False  # decode tokens are appended one at a time
    sweep: tuple = field(default_factory=tuple)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 512, 512),
    "llama3_8b": Workload("llama3_8b", 8, 32, 8, 8192, 8192),
    "stream_32k": Workload("stream_32k", 16, 32, 8, 4096, 32768, streaming=True),
    "sweep_128k": Workload("sweep_128k", 2, 28, 4, 131072, 131072, sweep=(
        BitPoint(4, 2, 0), BitPoint(4, 2, 8), BitPoint(4, 2, 16), BitPoint(4, 2, 32),
        BitPoint(2, 1, 16), BitPoint(2, 1, 32))),
    "pipeline_32l": Workload("pipeline_32l", 32, 32, 8, 4096, 32768, layers=32, streaming=True),
}
