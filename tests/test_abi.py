"""The C ABI on the host: every declared symbol is exported and host-side
validation answers without a GPU (no compute call is made here)."""
import ctypes
import os
import re

import pytest
import torch

import decode_attention_prefill_b200 as pm
import oracle

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pnmix.h")


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"PNMIX_API\s+[\w\s\*]+?\b(pnmix_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared()
    assert len(names) >= 13
    lib = ctypes.CDLL(pm.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(pm.EXPORTED)


def test_version_and_status_strings():
    assert pm.version().startswith("pnmix")
    assert pm._lib.pnmix_status_string(0) == b"ok"
    assert pm._lib.pnmix_status_string(99) == b"unknown status"


@pytest.mark.parametrize("k,bhi,blo", [(0, 4, 2), (8, 4, 2), (16, 4, 2), (32, 4, 2), (64, 4, 2),
                                       (0, 2, 1), (16, 2, 1), (32, 2, 1), (64, 2, 1)])
def test_record_bytes_agree_with_the_layout_definition(k, bhi, blo):
    cfg = pm.Config.make(32, 8, bhi, blo, k)
    assert pm.record_bytes(cfg) == oracle.record_bytes(k, bhi, blo) > 0


@pytest.mark.parametrize("change,status", [
    (dict(n_salient_pairs=4), pm.ERR_UNSUPPORTED),
    (dict(n_salient_pairs=8, key_bits_hi=2, key_bits_lo=1), pm.ERR_UNSUPPORTED),
    (dict(key_bits_hi=8), pm.ERR_UNSUPPORTED),
    (dict(head_dim=64), pm.ERR_UNSUPPORTED),
    (dict(n_q_heads=36, n_kv_heads=4), pm.ERR_UNSUPPORTED),   # G = 9
    (dict(n_q_heads=30, n_kv_heads=4), pm.ERR_INVALID_ARG),   # not a multiple
    (dict(value_bits=4), pm.ERR_UNSUPPORTED),
    (dict(saliency_window=0), pm.ERR_UNSUPPORTED),
    (dict(saliency_score=3), pm.ERR_UNSUPPORTED),
    (dict(saliency_score=-1), pm.ERR_UNSUPPORTED),
    (dict(n_pruned_pairs=64), pm.ERR_UNSUPPORTED),
    (dict(n_pruned_pairs=-1), pm.ERR_UNSUPPORTED),
    (dict(decode_kernel=5), pm.ERR_UNSUPPORTED),
    (dict(decode_kernel=-1), pm.ERR_UNSUPPORTED),
    (dict(decode_kernel=pm.DECODE_SIMT, n_pruned_pairs=5), pm.ERR_UNSUPPORTED),   # simt has no pruning
    (dict(n_pruned_slices=9), pm.ERR_UNSUPPORTED),
    (dict(n_pruned_slices=-1), pm.ERR_UNSUPPORTED),
    (dict(n_pruned_slices=3, n_pruned_pairs=5), pm.ERR_UNSUPPORTED),   # one pruning at a time
    (dict(decode_kernel=pm.DECODE_SIMT, n_pruned_slices=2), pm.ERR_UNSUPPORTED),
])
def test_config_validation(change, status):
    cfg = pm.Config.make(32, 8)
    for k, v in change.items():
        setattr(cfg, k, v)
    out = ctypes.c_size_t(0)
    assert pm._lib.pnmix_cache_bytes(ctypes.byref(cfg), 2, 64, ctypes.byref(out)) == status


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_cache_init_carves_aligned_regions_without_touching_memory():
    cfg = pm.Config.make(32, 8)
    nbytes = pm.cache_bytes(cfg, 4, 1024)
    c = pm.Cache()
    fake = 1 << 40   # never dereferenced: cache_init is host-only
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), 4, 1024, ctypes.c_void_p(fake), nbytes,
                                    ctypes.byref(c)) == pm.OK
    ptrs = [c.records, c.k_resid, c.v_resid, c.len, c.pair_idx, c.pair_mask, c.perm, c.pair_scores,
            c.scratch, c.error]
    assert all(p % 256 == 0 for p in ptrs) and ptrs == sorted(ptrs)
    assert c.k_resid - c.records >= 4 * 8 * 32 * 3200
    assert c.total_bytes == nbytes
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), 4, 1024, ctypes.c_void_p(fake + 16), nbytes,
                                    ctypes.byref(c)) == pm.ERR_ALIGNMENT
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), 4, 1024, ctypes.c_void_p(fake), nbytes - 1,
                                    ctypes.byref(c)) == pm.ERR_CAPACITY
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), 4, 1000, ctypes.c_void_p(fake), nbytes,
                                    ctypes.byref(c)) == pm.ERR_INVALID_ARG


def _fake_cache(cfg, B=2, cap=256):
    c = pm.Cache()
    nbytes = pm.cache_bytes(cfg, B, cap)
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), B, cap, ctypes.c_void_p(1 << 40), nbytes,
                                    ctypes.byref(c)) == pm.OK
    return c


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_entry_points_reject_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2)
    c = _fake_cache(cfg)
    P = ctypes.c_void_p(1 << 41)
    odd = ctypes.c_void_p((1 << 41) + 2)
    L = pm._lib
    # window must be min(L, W)
    assert L.pnmix_select_pairs(ctypes.byref(cfg), P, 63, P, 100, 128, ctypes.byref(c), None) == pm.ERR_INVALID_ARG
    assert L.pnmix_select_pairs(ctypes.byref(cfg), P, 64, P, 100, 99, ctypes.byref(c), None) == pm.ERR_INVALID_ARG
    assert L.pnmix_select_pairs(ctypes.byref(cfg), odd, 64, P, 100, 128, ctypes.byref(c), None) == pm.ERR_ALIGNMENT
    assert L.pnmix_select_pairs(ctypes.byref(cfg), None, 64, P, 100, 128, ctypes.byref(c), None) == pm.ERR_INVALID_ARG
    assert L.pnmix_quantize_keys(ctypes.byref(cfg), P, 257, 300, ctypes.byref(c), None) == pm.ERR_CAPACITY
    assert L.pnmix_quantize_values(ctypes.byref(cfg), odd, 10, 10, ctypes.byref(c), None) == pm.ERR_ALIGNMENT
    assert L.pnmix_append(ctypes.byref(cfg), P, None, ctypes.byref(c), None) == pm.ERR_INVALID_ARG
    ws = pm.workspace_bytes(cfg, 2, 256)
    assert ws > 0
    assert L.pnmix_decode_attention(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, P, ws - 1, None) == pm.ERR_CAPACITY
    assert L.pnmix_decode_attention(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, odd, ws, None) == pm.ERR_ALIGNMENT
    other = pm.Config.make(8, 2, n_salient_pairs=16)   # record size differs from the cache's
    assert L.pnmix_decode_attention(ctypes.byref(other), P, ctypes.byref(c), 256, P, P, ws, None) == pm.ERR_INVALID_ARG


def test_multi_query_workspace_follows_the_rows():
    cfg = pm.Config.make(8, 2)                      # G = 4
    one = pm.workspace_bytes(cfg, 2, 256)
    assert pm.workspace_bytes_multi(cfg, 2, 256, 1) == one
    assert pm.workspace_bytes_multi(cfg, 2, 256, 2) > one
    assert pm.workspace_bytes_multi(cfg, 2, 256, 3) > pm.workspace_bytes_multi(cfg, 2, 256, 2)   # 12 rows
    assert pm.workspace_bytes_multi(cfg, 2, 256, 16) > 0       # 64 rows per KV head
    assert pm.workspace_bytes_multi(cfg, 2, 256, 32) > 0       # 128 rows: the most (tcgen05 kernel)
    assert pm.workspace_bytes_multi(cfg, 2, 256, 33) == 0      # 132 rows: unsupported
    assert pm.workspace_bytes_multi(cfg, 2, 256, 0) == 0
    rows_kernel = pm.Config.make(8, 2, decode_kernel=pm.DECODE_MMA)   # forced: 8-row warps, up to 64
    assert pm.workspace_bytes_multi(rows_kernel, 2, 256, 16) > 0
    assert pm.workspace_bytes_multi(rows_kernel, 2, 256, 17) == 0


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_multi_query_entry_rejects_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2)
    c = _fake_cache(cfg)
    P = ctypes.c_void_p(1 << 41)
    L = pm._lib
    ws = pm.workspace_bytes_multi(cfg, 2, 256, 2)
    assert L.pnmix_decode_attention_multi(ctypes.byref(cfg), P, 33, ctypes.byref(c), 256, P, P, ws,
                                          None) == pm.ERR_UNSUPPORTED      # 132 rows per KV head
    forced = pm.Config.make(8, 2, decode_kernel=pm.DECODE_MMA)
    assert L.pnmix_decode_attention_multi(ctypes.byref(forced), P, 17, ctypes.byref(c), 256, P, P, ws,
                                          None) == pm.ERR_UNSUPPORTED      # 68 rows off the tcgen05 kernel
    assert L.pnmix_decode_attention_multi(ctypes.byref(cfg), P, 3, ctypes.byref(c), 256, P, P, ws,
                                          None) == pm.ERR_CAPACITY         # a 12-row workspace is larger
    simt = pm.Config.make(8, 2, decode_kernel=pm.DECODE_SIMT)
    assert L.pnmix_decode_attention_multi(ctypes.byref(simt), P, 2, ctypes.byref(c), 256, P, P, ws,
                                          None) == pm.ERR_UNSUPPORTED
    assert L.pnmix_decode_attention_multi(ctypes.byref(cfg), P, 0, ctypes.byref(c), 256, P, P, ws,
                                          None) == pm.ERR_INVALID_ARG
    assert L.pnmix_decode_attention_multi(ctypes.byref(cfg), P, 2, ctypes.byref(c), 256, P, P, ws - 1,
                                          None) == pm.ERR_CAPACITY


def _fake_cache_at(cfg, base, B=2, cap=256):
    c = pm.Cache()
    nbytes = pm.cache_bytes(cfg, B, cap)
    assert pm._lib.pnmix_cache_init(ctypes.byref(cfg), B, cap, ctypes.c_void_p(base), nbytes,
                                    ctypes.byref(c)) == pm.OK
    return c


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_shrink_entry_rejects_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2, key_bits_hi=4, key_bits_lo=2, n_salient_pairs=8)
    small = cfg.without_salient()
    assert small.n_salient_pairs == 0 and cfg.n_salient_pairs == 8
    src = _fake_cache_at(cfg, 1 << 40)
    dst = _fake_cache_at(small, 1 << 42)
    L = pm._lib
    # the destination must have the no-salient layout, its own memory, the same shape
    assert L.pnmix_shrink_keys(ctypes.byref(cfg), ctypes.byref(src), ctypes.byref(src), None) == pm.ERR_INVALID_ARG
    same = _fake_cache_at(small, 1 << 40)
    assert L.pnmix_shrink_keys(ctypes.byref(cfg), ctypes.byref(src), ctypes.byref(same), None) == pm.ERR_INVALID_ARG
    tail = _fake_cache_at(small, (1 << 40) + pm.cache_bytes(cfg, 2, 256) - 256)   # overlaps src's end
    assert L.pnmix_shrink_keys(ctypes.byref(cfg), ctypes.byref(src), ctypes.byref(tail), None) == pm.ERR_INVALID_ARG
    wide = _fake_cache_at(small, 1 << 42, cap=512)
    assert L.pnmix_shrink_keys(ctypes.byref(cfg), ctypes.byref(src), ctypes.byref(wide), None) == pm.ERR_INVALID_ARG
    assert L.pnmix_shrink_keys(ctypes.byref(cfg), None, ctypes.byref(dst), None) == pm.ERR_INVALID_ARG
    # there must be salient pairs to shrink (both supported bit pairs have b_hi = 2 b_lo)
    s0 = _fake_cache_at(small, 1 << 40)
    assert L.pnmix_shrink_keys(ctypes.byref(small), ctypes.byref(s0), ctypes.byref(dst), None) == pm.ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_split_groups_rejects_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2)
    P = ctypes.c_void_p(1 << 41)
    odd = ctypes.c_void_p((1 << 41) + 2)
    L = pm._lib
    def call(q=P, nw=64, k=P, v=P, n=300, ld=300, pct=50, sc=P, rt=P, ds=P, kh=P, vh=P, kl=P, vl=P, cf=cfg):
        return L.pnmix_split_groups(ctypes.byref(cf), 2, q, nw, k, v, n, ld, pct, sc, rt, ds, kh, vh, kl, vl, None)
    assert call(nw=63) == pm.ERR_INVALID_ARG                  # window must be min(L, W)
    assert call(ld=299) == pm.ERR_INVALID_ARG
    assert call(pct=101) == pm.ERR_INVALID_ARG
    assert call(pct=-1) == pm.ERR_INVALID_ARG
    assert call(n=0, nw=0) == pm.ERR_INVALID_ARG
    assert call(sc=None) == pm.ERR_INVALID_ARG                # 9 full groups need the outputs
    assert call(kh=None) == pm.ERR_INVALID_ARG                # 4 groups go to the high part
    assert call(pct=0, kh=None, vh=None, n=20, nw=20, ld=20, sc=None, rt=None, ds=None, kl=odd) == pm.ERR_ALIGNMENT
    assert call(v=odd) == pm.ERR_ALIGNMENT
    bad = pm.Config.make(8, 3)                                # 8 query heads over 3 KV heads
    assert call(cf=bad) == pm.ERR_INVALID_ARG
    assert pm.split_sizes(300, 50) == (128, 172)
    assert pm.split_sizes(64, 100) == (64, 0)
    assert pm.split_sizes(20, 100) == (0, 20)


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_is_plain_c_and_cxx(lang, std, tmp_path):
    """include/pnmix.h parses on its own as C99 and as C++ (no torch or CUDA types)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    r = subprocess.run([cc, "-fsyntax-only", "-Wall", "-Wextra", "-Werror", std, "-x", lang, HEADER],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors of pnmix_config and pnmix_cache have the header's size and field
    offsets (a C program built against include/pnmix.h prints them)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host compiler")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "pnmix.h"', 'int main(void) {']
    for cname, cls in (("pnmix_config", pm.Config), ("pnmix_cache", pm.Cache)):
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in cls._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ['  return 0;', '}']
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    r = subprocess.run([cc, "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    got = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    for line in filter(None, got):
        cname, field, value = line.split()
        cls = pm.Config if cname == "pnmix_config" else pm.Cache
        want = ctypes.sizeof(cls) if field == "size" else getattr(cls, field).offset
        assert int(value) == want, (cname, field)


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_noalloc_entry_rejects_bad_arguments_before_any_cuda_call():
    """Every rejection of the no-workspace decode happens on the host, before its scratch
    address is looked up or its memset is enqueued (none of these calls reaches CUDA)."""
    cfg = pm.Config.make(8, 2)
    c = _fake_cache(cfg)
    P = ctypes.c_void_p(1 << 41)
    odd = ctypes.c_void_p((1 << 41) + 2)
    f = pm._lib.pnmix_decode_attention_noalloc
    assert f(None, P, ctypes.byref(c), 256, P, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), None, ctypes.byref(c), 256, P, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, None, 256, P, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, None, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), -1, P, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), odd, ctypes.byref(c), 256, P, None) == pm.ERR_ALIGNMENT
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, odd, None) == pm.ERR_ALIGNMENT
    other = pm.Config.make(8, 2, n_salient_pairs=16)   # record size differs from the cache's
    assert f(ctypes.byref(other), P, ctypes.byref(c), 256, P, None) == pm.ERR_INVALID_ARG
    bad = pm.Cache.from_buffer_copy(c)
    bad.capacity_tokens = -32
    assert f(ctypes.byref(cfg), P, ctypes.byref(bad), 256, P, None) == pm.ERR_INVALID_ARG
    unsupported = pm.Config.make(8, 2, key_bits_hi=8)
    assert f(ctypes.byref(unsupported), P, ctypes.byref(c), 256, P, None) == pm.ERR_UNSUPPORTED
    big_cfg = pm.Config.make(64, 8)                     # G = 8, 1024 units: > 4 MiB of partials
    big = _fake_cache(big_cfg, B=128, cap=32)
    assert pm.workspace_bytes(big_cfg, 128, 32) > (4 << 20)
    assert f(ctypes.byref(big_cfg), P, ctypes.byref(big), 32, P, None) == pm.ERR_CAPACITY


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_stall_hook_rejects_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2)
    c = _fake_cache(cfg)                    # 2 x 2 units
    P = ctypes.c_void_p(1 << 41)
    ws = pm.workspace_bytes(cfg, 2, 256)
    f = pm._lib.pnmix_debug_decode_stall
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, P, ws, 4, 16, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, P, ws, -1, 16, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, P, ws, 0, 0, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, P, ws - 1, 0, 16, None) == pm.ERR_CAPACITY
    assert f(ctypes.byref(cfg), P, ctypes.byref(c), 256, P, None, ws, 0, 16, None) == pm.ERR_INVALID_ARG
    simt = pm.Config.make(8, 2, decode_kernel=pm.DECODE_SIMT)
    assert f(ctypes.byref(simt), P, ctypes.byref(c), 256, P, P, ws, 0, 16, None) == pm.ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_two_part_decode_rejects_bad_arguments_before_launching():
    hi, lo = pm.Config.make(8, 2, n_salient_pairs=16), pm.Config.make(8, 2, n_salient_pairs=8)
    a, b = _fake_cache(hi), _fake_cache(lo)
    P = ctypes.c_void_p(1 << 41)
    odd = ctypes.c_void_p((1 << 41) + 16)
    n = pm.workspace_bytes_two(hi, lo, 2, 256, 256)
    assert n >= max(pm.workspace_bytes(hi, 2, 256), pm.workspace_bytes(lo, 2, 256)) + 2 * 8 * 128 * 4
    assert pm.workspace_bytes_two(hi, pm.Config.make(8, 4), 2, 256, 256) == 0      # other head layout
    f = pm._lib.pnmix_decode_attention_two
    args = lambda cfg_a, ca, cfg_b, cb, ws, nb: (ctypes.byref(cfg_a), ctypes.byref(ca), 256, ctypes.byref(cfg_b),  # noqa: E731
                                                 ctypes.byref(cb), 256, P, P, ws, nb, None)
    assert f(*args(hi, a, lo, b, P, n - 1)) == pm.ERR_CAPACITY
    assert f(*args(hi, a, lo, b, odd, n)) == pm.ERR_ALIGNMENT
    assert f(*args(hi, a, lo, b, None, n)) == pm.ERR_INVALID_ARG
    assert f(*args(lo, a, lo, b, P, n)) == pm.ERR_INVALID_ARG          # cache a laid out for another config
    other = pm.Config.make(16, 4)
    assert f(*args(hi, a, other, _fake_cache(other), P, n)) == pm.ERR_INVALID_ARG   # head counts differ
    pruned = pm.Config.make(8, 2, n_salient_pairs=8, n_pruned_slices=2)
    assert f(*args(hi, a, pruned, b, P, n)) == pm.ERR_UNSUPPORTED      # no key-slice pruning across parts


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="uses fake device pointers; runs only where no kernel can launch")
def test_append_decode_rejects_bad_arguments_before_launching():
    cfg = pm.Config.make(8, 2)
    c = _fake_cache(cfg)
    P = ctypes.c_void_p(1 << 41)
    odd = ctypes.c_void_p((1 << 41) + 2)
    ws = pm.workspace_bytes(cfg, 2, 256)
    f = pm._lib.pnmix_append_decode
    assert f(ctypes.byref(cfg), None, P, P, ctypes.byref(c), 256, P, P, ws, None) == pm.ERR_INVALID_ARG
    assert f(ctypes.byref(cfg), P, odd, P, ctypes.byref(c), 256, P, P, ws, None) == pm.ERR_ALIGNMENT
    assert f(ctypes.byref(cfg), P, P, P, ctypes.byref(c), 256, P, P, ws - 1, None) == pm.ERR_CAPACITY
    assert f(ctypes.byref(cfg), P, P, P, ctypes.byref(c), -1, P, P, ws, None) == pm.ERR_INVALID_ARG
