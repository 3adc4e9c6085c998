"""The decode entry point that allocates nothing (pnmix_decode_attention_noalloc).

Callers that cannot allocate device memory -- a plugin whose host runtime owns
every byte of device memory, or an interface with no slot for a workspace
pointer -- use this call; its split-K scratch is a fixed 4 MiB array inside the
library.  These checks call it through the C ABI and compare it with
pnmix_decode_attention (caller workspace) and with the CPU oracle on two calls in a
row, with a call of another shape in between that leaves different contents in the
shared array.
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_harness import Case, assert_close, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(pm, cfg, q, cache, out, max_context=None):
    return pm._lib.pnmix_decode_attention_noalloc(
        ctypes.byref(cfg), q.data_ptr(), ctypes.byref(cache.c),
        cache.max_context if max_context is None else max_context, out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def test_noalloc_decode_matches_the_workspace_entry_point_twice():
    a = Case(2, 8, 2, 300, seed=21)
    a.prefill(check=False)
    b = Case(3, 28, 4, 700, seed=22)     # another geometry: other split count and units
    b.prefill(check=False)
    pm = a.pm
    qa, qb = to_dev(a.query(300)), to_dev(b.query(700))
    ref_a = torch.empty(2, 8, 128, dtype=torch.float32, device="cuda")
    ref_b = torch.empty(3, 28, 128, dtype=torch.float32, device="cuda")
    pm.pnmix_decode_attention(a.cfg, qa, a.cache, ref_a)
    pm.pnmix_decode_attention(b.cfg, qb, b.cache, ref_b)
    torch.cuda.synchronize()
    ref_a, ref_b = ref_a.cpu().numpy().astype(np.float64), ref_b.cpu().numpy().astype(np.float64)
    want_a, want_b = a.ocache.attend(a.query(300)), b.ocache.attend(b.query(700))
    for _ in range(2):
        out = torch.full((2, 8, 128), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(pm, a.cfg, qa, a.cache, out) == pm.OK
        torch.cuda.synchronize()
        assert_close(out.cpu().numpy(), ref_a)
        assert_close(out.cpu().numpy(), want_a)
        out_b = torch.full((3, 28, 128), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(pm, b.cfg, qb, b.cache, out_b) == pm.OK
        torch.cuda.synchronize()
        assert_close(out_b.cpu().numpy(), ref_b)
        assert_close(out_b.cpu().numpy(), want_b)


def test_noalloc_rejects_a_workspace_beyond_its_scratch():
    import decode_attention_prefill_b200 as pm
    cfg = pm.Config.make(64, 8)           # G = 8
    cache = pm.PNMixCache(cfg, 128, 32)   # 1024 units -> > 4 MiB of partials
    assert pm.workspace_bytes(cfg, 128, 32) > (4 << 20)
    q = torch.zeros(128, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(128, 64, 128, dtype=torch.float32, device="cuda")
    assert _noalloc(pm, cfg, q, cache, out, max_context=32) == pm.ERR_CAPACITY
