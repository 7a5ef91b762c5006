"""The allocation-free decode entry point (kvq_decode_attention_static) against the
workspace one (kvq_decode_attention) on the same cache and queries, two calls in a row
(the second reuses the library's fixed scratch array), and its size limit."""
import numpy as np
import pytest
import torch

import synth
from kvq_testlib import D, make_cache, oracle_patterns, to_torch

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


@pytest.fixture(scope="module")
def filled():
    w = W["llama3_8b_32k"].with_(B=3, S=700, Hkv=2, Hq=8, P=16)
    k, v = synth.gen_kv(w)
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    MK, MV, cK, cV = oracle_patterns(w, Kf, Vf)
    cache = make_cache(w, MK, MV, cK, cV)
    cache.append(to_torch(k, w.dtype), to_torch(v, w.dtype))
    torch.cuda.synchronize()
    assert cache.read_status() == 0
    return w, cache


def test_static_scratch_matches_workspace_twice(filled):
    import bit_kv_cache_26_b200 as kvq
    w, cache = filled
    scale = D ** -0.5
    for seed_shift in (0, 1):  # two different queries, each checked on two calls in a row
        q = to_torch(synth.gen_q(w.with_(seed=w.seed + seed_shift)), w.dtype)
        ref = torch.empty(w.B, w.Hq, D, device="cuda")
        kvq.kvq_decode_attention(cache.c, q, w.Hq, scale, ref, cache.decode_workspace(w.Hq))
        for _ in range(2):
            got = torch.full((w.B, w.Hq, D), float("nan"), device="cuda")
            kvq.kvq_decode_attention_static(cache.c, q, w.Hq, scale, got)
            torch.cuda.synchronize()
            assert torch.equal(got, ref)
    assert cache.read_status() == 0


def test_static_scratch_rejects_oversize_before_launch():
    import bit_kv_cache_26_b200 as kvq
    # 1024 sequences x 64 query heads: the split partials alone exceed the fixed array
    cache = kvq.PagedKVCache(1024, 4, 32, 2, 64)
    assert kvq.kvq_decode_workspace_bytes(cache.c, 64) > kvq.KVQ_DECODE_STATIC_SCRATCH_BYTES
    q = torch.zeros(1024, 64, D, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(1024, 64, D, device="cuda")
    with pytest.raises(kvq.KvqError) as ei:
        kvq.kvq_decode_attention_static(cache.c, q, 64, D ** -0.5, out)
    assert ei.value.status == kvq.KVQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (out == 0).all()
