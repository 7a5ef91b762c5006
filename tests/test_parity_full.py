"""GPU parity at the workloads' full sizes, on sampled outputs the oracle computes one by
one: the Llama-shaped workload (llama3_8b_32k, 2- and 4-bit), the Qwen-shaped 128K workload
with and without the pre-transform, the breadth workload (all 256 samples with per-sample
perturbed centers, each at the full 16K context: the launched grids are the benchmark's) and
the long chain-of-thought decode loop (8K prefill, then 4096 decode steps, each one
kvq_decode_step launch: a one-token append and decode attention).

Per case: mining of one KV head (K and V) against the oracle's Lloyd on the same pooled
prefill; page bytes, pattern indices and the K tail of sampled (sequence, KV head) units
against the oracle's encoding with the mined patterns; decode outputs of those units against
the oracle's attention over its encoding."""
import numpy as np
import pytest
import torch

import oracle
import synth
from kvq_testlib import D, attention_ok, check_pages, check_tail, gpu_v_rho, to_torch

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _gpu_mine(cache, w, kt, vt):
    import bit_kv_cache_26_b200 as kvq
    n = kt.shape[0] * kt.shape[1]
    for x, pat, col in ((kt, cache.k_patterns, cache.k_colscale), (vt, cache.v_patterns, cache.v_colscale)):
        xs = x.reshape(1, n, w.Hkv, D)
        ws = kvq._alloc_aligned(kvq.kvq_mine_workspace_bytes(n, 1, w.Hkv, w.P, w.transform), x.device)
        kvq.kvq_mine_patterns(xs, w.dtype, n, 1, w.Hkv, w.Hkv * D, D, n * w.Hkv * D, w.P, w.iters, w.transform,
                              pat, col, None, ws)


def _patterns(cache, w):
    MK = cache.k_patterns.cpu().numpy()[0]
    MV = cache.v_patterns.cpu().numpy()[0]
    if w.transform:
        return MK, MV, cache.k_colscale.cpu().numpy()[0], cache.v_colscale.cpu().numpy()[0]
    return MK, MV, None, None


def _check_mining_head(w, k, v, h, MK, MV, cK, cV):
    for x, M, c in ((k, MK, cK), (v, MV, cV)):
        xf = synth.to_float(x[:, :, h], w.dtype).reshape(-1, D)
        mo, co, _ = oracle.mine_set(xf, w.P, w.iters, w.transform)
        if w.transform:
            assert np.allclose(c[h], co, rtol=1e-6, atol=0)
            assert np.abs(M[h] - mo).max() <= 1e-3
        else:
            assert np.array_equal(M[h], mo), f"head {h}: max diff {np.abs(M[h] - mo).max()}"


def _check_unit(cache, w, k, v, b, h, N, MK, MV, cK, cV, q=None, out=None):
    Kf = synth.to_float(k[b, :N, h], w.dtype)
    Vf = synth.to_float(v[b, :N, h], w.dtype)
    e = oracle.encode(Kf, Vf, w.bits, MK[h], MV[h], None if cK is None else cK[h], None if cV is None else cV[h],
                      v_rho=oracle.v_rho(w.v_alpha))
    check_pages(cache, w, e, b, h)
    check_tail(cache, w, k, b, h, N)
    if q is not None:
        Gq = w.Hq // w.Hkv
        qf = synth.to_float(q[b, h * Gq:(h + 1) * Gq], w.dtype)
        want = oracle.attention_unit(qf, Kf, e, MK[h], MV[h], None if cK is None else cK[h],
                                     None if cV is None else cV[h])
        ok, rel = attention_ok(out[b, h * Gq:(h + 1) * Gq], want)
        assert ok.all(), f"seq {b} kv head {h}: relative errors {rel}"


FULL = {
    "llama3_8b_32k_2bit": W["llama3_8b_32k"],
    "llama3_8b_32k_4bit": W["llama3_8b_32k"].with_(bits=4),
    "qwen25_7b_128k": W["qwen25_7b_128k"],
    "qwen25_7b_128k_transform": W["qwen25_7b_128k"].with_(transform=1),
    "breadth_256x16k": W["breadth_256x16k"],
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_prefill_and_decode(name):
    import bit_kv_cache_26_b200 as kvq
    w = FULL[name]
    k, v = synth.gen_kv(w)
    kt, vt = to_torch(k, w.dtype), to_torch(v, w.dtype)
    cache = kvq.PagedKVCache(w.B, w.Hkv, w.S, w.bits, w.P, dtype=w.dtype, transform=w.transform, v_rho=gpu_v_rho(w))
    _gpu_mine(cache, w, kt, vt)
    cache.append(kt, vt)
    q = synth.gen_q(w)
    out = torch.empty(w.B, w.Hq, D, device="cuda")
    cache.decode(to_torch(q, w.dtype), out, cache.decode_workspace(w.Hq))
    out = out.cpu().numpy()
    assert cache.read_status() == 0
    del kt, vt
    MK, MV, cK, cV = _patterns(cache, w)
    _check_mining_head(w, k, v, w.Hkv - 1, MK, MV, cK, cV)
    for b, h in ((0, 0), (w.B - 1, w.Hkv - 1)):
        _check_unit(cache, w, k, v, b, h, w.S, MK, MV, cK, cV, q, out)


def test_long_cot_decode_loop():
    """8192-token prefill, patterns mined once and frozen, then 4096 decode steps, each one
    kvq_decode_step launch (a one-token quantize-append per sequence and decode attention with a
    new query), as the benchmark runs them."""
    import bit_kv_cache_26_b200 as kvq
    w = W["long_cot_8k"]
    total = w.S + w.steps
    k, v = synth.gen_kv(w.with_(S=total))
    kt, vt = to_torch(k, w.dtype), to_torch(v, w.dtype)
    cache = kvq.PagedKVCache(w.B, w.Hkv, total, w.bits, w.P, dtype=w.dtype, transform=w.transform, v_rho=gpu_v_rho(w))
    _gpu_mine(cache, w, kt[:, :w.S].contiguous(), vt[:, :w.S].contiguous())
    cache.append(kt[:, :w.S].contiguous(), vt[:, :w.S].contiguous())
    MK, MV, cK, cV = _patterns(cache, w)
    _check_mining_head(w, k[:, :w.S], v[:, :w.S], w.Hkv - 1, MK, MV, cK, cV)
    ws = cache.step_workspace(w.Hq)
    out = torch.empty(w.B, w.Hq, D, device="cuda")
    check_at = {0, 31, 1000, w.steps - 1}
    units = ((0, 0), (w.B - 1, w.Hkv - 1))
    for t in range(w.steps):
        q = synth.gen_q(w, step=t)
        cache.step(kt[:, w.S + t].contiguous(), vt[:, w.S + t].contiguous(), to_torch(q, w.dtype), out, ws)
        if t in check_at:
            got = out.cpu().numpy()
            for b, h in units:
                _check_unit(cache, w, k, v, b, h, w.S + t + 1, MK, MV, cK, cV, q, got)
    torch.cuda.synchronize()
    assert cache.read_status() == 0
