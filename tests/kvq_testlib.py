"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI and the
CPU oracle on the same seeded inputs, and compare (indices / codes / bytes bit-exact;
floats within the stated tolerances)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

D = 128
ATT_RTOL = 2e-3      # attention: ||o - o_ref||_inf <= 2e-3 * max(||o_ref||_inf, 1e-6) per (sequence, query head)
DEQ_ATOL = 1e-3      # dequantized values: max-abs
MINE_ATOL = 1e-3     # mining fallback tolerance (bit-exact is the target)


def to_torch(bits: np.ndarray, dtype: int, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device)
    return t.view(torch.bfloat16 if dtype == synth.BF16 else torch.float16)


def oracle_patterns(w: synth.Workload, Kf: np.ndarray, Vf: np.ndarray):
    """Oracle patterns (and column factors) per KV head, mined on the pooled prefill of all sequences."""
    MK, MV, cK, cV = [], [], [], []
    for h in range(w.Hkv):
        mk, ck, _ = oracle.mine_set(Kf[:, :, h].reshape(-1, D), w.P, w.iters, w.transform)
        mv, cv, _ = oracle.mine_set(Vf[:, :, h].reshape(-1, D), w.P, w.iters, w.transform)
        MK.append(mk); MV.append(mv); cK.append(ck); cV.append(cv)
    MK, MV = np.stack(MK), np.stack(MV)
    if w.transform:
        return MK, MV, np.stack(cK), np.stack(cV)
    return MK, MV, None, None


def gpu_v_rho(w: synth.Workload) -> float:
    """The library's fp32 rho* for the workload's V threshold (0 = off)."""
    import bit_kv_cache_26_b200 as kvq
    return kvq.kvq_v_rho_star(D, w.v_alpha)


def make_cache(w: synth.Workload, MK, MV, cK, cV, max_tokens=None, page_order=None):
    import bit_kv_cache_26_b200 as kvq
    cache = kvq.PagedKVCache(w.B, w.Hkv, max_tokens or max(w.S, 1), w.bits, w.P, dtype=w.dtype,
                             transform=w.transform, page_order=page_order, v_rho=gpu_v_rho(w))
    cache.k_patterns.copy_(torch.from_numpy(MK[None]))
    cache.v_patterns.copy_(torch.from_numpy(MV[None]))
    if w.transform:
        cache.k_colscale.copy_(torch.from_numpy(cK[None]))
        cache.v_colscale.copy_(torch.from_numpy(cV[None]))
    return cache


def encode_unit(w, Kf, Vf, b, h, MK, MV, cK, cV, N=None):
    N = w.S if N is None else N
    return oracle.encode(Kf[b, :N, h], Vf[b, :N, h], w.bits, MK[h], MV[h],
                         None if cK is None else cK[h], None if cV is None else cV[h], v_rho=oracle.v_rho(w.v_alpha))


def check_pages(cache, w, e: oracle.Encoded, b: int, h: int):
    """Bit-exact comparison of every defined byte of the unit's pages."""
    npages = (e.N + 31) // 32
    for pg in range(npages):
        want, defined = oracle.subblock(e, pg, w.transform)
        got = cache.subblock(b, pg, h).cpu().numpy()
        bad = np.flatnonzero((got != want) & defined)
        assert bad.size == 0, f"seq {b} head {h} page {pg}: {bad.size} bytes differ, first at {bad[:8]}"


def check_tail(cache, w, k_bits: np.ndarray, b: int, h: int, N: int):
    nt = N % 32
    if nt == 0:
        return
    got = cache.k_tail[b, h, :nt].view(torch.int16).cpu().numpy().view(np.uint16)
    want = k_bits[b, N - nt:N, h]
    assert np.array_equal(got, want), f"K tail of seq {b} head {h} differs"


def attention_ok(got: np.ndarray, want: np.ndarray):
    err = np.abs(got - want).max(axis=-1)
    ref = np.maximum(np.abs(want).max(axis=-1), 1e-6)
    return err <= ATT_RTOL * ref, err / ref
