"""kvq_decode_step (one-token quantize-append + decode attention in one launch) against the CPU
oracle, step by step: page bytes, indices and the K tail bit-exact, seq_len, and the decode
output of every step within 2e-3 relative.  Ragged prefills, steps that complete pages, 2- and
4-bit, the pre-transform, the V adaptive threshold, and decode-time Chebyshev-center insertion
with per-sequence pattern sets ("PatternKV", Section 3.1 Eq. 5, Section 3.2, Section 3.4)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from kvq_testlib import D, attention_ok, check_pages, check_tail, gpu_v_rho, to_torch

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS

CASES = {
    # prefill 100 (a partial page), 70 steps: pages complete at tokens 128 and 160
    "gqa4_2bit": (W["llama3_8b_32k"].with_(B=3, S=100, Hkv=2, Hq=8, P=16), 70),
    "gqa4_4bit": (W["llama3_8b_32k"].with_(B=2, S=64, Hkv=2, Hq=8, P=16, bits=4), 40),
    # GQA 7 with the Hadamard + dual-axis pre-transform, prefill 31 (tail only)
    "gqa7_transform": (W["qwen25_7b_128k"].with_(B=2, S=31, Hkv=2, Hq=14, P=8, transform=1), 45),
    # empty prefill: the first step opens the first page; the threshold off
    "from_empty": (W["llama3_8b_32k"].with_(B=2, S=0, Hkv=1, Hq=4, P=4, v_alpha=0.0), 40),
}


def _setup(w, steps, insertion=0, P_cap=None, per_seq_sets=False):
    import bit_kv_cache_26_b200 as kvq
    total = w.S + steps
    k, v = synth.gen_kv(w.with_(S=total))
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    nsets = w.B if per_seq_sets else 1
    # patterns: the oracle's, mined on (each sequence's or the pooled) prefill; a small prefill
    # borrows the first tokens of the whole stream
    src = max(w.S, 64)
    MK = np.zeros((nsets, w.Hkv, w.P, D), np.float32)
    MV = np.zeros_like(MK)
    CK = np.ones((nsets, w.Hkv, D), np.float32)
    CV = np.ones_like(CK)
    for s_ in range(nsets):
        for h in range(w.Hkv):
            xk = Kf[s_, :src, h] if per_seq_sets else Kf[:, :src, h].reshape(-1, D)
            xv = Vf[s_, :src, h] if per_seq_sets else Vf[:, :src, h].reshape(-1, D)
            MK[s_, h], ck, _ = oracle.mine_set(xk, w.P, w.iters, w.transform)
            MV[s_, h], cv, _ = oracle.mine_set(xv, w.P, w.iters, w.transform)
            if w.transform:
                CK[s_, h], CV[s_, h] = ck, cv
    P_cap = P_cap or w.P
    cache = kvq.PagedKVCache(w.B, w.Hkv, total, w.bits, P_cap, dtype=w.dtype, transform=w.transform,
                             num_sets=nsets, v_rho=gpu_v_rho(w),
                             seq_to_set=torch.arange(w.B, dtype=torch.int32) if per_seq_sets else None,
                             patterns_in_use=w.P if P_cap != w.P else None, insertion_window=insertion)
    cache.k_patterns[:, :, :w.P].copy_(torch.from_numpy(MK))
    cache.v_patterns[:, :, :w.P].copy_(torch.from_numpy(MV))
    if w.transform:
        cache.k_colscale.copy_(torch.from_numpy(CK))
        cache.v_colscale.copy_(torch.from_numpy(CV))
    kt, vt = to_torch(k, w.dtype), to_torch(v, w.dtype)
    if w.S:
        cache.append(kt[:, :w.S].contiguous(), vt[:, :w.S].contiguous())
    return dict(k=k, v=v, Kf=Kf, Vf=Vf, MK=MK, MV=MV, CK=CK if w.transform else None, CV=CV if w.transform else None,
                kt=kt, vt=vt, cache=cache)


def _check(w, d, b, h, N, q, out, MKs, MVs, e):
    cache = d["cache"]
    cK = None if d["CK"] is None else d["CK"][min(b, len(d["CK"]) - 1)][h]
    cV = None if d["CV"] is None else d["CV"][min(b, len(d["CV"]) - 1)][h]
    check_pages(cache, w, e, b, h)
    check_tail(cache, w, d["k"], b, h, N)
    Gq = w.Hq // w.Hkv
    qf = synth.to_float(q[b, h * Gq:(h + 1) * Gq], w.dtype)
    want = oracle.attention_unit(qf, d["Kf"][b, :N, h], e, MKs, MVs, cK, cV)
    ok, rel = attention_ok(out[b, h * Gq:(h + 1) * Gq], want)
    assert ok.all(), f"N={N} seq {b} kv head {h}: relative errors {rel}"


@pytest.mark.parametrize("name", list(CASES))
def test_decode_step_matches_oracle(name):
    w, steps = CASES[name]
    d = _setup(w, steps)
    cache = d["cache"]
    ws = cache.step_workspace(w.Hq)
    out = torch.empty(w.B, w.Hq, D, device="cuda")
    rho = oracle.v_rho(w.v_alpha)
    check_at = {0, 1, steps // 2, steps - 1} | {t for t in range(steps) if (w.S + t + 1) % 32 in (0, 1)}
    for t in range(steps):
        q = synth.gen_q(w, step=t)
        cache.step(d["kt"][:, w.S + t].contiguous(), d["vt"][:, w.S + t].contiguous(), to_torch(q, w.dtype), out, ws)
        if t in check_at:
            torch.cuda.synchronize()
            N = w.S + t + 1
            assert (cache.seq_len.cpu().numpy() == N).all()
            got = out.cpu().numpy()
            for b in range(w.B):
                for h in range(w.Hkv):
                    cK = None if d["CK"] is None else d["CK"][0][h]
                    cV = None if d["CV"] is None else d["CV"][0][h]
                    e = oracle.encode(d["Kf"][b, :N, h], d["Vf"][b, :N, h], w.bits, d["MK"][0][h], d["MV"][0][h],
                                      cK, cV, v_rho=rho)
                    _check(w, d, b, h, N, q, got, d["MK"][0][h], d["MV"][0][h], e)
    assert cache.read_status() == 0
    # the workspace's counters are back at zero after every step
    tail = ws.view(torch.int32)[-(w.B * w.Hkv + w.B + 64):]
    assert int(tail.abs().sum()) == 0


def test_decode_step_with_chebyshev_insertion():
    # per-sequence pattern sets of 8 patterns and room for 3 more; windows of 64 tokens after a
    # 128-token prefill: 4 windows in 256 steps, the capacity keeps 3 new patterns
    w = W["llama3_8b_32k"].with_(B=2, S=128, Hkv=2, Hq=8, P=8)
    steps, G, P_cap = 256, 64, 11
    d = _setup(w, steps, insertion=G, P_cap=P_cap, per_seq_sets=True)
    cache = d["cache"]
    ws = cache.step_workspace(w.Hq)
    out = torch.empty(w.B, w.Hq, D, device="cuda")
    rho = oracle.v_rho(w.v_alpha)
    for t in range(steps):
        q = synth.gen_q(w, step=t)
        cache.step(d["kt"][:, w.S + t].contiguous(), d["vt"][:, w.S + t].contiguous(), to_torch(q, w.dtype), out, ws)
        N = w.S + t + 1
        if t in (G - 2, G - 1, G, 2 * G, steps - 1):
            torch.cuda.synchronize()
            got = out.cpu().numpy()
            counts = cache.pattern_counts.cpu().numpy()
            for b in range(w.B):
                for h in range(w.Hkv):
                    e, MKs, MVs = oracle.encode_stream(d["Kf"][b, :N, h], d["Vf"][b, :N, h], w.S, w.bits,
                                                       d["MK"][b][h], d["MV"][b][h], Pmax=P_cap, G=G, v_rho=rho)
                    assert counts[b, h] == MKs.shape[0], (t, b, h, counts[b, h], MKs.shape[0])
                    gk = cache.k_patterns[b, h, :MKs.shape[0]].cpu().numpy()
                    gv = cache.v_patterns[b, h, :MVs.shape[0]].cpu().numpy()
                    assert np.array_equal(gk, MKs) and np.array_equal(gv, MVs), (t, b, h)
                    _check(w, d, b, h, N, q, got, MKs, MVs, e)
    assert (cache.pattern_counts.cpu().numpy() == P_cap).all()
    assert cache.read_status() == 0
