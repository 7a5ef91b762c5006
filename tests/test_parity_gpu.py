"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle on identical
seeded inputs.  Pattern indices, codes, scales and the K tail are compared bit for bit;
dequantized values to max-abs 1e-3; attention outputs to 2e-3 relative per output vector."""
import numpy as np
import pytest
import torch

import oracle
import synth
from kvq_testlib import (D, DEQ_ATOL, attention_ok, check_pages, check_tail, encode_unit, make_cache,
                         oracle_patterns, to_torch)

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS

CASES = {
    # the tiny reference workload, exactly: 1 x 4096 tokens, 1 KV head, fp16, P=16, 2-bit
    "tiny_ref": (W["tiny_ref_4k"], [4096]),
    # Llama-shaped heads at small size: GQA 4, P=64, ragged length, appended in uneven chunks
    "gqa4_2bit_ragged": (W["llama3_8b_32k"].with_(B=2, S=1000, Hkv=2, Hq=8), [37, 1, 462, 500]),
    "gqa4_4bit_ragged": (W["llama3_8b_32k"].with_(B=2, S=1000, Hkv=2, Hq=8, bits=4), [1000]),
    # Qwen-shaped heads, GQA 7, with the Hadamard + dual-axis pre-transform
    "gqa7_transform": (W["qwen25_7b_128k"].with_(B=2, S=777, Hkv=2, Hq=14, P=16, transform=1), [700, 77]),
    # tail only (fewer than 32 tokens), one pattern
    "tail_only_p1": (W["llama3_8b_32k"].with_(B=1, S=20, Hkv=1, Hq=1, P=1), [20]),
    # exact multiple of the group: no tail; one-token appends across a page boundary
    "no_tail_token_steps": (W["llama3_8b_32k"].with_(B=3, S=64, Hkv=1, Hq=2, P=8), [30, 1, 1, 32]),
    # many sequences, per-sample perturbed centers
    "breadth_small": (W["breadth_256x16k"].with_(B=16, S=100, Hkv=2, Hq=8, P=32), [100]),
    # more than 64 patterns: the tcgen05 assignment with 7-bit tags, 224 score columns and one
    # CTA per SM, the cluster sums with 8 clusters per warp, the fix-up with 128 threads a token
    "gqa4_p100": (W["llama3_8b_32k"].with_(B=2, S=1000, Hkv=2, Hq=8, P=100), [1000]),
    # pattern counts that pad the tcgen05 tile: 17 (32-column accumulators), 48 (48 of 64
    # columns used), 128 (the largest tcgen05 tile: four 128-column buffers, all of TMEM)
    "gqa4_p17": (W["llama3_8b_32k"].with_(B=1, S=500, Hkv=1, Hq=4, P=17), [250, 250]),
    "gqa4_p48": (W["llama3_8b_32k"].with_(B=2, S=600, Hkv=2, Hq=8, P=48), [600]),
    "gqa4_p128": (W["llama3_8b_32k"].with_(B=1, S=700, Hkv=1, Hq=4, P=128), [700]),
    # the largest pattern count the u8 indices allow: float64 assignment, 16 clusters per warp
    "p255": (W["llama3_8b_32k"].with_(B=1, S=600, Hkv=1, Hq=4, P=255), [300, 300]),
    # V adaptive threshold: every fourth V vector replaced by one far from every pattern (planted
    # rejections, index 255, quantized raw), with and without the pre-transform, at 2 and 4 bits
    "v_threshold_planted": (W["llama3_8b_32k"].with_(B=2, S=700, Hkv=2, Hq=8, P=32), [350, 350]),
    "v_threshold_planted_4bit_tx": (W["qwen25_7b_128k"].with_(B=1, S=500, Hkv=2, Hq=14, P=16, bits=4, transform=1),
                                    [500]),
    # the threshold off: every V vector keeps its nearest pattern
    "v_threshold_off": (W["llama3_8b_32k"].with_(B=2, S=300, Hkv=2, Hq=8, P=16, v_alpha=0.0), [300]),
}
PLANT_V = {"v_threshold_planted", "v_threshold_planted_4bit_tx"}


def plant_far_v(v: np.ndarray, dtype: int, seed: int) -> np.ndarray:
    """Every fourth token's V vectors replaced by N(0, 3^2) values (bit patterns of the dtype)."""
    rng = np.random.default_rng(seed)
    v = v.copy()
    x = (rng.standard_normal(v[:, ::4].shape) * 3).astype(np.float32)
    v[:, ::4] = (x.view(np.uint32) >> 16).astype(np.uint16) if dtype == synth.BF16 else \
        x.astype(np.float16).view(np.uint16)
    return v


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    w, chunks = CASES[request.param]
    assert sum(chunks) == w.S
    k, v = synth.gen_kv(w)
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    # patterns mined before any planting: the planted V vectors lie away from every pattern
    MK, MV, cK, cV = oracle_patterns(w, Kf, Vf) if w.B * w.S >= w.P else (None,) * 4
    if request.param in PLANT_V:
        v = plant_far_v(v, w.dtype, seed=w.seed)
        Vf = synth.to_float(v, w.dtype)
    cache = make_cache(w, MK, MV, cK, cV)
    kt, vt = to_torch(k, w.dtype), to_torch(v, w.dtype)
    s0 = 0
    for n in chunks:
        cache.append(kt[:, s0:s0 + n].contiguous(), vt[:, s0:s0 + n].contiguous())
        s0 += n
    torch.cuda.synchronize()
    assert cache.read_status() == 0
    return dict(name=request.param, w=w, k=k, v=v, Kf=Kf, Vf=Vf, MK=MK, MV=MV, cK=cK, cV=cV, cache=cache)


def test_seq_len(case):
    assert (case["cache"].seq_len.cpu().numpy() == case["w"].S).all()


def test_pages_and_tail_bit_exact(case):
    w = case["w"]
    for b in range(w.B):
        for h in range(w.Hkv):
            e = encode_unit(w, case["Kf"], case["Vf"], b, h, case["MK"], case["MV"], case["cK"], case["cV"])
            check_pages(case["cache"], w, e, b, h)
            check_tail(case["cache"], w, case["k"], b, h, w.S)


def test_v_threshold_rejections(case):
    # the oracle's encoding (which the page bytes match bit for bit) rejects many more of the
    # planted vectors than of the others, and the threshold decides both ways in every case
    w = case["w"]
    if w.B * w.S < w.P:
        pytest.skip("no patterns")
    raw = np.concatenate([encode_unit(w, case["Kf"], case["Vf"], b, h, case["MK"], case["MV"], case["cK"],
                                      case["cV"]).vidx == 255 for b in range(w.B) for h in range(w.Hkv)])
    if case["name"] in PLANT_V:
        planted = np.zeros(w.S, bool)
        planted[::4] = True
        planted = np.tile(planted, w.B * w.Hkv)
        fp, fu = raw[planted].mean(), raw[~planted].mean()
        assert fp > fu + 0.3 and 0 < fu < 0.5, (fp, fu)
    elif w.v_alpha == 0:
        assert not raw.any()


def test_dequantize(case):
    import bit_kv_cache_26_b200 as kvq
    w, cache = case["w"], case["cache"]
    for b in range(min(w.B, 3)):
        ko = torch.empty(w.S, w.Hkv, D, device="cuda")
        vo = torch.empty(w.S, w.Hkv, D, device="cuda")
        kvq.kvq_dequantize(cache.c, b, w.S, 0, w.S, ko, vo)
        ko, vo = ko.cpu().numpy(), vo.cpu().numpy()
        for h in range(w.Hkv):
            e = encode_unit(w, case["Kf"], case["Vf"], b, h, case["MK"], case["MV"], case["cK"], case["cV"])
            Kh, Vh = oracle.dequant(e, case["MK"][h], case["MV"][h], None if case["cK"] is None else case["cK"][h],
                                    None if case["cV"] is None else case["cV"][h])
            G = (w.S // 32) * 32
            Kfull = np.concatenate([Kh, case["Kf"][b, G:w.S, h]])
            assert np.abs(ko[:, h] - Kfull).max() <= DEQ_ATOL
            assert np.abs(vo[:, h] - Vh).max() <= DEQ_ATOL


def test_decode_attention(case):
    w, cache = case["w"], case["cache"]
    q = synth.gen_q(w)
    qt = to_torch(q, w.dtype)
    out = torch.empty(w.B, w.Hq, D, device="cuda")
    ws = cache.decode_workspace(w.Hq)
    cache.decode(qt, out, ws)
    got = out.cpu().numpy()
    qf = synth.to_float(q, w.dtype)
    Gq = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hkv):
            e = encode_unit(w, case["Kf"], case["Vf"], b, h, case["MK"], case["MV"], case["cK"], case["cV"])
            want = oracle.attention_unit(qf[b, h * Gq:(h + 1) * Gq], case["Kf"][b, :, h], e, case["MK"][h],
                                         case["MV"][h], None if case["cK"] is None else case["cK"][h],
                                         None if case["cV"] is None else case["cV"][h])
            ok, rel = attention_ok(got[b, h * Gq:(h + 1) * Gq], want)
            assert ok.all(), f"seq {b} kv head {h}: relative errors {rel}"


def test_mining_matches_oracle(case):
    import bit_kv_cache_26_b200 as kvq
    w = case["w"]
    if w.B * w.S < w.P:
        pytest.skip("fewer tokens than patterns")
    x = to_torch(case["k"], w.dtype).reshape(1, w.B * w.S, w.Hkv, D).contiguous()
    pats, col, _ = kvq.mine(x, w.P, w.iters, w.transform)
    pats = pats.cpu().numpy()[0]
    if w.transform:
        col = col.cpu().numpy()[0]
        assert np.allclose(col, case["cK"], rtol=1e-6, atol=0)
        assert np.abs(pats - case["MK"]).max() <= 1e-3
    else:
        assert np.array_equal(pats, case["MK"]), f"max diff {np.abs(pats - case['MK']).max()}"


def test_empty_sequence_decodes_to_zero():
    import bit_kv_cache_26_b200 as kvq
    w = W["llama3_8b_32k"].with_(B=2, S=64, Hkv=1, Hq=4, P=4)
    cache = kvq.PagedKVCache(w.B, w.Hkv, 64, 2, 4)
    out = torch.full((w.B, w.Hq, D), 7.0, device="cuda")
    q = to_torch(synth.gen_q(w), w.dtype)
    cache.decode(q, out, cache.decode_workspace(w.Hq))
    assert (out == 0).all()


def test_overflow_flags_device_status():
    import bit_kv_cache_26_b200 as kvq
    w = W["llama3_8b_32k"].with_(B=1, S=40, Hkv=1, Hq=1, P=2)
    cache = kvq.PagedKVCache(1, 1, 32, 2, 2)
    k, v = synth.gen_kv(w)
    cache.append(to_torch(k, w.dtype)[:, :30].contiguous(), to_torch(v, w.dtype)[:, :30].contiguous())
    cache.append(to_torch(k, w.dtype)[:, 30:40].contiguous(), to_torch(v, w.dtype)[:, 30:40].contiguous())
    torch.cuda.synchronize()
    assert cache.read_status(clear=True) == kvq.KVQ_DEV_OVERFLOW
    assert int(cache.seq_len[0]) == 30
    assert cache.read_status() == 0


def test_identical_patterns_resolve_ties_to_lowest_index():
    # Every pattern equal: the min-max distances all tie, the pruning bound excludes nothing
    # (the kernel falls back to evaluating every pattern) and index 0 must win everywhere.
    # (the V threshold off: with every pattern equal to one vector it would reject the others)
    w = W["llama3_8b_32k"].with_(B=1, S=96, Hkv=1, Hq=2, P=64, v_alpha=0.0)
    k, v = synth.gen_kv(w)
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    MK = np.repeat(Kf[0, :1, 0], 64, axis=0)[None]
    MV = np.repeat(Vf[0, :1, 0], 64, axis=0)[None]
    cache = make_cache(w, MK, MV, None, None)
    cache.append(to_torch(k, w.dtype), to_torch(v, w.dtype))
    torch.cuda.synchronize()
    e = encode_unit(w, Kf, Vf, 0, 0, MK, MV, None, None)
    assert (e.kidx == 0).all() and (e.vidx == 0).all()
    check_pages(cache, w, e, 0, 0)


@pytest.mark.parametrize("bits", [2, 4])
def test_subnormal_scales_bit_exact(bits):
    # Groups and channels whose residuals differ only by subnormal amounts: the scale
    # s = (max - min) / maxc is subnormal (or 0), its reciprocal inexact or infinite, and every
    # code must still be the definition's rne(fl32(t / s)), clamped ("PatternKV", Section 3.2,
    # Eq. 1).  Two whole pages (codes from the one-FMA path, whose tiny-scale exception divides)
    # and a 20-token partial page (the per-word path), the patterns zero where the tiny values sit.
    w = W["llama3_8b_32k"].with_(B=1, S=84, Hkv=1, Hq=2, P=4, bits=bits, v_alpha=0.0)
    k, v = synth.gen_kv(w)
    rng = np.random.default_rng(7)
    tiny = np.float32(2.0 ** -130)

    def bf16_bits(a):
        return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)

    k, v = k.copy(), v.copy()
    # V: group 0 (channels 0..31) of every token: zeros and small multiples of 2^-130
    v[0, :, 0, :32] = bf16_bits(tiny * rng.integers(0, 4, size=(w.S, 32)).astype(np.float32))
    # V: group 2 of the even tokens: one value 3 * 2^-133 (2^-133: the smallest bf16 subnormal),
    # the rest 0
    g2 = np.zeros((w.S, 32), np.float32)
    g2[::2, 5] = np.float32(3 * 2.0 ** -133)
    v[0, :, 0, 64:96] = bf16_bits(g2)
    # K: channels 7 and 100 over every token: tiny values (per-channel scales of the pages)
    k[0, :, 0, 7] = bf16_bits(tiny * rng.integers(0, 9, size=w.S).astype(np.float32))
    k[0, :, 0, 100] = bf16_bits(np.where(np.arange(w.S) % 3 == 0, np.float32(2.0 ** -132), np.float32(0)))
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    MK, MV, _, _ = oracle_patterns(w, Kf, Vf)
    MK[:, :, [7, 100]] = 0.0
    MV[:, :, :32] = 0.0
    MV[:, :, 64:96] = 0.0
    cache = make_cache(w, MK, MV, None, None)
    cache.append(to_torch(k, w.dtype), to_torch(v, w.dtype))
    torch.cuda.synchronize()
    assert cache.read_status() == 0
    e = encode_unit(w, Kf, Vf, 0, 0, MK, MV, None, None)
    assert np.any(e.vs[:, 0] != 0) and np.all(np.abs(e.vs[:, 0]) < 2.0 ** -126)
    assert np.any((e.ks != 0) & (np.abs(e.ks) < 2.0 ** -126))
    assert np.any(e.vs[:, 2] != 0) and np.any(e.ks[:, 100] != 0)
    check_pages(cache, w, e, 0, 0)
    check_tail(cache, w, k, 0, 0, w.S)


@pytest.mark.parametrize("bits", [2, 4])
def test_code_ties_round_half_even(bits):
    # Residuals placed exactly on rounding boundaries: in V group 1 and K channel 9 the values
    # are 0, maxc and half-integers in between, so (R - z) / s is a half-integer (exactly) and the
    # definition rounds it half to even ("PatternKV", Section 3.2, Eq. 1).  Whole pages (the
    # one-FMA codes, whose boundary exception divides) and a partial page.
    w = W["llama3_8b_32k"].with_(B=1, S=80, Hkv=1, Hq=2, P=4, bits=bits, v_alpha=0.0)
    k, v = synth.gen_kv(w)
    maxc = (1 << bits) - 1
    rng = np.random.default_rng(11)
    ladder = np.array([0.0, maxc] + [h + 0.5 for h in range(maxc)], np.float32)  # s = 1 when 0 and maxc occur

    def bf16_bits(a):
        return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)

    k, v = k.copy(), v.copy()
    g1 = ladder[rng.integers(0, len(ladder), size=(w.S, 32))]
    g1[:, 0], g1[:, 1] = 0.0, maxc
    v[0, :, 0, 32:64] = bf16_bits(g1)
    kc = ladder[rng.integers(0, len(ladder), size=w.S)]
    kc[::32], kc[1::32] = 0.0, maxc
    k[0, :, 0, 9] = bf16_bits(kc)
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    MK, MV, _, _ = oracle_patterns(w, Kf, Vf)
    MK[:, :, 9] = 0.0
    MV[:, :, 32:64] = 0.0
    cache = make_cache(w, MK, MV, None, None)
    cache.append(to_torch(k, w.dtype), to_torch(v, w.dtype))
    torch.cuda.synchronize()
    assert cache.read_status() == 0
    e = encode_unit(w, Kf, Vf, 0, 0, MK, MV, None, None)
    assert np.all(e.vs[:, 1] == 1.0) and np.all(e.ks[:, 9] == 1.0)
    # the half-integers did round to even codes
    half = (g1 % 1.0) == 0.5
    assert half.any() and np.all(e.vcode[:, 32:64][half] % 2 == 0)
    check_pages(cache, w, e, 0, 0)
    check_tail(cache, w, k, 0, 0, w.S)
