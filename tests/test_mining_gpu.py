"""GPU mining against the oracle on inputs built to stress the certified argmin.

The tensor-core assignment ("PatternKV", Section 3.1, Eq. 4: Lloyd k-means under the
Euclidean metric) decides a token on the spot only when its two best approximate scores are
further apart than an error bound; the rest go to an exact float64 decision.  Here the
tokens sit between pairs of nearby patterns, with gaps spread from exact ties through
one-ulp differences to about ten times the bound, so a bound that is too tight, or an exact
path that breaks ties differently, shows up as a mismatch.

Also here: the pre-transform mode (fp32 rows after the KVarN Hadamard + dual-axis
normalisation), whose float64 centroid sums depend on the order of the additions: the GPU
result must be the same on every run, its assignment must be the exact argmin of its own
inputs, and every difference from the oracle must be a certified near-tie."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

D = 128


def _bf16(a):
    """float -> nearest bf16 (ties to even), as float32."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def _round16(a, fp16: bool):
    """float -> nearest value of the 16-bit input type (fp16 or bf16), as float32."""
    return np.asarray(a, np.float32).astype(np.float16).astype(np.float32) if fp16 else _bf16(a)


def planted_ties(n: int, P: int, seed: int, fp16: bool = False):
    """n bf16 rows whose strided-initial patterns (rows floor(j n / P)) come in pairs (2i, 2i+1):
    even pairs are one-channel twins (equal except channel d0, 1.0 vs 1.5), odd pairs differ by
    N(0, 0.3^2) noise.  Other rows: 10 % exact ties between twins (channel d0 at the midpoint
    1.25), 5 % one bf16 ulp off the midpoint, the rest a + t (b - a) + N(0, 0.05^2) with t
    within 10^-5 .. 10^-1 of one half."""
    rng = np.random.default_rng(seed)
    npair = (P + 1) // 2
    base = rng.standard_normal((npair, D)) * 2.0
    d0 = rng.integers(0, D, npair)
    pats = np.zeros((P, D))
    for j in range(P):
        i = j // 2
        pats[j] = base[i]
        if i % 2 == 0:
            pats[j, d0[i]] = 1.5 if j % 2 else 1.0
        elif j % 2:
            pats[j] += rng.standard_normal(D) * 0.3
    pats = _round16(pats, fp16)
    x = np.zeros((n, D), np.float32)
    for r in range(n):
        i = int(rng.integers(0, npair))
        j = 2 * i
        a = pats[j].astype(np.float64)
        b = pats[min(j + 1, P - 1)].astype(np.float64)
        u = rng.random()
        if i % 2 == 0 and j + 1 < P and u < 0.15:
            v = a.copy()
            v[d0[i]] = 1.25 if u < 0.10 else 1.25 + (2.0 ** -7 if u < 0.125 else -2.0 ** -7)
        else:
            t = 0.5 + rng.standard_normal() * 10 ** rng.uniform(-5, -1)
            v = a + t * (b - a) + rng.standard_normal(D) * 0.05
        x[r] = _round16(v, fp16)
    for j in range(P):
        x[(j * n) // P] = pats[j]
    return x


def _to_dev(x32: np.ndarray, dtype):
    t = torch.from_numpy(x32).to(dtype)
    assert torch.equal(t.float(), torch.from_numpy(x32)), "rows must be exact in the input dtype"
    return t.reshape(1, -1, 1, D).contiguous().cuda()


@pytest.mark.parametrize("P,n,dtype", [
    (64, 8192, torch.bfloat16),    # tcgen05 assignment, 128 score columns, two CTAs per SM
    (100, 8192, torch.bfloat16),   # tcgen05 assignment, 224 score columns, one CTA per SM
    (32, 4096, torch.float16),     # mma.sync assignment (fp16 rows split into hi + lo)
    (48, 8192, torch.bfloat16),    # tcgen05 assignment, 48 of a 64-column accumulator used
    (128, 8192, torch.bfloat16),   # tcgen05 assignment, four 128-column accumulators
])
@pytest.mark.parametrize("iters", [1, 4])
def test_planted_near_ties_bit_exact(P, n, dtype, iters):
    import bit_kv_cache_26_b200 as kvq
    x = planted_ties(n, P, seed=P + n, fp16=dtype == torch.float16)
    xd = _to_dev(x, dtype)
    pats, _, asg = kvq.mine(xd, P, iters, want_assign=True)
    M, a = oracle.mine(x, P, iters)
    ga = asg.cpu().numpy()[0, 0]
    bad = np.flatnonzero(ga != a)
    assert bad.size == 0, f"{bad.size} assignments differ, first tokens {bad[:8]}"
    assert np.array_equal(pats.cpu().numpy()[0, 0], M)
    if iters == 1:
        # the planted exact ties are there (the first 1024 rows against the initial patterns)
        init = x[[(j * n) // P for j in range(P)]].astype(np.float64)
        d = ((x[:1024, None, :].astype(np.float64) - init[None]) ** 2).sum(axis=2)
        srt = np.sort(d, axis=1)
        assert (srt[:, 1] == srt[:, 0]).sum() > 1024 // 20


def _margin(y, yg, M, Mg, j):
    """Bound on |d(y, M_j) - d(yg, Mg_j)| from the input differences (norms, float64)."""
    e = np.linalg.norm(y.astype(np.float64) - yg) + np.linalg.norm(M[j].astype(np.float64) - Mg[j])
    r = np.linalg.norm(y.astype(np.float64) - M[j])
    return 2 * r * e + e * e


def test_transform_mining_deterministic_exact_and_certified():
    import bit_kv_cache_26_b200 as kvq
    w = synth.WORKLOADS["qwen25_7b_128k"].with_(B=2, S=1500, Hkv=1, Hq=7, P=16, transform=1)
    k, _ = synth.gen_kv(w, want_v=False)
    xf = synth.to_float(k, w.dtype).reshape(-1, D)
    xd = torch.from_numpy(np.ascontiguousarray(k).view(np.int16)).view(torch.bfloat16).reshape(1, -1, 1, D).cuda()
    it = w.iters
    runs = [kvq.mine(xd, w.P, it, transform=1, want_assign=True) for _ in range(2)]
    for t0, t1 in zip(runs[0], runs[1]):
        assert torch.equal(t0, t1), "transform-mode mining differs between two runs on the same input"
    pats, col, asg = (t.cpu().numpy()[0, 0] for t in runs[0])
    prev, colp, _ = (None if t is None else t.cpu().numpy()[0, 0]
                     for t in kvq.mine(xd, w.P, it - 1, transform=1, want_assign=False))
    assert np.array_equal(colp, col)
    # column factors: the oracle's float64 fit, up to the order of its sums
    Mo, co, ao = oracle.mine_set(xf, w.P, it, transform=1)
    assert np.allclose(col, co, rtol=1e-6, atol=0)
    # the GPU's rows y (same fp32 operations as the oracle's, with the GPU's column factors) and
    # its last assignment: the exact float64 argmin against its own patterns of the iteration before
    yg, _ = oracle.apply_transform(xf, col)
    want = np.array([oracle.nearest_euclid(yg[i], prev) for i in range(len(yg))], np.int32)
    assert np.array_equal(asg, want)
    # against the oracle: patterns within 1e-3, and every differing assignment is a near-tie that
    # the differences between the two sides' rows and patterns account for
    assert np.abs(pats - Mo).max() <= 1e-3
    yo, _ = oracle.apply_transform(xf, co)
    Mprev_o, _, _ = oracle.mine_set(xf, w.P, it - 1, transform=1)
    for i in np.flatnonzero(asg != ao):
        ga, oa = int(asg[i]), int(ao[i])
        gap = oracle.sqdist(yo[i], Mprev_o[ga]) - oracle.sqdist(yo[i], Mprev_o[oa])
        assert 0 <= gap <= _margin(yo[i], yg[i], Mprev_o, prev, ga) + _margin(yo[i], yg[i], Mprev_o, prev, oa), i


def test_mining_status_clear_after_a_normal_run():
    import bit_kv_cache_26_b200 as kvq
    x = planted_ties(2048, 16, seed=7)
    xd = _to_dev(x, torch.bfloat16)
    ws = kvq._alloc_aligned(kvq.kvq_mine_workspace_bytes(2048, 1, 1, 16, 0), xd.device)
    ws[:4].fill_(0xFF)  # the call itself clears the word
    pats = torch.empty(1, 1, 16, D, device="cuda")
    kvq.kvq_mine_patterns(xd, kvq.KVQ_BF16, 2048, 1, 1, D, D, 2048 * D, 16, 4, 0, pats, None, None, ws)
    assert kvq.kvq_mine_read_status(ws) == 0
