"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test checks the oracle against something the pages or the mathematics
fix: hand-worked examples of the cited equations (tests/golden), closed forms,
invariants, special cases that reduce to a library routine, and error bounds.
"""
import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle
import synth

D = 128
rng = np.random.default_rng(1234)


def sparse_vec(spec):
    v = np.zeros(D, np.float32)
    for k, val in spec.items():
        v[int(k)] = val
    return v


# ---------------------------------------------------------------- Eq. 1 quantizer

def test_quant_worked_examples(golden):
    g = golden("quant_eq1.json")
    for case in g["cases"]:
        s, z, q = oracle.quant_group(np.array(case["R"], np.float32), case["bits"])
        if "s_fp32_hex" in case:
            assert np.float32(s).view(np.uint32) == int(case["s_fp32_hex"], 16), case
        else:
            assert s == case["s"], case
        assert z == case["z"], case
        assert list(q) == case["codes"], case


def _bound(s, bits, R):
    # half a step, plus the fp32 roundings of s (relative 2^-24, times up to 2^bits levels), of the
    # quotient (R - z)/s (half an ulp of a number below 2^bits) and of R - z (relative 2^-24).
    return s / 2 + s * (2.0 ** bits) * 2.0 ** -23 + float(np.abs(R).max()) * 2.0 ** -23


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_quant_error_bound_and_range(bits):
    # |x - (s*q + z)| <= s/2 (plus fp32 rounding of the division), codes in range, extremes hit the ends.
    for trial in range(200):
        n = int(rng.integers(2, 64))
        R = (rng.standard_normal(n) * rng.uniform(0.01, 50)).astype(np.float32)
        s, z, q = oracle.quant_group(R, bits)
        assert q.min() >= 0 and q.max() <= (1 << bits) - 1
        assert q[np.argmin(R)] == 0 and q[np.argmax(R)] == (1 << bits) - 1
        xh = np.float64(s) * q + np.float64(z)
        err = np.abs(xh - R.astype(np.float64))
        assert err.max() <= _bound(s, bits, R), (trial, err.max(), s)


def test_quant_16bit_round_trip_near_exact():
    for _ in range(50):
        R = (rng.standard_normal(32) * 3).astype(np.float32)
        s, z, q = oracle.quant_group(R, 16)
        xh = np.float64(s) * q + np.float64(z)
        span = float(R.max() - R.min())
        assert np.abs(xh - R).max() <= _bound(s, 16, R)
        assert np.abs(xh - R).max() <= span * 1e-5


# ---------------------------------------------------------------- d_mm and Eq. 6

def test_dmm_worked_example(golden):
    g = golden("dmm_eq6.json")
    x = sparse_vec(g["x"])
    M = np.stack([sparse_vec(p) for p in g["patterns"]])
    for j, want in enumerate(g["dmm"]):
        assert oracle.dmm(x, M[j]) == want
    assert oracle.assign(x, M) == g["nearest"]


def test_dmm_is_shift_invariant_and_homogeneous():
    # d_mm(x + a*1, m) = d_mm(x, m) (a range ignores a common offset) and d_mm(2x, 2m) = 2 d_mm(x, m),
    # exactly, on small-integer vectors where no rounding happens.
    for _ in range(100):
        x = rng.integers(-50, 50, D).astype(np.float32)
        m = rng.integers(-50, 50, D).astype(np.float32)
        a = np.float32(rng.integers(-20, 20))
        d0 = oracle.dmm(x, m)
        assert oracle.dmm(x + a, m) == d0
        assert oracle.dmm(2 * x, 2 * m) == 2 * d0
        r = (x - m).astype(np.float64)
        # width <= 2 * sup-norm (PatternKV, Appendix C)
        assert d0 <= 2 * np.abs(r).max()


def test_assign_brute_force_small_patterns():
    # Brute force over all P patterns on small-integer data: the chosen index has the smallest range
    # of x - m and no lower index ties with it.  Ranges here come from numpy's ptp (a library routine).
    for _ in range(200):
        P = int(rng.integers(1, 6))
        M = rng.integers(-4, 5, (P, D)).astype(np.float32)
        if P > 1 and rng.random() < 0.3:
            M[rng.integers(P)] = M[rng.integers(P)]  # plant an exact duplicate -> a tie
        x = rng.integers(-4, 5, D).astype(np.float32)
        widths = np.ptp((x[None, :] - M).astype(np.float64), axis=1)
        want = int(np.flatnonzero(widths == widths.min())[0])
        assert oracle.assign(x, M) == want


# ---------------------------------------------------------------- mining, Eq. 4

def test_mine_strided_init_with_zero_iterations():
    x = rng.standard_normal((100, D)).astype(np.float32)
    M, _ = oracle.mine(x, 7, iters=0)
    for j in range(7):
        assert np.array_equal(M[j], x[(j * 100) // 7])


def test_mine_two_blobs_recover_means():
    a = rng.integers(-8, 8, D).astype(np.float32)
    b = a + 40.0
    xa = a + rng.integers(-2, 3, (50, D)).astype(np.float32) * 0.25
    xb = b + rng.integers(-2, 3, (70, D)).astype(np.float32) * 0.25
    x = np.concatenate([xa, xb])
    M, assign = oracle.mine(x, 2, iters=4)
    assert (assign[:50] == 0).all() and (assign[50:] == 1).all()
    # dyadic data: float64 sums are exact, so the centroid is the correctly rounded mean
    assert np.array_equal(M[0], xa.astype(np.float64).mean(axis=0).astype(np.float32))
    assert np.array_equal(M[1], xb.astype(np.float64).mean(axis=0).astype(np.float32))


def test_mine_single_pattern_is_the_mean():
    x = (rng.integers(-100, 100, (64, D)) / 8).astype(np.float32)
    M, _ = oracle.mine(x, 1, iters=3)
    assert np.array_equal(M[0], x.astype(np.float64).mean(axis=0).astype(np.float32))


def test_mine_empty_cluster_keeps_pattern_and_ties_go_low():
    a = np.full(D, 1.0, np.float32)
    b = np.full(D, 5.0, np.float32)
    x = np.stack([a, a, a, b])  # init: x[0] = a and x[2] = a -> identical patterns
    M, assign = oracle.mine(x, 2, iters=1)
    assert list(assign) == [0, 0, 0, 0]       # every point ties between the two -> index 0
    assert np.array_equal(M[1], a)             # pattern 1 got no member and keeps its value
    assert np.array_equal(M[0], np.full(D, 2.0, np.float32))  # mean of (1, 1, 1, 5)


def test_mine_objective_non_increasing():
    w = synth.WORKLOADS["tiny_ref_4k"]
    k, _ = synth.gen_kv(w, p1=1024)
    x = synth.to_float(k, w.dtype).reshape(-1, D)
    prev = np.inf
    for it in range(1, 6):
        M, _ = oracle.mine(x, 16, iters=it)
        a = np.array([oracle._load().kvqo_nearest_euclid(oracle._p(x[i]), oracle._p(M), 16) for i in range(len(x))],
                     np.int32)
        J = oracle.objective(x, M, a)
        assert J <= prev * (1 + 1e-9), (it, J, prev)
        prev = J


def test_sqdist_matches_library_norm():
    for _ in range(20):
        x = rng.standard_normal(D).astype(np.float32)
        m = rng.standard_normal(D).astype(np.float32)
        want = float(np.linalg.norm(x.astype(np.float64) - m.astype(np.float64)) ** 2)
        assert abs(oracle.sqdist(x, m) - want) <= 1e-12 * want


# ---------------------------------------------------------------- pre-transform (KVarN)

def test_fwht_is_sylvester_hadamard():
    H = oracle.fwht(np.eye(D, dtype=np.float32))
    assert np.array_equal(H, scipy.linalg.hadamard(D).astype(np.float32))
    assert np.array_equal(H.astype(np.float64) @ H.astype(np.float64), 128 * np.eye(D))
    x = rng.standard_normal((10, D))
    assert np.allclose(oracle.fwht64(oracle.fwht64(x)) / 128, x, atol=1e-12)


def test_fwht_preserves_norm_up_to_scale():
    x = rng.standard_normal((20, D)).astype(np.float32)
    y = oracle.fwht(x).astype(np.float64)
    assert np.allclose((y ** 2).sum(1), 128 * (x.astype(np.float64) ** 2).sum(1), rtol=1e-5)


def test_halving_sum():
    v = rng.integers(-1000, 1000, D).astype(np.float32)
    assert oracle.halving_sum(v) == float(v.astype(np.int64).sum())
    w = rng.standard_normal(D).astype(np.float32)
    assert abs(oracle.halving_sum(w) - w.astype(np.float64).sum()) <= 1e-5 * np.abs(w).sum()


def test_transform_normalises_rows_and_columns():
    w = synth.WORKLOADS["tiny_ref_4k"]
    k, _ = synth.gen_kv(w, p1=2048)
    x = synth.to_float(k, w.dtype).reshape(-1, D)
    xp = oracle.fwht(x)
    c = oracle.fit_colscale(xp)
    y, r = oracle.apply_transform(x, c)
    y64 = y.astype(np.float64)
    assert np.allclose(y64.std(axis=1), 1.0, atol=1e-5)          # every row: population std 1
    col = y64.std(axis=0)
    assert col.max() / col.min() < 1.05                           # fitted columns: equalised
    assert 0.8 < col.mean() < 1.2                                 # (up to the per-token re-normalisation)
    raw_col = xp.astype(np.float64).std(axis=0)
    assert raw_col.max() / raw_col.min() > 1.5                    # the rotated input was not
    # the transform is invertible: x = r * (y * c) H / 128
    back = oracle.fwht64(r[:, None].astype(np.float64) * (y64 * c.astype(np.float64))) / 128
    assert np.abs(back - x).max() <= 1e-5 * np.abs(x).max()


def test_colscale_equivariance():
    xp = (rng.standard_normal((512, D)) * rng.uniform(0.5, 4, D)).astype(np.float32)
    c0 = oracle.fit_colscale(xp)
    xs = xp.copy()
    xs[:, 3] *= 4.0   # scaling a column scales its factor
    xs[7, :] *= 8.0   # scaling a row changes nothing after the row passes... only through column stds
    c1 = oracle.fit_colscale(xs)
    assert abs(c1[3] / c0[3] / 4.0 - 1) < 0.05
    ratio = np.delete(c1 / c0, 3)
    assert np.allclose(ratio, np.median(ratio), rtol=0.05)


def _block_signed(m):
    """256 x 128 matrix with magnitudes m[token type][channel type] (tokens 0..127 type 0, 128..255
    type 1; channels 0..63 type 0, 64..127 type 1) and signs (-1)^(t + d): every row and every
    column has mean zero, so each population std is the root mean square of its magnitudes."""
    t = np.arange(256)[:, None]
    d = np.arange(D)[None, :]
    mag = np.asarray(m, np.float64)[(t >= 128).astype(int), (d >= 64).astype(int)]
    return mag * np.where((t + d) % 2 == 0, 1.0, -1.0)


def _block_fit_closed_form(m, passes):
    """Alternating row / column std normalisation of the block matrix above, reduced to its 2 x 2
    magnitudes: the sign pattern keeps every mean at zero through each division, so a row's std is
    sqrt((a^2 + b^2) / 2) of its two magnitudes and a column's the same over its two (equal counts)."""
    M = np.array(m, np.float64)
    C = np.ones(2)
    for _ in range(passes):
        M /= np.sqrt((M ** 2).mean(axis=1))[:, None]
        s = np.sqrt((M ** 2).mean(axis=0))
        M /= s[None, :]
        C *= s
    return np.repeat(C, 64)


def test_fit_pass_count_block_closed_form():
    # The 2 x 2 reduction converges slowly, so 1, 2 and 3 passes give factors about 1 % apart: the
    # oracle's fit matches the closed form for each pass count, and the mining pipeline uses 3.
    m = [[1.0, 4.0], [3.0, 0.5]]
    xp = _block_signed(m).astype(np.float32)
    forms = {p: _block_fit_closed_form(m, p) for p in (1, 2, 3)}
    for p, want in forms.items():
        c = oracle.fit_colscale(xp, passes=p).astype(np.float64)
        assert np.abs(c / want - 1).max() < 2 ** -22, (p, c[[0, 127]], want[[0, 127]])
    assert np.abs(forms[3] / forms[2] - 1).min() > 5e-3 and np.abs(forms[2] / forms[1] - 1).min() > 5e-3
    # mine_set rotates its input first: feed it the block matrix rotated back (x = xp H / 128)
    x = (oracle.fwht64(xp.astype(np.float64)) / 128).astype(np.float32)
    _, c, _ = oracle.mine_set(x, 4, iters=0, transform=1)
    rel = {p: np.abs(c / f - 1).max() for p, f in forms.items()}
    assert rel[3] < 1e-5 and rel[2] > 1e-3 and rel[1] > 1e-3, rel


def _encoded_const(N, bits, kidx, vidx, krow, vrow, kz=0.0, vz=0.0):
    """An encoding whose residual codes and scales are zero: reconstruction = z + pattern."""
    G = N // 32
    return oracle.Encoded(N, bits, np.zeros((G, 32, D), np.uint8), np.zeros((G, D), np.float32),
                          np.full((G, D), kz, np.float32), np.asarray(kidx, np.uint8),
                          np.asarray(krow, np.float32), np.zeros((N, D), np.uint8), np.zeros((N, 4), np.float32),
                          np.full((N, 4), vz, np.float32), np.asarray(vidx, np.uint8), np.asarray(vrow, np.float32))


def test_dequant_inverse_transform_is_the_library_hadamard():
    # x = r * (y (.) c) H / 128 with H the Sylvester Hadamard matrix (scipy): hand-chosen, non-uniform
    # c, row factors r != 1 and nonzero zero points, so a missing 1/128, a divided c or a dropped r fails.
    H = scipy.linalg.hadamard(D).astype(np.float64)
    P = 3
    MK = np.stack([np.linspace(-2, 2, D), np.cos(np.arange(D)), np.where(np.arange(D) % 3 == 0, 5.0, -1.0)])
    MV = MK[::-1].copy() * 0.5
    MK, MV = MK.astype(np.float32), MV.astype(np.float32)
    cK = (1.0 + np.arange(D) / 64.0).astype(np.float32)
    cV = (3.0 - np.arange(D) / 80.0).astype(np.float32)
    N = 64
    kidx = np.arange(N) % P
    vidx = (np.arange(N) + 1) % P
    krow = 0.5 + np.arange(N) / 16.0
    vrow = 2.0 - np.arange(N) / 50.0
    e = _encoded_const(N, 2, kidx, vidx, krow, vrow, kz=0.25, vz=-0.125)
    Kh, Vh = oracle.dequant(e, MK, MV, cK, cV)
    for t in range(N):
        yk = MK[kidx[t]].astype(np.float64) + 0.25
        yv = MV[vidx[t]].astype(np.float64) - 0.125
        wk = float(e.krow[t]) * (yk * cK) @ H / 128  # the stored (fp32) row factors
        wv = float(e.vrow[t]) * (yv * cV) @ H / 128
        assert np.allclose(Kh[t], wk, rtol=1e-12, atol=1e-12)
        assert np.allclose(Vh[t], wv, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 4])
def test_encode_round_trip_bound_with_transform(bits):
    # Eq. 1 bounds the error of every normalised value y_e by half its group's step s_e / 2; the inverse
    # x = r (y (.) c) H / 128 has entries of magnitude r c_e / 128, so per element of x
    #   |x_hat_d - x_d| <= r / 128 * sum_e c_e s_e / 2   (+ fp32 rounding of the forward transform).
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 1024 + 9)
    MK, cK, _ = oracle.mine_set(K[:1024], 16, transform=1)
    MV, cV, _ = oracle.mine_set(V[:1024], 16, transform=1)
    e = oracle.encode(K, V, bits, MK, MV, cK, cV)
    Kh, Vh = oracle.dequant(e, MK, MV, cK, cV)
    G = e.N // 32
    c64k, c64v = cK.astype(np.float64), cV.astype(np.float64)
    worst = 0.0
    for t in range(G * 32):
        s = e.ks[t // 32].astype(np.float64)
        bound = e.krow[t] / 128 * (c64k * s / 2).sum() * (1 + 2 ** -18) + 1e-5 * (1 + np.abs(K[t]).sum() / 128)
        err = np.abs(Kh[t] - K[t]).max()
        assert err <= bound, (t, err, bound)
        worst = max(worst, err / bound)
    for t in range(e.N):
        s = np.repeat(e.vs[t], 32).astype(np.float64)
        bound = e.vrow[t] / 128 * (c64v * s / 2).sum() * (1 + 2 ** -18) + 1e-5 * (1 + np.abs(V[t]).sum() / 128)
        err = np.abs(Vh[t] - V[t]).max()
        assert err <= bound, (t, err, bound)
    assert worst > 1 / 16, worst  # not vacuous: a missing 1/128 or a dropped r would break it
    # the round trip really passes through the inverse: without it the values would be y, not x
    y, _ = oracle.apply_transform(V[:4], cV)
    assert np.abs(y - V[:4]).max() > 1.0


# ---------------------------------------------------------------- encode / dequant

def _unit(w, p1, seed_h=0):
    k, v = synth.gen_kv(w, p1=p1)
    K = synth.to_float(k, w.dtype)[0, :, seed_h]
    V = synth.to_float(v, w.dtype)[0, :, seed_h]
    return K, V


@pytest.mark.parametrize("bits", [2, 4])
def test_encode_round_trip_bound(bits):
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 1024 + 7)
    MK, _, _ = oracle.mine_set(K[:1024], 16)
    MV, _, _ = oracle.mine_set(V[:1024], 16)
    e = oracle.encode(K, V, bits, MK, MV)
    Kh, Vh = oracle.dequant(e, MK, MV)
    G = e.N // 32
    for g in range(G):
        err = np.abs(Kh[g * 32:(g + 1) * 32] - K[g * 32:(g + 1) * 32])
        bound = e.ks[g][None, :].astype(np.float64) / 2 * (1 + 2 ** -20) + 2e-6 * (1 + np.abs(K[g * 32:(g + 1) * 32]))
        assert (err <= bound).all()
    errv = np.abs(Vh - V)
    boundv = np.repeat(e.vs, 32, axis=1).astype(np.float64) / 2 * (1 + 2 ** -20) + 2e-6 * (1 + np.abs(V))
    assert (errv <= boundv).all()
    # residual quantization is tighter than raw quantization on this clustered data
    assert e.vs.mean() < 0.7 * np.mean([oracle.quant_group(V[t, 32 * g:32 * g + 32], bits)[0]
                                        for t in range(64) for g in range(4)])


def test_single_zero_pattern_reduces_to_plain_quantization():
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 64)
    Z = np.zeros((1, D), np.float32)
    e = oracle.encode(K, V, 2, Z, Z)
    assert (e.kidx == 0).all() and (e.vidx == 0).all()
    for t in range(64):
        for g in range(4):
            s, z, q = oracle.quant_group(V[t, 32 * g:32 * g + 32], 2)
            assert e.vs[t, g] == s and e.vz[t, g] == z and np.array_equal(e.vcode[t, 32 * g:32 * g + 32], q)
    for grp in range(2):
        for d in range(D):
            s, z, q = oracle.quant_group(K[32 * grp:32 * grp + 32, d], 2)
            assert e.ks[grp, d] == s and np.array_equal(e.kcode[grp, :, d], q)


def test_encode_indices_are_nearest_under_dmm():
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 256)
    MK, _, _ = oracle.mine_set(K, 16)
    e = oracle.encode(K, V, 2, MK, MK[:1].repeat(3, 0))
    for t in range(0, 256, 17):
        widths = np.array([oracle.dmm(K[t], MK[j]) for j in range(16)])
        assert e.kidx[t] == int(np.flatnonzero(widths == widths.min())[0])


# ---------------------------------------------------------------- attention

def test_attention_matches_library_softmax():
    for Gq, N in [(1, 1), (4, 37), (7, 300)]:
        q = rng.standard_normal((Gq, D))
        K = rng.standard_normal((N, D)) * 3
        V = rng.standard_normal((N, D))
        out = oracle.attention(q, K, V, 1 / np.sqrt(D))
        want = scipy.special.softmax(q @ K.T / np.sqrt(D), axis=1) @ V
        assert np.allclose(out, want, rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    V = rng.standard_normal((50, D))
    K = np.tile(rng.standard_normal(D), (50, 1))  # identical keys -> uniform weights -> mean of V
    q = rng.standard_normal((2, D))
    assert np.allclose(oracle.attention(q, K, V, 0.1), np.tile(V.mean(0), (2, 1)), atol=1e-12)
    one = oracle.attention(q, K[:1], V[:1], 0.1)  # a single key returns its value
    assert np.allclose(one, np.tile(V[0], (2, 1)), atol=1e-14)


def test_attention_unit_with_exact_cache_is_plain_attention():
    # 16-bit-like exactness: feed the reconstruction the exact values and the unit result is plain attention.
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 96 + 5)
    q = rng.standard_normal((1, D))
    MK, _, _ = oracle.mine_set(K, 4)
    MV, _, _ = oracle.mine_set(V, 4)
    e = oracle.encode(K, V, 4, MK, MV)
    got = oracle.attention_unit(q, K, e, MK, MV)
    Kh, Vh = oracle.dequant(e, MK, MV)
    Kfull = np.concatenate([Kh, K[96:]])
    want = scipy.special.softmax(q @ Kfull.T / np.sqrt(D), axis=1) @ Vh
    assert np.allclose(got, want, rtol=1e-6, atol=1e-6)
    exact = scipy.special.softmax(q @ K.T.astype(np.float64) / np.sqrt(D), axis=1) @ V
    assert np.abs(got - exact).max() < 0.1 * np.abs(exact).max()


# ---------------------------------------------------------------- layout

def test_layout_positions_hand_worked(golden):
    g = golden("layout_positions.json")
    for bits, wk, bk in [(2, "w2", "b2"), (4, "w4", "b4")]:
        for case in g["k_codes"]:
            X = np.zeros((32, D), np.uint8)
            X[case["token"], case["channel"]] = 1
            words = oracle.pack_codes(X, 2, 8, bits).view("<u4")
            nz = np.flatnonzero(words)
            assert list(nz) == [case[wk]] and words[nz[0]] == 1 << case[bk], (bits, case)
        for case in g["v_codes"]:
            X = np.zeros((D, 32), np.uint8)
            X[case["channel"], case["token"]] = 1
            words = oracle.pack_codes(X, 8, 2, bits).view("<u4")
            nz = np.flatnonzero(words)
            assert list(nz) == [case[wk]] and words[nz[0]] == 1 << case[bk], (bits, case)
    for c in g["k_scale_index"]:
        assert oracle.KSC[c["i"]] == c["channel"]
    for c in g["v_scale_index"]:
        assert oracle.VSC[0][c["i"]] == c["token"] and oracle.VSC[1][c["i"]] == c["group"]
    for c in g["v_zero_index"]:
        assert oracle.VZC[0][c["i"]] == c["token"] and oracle.VZC[1][c["i"]] == c["group"]
    for c in g["token_index"]:
        assert oracle.TOK[c["i"]] == c["token"]


@pytest.mark.parametrize("bits,transform", [(2, 0), (4, 0), (2, 1)])
def test_pack_round_trip(bits, transform):
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 64 + 11)
    MK, cK, _ = oracle.mine_set(K, 8, transform=transform)
    MV, cV, _ = oracle.mine_set(V, 8, transform=transform)
    e = oracle.encode(K, V, bits, MK, MV, cK, cV)
    for page in range(2):
        buf, defined = oracle.subblock(e, page, transform)
        assert buf.size == oracle.subblock_bytes(bits, transform)
        back = oracle.parse_subblock(buf, bits, transform)
        assert np.array_equal(back["kcode"], e.kcode[page])
        assert np.array_equal(back["vcode"], e.vcode[page * 32:page * 32 + 32])
        assert np.array_equal(back["ks"], e.ks[page]) and np.array_equal(back["kz"], e.kz[page])
        assert np.array_equal(back["vs"], e.vs[page * 32:page * 32 + 32])
        assert np.array_equal(back["kidx"], e.kidx[page * 32:page * 32 + 32])
        assert np.array_equal(back["vidx"], e.vidx[page * 32:page * 32 + 32])
        if transform:
            assert np.array_equal(back["krow"], e.krow[page * 32:page * 32 + 32])
    buf, defined = oracle.subblock(e, 2, transform)  # partial page: 11 tokens, K undefined
    back = oracle.parse_subblock(buf, bits, transform)
    assert np.array_equal(back["vcode"][:11], e.vcode[64:75]) and not back["vcode"][11:].any()
    assert not defined[:oracle.code_bytes(bits)].any()


# ---------------------------------------------------------------- V adaptive threshold (Eq. 7-10)

def test_rho_star_worked_values_and_closed_form(golden):
    import scipy.stats
    for case in golden("rho_star_eq10.json")["cases"]:
        r = oracle.rho_star(case["d"], case["alpha"])
        assert abs(r - case["rho_star"]) < 6e-6, case
    for d in (64, 96, 128, 256):
        for a in (0.1, 0.05, 0.01):
            z = scipy.stats.norm.isf(a)                       # library quantile
            assert abs(oracle.normal_upper_quantile(a) - z) < 1e-12
            k = 2 * z / np.sqrt(5 * d)                        # closed-form root of the quadratic in rho^2
            A = 1 - k * k
            u = (1 - np.sqrt(1 - A * A)) / A
            r = oracle.rho_star(d, a)
            assert abs(r - np.sqrt(u)) < 1e-12
            assert abs((1 - r * r) - k * np.sqrt(1 + r ** 4)) < 1e-12   # Eq. 10 holds with equality
            assert r > oracle.rho_star(d, a / 2)              # a smaller alpha asks for more contraction


def _vec_with_ranges(raw, flat):
    """A V vector with range `raw` (channels 0 and 1) and a pattern whose residual range is `flat`
    (the residual is 0 except channel 2 = flat); small dyadic values, so every fp32 step is exact."""
    v = np.zeros(D, np.float32)
    v[0], v[1] = raw / 2, -raw / 2
    m = v.copy()
    m[2] -= flat
    return v, m


def test_v_threshold_decision_and_raw_fallback():
    rho = oracle.v_rho(0.05)
    assert rho == np.float32(0.91155338)
    raw = np.float32(8.0)
    limit = float(np.float32(rho) * raw)                      # fl32(rho* x R_raw)
    on_edge = np.float32(limit)
    above = np.nextafter(on_edge, np.float32(np.inf))
    K = np.zeros((32, D), np.float32)
    MK = np.zeros((1, D), np.float32)
    for flat, want_use in ((np.float32(1.0), True), (on_edge, True), (above, False), (np.float32(7.99), False)):
        v, m = _vec_with_ranges(raw, flat)
        assert oracle.dmm(v, m) == flat and oracle.vrange(v) == raw
        V = np.tile(v, (32, 1))
        e = oracle.encode(K, V, 2, MK, m[None], v_rho=rho)
        assert (e.vidx == (0 if want_use else 255)).all(), (flat, want_use)
        # with the threshold off the pattern is always used
        assert (oracle.encode(K, V, 2, MK, m[None]).vidx == 0).all()
        if not want_use:
            # quantized raw: the codes and scales of plain Eq. 1 on v itself, and dequant adds no pattern
            for g in range(4):
                s, z, q = oracle.quant_group(v[32 * g:32 * g + 32], 2)
                assert e.vs[0, g] == s and e.vz[0, g] == z and np.array_equal(e.vcode[0, 32 * g:32 * g + 32], q)
            _, Vh = oracle.dequant(e, MK, m[None])
            assert np.abs(Vh[0] - v).max() <= e.vs[0].max() / 2 * (1 + 2 ** -20)


def test_v_threshold_matches_eq10_on_clustered_data():
    # Every accepted V vector has rho = R_flat / R_raw <= rho* (up to the fp32 product), every
    # rejected one has rho > rho*; on data with a planted fraction of unclustered vectors the
    # rejections are about that fraction.
    w = synth.WORKLOADS["llama3_8b_32k"].with_(B=1, S=512, Hkv=1, Hq=4, P=16, ncv=4)
    k, v = synth.gen_kv(w)
    K = synth.to_float(k, w.dtype)[0, :, 0]
    V = synth.to_float(v, w.dtype)[0, :, 0]
    MV, _, _ = oracle.mine_set(V, 16)
    MK, _, _ = oracle.mine_set(K, 16)
    V2 = V.copy()
    V2[::4] = (rng.standard_normal((128, D)) * 3).astype(np.float32)  # a quarter far from every pattern
    rho = oracle.v_rho(0.05)
    e = oracle.encode(K, V2, 2, MK, MV, v_rho=rho)
    rs = oracle.rho_star(128, 0.05)
    for t in range(len(V2)):
        j = oracle.assign(V2[t], MV)
        ratio = oracle.dmm(V2[t], MV[j]) / oracle.vrange(V2[t])
        if e.vidx[t] == 255:
            assert ratio > rs * (1 - 1e-6)
        else:
            assert e.vidx[t] == j and ratio <= rs * (1 + 1e-6)
    planted = np.zeros(len(V2), bool)
    planted[::4] = True
    assert (e.vidx[planted] == 255).mean() > 0.9       # far from every pattern: flattening rejected
    assert (e.vidx[~planted] == 255).mean() < 0.1      # near their pattern: flattening kept


# ---------------------------------------------------------------- decode-time pattern insertion (Eq. 5)

def test_chebyshev_center_worked_example(golden):
    g = golden("chebyshev_eq5.json")
    X = np.stack([sparse_vec(v) for v in g["X"]])
    assert np.array_equal(oracle.chebyshev_center(X), sparse_vec(g["center"]))


def test_chebyshev_center_is_the_minimax_point():
    # Per channel the midrange minimises the largest deviation of the window's values (the l-inf
    # Chebyshev center, PatternKV Appendix C): no other point has a smaller maximum |X - M|.
    for _ in range(50):
        X = (rng.standard_normal((int(rng.integers(1, 40)), D)) * rng.uniform(0.1, 10)).astype(np.float32)
        M = oracle.chebyshev_center(X).astype(np.float64)
        X64 = X.astype(np.float64)
        radius = np.abs(X64 - M).max(axis=0)
        assert np.allclose(radius, (X64.max(0) - X64.min(0)) / 2, rtol=1e-6, atol=1e-6)
        for _ in range(5):
            Mp = M + rng.standard_normal(D) * 0.01
            assert (np.abs(X64 - Mp).max(axis=0) >= radius - 1e-6).all()


def test_stream_without_insertion_equals_batch_encoding():
    # Appending one token at a time with fixed patterns gives the same encoding as one bulk call.
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 320 + 5)
    MK, _, _ = oracle.mine_set(K[:256], 8)
    MV, _, _ = oracle.mine_set(V[:256], 8)
    rho = oracle.v_rho(0.05)
    for L0 in (0, 100, 256):
        e0 = oracle.encode(K, V, 2, MK, MV, v_rho=rho)
        e1, MK1, MV1 = oracle.encode_stream(K, V, L0, 2, MK, MV, Pmax=20, G=0, v_rho=rho)
        assert MK1.shape[0] == 8 and np.array_equal(MK1, MK)
        for f in ("kcode", "ks", "kz", "kidx", "vcode", "vs", "vz", "vidx"):
            assert np.array_equal(getattr(e0, f), getattr(e1, f)), (L0, f)


def test_stream_insertion_adds_window_centers():
    w = synth.WORKLOADS["tiny_ref_4k"]
    K, V = _unit(w, 128 * 5 + 17)
    L0, G = 128, 128
    MK, _, _ = oracle.mine_set(K[:L0], 4)
    MV, _, _ = oracle.mine_set(V[:L0], 4)
    e, MKf, MVf = oracle.encode_stream(K, V, L0, 2, MK, MV, Pmax=6, G=G)
    # windows [128, 256), [256, 384), ... complete at 256, 384, 512, 640: capacity 6 keeps the first two
    assert MKf.shape[0] == 6
    for i, w0 in enumerate((128, 256)):
        assert np.array_equal(MKf[4 + i], ((K[w0:w0 + G].min(0) + K[w0:w0 + G].max(0)) * np.float32(0.5)))
        assert np.array_equal(MVf[4 + i], ((V[w0:w0 + G].min(0) + V[w0:w0 + G].max(0)) * np.float32(0.5)))
    # every token is assigned among the patterns present when it (V) or its group (K) arrived
    for t in range(L0, e.N):
        P_t = 4 + min(2, (t - L0) // G)
        assert e.vidx[t] == oracle.assign(V[t], MVf[:P_t]), t
    for grp in range(L0 // 32, e.N // 32):
        last = 32 * grp + 31
        P_t = 4 + min(2, max(0, last - L0) // G) if last >= L0 else 4
        for t in range(32 * grp, 32 * grp + 32):
            assert e.kidx[t] == oracle.assign(K[t], MKf[:P_t]), (grp, t)
    # the inserted patterns are used
    assert (e.vidx[L0 + G:] >= 4).any()
