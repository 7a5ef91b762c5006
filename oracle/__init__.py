"""CPU oracle for pattern-aligned residual KV quantization and decode attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``bit_kv_cache_26_b200``) never imports, loads or calls it, and shares no code,
header, table or constant generator with it.

The arithmetic lives in ``kvq_oracle.c`` (plain C: float64, except the fp32
quantization step).  This module adds the ctypes binding and an independent
restatement of the paged-cache byte layout, written from the layout
description (not from the CUDA sources), so that tests can compare the GPU's
cache bytes with the oracle's.

Sources: "PatternKV: Flattening KV Representation Expands Quantization
Headroom" (Sections 2.1, 3.1, 3.2, 4.1) and "KVarN: Variance-Normalized KV-Cache
Quantization ..." (abstract).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_build", "libkvq_oracle.so")
_lib = None
D = 128
GROUP = 32


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c (gcc, OpenMP, no FMA contraction, no fast-math)."""
    src = os.path.join(_HERE, "kvq_oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11",
                               "-fPIC", "-shared", "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_vp = ctypes.c_void_p


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        sig = {
            "kvqo_sqdist": (f64, [_vp, _vp]),
            "kvqo_nearest_euclid": (i32, [_vp, _vp, i32]),
            "kvqo_mine": (ctypes.c_int, [_vp, i64, i32, i32, _vp, _vp]),
            "kvqo_objective": (f64, [_vp, i64, _vp, _vp]),
            "kvqo_fwht": (None, [_vp]),
            "kvqo_fwht64": (None, [_vp]),
            "kvqo_halving_sum": (ctypes.c_float, [_vp]),
            "kvqo_fit_colscale": (ctypes.c_int, [_vp, i64, i32, _vp]),
            "kvqo_apply_row": (None, [_vp, _vp, _vp, _vp]),
            "kvqo_dmm": (ctypes.c_float, [_vp, _vp]),
            "kvqo_assign": (i32, [_vp, _vp, i32]),
            "kvqo_quant_group": (None, [_vp, i64, i64, i32, _vp, _vp, _vp, i64]),
            "kvqo_encode": (ctypes.c_int, [_vp, _vp, i64, i32, i32, _vp, _vp, _vp, _vp, ctypes.c_float] + [_vp] * 10),
            "kvqo_normal_upper_quantile": (f64, [f64]),
            "kvqo_rho_star": (f64, [i32, f64]),
            "kvqo_range": (ctypes.c_float, [_vp]),
            "kvqo_chebyshev_center": (None, [_vp, i64, _vp]),
            "kvqo_encode_stream": (ctypes.c_int, [_vp, _vp, i64, i64, i32, i32, i32, i32, _vp, _vp, _vp, _vp,
                                                  ctypes.c_float, _vp] + [_vp] * 10),
            "kvqo_dequant": (None, [i64, _vp, _vp, _vp, _vp] + [_vp] * 10 + [_vp, _vp]),
            "kvqo_attention": (None, [_vp, i32, _vp, _vp, i64, f64, _vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# Mining (PatternKV Section 3.1, Eq. 4) and the pre-transform (KVarN abstract)
# ---------------------------------------------------------------------------

def sqdist(x, m) -> float:
    x, m = _f32(x), _f32(m)
    return _load().kvqo_sqdist(_p(x), _p(m))


def nearest_euclid(x, M) -> int:
    """Index of the nearest pattern under the float64 squared distance (lowest index on ties)."""
    x, M = _f32(x), _f32(M)
    return int(_load().kvqo_nearest_euclid(_p(x), _p(M), M.shape[0]))


def mine(x: np.ndarray, P: int, iters: int = 4):
    """Lloyd k-means on rows of x (n x 128 fp32).  Returns (patterns[P,128] fp32, assign[n] int32)."""
    x = _f32(x)
    n = x.shape[0]
    M = np.zeros((P, D), np.float32)
    a = np.zeros(n, np.int32)
    rc = _load().kvqo_mine(_p(x), n, P, iters, _p(M), _p(a))
    if rc != 0:
        raise ValueError(f"kvqo_mine rc={rc}")
    return M, a


def objective(x, M, a) -> float:
    x, M, a = _f32(x), _f32(M), np.ascontiguousarray(a, np.int32)
    return _load().kvqo_objective(_p(x), x.shape[0], _p(M), _p(a))


def fwht(v: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester Walsh-Hadamard transform of each 128-row (fp32 butterfly)."""
    v = _f32(v).copy()
    rows = v.reshape(-1, D)
    lib = _load()
    for r in rows:
        lib.kvqo_fwht(_p(r))
    return v


def fwht64(v: np.ndarray) -> np.ndarray:
    v = _f64(v).copy()
    rows = v.reshape(-1, D)
    lib = _load()
    for r in rows:
        lib.kvqo_fwht64(_p(r))
    return v


def halving_sum(v) -> float:
    v = _f32(v)
    return float(_load().kvqo_halving_sum(_p(v)))


def fit_colscale(xp: np.ndarray, passes: int = 3) -> np.ndarray:
    """Column factors c[128] from rows already rotated by fwht (float64 fit, fp32 result)."""
    xp = _f32(xp)
    c = np.zeros(D, np.float32)
    rc = _load().kvqo_fit_colscale(_p(xp), xp.shape[0], passes, _p(c))
    if rc != 0:
        raise ValueError(f"kvqo_fit_colscale rc={rc}")
    return c


def apply_transform(x: np.ndarray, c: np.ndarray):
    """Per row: y = (fwht(x) / c) / r, r = population std (fp32).  Returns (y[n,128], r[n])."""
    x, c = _f32(x).reshape(-1, D), _f32(c)
    y = np.zeros_like(x)
    r = np.zeros(x.shape[0], np.float32)
    lib = _load()
    for i in range(x.shape[0]):
        lib.kvqo_apply_row(_p(x[i]), _p(c), _p(y[i]), ctypes.c_void_p(r.ctypes.data + 4 * i))
    return y, r


def mine_set(x: np.ndarray, P: int, iters: int = 4, transform: int = 0):
    """Mining of one (set, KV head): optional pre-transform fit, then Lloyd.

    Returns (patterns, colscale or None, assign).  With the transform, patterns
    live in the normalised space y.
    """
    x = _f32(x)
    if transform:
        xp = fwht(x)
        c = fit_colscale(xp)
        y, _ = apply_transform(x, c)
        M, a = mine(y, P, iters)
        return M, c, a
    M, a = mine(x, P, iters)
    return M, None, a


# ---------------------------------------------------------------------------
# Alignment (Section 3.2, Eq. 6) and quantization (Section 2.1, Eq. 1)
# ---------------------------------------------------------------------------

def dmm(x, m) -> float:
    x, m = _f32(x), _f32(m)
    return float(_load().kvqo_dmm(_p(x), _p(m)))


def assign(x, M) -> int:
    x, M = _f32(x), _f32(M)
    return int(_load().kvqo_assign(_p(x), _p(M), M.shape[0]))


def quant_group(R, bits: int):
    """Quantize one group of values (1 <= bits <= 16).  Returns (s, z, codes int32)."""
    R = _f32(R)
    n = R.shape[0]
    s = np.zeros(1, np.float32)
    z = np.zeros(1, np.float32)
    q = np.zeros(n, np.int32)
    _load().kvqo_quant_group(_p(R), n, 1, bits, _p(s), _p(z), _p(q), 1)
    return float(s[0]), float(z[0]), q


@dataclass
class Encoded:
    """Quantized form of one (sequence, KV head) stream of N tokens, natural order."""
    N: int
    bits: int
    kcode: np.ndarray  # [G, 32, 128] uint8
    ks: np.ndarray     # [G, 128] fp32
    kz: np.ndarray     # [G, 128]
    kidx: np.ndarray   # [G*32] uint8
    krow: np.ndarray   # [G*32] fp32
    vcode: np.ndarray  # [N, 128] uint8
    vs: np.ndarray     # [N, 4]
    vz: np.ndarray     # [N, 4]
    vidx: np.ndarray   # [N] uint8
    vrow: np.ndarray   # [N] fp32


def normal_upper_quantile(a: float) -> float:
    """z with P(Z > z) = a for a standard normal Z (bisection)."""
    return float(_load().kvqo_normal_upper_quantile(a))


def rho_star(d: int, alpha: float) -> float:
    """rho*(d, alpha) of PatternKV Eq. 10 (float64, bisection)."""
    return float(_load().kvqo_rho_star(d, alpha))


def v_rho(alpha: float, d: int = D) -> float:
    """The fp32 threshold the encoder compares with (0 = adaptive threshold off)."""
    return 0.0 if alpha <= 0 else float(np.float32(rho_star(d, alpha)))


def vrange(x) -> float:
    x = _f32(x)
    return float(_load().kvqo_range(_p(x)))


def encode(K: np.ndarray, V: np.ndarray, bits: int, MK, MV, cK=None, cV=None, v_rho: float = 0.0) -> Encoded:
    """Encode N tokens of one (sequence, KV head): K, V are [N,128] fp32 (exact input values).

    v_rho > 0 enables the V adaptive threshold (PatternKV Section 3.3): a V vector whose
    residual range exceeds fl32(v_rho * its own range) is quantized raw, with index 255."""
    K, V, MK, MV = _f32(K), _f32(V), _f32(MK), _f32(MV)
    cK = None if cK is None else _f32(cK)
    cV = None if cV is None else _f32(cV)
    N = K.shape[0]
    G = N // GROUP
    e = Encoded(N, bits, np.zeros((G, GROUP, D), np.uint8), np.zeros((G, D), np.float32),
                np.zeros((G, D), np.float32), np.zeros(G * GROUP, np.uint8), np.zeros(G * GROUP, np.float32),
                np.zeros((N, D), np.uint8), np.zeros((N, 4), np.float32), np.zeros((N, 4), np.float32),
                np.zeros(N, np.uint8), np.zeros(N, np.float32))
    rc = _load().kvqo_encode(_p(K), _p(V), N, bits, MK.shape[0], _p(MK), _p(MV), _p(cK), _p(cV), float(v_rho),
                             _p(e.kcode), _p(e.ks), _p(e.kz), _p(e.kidx), _p(e.krow),
                             _p(e.vcode), _p(e.vs), _p(e.vz), _p(e.vidx), _p(e.vrow))
    if rc != 0:
        raise ValueError(f"kvqo_encode rc={rc}")
    return e


def chebyshev_center(X) -> np.ndarray:
    """Per channel the mean of the minimum and maximum of the rows of X (PatternKV Eq. 5), fp32."""
    X = _f32(X).reshape(-1, D)
    M = np.zeros(D, np.float32)
    _load().kvqo_chebyshev_center(_p(X), X.shape[0], _p(M))
    return M


def encode_stream(K: np.ndarray, V: np.ndarray, L0: int, bits: int, MK0, MV0, Pmax: int, G: int = 0,
                  cK=None, cV=None, v_rho: float = 0.0):
    """Streaming encoding with decode-time pattern insertion (PatternKV Section 3.1, Eq. 5).

    Tokens [0, L0) are the prefill (the initial P0 patterns); tokens from L0 on arrive one at a
    time, and with G > 0 every window of G tokens (aligned to multiples of G) adds the Chebyshev
    centers of its K and V vectors to the pattern sets (up to Pmax patterns), used from the next
    token on.  Returns (Encoded, MK [P, 128], MV [P, 128]) with the final pattern count P."""
    K, V = _f32(K), _f32(V)
    MK0, MV0 = _f32(MK0), _f32(MV0)
    cK = None if cK is None else _f32(cK)
    cV = None if cV is None else _f32(cV)
    N, P0 = K.shape[0], MK0.shape[0]
    MK = np.zeros((Pmax, D), np.float32)
    MV = np.zeros((Pmax, D), np.float32)
    MK[:P0], MV[:P0] = MK0, MV0
    G32 = N // GROUP
    e = Encoded(N, bits, np.zeros((G32, GROUP, D), np.uint8), np.zeros((G32, D), np.float32),
                np.zeros((G32, D), np.float32), np.zeros(G32 * GROUP, np.uint8), np.zeros(G32 * GROUP, np.float32),
                np.zeros((N, D), np.uint8), np.zeros((N, 4), np.float32), np.zeros((N, 4), np.float32),
                np.zeros(N, np.uint8), np.zeros(N, np.float32))
    P = ctypes.c_int32(0)
    rc = _load().kvqo_encode_stream(_p(K), _p(V), N, L0, G, bits, P0, Pmax, _p(MK), _p(MV), _p(cK), _p(cV),
                                    float(v_rho), ctypes.byref(P), _p(e.kcode), _p(e.ks), _p(e.kz), _p(e.kidx),
                                    _p(e.krow), _p(e.vcode), _p(e.vs), _p(e.vz), _p(e.vidx), _p(e.vrow))
    if rc != 0:
        raise ValueError(f"kvqo_encode_stream rc={rc}")
    return e, MK[:P.value].copy(), MV[:P.value].copy()


def dequant(e: Encoded, MK, MV, cK=None, cV=None):
    """Reconstruct (Khat[G*32,128], Vhat[N,128]) in float64, original space."""
    MK, MV = _f32(MK), _f32(MV)
    cK = None if cK is None else _f32(cK)
    cV = None if cV is None else _f32(cV)
    G = e.N // GROUP
    Kh = np.zeros((G * GROUP, D), np.float64)
    Vh = np.zeros((e.N, D), np.float64)
    _load().kvqo_dequant(e.N, _p(MK), _p(MV), _p(cK), _p(cV), _p(e.kcode), _p(e.ks), _p(e.kz), _p(e.kidx),
                         _p(e.krow), _p(e.vcode), _p(e.vs), _p(e.vz), _p(e.vidx), _p(e.vrow), _p(Kh), _p(Vh))
    return Kh, Vh


def attention(q: np.ndarray, Kfull: np.ndarray, Vfull: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q K^T) V in float64 for q [Gq,128] against N keys/values."""
    q, Kfull, Vfull = _f64(q).reshape(-1, D), _f64(Kfull).reshape(-1, D), _f64(Vfull).reshape(-1, D)
    out = np.zeros_like(q)
    _load().kvqo_attention(_p(q), q.shape[0], _p(Kfull), _p(Vfull), Kfull.shape[0], scale, _p(out))
    return out


def attention_unit(q: np.ndarray, K: np.ndarray, e: Encoded, MK, MV, cK=None, cV=None, scale=None) -> np.ndarray:
    """Decode attention of the query heads of one KV head over its quantized stream.

    Keys: reconstructed K for complete groups, exact K for the N % 32 newest
    tokens (the full-precision window).  Values: reconstructed V for all tokens.
    Returns fp32 [Gq, 128].
    """
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    Kh, Vh = dequant(e, MK, MV, cK, cV)
    G = e.N // GROUP
    Kfull = np.concatenate([Kh, _f64(K)[G * GROUP: e.N]], axis=0)
    return attention(q, Kfull, Vh, scale).astype(np.float32)


# ---------------------------------------------------------------------------
# Paged-cache byte layout, restated independently from its description.
#
# A page holds 32 consecutive tokens of one sequence for every KV head; the
# sub-block of one KV head (bits b, CB = 32*128*b/8 bytes of codes) is:
#   [0, CB)                 K codes      (fragment order, rows = tokens)
#   [CB, CB+512)            K scales s   (channel order KSC below)
#   [CB+512, CB+1024)       K zeros  z   (same order)
#   [CB+1024, 2CB+1024)     V codes      (fragment order, rows = channels)
#   [2CB+1024, 2CB+1536)    V scales s   (order VSC below, 4 channel groups)
#   [2CB+1536, 2CB+2048)    V zeros  z   (order VZC below)
#   [2CB+2048, 2CB+2080)    K pattern indices (order TOK below)
#   [2CB+2080, 2CB+2112)    V pattern indices (order TOK below)
#   with the pre-transform: K row factors then V row factors, fp32, order TOK.
#
# Fragment order of a (16*MT) x (16*KS) code matrix X (K: X[token][channel],
# MT=2, KS=8; V: X[channel][token], MT=8, KS=2): element (row, col) has
#   lane = (row%16 % 8)*4 + (col%16 % 8)//2,  odd = col % 2,
#   reg  = ((row//16)*KS + col//16)*4 + (row%16)//8 + 2*((col%16)//8)
# and belongs to the lane's word w = reg//8 at bit 2*(reg%8) + 16*odd (2-bit), or
# w = reg//4 at bit 4*(reg%4) + 16*odd (4-bit); word w of lane l is the little-endian
# 32-bit word (w//4)*128 + l*4 + w%4 of the block (lane-interleaved 16-byte chunks).
# Orders:  KSC[i], i = ks*16 + tig*4 + e      -> channel 16ks + 2tig + (e&1) + 8(e>>1)
#          VSC[i], i = ((ks*4+e)*4+tig)*4+grp -> (token 16ks + 2tig + (e&1) + 8(e>>1), group grp)
#          VZC[i], i = (j*8 + g)*4 + grp      -> (token g + 8j, group grp)
#          TOK[i], i = g*4 + j                -> token g + 8j
# Entries of tokens not yet appended are zero; the K part of a page is
# undefined until its 32nd token arrives.
# ---------------------------------------------------------------------------

def code_bytes(bits: int) -> int:
    return GROUP * D * bits // 8


def subblock_bytes(bits: int, transform: int) -> int:
    return 2 * code_bytes(bits) + 2112 + (256 if transform else 0)


def _frag_words(MT: int, KS: int, bits: int):
    rows, cols = np.meshgrid(np.arange(16 * MT), np.arange(16 * KS), indexing="ij")
    rr, cc = rows % 16, cols % 16
    lane = (rr % 8) * 4 + (cc % 8) // 2
    reg = ((rows // 16) * KS + cols // 16) * 4 + rr // 8 + 2 * (cc // 8)
    odd = cols % 2
    if bits == 2:
        w, bit = reg // 8, 2 * (reg % 8) + 16 * odd
    else:
        w, bit = reg // 4, 4 * (reg % 4) + 16 * odd
    word = (w // 4) * 128 + lane * 4 + w % 4
    return word, bit


def pack_codes(X: np.ndarray, MT: int, KS: int, bits: int) -> np.ndarray:
    word, bit = _frag_words(MT, KS, bits)
    words = np.zeros(code_bytes(bits) // 4, np.uint32)
    np.bitwise_or.at(words, word.ravel(), (X.astype(np.uint32) << bit.astype(np.uint32)).ravel())
    return words.astype("<u4").view(np.uint8)


def unpack_codes(buf: np.ndarray, MT: int, KS: int, bits: int) -> np.ndarray:
    words = np.frombuffer(np.ascontiguousarray(buf).tobytes(), "<u4")
    word, bit = _frag_words(MT, KS, bits)
    return ((words[word] >> bit.astype(np.uint32)) & ((1 << bits) - 1)).astype(np.uint8)


def _orders():
    i = np.arange(128)
    ks, tig, e = i // 16, (i // 4) % 4, i % 4
    ksc = 16 * ks + 2 * tig + (e & 1) + 8 * (e >> 1)
    grp = i % 4
    tig2 = (i // 4) % 4
    e2 = (i // 16) % 4
    ks2 = i // 64
    vsc_tok = 16 * ks2 + 2 * tig2 + (e2 & 1) + 8 * (e2 >> 1)
    g = (i // 4) % 8
    j = i // 32
    vzc_tok = g + 8 * j
    t = np.arange(32)
    tok = (t // 4) + 8 * (t % 4)
    return ksc, (vsc_tok, grp), (vzc_tok, grp), tok


KSC, VSC, VZC, TOK = _orders()


def subblock(e: Encoded, page: int, transform: int):
    """Expected bytes of logical page `page` of an encoded stream, and a mask of the defined bytes."""
    bits = e.bits
    CB = code_bytes(bits)
    size = subblock_bytes(bits, transform)
    out = np.zeros(size, np.uint8)
    defined = np.zeros(size, bool)
    t0 = page * GROUP
    n_present = max(0, min(GROUP, e.N - t0))
    sealed = n_present == GROUP
    if sealed:
        out[0:CB] = pack_codes(e.kcode[page], 2, 8, bits)
        out[CB:CB + 512] = e.ks[page][KSC].astype("<f4").view(np.uint8)
        out[CB + 512:CB + 1024] = e.kz[page][KSC].astype("<f4").view(np.uint8)
        out[2 * CB + 2048:2 * CB + 2080] = e.kidx[t0 + TOK]
        defined[0:CB + 1024] = True
        defined[2 * CB + 2048:2 * CB + 2080] = True
        if transform:
            out[2 * CB + 2112:2 * CB + 2240] = e.krow[t0 + TOK].astype("<f4").view(np.uint8)
            defined[2 * CB + 2112:2 * CB + 2240] = True
    present = np.arange(GROUP) < n_present
    vt = np.zeros((D, GROUP), np.uint8)
    vt[:, :n_present] = e.vcode[t0:t0 + n_present].T
    out[CB + 1024:2 * CB + 1024] = pack_codes(vt, 8, 2, bits)

    def per_token(arr, tokens, grp=None):
        vals = np.zeros(len(tokens), np.float32)
        ok = present[tokens]
        src = t0 + tokens[ok]
        vals[ok] = arr[src] if grp is None else arr[src, grp[ok]]
        return vals

    out[2 * CB + 1024:2 * CB + 1536] = per_token(e.vs, VSC[0], VSC[1]).astype("<f4").view(np.uint8)
    out[2 * CB + 1536:2 * CB + 2048] = per_token(e.vz, VZC[0], VZC[1]).astype("<f4").view(np.uint8)
    vid = np.zeros(GROUP, np.uint8)
    vid[present[TOK]] = e.vidx[t0 + TOK[present[TOK]]]
    out[2 * CB + 2080:2 * CB + 2112] = vid
    defined[CB + 1024:2 * CB + 2048] = True
    defined[2 * CB + 2080:2 * CB + 2112] = True
    if transform:
        out[2 * CB + 2240:2 * CB + 2368] = per_token(e.vrow, TOK).astype("<f4").view(np.uint8)
        defined[2 * CB + 2240:2 * CB + 2368] = True
    return out, defined


def parse_subblock(buf: np.ndarray, bits: int, transform: int):
    """Inverse of subblock() for a sealed page: natural-order arrays (for pack/unpack round-trip tests)."""
    CB = code_bytes(bits)
    buf = np.ascontiguousarray(buf, np.uint8)
    kcode = unpack_codes(buf[0:CB], 2, 8, bits)
    ks = np.zeros(D, np.float32)
    kz = np.zeros(D, np.float32)
    ks[KSC] = buf[CB:CB + 512].view("<f4")
    kz[KSC] = buf[CB + 512:CB + 1024].view("<f4")
    vcode = unpack_codes(buf[CB + 1024:2 * CB + 1024], 8, 2, bits).T
    vs = np.zeros((GROUP, 4), np.float32)
    vz = np.zeros((GROUP, 4), np.float32)
    vs[VSC[0], VSC[1]] = buf[2 * CB + 1024:2 * CB + 1536].view("<f4")
    vz[VZC[0], VZC[1]] = buf[2 * CB + 1536:2 * CB + 2048].view("<f4")
    kidx = np.zeros(GROUP, np.uint8)
    vidx = np.zeros(GROUP, np.uint8)
    kidx[TOK] = buf[2 * CB + 2048:2 * CB + 2080]
    vidx[TOK] = buf[2 * CB + 2080:2 * CB + 2112]
    out = dict(kcode=kcode, ks=ks, kz=kz, vcode=vcode, vs=vs, vz=vz, kidx=kidx, vidx=vidx)
    if transform:
        krow = np.zeros(GROUP, np.float32)
        vrow = np.zeros(GROUP, np.float32)
        krow[TOK] = buf[2 * CB + 2112:2 * CB + 2240].view("<f4")
        vrow[TOK] = buf[2 * CB + 2240:2 * CB + 2368].view("<f4")
        out.update(krow=krow, vrow=vrow)
    return out
