"""Seeded synthetic inputs shaped like the PatternKV / KVarN workloads.

This package draws inputs only: it holds none of the quantization, pattern or
attention arithmetic.  The CUDA path and the CPU oracle both take their K, V and
q from here, so the two sides always see identical values.

The five workloads mirror the shapes the pages evaluate on (head_dim 128, GQA,
8K-131K contexts, long chain-of-thought decode, many parallel samples).  The
pages evaluate on LongBench / GSM8K / AIME / AMC with trained Llama and Qwen
weights; none of that is available or used here: mixtures of Gaussian centers
with K outlier channels and RoPE rotation stand in for real K/V activations
(PatternKV, Section 2.2: K has stable outlier channels and drifts smoothly under
RoPE; V clusters around semantic centers).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_build", "libsynth.so")
_lib = None

FP16, BF16 = 0, 1


class _Params(ctypes.Structure):
    _fields_ = [
        ("seed", ctypes.c_uint64),
        ("B", ctypes.c_int32), ("S", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
        ("nck", ctypes.c_int32), ("ncv", ctypes.c_int32),
        ("sigma_k", ctypes.c_double), ("sigma_v", ctypes.c_double),
        ("n_outlier", ctypes.c_int32),
        ("out_lo", ctypes.c_double), ("out_hi", ctypes.c_double),
        ("rope", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("sample_sigma", ctypes.c_double),
        ("drift_start", ctypes.c_int32),
        ("drift_block", ctypes.c_int32),
        ("drift_step", ctypes.c_double),
        ("dtype", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile the generator into synth/_build/libsynth.so (host C, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=gnu11",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_kv.restype = ctypes.c_int
        lib.synth_kv.argtypes = [ctypes.POINTER(_Params), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                 ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_q.restype = None
        lib.synth_q.argtypes = [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
        lib.synth_uniform.restype = ctypes.c_double
        lib.synth_uniform.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_outliers.restype = None
        lib.synth_outliers.argtypes = [ctypes.POINTER(_Params), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
        _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: cache shape, generator recipe and method knobs."""
    name: str
    seed: int
    B: int              # sequences (batch)
    S: int              # context (prefill) tokens per sequence
    Hkv: int            # KV heads
    Hq: int             # query heads
    D: int = 128        # head_dim
    nck: int = 64       # K mixture centers
    ncv: int = 64       # V mixture centers
    sigma_k: float = 0.3
    sigma_v: float = 0.5
    n_outlier: int = 8
    out_lo: float = 10.0
    out_hi: float = 20.0
    rope: bool = True
    rope_base: float = 10000.0
    sample_sigma: float = 0.0
    drift_start: int = -1
    drift_block: int = 512
    drift_step: float = 0.01
    dtype: int = BF16
    P: int = 64         # patterns per (set, KV head)
    iters: int = 4      # Lloyd iterations
    bits: int = 2
    transform: int = 0  # 0 = pattern residual only, 1 = Hadamard + dual-axis variance normalisation
    steps: int = 0      # decode steps after the prefill (long chain-of-thought workload)
    v_alpha: float = 0.05  # significance level of the V adaptive threshold (0 = threshold off)

    def params(self) -> _Params:
        return _Params(self.seed, self.B, self.S, self.Hkv, self.D, self.nck, self.ncv, self.sigma_k,
                       self.sigma_v, self.n_outlier, self.out_lo, self.out_hi, int(self.rope), self.rope_base,
                       self.sample_sigma, self.drift_start, self.drift_block, self.drift_step, self.dtype)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 1 layer, 1 KV head, 1 query head, 4096 tokens, fp16; 16-center mixtures, 4 outlier channels x15.
    "tiny_ref_4k": Workload("tiny_ref_4k", seed=0, B=1, S=4096, Hkv=1, Hq=1, nck=16, ncv=16,
                            n_outlier=4, out_lo=15.0, out_hi=15.0, rope=False, dtype=FP16, P=16),
    # Llama-3-8B-shaped layer: 32 q heads / 8 KV heads, 8 x 32768 tokens, bf16.
    "llama3_8b_32k": Workload("llama3_8b_32k", seed=2, B=8, S=32768, Hkv=8, Hq=32),
    # Long chain-of-thought decode: 32 x 8192 prefill then 4096 one-token steps with slow center drift.
    "long_cot_8k": Workload("long_cot_8k", seed=3, B=32, S=8192, Hkv=8, Hq=32, drift_start=8192, steps=4096),
    # Qwen2.5-7B-shaped layer: 28 q heads / 4 KV heads, 4 x 131072 tokens.
    "qwen25_7b_128k": Workload("qwen25_7b_128k", seed=4, B=4, S=131072, Hkv=4, Hq=28),
    # Breadth test-time scaling: 256 samples x 16384 tokens, per-sample centers perturbed by N(0, 0.1^2).
    "breadth_256x16k": Workload("breadth_256x16k", seed=5, B=256, S=16384, Hkv=8, Hq=32, sample_sigma=0.1),
}


def gen_kv(w: Workload, b0: int = 0, b1: int | None = None, p0: int = 0, p1: int | None = None,
           want_k: bool = True, want_v: bool = True):
    """K, V as uint16 bit patterns (fp16 or bf16) shaped [b1-b0, p1-p0, Hkv, D]."""
    b1 = w.B if b1 is None else b1
    p1 = w.S if p1 is None else p1
    shape = (b1 - b0, p1 - p0, w.Hkv, w.D)
    k = np.empty(shape, np.uint16) if want_k else None
    v = np.empty(shape, np.uint16) if want_v else None
    prm = w.params()
    rc = _load().synth_kv(ctypes.byref(prm), b0, b1, p0, p1,
                          k.ctypes.data if k is not None else None, v.ctypes.data if v is not None else None)
    if rc != 0:
        raise ValueError(f"synth_kv: unsupported workload shape (rc={rc})")
    return k, v


def gen_q(w: Workload, step: int = 0, b0: int = 0, b1: int | None = None) -> np.ndarray:
    """Decode queries as uint16 bit patterns shaped [b1-b0, Hq, D], N(0,1) before rounding."""
    b1 = w.B if b1 is None else b1
    out = np.empty((b1 - b0, w.Hq, w.D), np.uint16)
    _load().synth_q(w.seed, step, w.B, b0, b1, w.Hq, w.D, w.dtype, out.ctypes.data)
    return out


def outliers(w: Workload, h: int):
    """(channels, scales) of the K outlier channels of KV head h."""
    ch = np.zeros(max(w.n_outlier, 1), np.int32)
    sc = np.zeros(max(w.n_outlier, 1), np.float64)
    prm = w.params()
    _load().synth_outliers(ctypes.byref(prm), h, ch.ctypes.data, sc.ctypes.data)
    return ch[: w.n_outlier], sc[: w.n_outlier]


def uniform(seed: int, stream: int, ctr: int) -> float:
    return _load().synth_uniform(seed, stream, ctr)


def normal(seed: int, stream: int, i: int) -> float:
    return _load().synth_normal(seed, stream, i)


def to_float(bits: np.ndarray, dtype: int) -> np.ndarray:
    """fp16 / bf16 bit patterns -> float32 (exact)."""
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << 16).view(np.float32)
