"""Python binding of libkvq (include/kvq.h): pattern-aligned residual 2/4-bit KV-cache
quantization and decode attention over the quantized paged cache, on NVIDIA B200.

Argument marshalling only: every step of the computation runs in the CUDA kernels of
``libkvq.so``.  PyTorch is used for device memory and streams.  There is no CPU or
PyTorch fallback: importing this package fails if the library is missing.

Functions keep the C names (``kvq_mine_patterns``, ``kvq_quantize_append``,
``kvq_decode_attention``, ``kvq_dequantize`` ...); tensors are passed as torch CUDA
tensors and the call is enqueued on the current torch stream unless ``stream`` is given.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libkvq.so not found at {LIB_PATH}; build it with `python bit_kv_cache_26_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, KVQ_ERR_CUDA, KVQ_ERR_DEVICE = range(7)
KVQ_DECODE_STATIC_SCRATCH_BYTES = 16 << 20  # size of the fixed scratch of kvq_decode_attention_static
KVQ_DEV_BAD_PAGE, KVQ_DEV_OVERFLOW, KVQ_DEV_BAD_SET, KVQ_DEV_TIMEOUT, KVQ_DEV_RANGE = 0x1, 0x2, 0x4, 0x8, 0x10
KVQ_F16, KVQ_BF16 = 0, 1
KVQ_TX_NONE, KVQ_TX_HADAMARD_VARNORM = 0, 1
HEAD_DIM, GROUP = 128, 32


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"kvq status {status}: {message}")
        self.status = status


class kvq_cache(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("group", ctypes.c_int32), ("bits", ctypes.c_int32), ("num_patterns", ctypes.c_int32),
        ("num_sets", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("transform", ctypes.c_int32), ("v_rho", ctypes.c_float),
        ("page_pool", ctypes.c_void_p), ("page_table", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
        ("k_tail", ctypes.c_void_p), ("k_patterns", ctypes.c_void_p), ("v_patterns", ctypes.c_void_p),
        ("seq_to_set", ctypes.c_void_p), ("k_colscale", ctypes.c_void_p), ("v_colscale", ctypes.c_void_p),
        ("status", ctypes.c_void_p),
        ("pattern_counts", ctypes.c_void_p), ("pattern_window", ctypes.c_void_p),
        ("pattern_window_len", ctypes.c_int32), ("reserved", ctypes.c_int32),
    ]


_P = ctypes.POINTER(kvq_cache)
_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "kvq_page_bytes": (_sz, [_P]),
    "kvq_subblock_bytes": (_sz, [_i32, _i32]),
    "kvq_v_rho_star": (_f32, [_i32, ctypes.c_double]),
    "kvq_mine_workspace_bytes": (_sz, [_i64, _i32, _i32, _i32, _i32]),
    "kvq_mine_patterns": (ctypes.c_int, [_vp, _i32, _i64, _i32, _i32, _i64, _i64, _i64, _i32, _i32, _i32,
                                         _vp, _vp, _vp, _vp, _sz, _vp]),
    "kvq_append_workspace_bytes": (_sz, [_P, _i32]),
    "kvq_quantize_append": (ctypes.c_int, [_P, _vp, _vp, _i32, _vp, _sz, _vp]),
    "kvq_decode_workspace_bytes": (_sz, [_P, _i32]),
    "kvq_decode_attention": (ctypes.c_int, [_P, _vp, _i32, _f32, _vp, _vp, _sz, _vp]),
    "kvq_decode_attention_static": (ctypes.c_int, [_P, _vp, _i32, _f32, _vp, _vp]),
    "kvq_step_workspace_bytes": (_sz, [_P, _i32]),
    "kvq_decode_step": (ctypes.c_int, [_P, _vp, _vp, _vp, _i32, _f32, _vp, _vp, _sz, _vp]),
    "kvq_dequantize": (ctypes.c_int, [_P, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "kvq_read_status": (ctypes.c_int, [_P, ctypes.POINTER(_i32), _i32, _vp]),
    "kvq_mine_read_status": (ctypes.c_int, [_vp, ctypes.POINTER(_i32), _vp]),
    "kvq_last_error": (ctypes.c_char_p, []),
    "kvq_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int):
    if rc != KVQ_OK:
        raise KvqError(rc, kvq_last_error())


def kvq_last_error() -> str:
    return _lib.kvq_last_error().decode()


def kvq_version() -> str:
    return _lib.kvq_version().decode()


def kvq_subblock_bytes(bits: int, transform: int) -> int:
    return int(_lib.kvq_subblock_bytes(bits, transform))


def kvq_v_rho_star(head_dim: int, alpha: float) -> float:
    """rho*(d, alpha) of PatternKV Eq. 10 as the fp32 value the kernels compare with (0 = off)."""
    return float(_lib.kvq_v_rho_star(head_dim, alpha))


def kvq_page_bytes(cache: kvq_cache) -> int:
    return int(_lib.kvq_page_bytes(ctypes.byref(cache)))


def kvq_mine_workspace_bytes(n: int, num_sets: int, num_kv_heads: int, P: int, transform: int) -> int:
    return int(_lib.kvq_mine_workspace_bytes(n, num_sets, num_kv_heads, P, transform))


def kvq_mine_patterns(x: torch.Tensor, dtype: int, n: int, num_sets: int, num_kv_heads: int, tok_stride: int,
                      head_stride: int, set_stride: int, P: int, iters: int, transform: int,
                      patterns_out: torch.Tensor, colscale_out: torch.Tensor | None, assign_out: torch.Tensor | None,
                      ws: torch.Tensor | None, stream=None) -> None:
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.kvq_mine_patterns(_ptr(x), dtype, n, num_sets, num_kv_heads, tok_stride, head_stride, set_stride, P,
                                  iters, transform, _ptr(patterns_out), _ptr(colscale_out), _ptr(assign_out),
                                  _ptr(ws), ws_bytes, _stream(stream)))


def kvq_mine_read_status(ws: torch.Tensor, stream=None) -> int:
    """Status bits of the mining call that used workspace `ws` (synchronises the stream)."""
    bits = ctypes.c_int32(0)
    rc = _lib.kvq_mine_read_status(_ptr(ws), ctypes.byref(bits), _stream(stream))
    if rc not in (KVQ_OK, KVQ_ERR_DEVICE):
        _check(rc)
    return int(bits.value)


def kvq_append_workspace_bytes(cache: kvq_cache, n_new: int) -> int:
    return int(_lib.kvq_append_workspace_bytes(ctypes.byref(cache), n_new))


def kvq_quantize_append(cache: kvq_cache, k_new: torch.Tensor, v_new: torch.Tensor, n_new: int,
                        ws: torch.Tensor | None = None, stream=None) -> None:
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.kvq_quantize_append(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), n_new, _ptr(ws), ws_bytes,
                                    _stream(stream)))


def kvq_decode_workspace_bytes(cache: kvq_cache, num_q_heads: int) -> int:
    return int(_lib.kvq_decode_workspace_bytes(ctypes.byref(cache), num_q_heads))


def kvq_decode_attention(cache: kvq_cache, q: torch.Tensor, num_q_heads: int, sm_scale: float, out: torch.Tensor,
                         ws: torch.Tensor, stream=None) -> None:
    _check(_lib.kvq_decode_attention(ctypes.byref(cache), _ptr(q), num_q_heads, sm_scale, _ptr(out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)))


def kvq_decode_attention_static(cache: kvq_cache, q: torch.Tensor, num_q_heads: int, sm_scale: float,
                                out: torch.Tensor, stream=None) -> None:
    """kvq_decode_attention with its partials in the library's fixed device array (no workspace)."""
    _check(_lib.kvq_decode_attention_static(ctypes.byref(cache), _ptr(q), num_q_heads, sm_scale, _ptr(out),
                                            _stream(stream)))


def kvq_step_workspace_bytes(cache: kvq_cache, num_q_heads: int) -> int:
    return int(_lib.kvq_step_workspace_bytes(ctypes.byref(cache), num_q_heads))


def kvq_decode_step(cache: kvq_cache, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, num_q_heads: int,
                    sm_scale: float, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """One-token quantize-append + decode attention in one launch (workspace zero-filled before first use)."""
    _check(_lib.kvq_decode_step(ctypes.byref(cache), _ptr(k_new), _ptr(v_new), _ptr(q), num_q_heads, sm_scale,
                                _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def kvq_dequantize(cache: kvq_cache, seq: int, seq_len_host: int, start: int, count: int,
                   k_out: torch.Tensor | None, v_out: torch.Tensor | None, stream=None) -> None:
    _check(_lib.kvq_dequantize(ctypes.byref(cache), seq, seq_len_host, start, count, _ptr(k_out), _ptr(v_out),
                               _stream(stream)))


def kvq_read_status(cache: kvq_cache, clear: bool = False, stream=None) -> int:
    bits = ctypes.c_int32(0)
    rc = _lib.kvq_read_status(ctypes.byref(cache), ctypes.byref(bits), int(clear), _stream(stream))
    if rc not in (KVQ_OK, KVQ_ERR_DEVICE):
        _check(rc)
    return int(bits.value)


# ---------------------------------------------------------------------------
# Device-memory plumbing: a paged cache whose buffers are torch tensors.
# ---------------------------------------------------------------------------

def _alloc_aligned(nbytes: int, device, align: int = 256, zero: bool = False) -> torch.Tensor:
    buf = (torch.zeros if zero else torch.empty)(nbytes + align, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % align
    return buf[off:off + nbytes]


class PagedKVCache:
    """Owns the device buffers of one quantized KV cache and the matching kvq_cache struct.

    page_order: optional permutation of the physical pages (default: sequence-major,
    page i of sequence b at b * max_pages_per_seq + i).
    v_rho: V adaptive threshold (PatternKV Section 3.3); kvq_v_rho_star(128, alpha) for a
    significance level alpha, 0 = off.
    patterns_in_use / insertion_window: decode-time pattern insertion (PatternKV Section 3.1,
    Eq. 5): every set starts with `patterns_in_use` of its `num_patterns` rows in use, and each
    kvq_decode_step that brings a sequence to a multiple of `insertion_window` tokens adds the
    window's Chebyshev centers as the next pattern (sequences need sets of their own).
    """

    def __init__(self, num_seqs: int, num_kv_heads: int, max_tokens: int, bits: int, num_patterns: int,
                 dtype: int = KVQ_BF16, transform: int = KVQ_TX_NONE, num_sets: int = 1, device="cuda",
                 page_order: torch.Tensor | None = None, seq_to_set: torch.Tensor | None = None,
                 v_rho: float = 0.0, patterns_in_use: int | None = None, insertion_window: int = 0):
        self.device = torch.device(device)
        self.B, self.H, self.bits, self.P, self.S = num_seqs, num_kv_heads, bits, num_patterns, num_sets
        self.dtype, self.transform = dtype, transform
        self.maxp = (max_tokens + GROUP - 1) // GROUP
        self.num_pages = self.B * self.maxp
        c = kvq_cache()
        c.num_seqs, c.num_kv_heads, c.head_dim, c.group = num_seqs, num_kv_heads, HEAD_DIM, GROUP
        c.bits, c.num_patterns, c.num_sets = bits, num_patterns, num_sets
        c.max_pages_per_seq, c.num_pages, c.dtype, c.transform = self.maxp, self.num_pages, dtype, transform
        c.v_rho = v_rho
        self.page_bytes = kvq_page_bytes(c)
        if self.page_bytes == 0:
            raise KvqError(KVQ_ERR_UNSUPPORTED, f"unsupported cache shape (bits={bits})")
        self.pool = _alloc_aligned(max(1, self.num_pages) * self.page_bytes, self.device)
        order = torch.arange(self.num_pages, dtype=torch.int32) if page_order is None else page_order.to(torch.int32)
        self.page_table = order.reshape(max(self.B, 1) if self.B else 0, self.maxp).to(self.device).contiguous() \
            if self.B else torch.zeros(0, dtype=torch.int32, device=self.device)
        self.seq_len = torch.zeros(self.B, dtype=torch.int32, device=self.device)
        tdt = torch.bfloat16 if dtype == KVQ_BF16 else torch.float16
        self.k_tail = torch.zeros(self.B, self.H, GROUP, HEAD_DIM, dtype=tdt, device=self.device)
        self.k_patterns = torch.zeros(num_sets, self.H, num_patterns, HEAD_DIM, dtype=torch.float32, device=self.device)
        self.v_patterns = torch.zeros_like(self.k_patterns)
        self.seq_to_set = None if seq_to_set is None else seq_to_set.to(torch.int32).to(self.device).contiguous()
        self.k_colscale = self.v_colscale = None
        if transform:
            self.k_colscale = torch.ones(num_sets, self.H, HEAD_DIM, dtype=torch.float32, device=self.device)
            self.v_colscale = torch.ones_like(self.k_colscale)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.pattern_counts = None
        self.pattern_window = None
        if patterns_in_use is not None or insertion_window:
            self.pattern_counts = torch.full((num_sets, self.H), num_patterns if patterns_in_use is None else patterns_in_use,
                                             dtype=torch.int32, device=self.device)
        if insertion_window:
            w = torch.empty(self.B, self.H, 4, HEAD_DIM, dtype=torch.float32, device=self.device)
            w[:, :, 0::2] = float("inf")
            w[:, :, 1::2] = float("-inf")
            self.pattern_window = w
        c.page_pool = self.pool.data_ptr()
        c.page_table = self.page_table.data_ptr() if self.B else None
        c.seq_len = self.seq_len.data_ptr()
        c.k_tail = self.k_tail.data_ptr()
        c.k_patterns = self.k_patterns.data_ptr()
        c.v_patterns = self.v_patterns.data_ptr()
        c.seq_to_set = None if self.seq_to_set is None else self.seq_to_set.data_ptr()
        c.k_colscale = None if self.k_colscale is None else self.k_colscale.data_ptr()
        c.v_colscale = None if self.v_colscale is None else self.v_colscale.data_ptr()
        c.status = self.status.data_ptr()
        c.pattern_counts = None if self.pattern_counts is None else self.pattern_counts.data_ptr()
        c.pattern_window = None if self.pattern_window is None else self.pattern_window.data_ptr()
        c.pattern_window_len = int(insertion_window)
        c.reserved = 0
        self.c = c

    @property
    def subblock_bytes(self) -> int:
        return kvq_subblock_bytes(self.bits, self.transform)

    def subblock(self, seq: int, page: int, head: int) -> torch.Tensor:
        """Bytes of one (sequence, logical page, KV head) sub-block (a view into the pool)."""
        phys = int(self.page_table[seq, page])
        o = phys * self.page_bytes + head * self.subblock_bytes
        return self.pool[o:o + self.subblock_bytes]

    def append_workspace(self) -> torch.Tensor:
        if getattr(self, "_append_ws", None) is None:
            self._append_ws = _alloc_aligned(max(256, kvq_append_workspace_bytes(self.c, 1)), self.device)
        return self._append_ws

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        kvq_quantize_append(self.c, k_new, v_new, int(k_new.shape[1]), self.append_workspace(), stream)

    def decode_workspace(self, num_q_heads: int) -> torch.Tensor:
        return _alloc_aligned(kvq_decode_workspace_bytes(self.c, num_q_heads), self.device)

    def decode(self, q: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, sm_scale: float | None = None,
               stream=None) -> None:
        scale = HEAD_DIM ** -0.5 if sm_scale is None else sm_scale
        kvq_decode_attention(self.c, q, int(q.shape[1]), scale, out, ws, stream)

    def step_workspace(self, num_q_heads: int) -> torch.Tensor:
        """Zero-filled workspace of kvq_decode_step (the kernel keeps its counters at zero)."""
        return _alloc_aligned(kvq_step_workspace_bytes(self.c, num_q_heads), self.device, zero=True)

    def step(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
             sm_scale: float | None = None, stream=None) -> None:
        """kvq_decode_step: k_new / v_new [num_seqs][num_kv_heads][128], q [num_seqs][num_q_heads][128]."""
        scale = HEAD_DIM ** -0.5 if sm_scale is None else sm_scale
        kvq_decode_step(self.c, k_new, v_new, q, int(q.shape[1]), scale, out, ws, stream)

    def read_status(self, clear: bool = False) -> int:
        return kvq_read_status(self.c, clear)


def mine(x: torch.Tensor, P: int, iters: int = 4, transform: int = KVQ_TX_NONE, num_sets: int = 1,
         want_assign: bool = False, stream=None, check: bool = True):
    """Mine patterns from x shaped [num_sets, n, H, 128] (fp16/bf16, contiguous).

    Returns (patterns [sets,H,P,128] fp32, colscale [sets,H,128] or None, assign [sets,H,n] or None).
    With `check`, the call's device status word is read back (a stream synchronisation) and a
    set bit raises KvqError.
    """
    assert x.dim() == 4 and x.shape[-1] == HEAD_DIM and x.is_contiguous()
    S, n, H, _ = x.shape
    dt = KVQ_BF16 if x.dtype == torch.bfloat16 else KVQ_F16
    pats = torch.empty(S, H, P, HEAD_DIM, dtype=torch.float32, device=x.device)
    col = torch.empty(S, H, HEAD_DIM, dtype=torch.float32, device=x.device) if transform else None
    asg = torch.empty(S, H, n, dtype=torch.int32, device=x.device) if want_assign else None
    ws = _alloc_aligned(kvq_mine_workspace_bytes(n, S, H, P, transform), x.device)
    kvq_mine_patterns(x, dt, n, S, H, H * HEAD_DIM, HEAD_DIM, n * H * HEAD_DIM, P, iters, transform, pats, col, asg,
                      ws, stream)
    if check:
        bits = kvq_mine_read_status(ws, stream)
        if bits:
            raise KvqError(KVQ_ERR_DEVICE, f"mining status bits 0x{bits:x}")
    return pats, col, asg
