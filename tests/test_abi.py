"""The C-ABI library loads and exports every entry point include/kvq.h declares, and its
host-side validation rejects bad arguments before touching a GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "kvq.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    syms = declared_symbols()
    for name in ["kvq_mine_patterns", "kvq_quantize_append", "kvq_decode_attention", "kvq_dequantize"]:
        assert name in syms


def test_library_exports_every_declared_symbol():
    import bit_kv_cache_26_b200 as kvq
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(kvq.EXPORTED)


def test_layout_sizes():
    import bit_kv_cache_26_b200 as kvq
    assert kvq.kvq_subblock_bytes(2, 0) == 4160
    assert kvq.kvq_subblock_bytes(4, 0) == 6208
    assert kvq.kvq_subblock_bytes(2, 1) == 4416
    assert kvq.kvq_subblock_bytes(3, 0) == 0
    c = kvq.kvq_cache()
    c.num_kv_heads, c.bits, c.head_dim, c.group = 8, 2, 128, 32
    assert kvq.kvq_page_bytes(c) == 8 * 4160


def _cache(**kw):
    import bit_kv_cache_26_b200 as kvq
    c = kvq.kvq_cache()
    c.num_seqs, c.num_kv_heads, c.head_dim, c.group, c.bits, c.num_patterns = 1, 1, 128, 32, 2, 16
    c.num_sets, c.max_pages_per_seq, c.num_pages, c.dtype = 1, 4, 4, 1
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, 2), ("group", 16, 2), ("bits", 3, 2), ("num_patterns", 0, 2), ("num_patterns", 256, 2),
    ("dtype", 7, 2), ("transform", 5, 2), ("v_rho", -1.0, 1), ("v_rho", float("nan"), 1),
    ("v_rho", float("inf"), 1),
])
def test_append_rejects_bad_cache_on_host(field, value, status):
    import bit_kv_cache_26_b200 as kvq
    c = _cache(**{field: value})
    rc = kvq._lib.kvq_quantize_append(ctypes.byref(c), None, None, 1, None, 0, None)
    assert rc == status
    assert kvq.kvq_last_error()


def test_null_pointers_rejected_on_host():
    import bit_kv_cache_26_b200 as kvq
    c = _cache()  # all device pointers NULL
    assert kvq._lib.kvq_quantize_append(ctypes.byref(c), None, None, 1, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert kvq._lib.kvq_quantize_append(None, None, None, 1, None, 0, None) == kvq.KVQ_ERR_INVALID_ARG
    assert kvq._lib.kvq_dequantize(ctypes.byref(c), 0, 0, 0, 1, None, None, None) == kvq.KVQ_ERR_INVALID_ARG


def test_mine_validation_on_host():
    import bit_kv_cache_26_b200 as kvq
    L = kvq._lib
    # n < P
    assert L.kvq_mine_patterns(ctypes.c_void_p(16), 1, 8, 1, 1, 128, 128, 0, 16, 4, 0, ctypes.c_void_p(16), None,
                               None, ctypes.c_void_p(256), 1 << 30, None) == kvq.KVQ_ERR_INVALID_ARG
    # P out of range
    assert L.kvq_mine_patterns(ctypes.c_void_p(16), 1, 8, 1, 1, 128, 128, 0, 300, 4, 0, ctypes.c_void_p(16), None,
                               None, None, 0, None) == kvq.KVQ_ERR_UNSUPPORTED
    # workspace too small
    assert L.kvq_mine_patterns(ctypes.c_void_p(16), 1, 100, 1, 1, 128, 128, 0, 16, 4, 0, ctypes.c_void_p(16), None,
                               None, ctypes.c_void_p(256), 8, None) == kvq.KVQ_ERR_WORKSPACE
    # transform without colscale output
    assert L.kvq_mine_patterns(ctypes.c_void_p(16), 1, 100, 1, 1, 128, 128, 0, 16, 4, 1, ctypes.c_void_p(16), None,
                               None, ctypes.c_void_p(256), 1 << 30, None) == kvq.KVQ_ERR_INVALID_ARG


def test_decode_validation_on_host():
    import bit_kv_cache_26_b200 as kvq
    c = _cache(num_kv_heads=2, page_pool=256, page_table=16, seq_len=16, k_tail=16, k_patterns=16, v_patterns=16,
               status=16)
    rc = kvq._lib.kvq_decode_attention(ctypes.byref(c), ctypes.c_void_p(16), 3, 0.1, ctypes.c_void_p(16),
                                       ctypes.c_void_p(256), 1 << 20, None)
    assert rc == kvq.KVQ_ERR_UNSUPPORTED  # 3 query heads over 2 KV heads
    rc = kvq._lib.kvq_decode_attention(ctypes.byref(c), ctypes.c_void_p(16), 4, 0.1, ctypes.c_void_p(16),
                                       ctypes.c_void_p(256), 8, None)
    assert rc == kvq.KVQ_ERR_WORKSPACE


def test_static_scratch_size_matches_header():
    import bit_kv_cache_26_b200 as kvq
    m = re.search(r"#define\s+KVQ_DECODE_STATIC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", open(HEADER).read())
    assert m and int(m.group(1)) << int(m.group(2)) == kvq.KVQ_DECODE_STATIC_SCRATCH_BYTES


def test_library_rho_star_equals_the_oracles():
    # The library's closed form and the oracle's bisection of Eq. 10 give the same fp32 threshold
    # (the two sides must take the keep-the-pattern decision in the same precision).
    import numpy as np

    import bit_kv_cache_26_b200 as kvq
    import oracle
    for d in (64, 96, 128, 256):
        for a in (0.2, 0.1, 0.05, 0.01, 0.001):
            assert kvq.kvq_v_rho_star(d, a) == np.float32(oracle.rho_star(d, a)), (d, a)
    assert kvq.kvq_v_rho_star(128, 0.0) == 0.0 and oracle.v_rho(0.0) == 0.0
