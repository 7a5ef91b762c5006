"""Failure detection on the device path, without a GPU fault.

Decode attention waits for each page copy with a bounded mbarrier wait.  In a child process
started with KVQ_TEST_WAIT_LIMIT=0 every page-loop wait gives up at once: the kernel must set
KVQ_DEV_TIMEOUT in the cache's status word, still wait (under the normal limit) for the copies
it issued, and return, leaving the CUDA context usable (a later kernel and copy succeed)."""
import os
import subprocess
import sys
import textwrap

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import torch
    import bit_kv_cache_26_b200 as kvq
    import synth
    from kvq_testlib import D, make_cache, oracle_patterns, to_torch

    w = synth.WORKLOADS["llama3_8b_32k"].with_(B=2, S=300, Hkv=2, Hq=8, P=8)
    k, v = synth.gen_kv(w)
    Kf, Vf = synth.to_float(k, w.dtype), synth.to_float(v, w.dtype)
    MK, MV, cK, cV = oracle_patterns(w, Kf, Vf)
    cache = make_cache(w, MK, MV, cK, cV)
    cache.append(to_torch(k, w.dtype), to_torch(v, w.dtype))
    torch.cuda.synchronize()
    assert cache.read_status(clear=True) == 0          # append has no page-copy waits
    out = torch.zeros(w.B, w.Hq, D, device="cuda")
    cache.decode(to_torch(synth.gen_q(w), w.dtype), out, cache.decode_workspace(w.Hq))
    bits = cache.read_status(clear=True)
    assert bits & kvq.KVQ_DEV_TIMEOUT, hex(bits)
    # the context still works: a plain kernel and a copy back
    t = torch.arange(1 << 20, device="cuda", dtype=torch.float32).sum().item()
    assert t == float((1 << 20) * ((1 << 20) - 1) // 2)
    print("timeout flagged", hex(bits))
""")


def test_decode_page_wait_expiry_flags_timeout():
    env = dict(os.environ, KVQ_TEST_WAIT_LIMIT="0")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "timeout flagged" in r.stdout
