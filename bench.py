"""Benchmark of the hot path on B200: pattern mining + quantize-append + decode attention.

One step = one pass of the whole path over one batch of synthetic input (by default the
breadth workload: 256 independent samples x 16384 tokens, 8 KV heads, 32 query heads,
head_dim 128, bf16, P=64, 2-bit, per-sample perturbed centers):
  mine K patterns, mine V patterns      (kvq_mine_patterns x2, pooled prefill of every sample)
  quantize-append the whole context     (kvq_quantize_append, into a freshly reset cache)
  one decode step of attention          (kvq_decode_attention)
All work runs in libkvq's CUDA kernels through the C ABI.  Inputs (16 GiB of K/V) exceed the
126 MB L2, so every step streams from HBM.  After the headline the same step is measured on the
Llama-shaped layer (2- and 4-bit) and the Qwen-shaped 128K layer (with and without the
pre-transform), and the long chain-of-thought loop is timed per decode step (`per_config`).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload NAME] [--bits 2|4]

Multi-GPU (torchrun): the batch's samples are sharded over the ranks (contiguous shards of the
same job); each rank mines, appends and decodes its shard, each step ends with an all-gather of
the decode outputs (NCCL), the step time is the max over ranks and value counts the whole job's
tokens (strong scaling: the total work is fixed).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "2-bit quantized-KV decode attn KV-tokens/s & HBM GB/s vs ~8 TB/s; quant-append GB/s"
DEFAULT_WORKLOAD = "breadth_256x16k"
D = 128


def bytes_per_token_head(bits: int, transform: int) -> int:
    """Algorithmic cache bytes per (token, KV head): K+V codes, fp32 scale/zero, indices (+ row factors)."""
    codes = 2 * D * bits // 8
    return codes + 64 + 2 + (8 if transform else 0)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def source_digest() -> str:
    """Digest of the CUDA sources and the layout header: DRAM traffic taken with ncu is only
    reported while the kernels it was taken on are unchanged."""
    import glob
    import hashlib
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "bit_kv_cache_26_b200", "csrc", "*"))) + \
        [os.path.join(ROOT, "include", "kvq.h")]
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def dram_traffic(workload: str, bits: int, batch: int):
    """DRAM bytes (read + write) per call of each phase, from profiles/dram_traffic.txt (one ncu
    capture per source digest); {} if there is none for the current sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    out = {}
    if not os.path.exists(path):
        return out
    digest = source_digest()
    with open(path) as f:
        for line in f:
            t = line.split()
            if len(t) == 6 and not line.startswith("#") and t[0] == digest and t[1] == workload and \
                    int(t[2]) == bits and int(t[3]) == batch:
                out[t[4]] = float(t[5])
    return out


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.strip().split(", ") for r in f if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample of the workload.
# ---------------------------------------------------------------------------

def sample_shape(w, target_s: float, unit_s: float):
    """(KV heads, sequences) of a sample of about target_s seconds, one (sequence, KV head) unit
    taking about unit_s: heads first (the generator makes every head of a sequence), then
    sequences."""
    units = max(1, min(w.B * w.Hkv, int(round(target_s / max(unit_s, 1e-3)))))
    heads = max(1, min(w.Hkv, units))
    return heads, max(1, min(w.B, -(-units // heads)))


def cpu_baseline(w, heads: int = 1, seqs: int | None = None, target_s: float | None = None):
    """The oracle, as it stands, on a bounded sample of the workload: every sequence (or the
    first `seqs`) of `heads` of the KV heads, the whole path (mining of K and V on the pooled
    prefill, encoding, decode attention of each sequence's query heads), scaled to KV-tokens/s
    of the whole job (all KV heads).  With target_s, one (sequence, KV head) unit is timed first
    and the sample is sized to about target_s seconds of oracle work."""
    import numpy as np

    import oracle
    import synth

    if target_s is not None:
        _, unit_s = cpu_baseline(w, heads=1, seqs=1)
        heads, seqs = sample_shape(w, target_s, unit_s)
    B = w.B if seqs is None else min(seqs, w.B)
    heads = max(1, min(heads, w.Hkv))
    sw = w.with_(B=B)
    k, v = synth.gen_kv(sw)
    q = synth.gen_q(sw)
    Gq = w.Hq // w.Hkv
    t0 = time.perf_counter()
    for h in range(heads):
        Kf, Vf = synth.to_float(k[:, :, h], w.dtype), synth.to_float(v[:, :, h], w.dtype)
        MK, cK, _ = oracle.mine_set(Kf.reshape(-1, D), w.P, w.iters, w.transform)
        MV, cV, _ = oracle.mine_set(Vf.reshape(-1, D), w.P, w.iters, w.transform)
        for b in range(B):
            e = oracle.encode(Kf[b], Vf[b], w.bits, MK, MV, cK, cV, v_rho=oracle.v_rho(w.v_alpha))
            qf = synth.to_float(q[b, h * Gq:(h + 1) * Gq], w.dtype)
            oracle.attention_unit(qf, Kf[b], e, MK, MV, cK, cV)
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    value = B * w.S * heads / (dt * w.Hkv)  # KV-tokens/s of the whole job: all KV heads take heads/Hkv longer
    sample = (f"oracle mining (K and V, pooled prefill), encoding and decode attention of {B} sequences x {w.S} tokens "
              f"for {heads} of {w.Hkv} KV heads ({Gq} query heads each), scaled to all KV heads; {dt:.2f} s")
    return {"value": value, "unit": "KV-tokens/s", "cores": cores, "kind": "oracle", "sample": sample}, dt


def run_reference(args):
    import synth

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload].with_(bits=args.bits, transform=args.transform)
    synth.build()
    import oracle
    oracle.build()
    vals, times = [], []
    for i in range(args.warmup + args.steps):
        cb, dt = cpu_baseline(w, heads=args.ref_heads, seqs=args.ref_seqs)
        if i >= args.warmup:
            vals.append(cb["value"])
            times.append(dt)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "KV-tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, args),
            "cpu_baseline": dict(cb, value=value),
            "e2e": {"value": value, "unit": "KV-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_shard(base, rank: int, world: int):
    """The sequences [b0, b1) of the job that rank `rank` processes (batch sharding: the samples
    are independent; total work fixed, strong scaling)."""
    from bit_kv_cache_26_b200.shard import shard_range
    return shard_range(base.B, rank, world)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity on a single process)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def workload_config(w, args):
    return {"workload": w.name, "batch": w.B, "context": w.S, "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": D,
            "patterns": w.P, "lloyd_iters": w.iters, "bits": w.bits, "group": 32,
            "transform": "hadamard+varnorm" if w.transform else "none",
            "input_dtype": "bf16" if w.dtype == 1 else "fp16",
            "parallelism": "single GPU" if args.gpus == 1 else
            f"batch-sharded x{args.gpus} (independent samples, per-rank patterns, decode outputs all-gathered)",
            "l2": f"inputs larger than L2 ({w.B * w.S * w.Hkv * D * 4 / 2**30:.1f} GiB of K/V per step, 126 MB L2)",
            "v_threshold_alpha": w.v_alpha}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

# Sub-records measured after the headline (each its own workload and roofline): the Llama-shaped
# layer at 2 and 4 bits, the Qwen-shaped 128K layer without and with the pre-transform.
PER_CONFIG = [("llama3_8b_32k", {"bits": 2}), ("llama3_8b_32k", {"bits": 4}),
              ("qwen25_7b_128k", {}), ("qwen25_7b_128k", {"transform": 1})]


def launches_per_step(w) -> int:
    """Kernels this library launches per step: per mining call init + per Lloyd iteration
    assignment (+ the float64 fix-up after the tcgen05 assignment), cluster sums and update (+8
    for the pre-transform: three fit passes with their finish kernels, the factors' output and
    apply); append: prep, pages, tail; decode: 1."""
    tc = w.dtype == 1 and not w.transform and w.P <= 128
    mine = 1 + (4 if tc else 3) * w.iters + (8 if w.transform else 0)
    return 2 * mine + 3 + 1


def measure_path(w, args, dev, world: int, rank: int, headline: bool, shard=None):
    """Time `args.steps` steps of the whole path on workload w (mine K and V patterns on the
    pooled prefill, quantize-append the whole context into a reset cache, one decode step).
    With `shard` = (b0, b1) this rank runs sequences [b0, b1) of w and each step ends with the
    all-gather of the decode outputs of every rank (NCCL).  Returns the record (and, for the
    headline, the end-to-end measurement through host buffers)."""
    import numpy as np
    import torch

    import bit_kv_cache_26_b200 as kvq
    import synth

    B_total = w.B
    b0, b1 = shard if shard else (0, w.B)
    k, v = synth.gen_kv(w, b0=b0, b1=b1)
    q = synth.gen_q(w, b0=b0, b1=b1)
    w = w.with_(B=b1 - b0)
    tdt = torch.bfloat16 if w.dtype == synth.BF16 else torch.float16

    def pinned(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(tdt).pin_memory()

    kh, vh, qh = pinned(k), pinned(v), pinned(q)
    del k, v
    kd, vd, qd = kh.to(dev), vh.to(dev), qh.to(dev)
    cache = kvq.PagedKVCache(w.B, w.Hkv, w.S, w.bits, w.P, dtype=w.dtype, transform=w.transform, device=dev,
                             v_rho=kvq.kvq_v_rho_star(D, w.v_alpha))
    n = w.B * w.S
    ws_m = kvq._alloc_aligned(kvq.kvq_mine_workspace_bytes(n, 1, w.Hkv, w.P, w.transform), dev)
    ws_d = cache.decode_workspace(w.Hq)
    ws_a = cache.append_workspace()
    out = torch.empty(w.B, w.Hq, D, device=dev)
    out_h = torch.empty(w.B, w.Hq, D).pin_memory()
    tok_stride, set_stride = w.Hkv * D, n * w.Hkv * D

    def step(kx, vx, qx, ev=None):
        if ev: ev[0].record()
        kvq.kvq_mine_patterns(kx, w.dtype, n, 1, w.Hkv, tok_stride, D, set_stride, w.P, w.iters, w.transform,
                              cache.k_patterns, cache.k_colscale, None, ws_m)
        kvq.kvq_mine_patterns(vx, w.dtype, n, 1, w.Hkv, tok_stride, D, set_stride, w.P, w.iters, w.transform,
                              cache.v_patterns, cache.v_colscale, None, ws_m)
        if ev: ev[1].record()
        cache.seq_len.zero_()
        kvq.kvq_quantize_append(cache.c, kx, vx, w.S, ws_a)
        if ev: ev[2].record()
        kvq.kvq_decode_attention(cache.c, qx, w.Hq, D ** -0.5, out, ws_d)
        if world > 1:
            from bit_kv_cache_26_b200.shard import gather_outputs
            gather_outputs(out, B_total)
        if ev: ev[3].record()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    for _ in range(args.warmup):
        step(kd, vd, qd)
    torch.cuda.synchronize()
    assert cache.read_status() == 0, "device status bits set"
    assert kvq.kvq_mine_read_status(ws_m) == 0, "mining status bits set"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(int(str(dev).split(":")[-1]) if ":" in str(dev) else 0) if headline else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        step(kd, vd, qd, evs[i])
    t_end.record()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    mine_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    append_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    decode_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    # V adaptive threshold: share of V vectors stored with their pattern (index != 255)
    sub = cache.subblock_bytes
    cb = 32 * D * w.bits // 8
    pool = cache.pool.view(-1, sub)
    vidx = pool[:, 2 * cb + 2080:2 * cb + 2112]
    utilisation = float((vidx != 255).float().mean()) if w.v_alpha > 0 else 1.0

    e2e = None
    if headline:
        # end to end through host buffers: every step copies its K, V and q from pinned memory
        # and reads its output back.  The inputs are double-buffered on the device: step i + 1's
        # copies run on a second stream while step i computes (a buffer is refilled only after
        # the step that read it has finished), as a caller streaming batches would run it.
        bufs = [(kd, vd, qd), (torch.empty_like(kd), torch.empty_like(vd), torch.empty_like(qd))]
        main = torch.cuda.current_stream(dev)
        cs = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        freed = [torch.cuda.Event() for _ in range(2)]

        def load(b):
            with torch.cuda.stream(cs):
                cs.wait_event(freed[b])
                bufs[b][0].copy_(kh, non_blocking=True)
                bufs[b][1].copy_(vh, non_blocking=True)
                bufs[b][2].copy_(qh, non_blocking=True)
                copied[b].record(cs)

        def run(nsteps):
            load(0)
            for i in range(nsteps):
                b = i % 2
                if i + 1 < nsteps:
                    load((i + 1) % 2)
                main.wait_event(copied[b])
                step(*bufs[b])
                out_h.copy_(out, non_blocking=True)
                freed[b].record(main)

        for b in range(2):
            freed[b].record(main)
        run(2)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(main)
        run(args.steps)
        e1.record(main)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        barrier()
        elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], device=dev)
        e2e = {"ms": e2e_ms, "h2d_bytes_per_step": int(kh.numel() * 2 + vh.numel() * 2 + qh.numel() * 2),
               "d2h_bytes_per_step": int(out_h.numel() * 4),
               "overlap": "step i+1's H2D copies on a second stream during step i (double-buffered device inputs)"}
        del bufs

    ms_per_step = elapsed_ms / args.steps
    pk = peaks()
    bpt = bytes_per_token_head(w.bits, w.transform)
    token_heads = n * w.Hkv
    dec_bytes = token_heads * bpt
    app_bytes = token_heads * (bpt + 2 * 2 * D)
    # mining: every vector read once per Lloyd iteration (K and V calls; the minimum for unfused Lloyd)
    mine_bytes = 2 * w.iters * n * w.Hkv * D * 2
    rooflines = {
        "decode_attention": {"bound": "hbm", "achieved": dec_bytes / (decode_ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "ms": decode_ms, "algorithmic_bytes": dec_bytes},
        "quantize_append": {"bound": "hbm", "achieved": app_bytes / (append_ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                            "unit": "GB/s", "ms": append_ms, "algorithmic_bytes": app_bytes},
        "mine_patterns": {"bound": "hbm", "achieved": mine_bytes / (mine_ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                          "unit": "GB/s", "ms": mine_ms, "algorithmic_bytes": mine_bytes},
    }
    traffic = dram_traffic(w.name, w.bits, w.B)
    for name, r in rooflines.items():
        r["traffic"] = traffic.get(name)
        r["frac"] = r["achieved"] / r["peak"]
    # The exact d_mm argmin by its definition costs 3 lane-ops (subtract, max, min) per channel and
    # pattern for K and for V; the kernel prunes it with exact bounds, so this is the rate at which
    # that definitional work gets done, against the fp32 lanes (128 per SM) at the sampled clock.
    sm_mhz = (clk or {}).get("sm_max_mhz") or 1965.0
    naive_ops = token_heads * 2 * w.P * D * 3
    alu_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * sm_mhz * 1e6
    rooflines["quantize_append"]["alu_naive_equivalent"] = {
        "lane_ops_per_token_head": 2 * w.P * D * 3, "achieved_tops": naive_ops / (append_ms * 1e-3) / 1e12,
        "peak_tops": alu_peak / 1e12, "frac": naive_ops / (append_ms * 1e-3) / alu_peak}
    dominant = max(rooflines, key=lambda kk: rooflines[kk]["ms"])
    dom = rooflines[dominant]
    roofline = {"bound": dom["bound"], "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
                "frac": dom["frac"], "traffic": dom["traffic"], "kernel": dominant, "peak_source": pk["source"]}
    tokens = B_total * w.S
    rec = {"workload": w.name, "bits": w.bits, "transform": bool(w.transform), "value": tokens / (ms_per_step * 1e-3),
           "unit": "KV-tokens/s", "ms_per_step": ms_per_step,
           "phases_ms": {"mine_patterns_KV": mine_ms, "quantize_append": append_ms, "decode_attention": decode_ms},
           "decode_kv_tokens_per_s": tokens / (decode_ms * 1e-3), "decode_hbm_gbs": rooflines["decode_attention"]["achieved"],
           "quant_append_gbs": rooflines["quantize_append"]["achieved"], "v_pattern_utilisation": utilisation,
           "roofline": roofline, "rooflines": rooflines,
           "gpu_launches": args.steps * launches_per_step(w)}
    del kd, vd, qd, kh, vh, qh, cache, ws_m, ws_d, ws_a
    torch.cuda.empty_cache()
    return rec, e2e, clk


def measure_decode_loop(w, args, dev, nsteps: int = 512, chunk: int = 64):
    """Long chain-of-thought decode: mine patterns on the 8192-token prefill (frozen after it),
    append the prefill, then decode steps -- kvq_decode_step, one launch that quantize-appends one
    token per sequence and runs decode attention with a new query.  Steps are captured `chunk` at a
    time in CUDA graphs and replayed (each replay appends `chunk` new tokens); the time per step is
    the median replay time / chunk.  Falls back to event-timed batches if capture is refused."""
    import numpy as np
    import torch

    import bit_kv_cache_26_b200 as kvq
    import synth

    warm = 2 * chunk
    total = w.S + nsteps + warm
    k, v = synth.gen_kv(w.with_(S=total))
    tdt = torch.bfloat16 if w.dtype == synth.BF16 else torch.float16
    kd = torch.from_numpy(np.ascontiguousarray(k).view(np.int16)).view(tdt).to(dev)
    vd = torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).view(tdt).to(dev)
    del k, v
    qs = torch.stack([torch.from_numpy(np.ascontiguousarray(synth.gen_q(w, step=t)).view(np.int16)).view(tdt)
                      for t in range(nsteps + warm)]).to(dev)
    cache = kvq.PagedKVCache(w.B, w.Hkv, total, w.bits, w.P, dtype=w.dtype, transform=w.transform, device=dev,
                             v_rho=kvq.kvq_v_rho_star(D, w.v_alpha))
    n = w.B * w.S
    pre_k, pre_v = kd[:, :w.S].contiguous(), vd[:, :w.S].contiguous()
    ws_m = kvq._alloc_aligned(kvq.kvq_mine_workspace_bytes(n, 1, w.Hkv, w.P, w.transform), dev)
    for x, pat, col in ((pre_k, cache.k_patterns, cache.k_colscale), (pre_v, cache.v_patterns, cache.v_colscale)):
        kvq.kvq_mine_patterns(x, w.dtype, n, 1, w.Hkv, w.Hkv * D, D, n * w.Hkv * D, w.P, w.iters, w.transform,
                              pat, col, None, ws_m)
    cache.append(pre_k, pre_v)
    del pre_k, pre_v
    steps_k = [kd[:, w.S + t].contiguous() for t in range(nsteps + warm)]
    steps_v = [vd[:, w.S + t].contiguous() for t in range(nsteps + warm)]
    ws_s = cache.step_workspace(w.Hq)
    out = torch.empty(w.B, w.Hq, D, device=dev)

    def run(t0, t1):
        for t in range(t0, t1):
            cache.step(steps_k[t], steps_v[t], qs[t], out, ws_s)

    run(0, chunk)  # warm-up outside any capture
    torch.cuda.synchronize()
    method = "cuda graph replay"
    us = []
    try:
        graphs = []
        for c0 in range(chunk, warm + nsteps, chunk):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph):
                run(c0, c0 + chunk)
            graphs.append(gph)
        # capture only records: seq_len has not moved; replay the chunks in order
        torch.cuda.synchronize()
        for i, gph in enumerate(graphs):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            gph.replay()
            e1.record()
            torch.cuda.synchronize()
            if i >= 1:
                us.append(1e3 * e0.elapsed_time(e1) / chunk)
        del graphs
    except Exception as exc:  # capture refused: time batches of eagerly launched steps instead
        method = f"event-timed batches ({type(exc).__name__} in capture)"
        torch.cuda.synchronize()
        cache.seq_len.fill_(w.S + chunk)
        us = []
        for c0 in range(chunk, warm + nsteps, chunk):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run(c0, c0 + chunk)
            e1.record()
            torch.cuda.synchronize()
            if c0 >= warm:
                us.append(1e3 * e0.elapsed_time(e1) / chunk)
    torch.cuda.synchronize()
    assert cache.read_status() == 0, "device status bits set"
    assert int(cache.seq_len.min()) == total, "every step appended its token"
    us.sort()
    med = us[len(us) // 2]
    ctx = w.S + warm + nsteps // 2
    pk = peaks()
    step_bytes = w.B * ctx * w.Hkv * bytes_per_token_head(w.bits, w.transform)
    rec = {"workload": w.name, "bits": w.bits, "metric": "us per decode step (1-token quantize-append + decode, one launch)",
           "us_per_step_median": med, "us_per_step_min": us[0], "us_per_step_max": us[-1],
           "steps_timed": len(us) * chunk, "timing": method, "context_tokens_mid": ctx, "launches_per_step": 1,
           "value": w.B * ctx / (med * 1e-6), "unit": "KV-tokens/s (decode, at the median step)",
           "roofline": {"bound": "hbm", "achieved": step_bytes / (med * 1e-6) / 1e9, "peak": pk["hbm_gbs"],
                        "unit": "GB/s", "frac": step_bytes / (med * 1e-6) / 1e9 / pk["hbm_gbs"], "traffic": None,
                        "kernel": "decode_mma_kernel (decode step)", "peak_source": pk["source"]}}
    del kd, vd, qs, cache, ws_m, ws_s, steps_k, steps_v
    torch.cuda.empty_cache()
    return rec


def cpu_baseline_step(w, ctx: int):
    """The oracle on one decode step of one (sequence, KV head) unit of the long-CoT workload:
    encode the new token against the frozen patterns and run decode attention over `ctx` tokens;
    scaled to every unit of the batch (us per step)."""
    import oracle
    import synth

    sw = w.with_(B=1, S=ctx)
    k, v = synth.gen_kv(sw, p1=ctx)
    Kf = synth.to_float(k[0, :, 0], w.dtype)
    Vf = synth.to_float(v[0, :, 0], w.dtype)
    MK, cK, _ = oracle.mine_set(Kf[:2048], w.P, w.iters, w.transform)
    MV, cV, _ = oracle.mine_set(Vf[:2048], w.P, w.iters, w.transform)
    e = oracle.encode(Kf, Vf, w.bits, MK, MV, cK, cV, v_rho=oracle.v_rho(w.v_alpha))
    Gq = w.Hq // w.Hkv
    qf = synth.to_float(synth.gen_q(sw)[0, :Gq], w.dtype)
    t0 = time.perf_counter()
    reps = 3
    for _ in range(reps):
        oracle.encode(Kf[-1:], Vf[-1:], w.bits, MK, MV, cK, cV, v_rho=oracle.v_rho(w.v_alpha))
        oracle.attention_unit(qf, Kf, e, MK, MV, cK, cV)
    dt = (time.perf_counter() - t0) / reps
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    us = dt * 1e6 * w.B * w.Hkv
    return {"value": us, "unit": "us per decode step", "cores": cores, "kind": "oracle",
            "sample": f"one (sequence, KV head) unit at {ctx} tokens ({dt * 1e3:.1f} ms: encode the new token, "
                      f"attention of {Gq} query heads), times the {w.B * w.Hkv} units of a step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--bits", type=int, default=2)
    ap.add_argument("--transform", type=int, default=0, choices=[0, 1],
                    help="the Hadamard + dual-axis pre-transform on the headline workload")
    ap.add_argument("--ref-heads", type=int, default=2, help="reference arm: KV heads per step (bounded sample)")
    ap.add_argument("--ref-seqs", type=int, default=24, help="reference arm: sequences per step (bounded sample)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle work in the headline's cpu_baseline sample (half that per configuration)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="headline workload only")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases of the same kernels, for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    import synth

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    base = synth.WORKLOADS[args.workload].with_(bits=args.bits, transform=args.transform)
    if args.batch:
        base = base.with_(B=args.batch)
    w = base
    shard = rank_shard(base, rank, world) if world > 1 else None
    rec, e2e, clk = measure_path(w, args, dev, world, rank, headline=True, shard=shard)

    per_config = []
    if world == 1 and not args.no_per_config and not args.batch:
        for name, kw in PER_CONFIG:
            wc = synth.WORKLOADS[name].with_(**kw)
            r, _, _ = measure_path(wc, args, dev, 1, 0, headline=False)
            if not args.no_cpu_baseline:
                r["cpu_baseline"], _ = cpu_baseline(wc, target_s=args.cpu_seconds / 2)
            per_config.append(r)
        wl = synth.WORKLOADS["long_cot_8k"]
        r = measure_decode_loop(wl, args, dev)
        if not args.no_cpu_baseline:
            r["cpu_baseline"] = cpu_baseline_step(wl, r["context_tokens_mid"])
        per_config.append(r)

    if rank == 0:
        line = {
            "metric": METRIC, "value": rec["value"], "unit": "KV-tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
            "scaling": "strong" if world > 1 else "weak",
            "vs_baseline": None, "dtype": "f32 (fp32 quantization, f64 mining distances, bf16 inputs)",
            "data": "synthetic (seeded Gaussian-mixture K/V with outlier channels and RoPE)",
            "config": workload_config(w, args),
            "phases_ms": rec["phases_ms"], "decode_kv_tokens_per_s": rec["decode_kv_tokens_per_s"],
            "decode_hbm_gbs": rec["decode_hbm_gbs"], "quant_append_gbs": rec["quant_append_gbs"],
            "v_pattern_utilisation": rec["v_pattern_utilisation"],
            "roofline": rec["roofline"], "rooflines": rec["rooflines"],
            "e2e": {"value": w.B * w.S / (e2e["ms"] / args.steps * 1e-3), "unit": "KV-tokens/s",
                    "h2d_bytes_per_step": e2e["h2d_bytes_per_step"], "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                    "overlap": e2e["overlap"]},
            "gpu_launches": rec["gpu_launches"],
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"], _ = cpu_baseline(w, target_s=args.cpu_seconds)
        if per_config:
            line["per_config"] = per_config
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
