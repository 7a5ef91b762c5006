"""Host-side pieces of bench.py, no GPU: the algorithmic byte counts the rooflines divide by,
the per-digest lookup of the ncu DRAM bytes, and the launch count a step claims."""
import bench
import synth


def test_bytes_per_token_head():
    # per (token, KV head): 2-bit K+V codes 64 B, fp32 scale/zero 64 B, two u8 indices; the
    # bulk append also reads the 512 B of bf16 K and V (642 B at 2-bit, 706 B at 4-bit)
    assert bench.bytes_per_token_head(2, 0) == 130
    assert bench.bytes_per_token_head(2, 0) + 512 == 642
    assert bench.bytes_per_token_head(4, 0) + 512 == 706
    assert bench.bytes_per_token_head(2, 1) == 138  # + fp32 row factors of K and V


def test_dram_traffic_lookup(monkeypatch):
    rows = [line.split() for line in open(bench.os.path.join(bench.ROOT, "profiles", "dram_traffic.txt"))
            if not line.startswith("#") and line.strip()]
    assert rows, "no DRAM rows"
    digest, wl, bits, batch = rows[0][0], rows[0][1], int(rows[0][2]), int(rows[0][3])
    monkeypatch.setattr(bench, "source_digest", lambda: digest)
    got = bench.dram_traffic(wl, bits, batch)
    want = {r[4]: float(r[5]) for r in rows if r[0] == digest and r[1] == wl and int(r[2]) == bits and int(r[3]) == batch}
    assert got == want and set(got) == {"mine_patterns", "quantize_append", "decode_attention"}
    monkeypatch.setattr(bench, "source_digest", lambda: "0" * 16)
    assert bench.dram_traffic(wl, bits, batch) == {}


def test_launches_per_step():
    W = synth.WORKLOADS
    # bf16, P <= 128: per mining call init + 4 x (assignment, fix-up, cluster sums, update)
    assert bench.launches_per_step(W["breadth_256x16k"]) == 2 * 17 + 4
    # pre-transform: the mma.sync assignment (no fix-up) and 8 fit / apply launches
    assert bench.launches_per_step(W["qwen25_7b_128k"].with_(transform=1)) == 2 * (1 + 3 * 4 + 8) + 4
