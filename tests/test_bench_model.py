"""bench.py's algorithmic byte counts (the roofline numerator) written out by hand
for the 8192-token workload, and the lookup of recorded DRAM traffic."""
import json

import bench
import workloads


def test_byte_model_of_the_8192_token_step():
    wl = workloads.BY_NAME["uniform_bs8192_h1536_k8_e64"]
    bs, k, h, e, E = 8192, 8, 1536, 2, 64
    pairs, row, r = bs * k, h * e, bs * k  # every pair routed: R = BS * K
    m = bench.byte_model(wl, r, 0)
    # ids, the slot maps both ways, counts and prefix (E + E + 1 int32)
    assert m["layout"] == 4 * pairs + 4 * (wl.a_capacity + pairs) + 4 * (2 * E + 1)
    # x once, the pair -> slot map, R rows written
    assert m["permute"] == bs * row + 4 * pairs + r * row
    # R rows read, weights + slot map, one output row per token
    assert m["combine_fwd"] == r * row + 4 * pairs + 4 * pairs + bs * row
    # grad_out, rows in and grad rows out, weights + slot map + grad_w
    assert m["combine_bwd"] == bs * row + 2 * r * row + 12 * pairs
    # grad rows in, grad_x out, slot map
    assert m["dispatch_bwd"] == r * row + bs * row + 4 * pairs
    assert sum(m.values()) == 1109918212


def test_byte_model_of_the_int8_variants():
    wl = workloads.BY_NAME["special_int8_bs8192_h2048_k8_n70"]
    bs, h, E, r = wl.bs, wl.h, wl.num_experts, 59867
    plain = bench.byte_model(wl, r, 0)["permute"]
    assert plain == bs * h * 2 + 4 * bs * wl.k + r * h + 4 * r  # codes + one scale per slot
    smooth = bench.byte_model(wl.scaled(smooth=True), r, 0)["permute"]
    # the smooth factors once, a pair and an expert id per slot instead of the pair map
    assert smooth == bs * h * 2 + 4 * E * h + 8 * r + r * h + 4 * r


def test_recorded_traffic_is_used_only_for_current_sources(tmp_path, monkeypatch):
    kernel = "combine_bwd"
    rec = {"w": {kernel: {"dram_bytes_per_launch": 123.0,
                          "source_hash": bench.kernel_source_hash(kernel)}},
           "stale": {kernel: {"dram_bytes_per_launch": 456.0, "source_hash": "0" * 16}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the sources under the fake root do not exist: fix the hash of "current" sources
    monkeypatch.setattr(bench, "kernel_source_hash",
                        lambda k: rec["w"][kernel]["source_hash"])
    assert bench.profiled_traffic(kernel, "w") == 123.0
    assert bench.profiled_traffic(kernel, "stale") is None
    assert bench.profiled_traffic(kernel, "missing") is None
