"""The benchmark's host-side arithmetic: the algorithmic bytes and flops its roofline divides
by, and the guard that drops a stale DRAM-traffic figure."""
import json
import os

import torch

import bench
import workloads


def test_decode_step_algorithmic_bytes_and_flops():
    w = workloads.WORKLOADS["v3_decode_b32_ctx4096"]
    a = bench.alg_step(w)
    tokens = 32 * 4096
    assert a["tokens"] == tokens
    assert a["cache_bytes"] == tokens * 1152                  # (512 + 64) bf16 per token
    # cache 151.0 MB + W_UK, W_UV 33.6 MB + queries 1.6 MB + output 1.0 MB
    assert a["bytes"] == tokens * 1152 + 2 * 128 * 128 * 512 * 2 + 32 * 128 * 192 * 2 + 32 * 128 * 128 * 2
    assert round(a["bytes"] / 1e6, 1) == 187.2
    # per attended token and head: 2 x 576 (scores) + 2 x 512 (P c) flops; plus the two absorptions
    assert a["attn_flops"] == tokens * 128 * (2 * 576 + 2 * 512)
    assert round(a["flops"] / 1e9, 1) == 37.6
    # the dominant kernel reads the cache and the absorbed and rotary queries once
    assert bench.alg_kernel_bytes("tc_flash_decode", w) == tokens * 1152 + 32 * 128 * 576 * 2
    # 2176 flops per attended token and head: 242 flop per cache byte, next to the measured
    # ridge of about 249 flop/B (1628.3 TFLOP/s over 6535.1 GB/s)
    f = bench.alg_kernel_flops("tc_flash_decode", w)
    assert f == tokens * 128 * 2176
    assert 240 < f / (tokens * 1152) < 243


def test_layer_and_prefill_steps_count_their_weights():
    lay = bench.alg_layer(workloads.WORKLOADS["v3_layer_b128_ctx8192"])
    # W_Q (352 MB) and W_O (235 MB) dominate the weights; the cache holds 128 x 8193 rows
    assert lay["bytes"] > 128 * 8193 * 1152 + 352e6 + 235e6
    pre = bench.alg_prefill(workloads.WORKLOADS["v2_prefill_b4_s4096"])
    assert pre["tokens"] == 4 * 4096
    assert 7.0e12 < pre["flops"] < 8.0e12


def test_multi_token_step_counts_the_window():
    w = workloads.WORKLOADS["v3_mtp_b32_ctx4096_q2"]
    a = bench.alg_multi(w)
    rows = 32 * (4096 + 2)
    assert a["tokens"] == rows and a["cache_bytes"] == rows * 1152
    # new token t attends to 4096 + t + 1 rows
    assert a["attn_flops"] == 32 * (4097 + 4098) * 128 * (2 * 576 + 2 * 512)
    inp = workloads.make_inputs(workloads.shrink(w, B=3, ctx=100, q_len=3))
    assert tuple(inp["q_nope"].shape) == (3, 3, 128, 128) and tuple(inp["q_rope"].shape) == (3, 3, 128, 64)
    assert inp["offsets"].tolist() == [0, 103, 206, 309]


def test_paged_layout_keeps_every_row():
    w = workloads.shrink(workloads.WORKLOADS["v3_mtp_b32_ctx4096_q2"], B=3, ctx=100, q_len=2)
    inp = workloads.make_inputs(w)
    pages, table, lens = bench.paged_layout(w, inp, 5)
    assert lens.tolist() == [102, 102, 102] and tuple(table.shape) == (3, 2)
    assert sorted(table.flatten().tolist()) == list(range(6))
    offs = inp["offsets"].tolist()
    for b in range(3):
        for t in (0, 63, 64, 101):
            assert bytes(pages[table[b, t // 64], t % 64].view(-1).view(torch.int16).numpy()) == \
                bytes(inp["cache"][offs[b] + t].view(torch.int16).numpy())


def test_traffic_figure_is_dropped_when_the_kernel_source_changed(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    digest = hashlib.sha256(b"kernel v1").hexdigest()
    (prof / "traffic.json").write_text(json.dumps({"tc_x": {"source": "k.cu", "sha256": digest,
                                                            "bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("tc_x") == 123
    src.write_text("kernel v2")
    assert bench.traffic_for("tc_x") is None
    assert bench.traffic_for("tc_other") is None


def test_cpu_baseline_runs_the_oracle_on_several_threads():
    """The CPU baseline's host logic: a fixed number of seeded units spread over two threads,
    each through the oracle, throughput scaled from the units to the full step."""
    w = workloads.shrink(workloads.WORKLOADS["v3_decode_b32_ctx4096"], B=2, ctx=64)
    inp = workloads.make_inputs(w)
    r = bench.time_oracle_units(w, inp, 0.0, min_units=6, max_units=6, threads=2)
    assert r["cores"] == 2 and r["kind"] == "oracle" and r["value"] > 0
    assert r["sample"].startswith("6 seeded (sequence, head) units")
    # a unit over its first 16 rows counts as 64 / 16 of a full unit
    s = bench.time_oracle_units(w, inp, 0.0, min_units=3, max_units=3, tokens=16)
    assert s["cores"] == 1 and "first 16 rows" in s["sample"]
    assert bench.host_cores() >= 1


def test_fp8_step_counts_656_bytes_per_token():
    w = workloads.WORKLOADS["v3_decode_fp8_b32_ctx4096"]
    a = bench.alg_step_fp8(w)
    tokens = 32 * 4096
    assert a["cache_bytes"] == tokens * 656
    assert a["bytes"] == tokens * 656 + 2 * 128 * 128 * 512 * 2 + 32 * 128 * 192 * 2 + 32 * 128 * 128 * 2
    assert a["flops"] == bench.alg_step(workloads.WORKLOADS["v3_decode_b32_ctx4096"])["flops"]
    assert bench.alg_kernel_bytes("tc_flash_decode_fp8", w) == tokens * 656 + 32 * 128 * 576 * 2
