"""Host-side logic without a GPU: the parity comparator's acceptance rules and
the benchmark's clock-sample parsing and traffic-record bookkeeping."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from tests import parity  # noqa: E402


def row(w):
    w = np.asarray(w, dtype=np.float64)
    return w / w.sum()


def test_equal_sets_pass_without_tolerance():
    ok, tol, _ = parity.compare_row([0, 3], [0, 3], row([5, 1, 1, 4]), [0.5, 0.3, 0.8], 0.75, 3)
    assert ok and tol == 0


def test_near_cut_swap_is_tolerated_and_counted():
    w = row([0.300000, 0.3000001, 0.1, 0.2999999])
    # oracle kept block 1 (score just above block 0's); the GPU kept block 0
    info = [w[1], w[3], w[3] + w[1]]
    ok, tol, _ = parity.compare_row([0, 3], [1, 3], w, info, 0.5, 3)
    assert ok and tol == 2


def test_far_mismatch_is_rejected():
    w = row([0.5, 0.05, 0.05, 0.4])
    info = [w[0], w[3], w[3] + w[0]]
    ok, _, msg = parity.compare_row([1, 3], [0, 3], w, info, 0.8, 3)
    assert not ok and "differs" in msg


def test_missing_diagonal_and_unsorted_lists_are_rejected():
    w = row([1, 1, 1])
    assert not parity.compare_row([0, 1], [0, 1, 2], w, [-1, 1, 1], 0.5, 2)[0]
    assert not parity.compare_row([2, 0], [0, 2], w, [-1, 1, 1], 0.5, 2)[0]


def test_gamma_one_requires_the_full_row():
    w = row([1, 1, 1])
    assert not parity.compare_row([0, 2], [0, 1, 2], w, [-1, 1, 1], 1.0, 2)[0]
    assert parity.compare_row([0, 1, 2], [0, 1, 2], w, [-1, 1, 1], 1.0, 2)[0]


def test_one_extra_block_allowed_only_when_oracle_barely_crossed_gamma():
    w = row([0.2, 0.1, 0.7])
    # oracle: diag 0.7 + block 0 0.2 = 0.9 reaches gamma exactly; the GPU took block 1 too
    info = [w[0], w[2], w[2] + w[0]]
    assert parity.compare_row([0, 1, 2], [0, 2], w, info, 0.9, 2)[0]
    assert not parity.compare_row([0, 1, 2], [0, 2], w, info, 0.85, 2)[0]


def test_clock_sampler_parses_reasons_and_median():
    import bench
    cs = bench.ClockSampler(0)
    cs.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    cs.lines = ["1800, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
                "1750, 1965, 950.2, 0x4, Not Active, Not Active, Not Active, Active",
                "1900, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
                "garbage"]
    out = cs.stop()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965 and out["reasons"] == ["sw_power_cap"]


def test_traffic_record_is_dropped_when_the_kernel_source_changes(tmp_path, monkeypatch):
    import bench
    rec = json.load(open(os.path.join(ROOT, "profiles", "attn_traffic.json")))
    assert set(rec) >= {"dram_bytes_per_launch", "kernel_src_sha256", "command"}
    fake = tmp_path / "attn.cuh"
    fake.write_text("// another kernel\n")
    monkeypatch.setattr(bench, "ATTN_SRC", str(fake))
    assert bench.attn_traffic_record() is None


def test_attention_peak_for_mixed_int8():
    import bench
    assert bench.attention_peak(1400.0) == 1400.0
    # W8A8: half the FLOPs at the int8 peak and half at the bf16 peak
    F, P, P8 = 1.0e15, 1400.0e12, 2600.0e12
    t = (F / 2) / P8 + (F / 2) / P
    assert abs(bench.attention_peak(1400.0, 2600.0) * 1e12 - F / t) < 1e-6 * P
    # int8 at exactly 2x bf16: 0.75 F / P, an effective peak of 4/3 P
    assert abs(bench.attention_peak(1400.0, 2800.0) - 1400.0 * 4.0 / 3.0) < 1e-9


def test_oracle_sample_extrapolates_items_to_the_layer():
    """The CPU baseline's sample: per-item thread CPU times scaled to every
    head and tile of the layer, divided over the threads used."""
    import bench
    from dynamic_block_sparse_last_b200 import synth
    from oracle import oracle as orc
    w = synth.Workload("t", S=512, Hq=4, Hkv=2, b=128, seed=0)
    x = synth.make_inputs(w)
    P = orc.OracleProblem(x["q"], x["k"], x["v"], w.b)
    res = bench.oracle_sample(w, P, 3, heads=2, tiles=6, threads=3)
    assert res["threads"] == 3 and res["layer_s"] > 0
    assert abs(res["layer_s"] * 3 - res["layer_cpu_s"]) < 1e-9
    lo, med, hi = res["spread_min_median_max"]["tile_s"]
    assert 0 <= lo <= med <= hi
    assert "extrapolated" in res["desc"]


def test_index_pass_floors():
    import bench
    # S = 2b: the last block's rows see b+1 .. 2b causal keys, sum = b(3b+1)/2 per head
    hbm, n_exp, mufu = bench.index_pass_floors(256, 2, 128, 6_550_000_000, 6550.0, 148, 1000.0)
    assert n_exp == 2 * (128 * (3 * 128 + 1) // 2)
    assert abs(hbm - 1.0) < 1e-12
    assert abs(mufu - n_exp / (16 * 148 * 1e9) * 1e3) < 1e-15
    # a partial last block of 3 rows: keys S-2, S-1, S
    _, n_exp, _ = bench.index_pass_floors(259, 1, 128, 1, 1.0, 1, 1.0)
    assert n_exp == 257 + 258 + 259


def csr(rows_per_head):
    rp, col = [0], []
    for rows in rows_per_head:
        for r in rows:
            col += r
            rp.append(len(col))
    return np.array(rp), np.array(col)


def test_computed_chunk_tiles():
    import bench
    # b = 128, S = 384, one head: rows [0], [0,1], [1,2] -> tiles compute 1 + 2 + 2 chunks
    rp, col = csr([[[0], [0, 1], [1, 2]]])
    assert bench.computed_chunk_tiles(rp, col, 1, 384, 128) == 5
    # b = 256, S = 512: block 0 = tiles 0,1, block 1 = tiles 2,3; lists [0], [0, 1]
    rp, col = csr([[[0], [0, 1]]])
    assert bench.computed_chunk_tiles(rp, col, 1, 512, 256) == 1 + 2 + 3 + 4
    # b = 64, S = 256: blocks 0..3, tile 0 = blocks 0,1, tile 1 = blocks 2,3
    # lists: [0], [1], [0, 2], [3]: tile 0 -> chunks {0}; tile 1 -> chunks {0, 1}
    rp, col = csr([[[0], [1], [0, 2], [3]]])
    assert bench.computed_chunk_tiles(rp, col, 1, 256, 64) == 1 + 2
    # b = 64 with a last tile holding one query block (S = 192: blocks 0..2)
    rp, col = csr([[[0], [0, 1], [2]]])
    assert bench.computed_chunk_tiles(rp, col, 1, 192, 64) == 1 + 1


def test_kernels_per_step_counts_the_tensor_core_logits_split():
    """Six launches per layer step, two more (the tf32 operand splits) where the
    q-bar . k-bar logits run on the tensor cores (n >= 640 blocks)."""
    import bench
    assert bench.kernels_per_step(131072, 128) == 8   # n = 1024
    assert bench.kernels_per_step(131072, 256) == 6   # n = 512
    assert bench.kernels_per_step(32768, 128) == 6    # n = 256
    assert bench.kernels_per_step(81920, 128) == 8    # n = 640, the switch
    assert bench.kernels_per_step(81792, 128) == 6    # n = 639


def test_load_peaks_reads_the_measured_file_and_falls_back(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops_sustained"] == 1400.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6550, "bf16_tflops": 1644.9, "bf16_tflops_sustained": 1403.3, "other": [1]}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6550.0 and p["bf16_tflops_sustained"] == 1403.3
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6550, "bf16_tflops": 1644.9}))
    assert bench.load_peaks()["bf16_tflops_sustained"] == 1644.9   # no sustained figure: the burst one
    for bad in ('{"hbm_gbs": {"value": 6550}, "bf16_tflops": 1644.9}', '{"bf16_tflops": 1}', 'not json',
                '{"hbm_gbs": 0, "bf16_tflops": 1644.9}'):
        (tmp_path / "MEASURED_PEAKS.json").write_text(bad)
        p = bench.load_peaks()
        assert p["source"].startswith("fallback") and p["hbm_gbs"] == 6650.0, bad
