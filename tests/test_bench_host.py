"""Host-side logic of bench.py, on CPU: the algorithmic byte counts behind the HBM
roofline entries, the choice of the bf16 peak by the length of the timed region,
the config dict both arms print, and the traffic record's source hash."""
import json
import os

import bench

N, K, G_SIZE = 4096, 4096, 64
NG = N * (K // G_SIZE)


def test_code_bytes_per_packing():
    assert bench.code_bytes(N, K, 2) == N * K // 4
    assert bench.code_bytes(N, K, 4) == N * K // 2
    assert bench.code_bytes(N, K, 3) == N * K  # 3-bit codes are stored one per byte


def test_hbm_bytes_read_and_write_every_tensor_once():
    w = N * K * 2  # bf16 W (and W-hat)
    assert bench.hbm_bytes("init", N, K, 2, G_SIZE) == w + 8 * NG                      # W; s, z fp32
    assert bench.hbm_bytes("pack", N, K, 2, G_SIZE) == w + 8 * NG + N * K // 4 + NG    # + codes, zq
    assert bench.hbm_bytes("prepass", N, K, 2, G_SIZE) == 2 * w + 8 * NG              # W in, W-hat out
    assert bench.hbm_bytes("dequant", N, K, 2, G_SIZE) == N * K // 4 + 5 * NG + w     # codes, zq, s; W-hat
    assert bench.hbm_bytes("init", N, K, 2, G_SIZE, wbytes=4) == 2 * w + 8 * NG


def test_peak_follows_the_length_of_the_timed_region():
    peaks = {"bf16_tflops": 1586.2, "bf16_tflops_sustained": 1372.0, "source": "measured"}
    p, kind = bench.choose_gemm_peak(peaks, 0.015)
    assert p == 1586.2 and "burst" in kind
    p, kind = bench.choose_gemm_peak(peaks, 1.7)
    assert p == 1372.0 and "sustained" in kind


def test_config_dict_is_the_workloads_and_the_same_for_both_arms():
    c1 = bench.bench_config(1)
    assert c1["M"] == c1["N"] == c1["K"] == 4096 and c1["bits"] == 2 and c1["group"] == 64
    assert c1["flops_per_step"] == 12 * 4096 ** 3
    assert c1["step"].split("+") == bench.PHASES and bench.DOMINANT in bench.PHASES
    assert c1["parallelism"] == "single-gpu" and bench.bench_config(8)["parallelism"] == "dp8"
    assert bench.bench_config(1) == c1  # deterministic: the reference arm prints this same dict


def test_traffic_record_is_keyed_by_the_kernel_sources():
    path = os.path.join(bench.ROOT, "profiles", "gemm_bwd_grouped_fused_ste_llama2-7b-q_proj_traffic.json")
    rec = json.load(open(path))
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    # used only while the sources hash to the recorded value
    expected = rec["dram_bytes_per_launch"] if rec["kernel_source_hash"] == bench.kernel_source_hash() else None
    assert bench.load_traffic() == expected
