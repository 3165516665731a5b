"""The benchmark's roofline arithmetic, against values worked out by hand.

Per (token, head), with chunk size C = 32 and head size d = 128: the whole method does
6 d^2 + 10 C d = 139,264 flops, the state-dependent part 6 d^2 + 2 C d = 106,496 and the chunk-parallel
part 8 C d = 32,768 (the two add up to the whole). A prefill of T = 4096 tokens and 32 heads moves
4 T H d bf16 values (q, k, v, out), 2 T H fp32 gates and one fp32 state of d x d per head:
137,363,456 bytes. With the 3xTF32 split, 3 x 139,264 x 4096 x 32 = 54.76 GFLOP take 48.67 us at the
nominal 1.125 PFLOP/s TF32 peak, while the bytes take 17.17 us at 8 TB/s: a tensor-bound roofline.
"""
import math

import bench

PEAKS = dict(hbm_gbs=6532.0, bf16_tflops=1656.9, bf16_tflops_sustained=1400.0, sm_max_mhz=1965.0,
             source="measured")


def test_flop_counts_per_token_head():
    assert bench.flops_whole(128) == 139264
    assert bench.flops_scan(128) == 106496
    assert bench.flops_prep(128) == 32768
    for d in (64, 128):
        assert bench.flops_scan(d) + bench.flops_prep(d) == bench.flops_whole(d)


def test_api_bytes_of_the_4k_prefill():
    assert bench.prefill_api_bytes(4096, 32, 128, 1, False) == 137363456
    # a resumed call also reads the initial states
    assert bench.prefill_api_bytes(4096, 32, 128, 1, True) - 137363456 == 32 * 128 * 128 * 4


def test_method_roofline_at_nominal_and_measured_peaks():
    r = bench.method_roofline_of(4096, 32, 128, 1, False, call_ms=0.2291, peaks=PEAKS)
    nom = r["nominal_peaks"]
    assert nom["bound"].startswith("tensor")
    assert math.isclose(nom["roofline_us"], 3 * 139264 * 4096 * 32 / 1.125e15 * 1e6, rel_tol=1e-12)
    assert math.isclose(nom["roofline_us"], 48.67, abs_tol=0.01)
    meas = r["measured_peaks"]
    # TF32 from the measured bf16 GEMM: 1656.9 x 1.1 / 2.25 = 810.0 TFLOP/s
    assert math.isclose(meas["tf32_peak_tflops"], 810.04, abs_tol=0.01)
    assert math.isclose(meas["roofline_us"], 67.6, abs_tol=0.05)
    assert math.isclose(meas["frac"], meas["roofline_us"] / 229.1, rel_tol=1e-9)


def test_peaks_of_each_bound():
    tf32, unit, _ = bench.peak_for("tensor", PEAKS)
    assert unit == "TFLOP/s" and math.isclose(tf32, 1656.9 * 1.1 / 2.25)
    alu, _, _ = bench.peak_for("alu", PEAKS)
    assert math.isclose(alu, 148 * 128 * 2 * 1965e6 / 1e12)      # 74.4 TFLOP/s of fp32 FMA
    hbm, unit, _ = bench.peak_for("hbm", PEAKS)
    assert unit == "GB/s" and hbm == 6532.0


def test_job_throughput_counts_every_rank():
    # 4096 tokens per rank and step, 10 steps, 2 ranks, slowest rank 20 ms
    assert math.isclose(bench.job_throughput(4096, 10, 2, 20.0), 4096 * 2 * 10 / 0.020)
