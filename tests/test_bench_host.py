"""bench.py's host arithmetic (no GPU): the roofline objects and the stored ncu
figures' source keys."""
import bench


def test_tensor_roofline_units_and_peak():
    peaks = {"hbm_gbs": 6556.2, "bf16_tflops": 1613.7, "bf16_tflops_sustained": 1342.7, "source": "measured"}
    # 2 * 4096 * 4096 * 11008 multiply-adds in 0.5 ms: 1.4777e18 / 5e-4 = 1477.5 TFLOP/s (int8 ops)
    r = bench.tensor_roofline(2 * 4096 * 4096 * 11008, 0.5, peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 2 * 2 * 4096 * 4096 * 11008 / 5e-4 / 1e12) < 0.1
    assert r["peak"] == round(2 * 1342.7, 1)                 # int8 dense = 2 x bf16 dense
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    fb = bench.tensor_roofline(1, 1.0, {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                                        "bf16_tflops_sustained": 1400.0, "source": "fallback"})
    assert fb["peak"] == 2800.0 and fb["peak_source"].startswith("fallback")


def test_measured_peaks_has_the_sustained_rate():
    p = bench.measured_peaks()
    assert p["bf16_tflops_sustained"] > 0 and p["hbm_gbs"] > 0


def test_kernel_source_hash_is_scoped():
    # the wquant kernel's key ignores host code that does not name it, the
    # whole-library key does not
    assert bench.kernel_source_hash("wquant_kernel") != bench.kernel_source_hash()
    assert bench.kernel_source_hash("no_such_kernel") == bench.kernel_source_hash()
    assert len(bench.kernel_source_hash("wquant_kernel")) == 16


def test_algorithmic_bytes():
    N, K, M = 6912, 2560, 1
    packed = N * -(-K // 5)
    assert bench.algorithmic_bytes("wquant", N, K, 0, 1) == 4 * N * K + packed
    assert bench.algorithmic_bytes("linear", N, K, M, 1) == packed + 4 * M * K + 4 * M * N
    assert bench.algorithmic_bytes("forward", N, K, M, 1) == 4 * N * K + packed + 4 * M * K + 4 * M * N
    assert bench.algorithmic_bytes("linear", N, K, M, 0) == N * K + 4 * M * K + 4 * M * N
