"""bench.py's host arithmetic (no GPU): the roofline objects and the stored ncu
figures' source keys."""
import bench


def test_tensor_roofline_units_and_peak():
    peaks = {"hbm_gbs": 6556.2, "bf16_tflops": 1613.7, "bf16_tflops_sustained": 1342.7, "source": "measured"}
    # 2 * 4096 * 4096 * 11008 multiply-adds in 0.5 ms: 1.4777e18 / 5e-4 = 1477.5 TFLOP/s (int8 ops)
    r = bench.tensor_roofline(2 * 4096 * 4096 * 11008, 0.5, peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - 2 * 2 * 4096 * 4096 * 11008 / 5e-4 / 1e12) < 0.1
    assert r["peak"] == round(2 * 1613.7, 1)                 # int8 dense = 2 x bf16 dense, burst
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    s = bench.tensor_roofline(2 * 4096 * 4096 * 11008, 0.5, peaks, burst=False)
    assert s["peak"] == round(2 * 1342.7, 1) and "sustained" in s["peak_source"]
    fb = bench.tensor_roofline(1, 1.0, {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                                        "bf16_tflops_sustained": 1400.0, "source": "fallback"})
    assert fb["peak"] == 3180.0 and fb["peak_source"].startswith("of fallback")


def test_hbm_roofline_and_replicas():
    peaks = {"hbm_gbs": 6556.2, "bf16_tflops": 1613.7, "bf16_tflops_sustained": 1342.7, "source": "measured"}
    r = bench.hbm_roofline(7_079_424 + 4 * (2560 + 6912) * 2, 0.002, peaks)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - (7_079_424 + 75_776) / 2e-6 / 1e9) < 0.1
    assert abs(r["frac"] - r["achieved"] / 6556.2) < 1e-4
    l2 = 126 * 2 ** 20
    R = bench.replicas_for(7_155_200, l2)
    assert R * 7_155_200 >= 4 * l2 and (R - 1) * 7_155_200 < 4 * l2
    assert bench.replicas_for(10 ** 10, l2) == 2


def test_time_graph_counts_exactly_the_requested_steps():
    """time_graph runs exactly `steps` issues after `warmup` (full graph replays
    plus one graph of the remainder), on any replica count."""
    calls = []

    class FakeGraph:
        def __init__(self):
            self.fns = []

        def replay(self):
            for f in self.fns:
                f()

    class FakeTorch:
        class cuda:
            _cur = None

            @staticmethod
            def CUDAGraph():
                return FakeGraph()

            class graph:
                def __init__(self, g, stream=None):
                    self.g = g

                def __enter__(self):
                    FakeTorch.cuda._cur = self.g

                def __exit__(self, *a):
                    FakeTorch.cuda._cur = None

            class stream:
                def __init__(self, s):
                    pass

                def __enter__(self):
                    return self

                def __exit__(self, *a):
                    pass

            class Event:
                def __init__(self, enable_timing=False):
                    pass

                def record(self, s=None):
                    calls.append("event")

                def elapsed_time(self, other):
                    return 1.0

            @staticmethod
            def synchronize():
                pass

    def make(i):
        def f():
            if FakeTorch.cuda._cur is not None:
                FakeTorch.cuda._cur.fns.append(lambda: calls.append(i))
        return f
    fns = [make(i) for i in range(7)]
    bench.time_graph(FakeTorch, None, fns, 23, 5)
    ev = [k for k, c in enumerate(calls) if c == "event"]
    timed = calls[ev[0] + 1:ev[1]]
    assert len(timed) == 23 and timed[:7] == list(range(7)) and timed[21:] == [0, 1]
    assert len(calls[:ev[0]]) == 7 + 5


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


def test_cpu_run_splits_rows_over_processes():
    """The oracle baseline's process pool (spawn): two processes together do
    every row of the tiny workload once per step."""
    gmacs, reps, dt = bench.cpu_run(1, 2, 0.2)
    assert gmacs > 0 and reps >= 1 and dt >= 0.2
    prepared = bench.oracle_prepare(1, (0.0, 1.0))
    assert bench.oracle_linear_step(prepared) == 8 * 256 * 128
    half = bench.oracle_prepare(1, (0.0, 0.5))
    assert bench.oracle_linear_step(half) == 8 * 128 * 128
