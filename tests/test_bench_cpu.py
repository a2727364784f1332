"""Host logic of bench.py that needs no GPU: the kernel-source hash that keys
the committed ncu traffic captures, and the kernel names the launch counts
refer to."""
import numpy as np

import bench
import workloads


def test_source_hash_ignores_comments_and_whitespace():
    code = b"__global__ void k(int* p) {\n  p[0] = 1;  // store\n}\n"
    same = [
        b"// leading comment\n__global__ void k(int* p) {\n  p[0] = 1;\n}\n",
        b"__global__ void k(int* p) { /* block\n comment */ p[0] = 1; }",
        b"__global__   void k(int* p)\n{\n\n    p[0] = 1;\n}\n",
    ]
    h = bench.source_hash({"a.cuh": code})
    for s in same:
        assert bench.source_hash({"a.cuh": s}) == h


def test_source_hash_sees_code_and_file_changes():
    code = b"__global__ void k(int* p) { p[0] = 1; }"
    h = bench.source_hash({"a.cuh": code})
    assert bench.source_hash({"a.cuh": code.replace(b"1", b"2")}) != h
    assert bench.source_hash({"b.cuh": code}) != h
    assert bench.source_hash({"a.cuh": code, "b.cuh": b"int x;"}) != h
    # the order files are listed in does not matter
    two = {"a.cuh": code, "b.cuh": b"int x;"}
    assert bench.source_hash(dict(reversed(list(two.items())))) == bench.source_hash(two)


def test_kernel_source_hash_is_stable():
    assert bench.kernel_source_hash() == bench.kernel_source_hash()
    assert len(bench.kernel_source_hash()) == 16


def test_gemm_kernel_names():
    d = workloads.DenseInputs(a=None, b=None, M=64, N=4096, K=7168)
    assert bench.gemm_kernel_name("dense", d, False) == "fp8_gemm_kernel"
    p = workloads.DenseInputs(a=None, b=None, M=4096, N=7168, K=2048)
    assert bench.gemm_kernel_name("dense", p, True) == "fp8_gemm_mx_kernel"
    # thin shapes take the promoted swapped kernel for power-of-two scales too
    assert bench.gemm_kernel_name("dense", d, True) == "fp8_gemm_kernel"


def test_quantizer_cpu_sample_reports_bytes_per_second():
    inp = workloads.quant(M=64, K=256, seed=1)
    for ue8m0 in (False, True):
        r = bench.quant_cpu_sample(inp, 0.01, ue8m0)
        assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0 and r["cores"] >= 1
        rows = int(r["sample"].split()[0])
        assert 16 <= rows <= 64


def test_both_arms_describe_the_same_problem():
    """The reference arm and the GPU arm build `config` with one function: the
    same keys and values for the same workload and options."""
    import argparse
    args = argparse.Namespace(workload="contiguous_8x4096x7168", with_weight_quant=False)
    inp = workloads.contiguous(N=256, K=256, counts=[130, 0, 5], seed=3)
    a = bench.step_config(args, "contiguous", inp, 1, False)
    b = bench.step_config(args, "contiguous", inp, 1, False)
    assert a == b
    assert a["M_total"] == inp.M_total and a["M_valid"] == 135 and a["G"] == 3
    assert "l2" not in a and "launch" not in a  # how a step is timed lives in `method`
    d = workloads.DenseInputs(a=None, b=None, M=64, N=4096, K=7168)
    assert bench.step_config(args, "dense", d, 1, False)["M"] == 64


def test_default_workload_is_the_largest_single_gpu_config():
    import sys
    old = sys.argv
    try:
        sys.argv = ["bench.py"]
        args = bench.parse_args()
    finally:
        sys.argv = old
    assert args.workload == "contiguous_8x4096x7168" and args.scales == "fp32"


def test_peaks_used_records_both_denominators():
    d = bench.peaks_used({"hbm_gbs": 6549.1, "bf16_tflops": 1654.5,
                         "clocks_under_load": {"sm_mhz_median": 1192.0}}, "measured")
    assert d["fp8_tflops"] == 2 * 1654.5 and d["rated_fp8_tflops"] == 4500.0
    assert d["rated_hbm_gbs"] == 8000.0 and d["sm_mhz_median_when_measured"] == 1192.0
    assert d["source"] == "MEASURED_PEAKS.json"
    # the committed in-library tensor-core rate rides along as a third denominator
    assert d["fp8_mma_in_library_tflops"] == bench.fp8_mma_rate() > 0


def test_peak_expected_matches_the_declared_sums():
    """The tensor-core rate kernel's check value against the declaration's
    definition summed element by element over one 128-wide K block."""
    import bench
    iters = 3
    want = np.zeros((128, 256))
    for m in (0, 1, 17, 127):
        for n in (0, 5, 16, 255):
            s = 0
            for k in range(128):
                j = k % 16
                s += ((2 * m + 3 * j) % 5 - 2) * ((3 * n + 2 * j + n // 16) % 5 - 2)
            want[m, n] = iters * s
            assert bench.peak_expected(iters)[m, n] == want[m, n]
    assert np.abs(bench.peak_expected(32768)).max() < 2 ** 24  # exact in fp32


def test_peak_reference_arm_is_unavailable(capsys):
    import json
    import sys

    import bench
    argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--workload", "peak_fp8_mma_16384"]
    try:
        bench.main()
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and "unavailable" in line


def test_other_configs_run_each_named_config_device_timed_only(monkeypatch):
    """The default run's extra configurations: every one of OTHER_CONFIGS in
    order, without the CPU baseline or the end-to-end leg, summarised from the
    same fields a full line carries."""
    import argparse
    seen = []

    def fake_run_ours(a, rank, world, local_rank):
        seen.append((a.workload, a.no_cpu_baseline, a.no_e2e, a.steps))
        return {"value": 1.0, "unit": "TFLOP/s", "ms_per_step": 0.5, "clocks": {"sm_mhz": 1965.0},
                "roofline": {"bound": "tensor", "achieved": 2.0, "peak": 3.0, "unit": "TFLOP/s",
                             "frac": 0.6, "frac_rated": 0.4, "kernel_ms": 0.4, "traffic": None,
                             "kernel": "k"}}
    monkeypatch.setattr(bench, "run_ours", fake_run_ours)
    args = argparse.Namespace(workload=bench.DEFAULT_WORKLOAD, no_cpu_baseline=False, no_e2e=False, steps=7)
    res = bench.run_other_configs(args, 0, 1, 0)
    assert [s[0] for s in seen] == list(bench.OTHER_CONFIGS)
    assert all(s[1] and s[2] and s[3] == 7 for s in seen)
    assert args.workload == bench.DEFAULT_WORKLOAD and not args.no_e2e  # the caller's args untouched
    assert [r["workload"] for r in res] == list(bench.OTHER_CONFIGS)
    assert res[0]["kernel_ms"] == 0.4 and res[0]["roofline"]["frac"] == 0.6
    assert "kernel" not in res[0]["roofline"]


def test_ep_reference_arm_is_unavailable(capsys):
    import json
    import sys
    argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--workload", "ep_32x512x8_4096x7168"]
    try:
        bench.main()
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and "unavailable" in line
