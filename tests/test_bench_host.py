"""Host logic of bench.py that needs no GPU."""


def test_kernel_hash_ignores_comments():
    """The profile key (hash of the device-code sources) changes with code, not comments."""
    import bench
    a = "int f(int x) {  // doubles x\n    return 2 * x; /* twice */\n}\n"
    b = "// header\nint f(int x) {\n\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n    return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_reference_arm_line_on_cpu():
    """`bench.py --impl reference` times the CPU oracle and prints the contract's JSON line:
    the same metric and unit, an e2e object with no host-device bytes, and a cpu_baseline
    of kind "oracle" (it needs no GPU)."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    import bench
    assert line["metric"] == bench.METRIC


def test_oracle_pinning_restores_affinity():
    """The CPU baseline runs pinned to one host core and leaves the process's
    affinity as it found it."""
    import os
    import bench
    before = os.sched_getaffinity(0)
    with bench.pinned_to_one_core() as pin:
        assert os.sched_getaffinity(0) == {pin.core}
        assert pin.core in before
    assert os.sched_getaffinity(0) == before


def test_kernel_figures_mean_and_median():
    import bench
    f = bench.kernel_figures([1.0, 2.0, 6.0], 3e9, 1000.0)
    assert abs(f["ms"] - 3.0) < 1e-12 and f["ms_median"] == 2.0
    assert abs(f["gbs"] - 1000.0) < 1e-9 and abs(f["frac"] - 1.0) < 1e-12
    assert abs(f["frac_median"] - 1.5) < 1e-12
