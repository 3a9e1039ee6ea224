"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
ties the recorded DRAM traffic to the code it was captured on."""
import bench


def _src():
    with open(bench.KERNEL_SOURCES[0]) as fh:
        return fh.read()


def test_kernel_source_text_covers_the_kernel_and_its_launch_path():
    t = bench.kernel_source_text(_src())
    assert "kq_packed_kernel(const uint4" in t and "kq_fast_apply" in t and "mx_quantize_pairs" in t
    for head in bench.LAUNCH_FUNCS:
        assert head in t
    assert "norm_kq_rows_kernel" not in t and "mxf4_gemm_kernel" not in t


def test_hash_follows_the_kernel_not_unrelated_code():
    src = _src()
    base = bench.kernel_source_text(src)
    # an edit inside the dominant kernel or its launch path changes the text
    edited = src.replace("kq_fast_apply(p, st);", "kq_fast_apply(p, st); /* edit */", 1)
    assert bench.kernel_source_text(edited) != base
    launch = src.replace("Geometry pinned_geometry(int64_t M, int64_t nb, int64_t target_threads)\n{",
                         "Geometry pinned_geometry(int64_t M, int64_t nb, int64_t target_threads)\n{ /* edit */", 1)
    assert launch != src and bench.kernel_source_text(launch) != base
    # an edit in an unrelated kernel later in the file does not
    other = src.replace("norm_kq_rows_kernel(", "norm_kq_rows_kernel /* edit */ (", 1)
    assert other != src and bench.kernel_source_text(other) == base


def test_every_mode_is_offered_on_the_command_line():
    import subprocess
    import sys

    out = subprocess.run([sys.executable, bench.__file__, "--help"], capture_output=True, text=True, check=True).stdout
    for mode in ("step", "kernel", "sweep", "sqnr", "gemm", "compare"):
        assert mode in out
    for flag in ("--shapes", "--reps", "--kernels", "--launches"):
        assert flag in out


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the CPU oracle on a bounded sample of the
    same workload and prints one JSON line with the contract's keys (no GPU)."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, bench.__file__, "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, check=True, timeout=600)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]
