"""Host-side logic of bench.py, without a GPU: the
source-text hash that ties the ncu traffic figure to the kernel it was
measured on, the parsing of the nvidia-smi clock samples, the algorithmic
bytes and ops per row, and the sweep definitions."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def test_function_text_finds_definitions_not_calls():
    b = _bench()
    src = """
int helper(int a);

// the kernel
template <typename T>
__global__ void kern(const T *x) {
  if (x) { helper(1); }
}

void launch() { kern<float><<<1, 1>>>(nullptr); }
"""
    t = b.function_text(src, "kern")
    assert t.startswith("// the kernel") and t.rstrip().endswith("}")
    assert "launch()" not in t
    assert b.function_text(src, "launch").startswith("void launch()")


def test_traffic_is_reported_only_for_the_measured_source(monkeypatch):
    b = _bench()
    entry = dict(b.TRAFFIC["absmax_cols_kernel"])
    current = b.src_hash(entry["source"], entry["functions"])
    monkeypatch.setitem(b.TRAFFIC, "absmax_cols_kernel", dict(entry, sha=current))
    assert b.traffic_for("absmax_cols_kernel", 1e9) == int(round(entry["ratio"] * 1e9))
    monkeypatch.setitem(b.TRAFFIC, "absmax_cols_kernel", dict(entry, sha="0" * 16))
    assert b.traffic_for("absmax_cols_kernel", 1e9) is None
    assert b.traffic_for("no_such_kernel", 1e9) is None


def test_clock_summary_keeps_this_gpu_and_collects_reasons():
    b = _bench()
    c = b.ClockSampler("0000:1B:00.0")
    row = lambda bus, mhz, pc: [bus, str(mhz), "1965", "500.0", "0x4", "Not Active", "Not Active", "Not Active", pc]
    c.rows = [row("00000000:1B:00.0", 1965, "Active"), row("00000000:1B:00.0", 1900, "Not Active"),
              row("00000000:3A:00.0", 600, "Not Active")]
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1932.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert b.ClockSampler(None).summary()["samples"] == 0


def test_row_work_counts_the_algorithmic_bytes():
    # one OPT-shaped linear: the per-row bytes and ops the bench divides by
    b = _bench()

    class L:
        M, K, N = 2048, 4096, 12288
        calib = type("T", (), {"shape": (65536, 4096)})()

    w = b.row_work([L])
    assert w["calib"] == 65536 * 4096 * 2 + 8 * 4096
    assert w["weight"] == 2 * 12288 * 4096 * 2 + 12288 * 4096 + 4 * 12288 + 16 * 4096  # 2 reads + int8 write
    assert w["act"] == 2048 * 4096 * 3 + 4 * 2048 + 4 * 4096  # 2 B read + 1 B write per element
    assert w["linear_ops"] == 2 * 2048 * 12288 * 4096


def test_profile_sweeps_name_known_ops():
    pc = _bench()
    known = {"calib", "weight", "act", "linear", "rmsnorm", "layernorm", "static", "act8", "weight8", "linear8",
             "rot"}
    for name, cases in pc.sweeps().items():
        assert cases, name
        for op, M, K, N, dt in cases:
            assert op in known, (name, op)
            assert dt in pc.DT and K % 16 == 0, (name, op, K, dt)
            if op == "rot":
                assert N & (N - 1) == 0 and K % N == 0, (name, K, N)


def test_both_arms_share_the_config_and_the_reference_is_labelled():
    import bench as b  # by its module name: the oracle processes are spawned and import it again
    c1, c2 = b.config_dict(1), b.config_dict(2)
    assert set(c1) == {"workload", "global_batch", "seq_len", "parallelism", "l2"}
    assert c2["global_batch"] == 2 * c1["global_batch"] and c2["parallelism"] == "dp2"

    class A:
        oracle_procs, warmup, steps = 2, 3, 1
    out = b.bench_reference(A, 0, 1)
    assert out["impl"] == "reference" and out["config"] == c1
    assert out["ms_per_step_kind"].startswith("extrapolated")
    assert out["cpu_baseline"]["cores"] == 2 and out["e2e"]["h2d_bytes_per_step"] == 0
    assert b.bench_reference(A, 1, 2) is None  # other ranks do no work
