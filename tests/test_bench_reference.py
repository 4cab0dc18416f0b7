"""bench.py's reference arm (the float64 oracle timed on the host cores) keeps
the bench contract on the CPU: one JSON line with the required keys from rank
0, nothing from the other ranks."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--workload", "llama60m"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return [line for line in r.stdout.splitlines() if line.strip()]


def test_reference_arm_prints_one_contract_line():
    lines = _run()
    assert len(lines) == 1
    out = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["unit"] == "tokens/s" and out["higher_is_better"] is True
    assert out["value"] > 0 and out["steps"] == 1 and out["warmup"] == 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["cpu_baseline"]["value"] == out["value"] and out["cpu_baseline"]["sample"]
    assert out["e2e"] == {"value": out["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in out["config"] and "model" not in out["config"]


def test_reference_arm_other_ranks_do_no_work():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_kernel_table_holds_each_launch_to_its_own_bound():
    """The per-kind roofline fraction: the roofline time of the tensor-bound
    launches' flops at the tensor peak plus the HBM-bound launches' bytes at
    the copy peak, over the measured time.  A kind with one launch of each
    kind gets the sum of both terms; `bound` names the larger."""
    sys.path.insert(0, ROOT)
    import bench

    peaks = bench.load_peaks()
    pt, ph = peaks["bf16_tflops_sustained"] * 1e12, peaks["hbm_gbs"] * 1e9
    t_tc, t_hbm = 1e-3, 3e-3  # seconds of roofline time in each term
    rows = {"mixed": {"launches": 2, "ms": 8.0, "flop": t_tc * pt + 1e9, "bytes": 5e9 + t_hbm * ph,
                      "flop_tc": t_tc * pt, "bytes_hbm": t_hbm * ph},
            "copy": {"launches": 1, "ms": 1.0, "flop": 0.0, "bytes": 0.5 * 1e-3 * ph, "flop_tc": 0.0,
                     "bytes_hbm": 0.5 * 1e-3 * ph}}
    tab = bench.kernel_table(rows, steps=1)
    assert abs(tab["mixed"]["frac"] - 0.5) < 1e-4 and tab["mixed"]["bound"] == "hbm"
    assert abs(tab["copy"]["frac"] - 0.5) < 1e-4 and tab["copy"]["bound"] == "hbm" and tab["copy"]["tflops"] is None
    rows["mixed"]["bytes_hbm"] = 0.0
    tab = bench.kernel_table(rows, steps=1)
    assert abs(tab["mixed"]["frac"] - 0.125) < 1e-4 and tab["mixed"]["bound"] == "tensor"
