"""bench.py's reference arm (the CPU oracle on a workload) and its JSON line,
on the host only: one line with the keys the benchmark contract names."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_fp32", "--steps", "2", "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_reference_arm_other_ranks_print_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_fp32", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr
    assert res.stdout.strip() == ""


def test_kernel_rooflines_fractions_and_stage_totals():
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops_sustained": 1000.0, "hbm_gbs": 5000.0}      # ridge: 200 FLOP per byte
    fl = {"gemm_a": 2e12, "gemm_b": 1e12, "router": 1e9}
    by = {"router": 1e8, "rows": 5e9, "meta_x": 1e6}
    # (total ms, launches) over 2 steps
    per = {"gemm_a": (8.0, 2), "gemm_b": (2.0, 2), "router": (0.1, 2), "rows": (2.0, 2),
           "meta_x": (0.02, 2), "other": (0.5, 2)}
    k, st = bench.kernel_rooflines(per, 2, 20.0, fl, by, peaks)
    assert k["gemm_a"]["tflops"] == 500.0 and k["gemm_a"]["bound"] == "tensor" and k["gemm_a"]["frac"] == 0.5
    assert k["gemm_b"]["frac"] == 1.0
    # router: 10 FLOP per byte, below the ridge, so rated against HBM: 1e8 B in 50 us = 2000 GB/s
    assert k["router"]["bound"] == "hbm" and k["router"]["gbs"] == 2000.0 and k["router"]["frac"] == 0.4
    assert k["rows"]["gbs"] == 5000.0 and k["rows"]["frac"] == 1.0
    assert "frac" not in k["other"] and k["other"]["share"] == 0.025
    assert k["meta_x"]["bound"] == "latency" and "frac" not in k["meta_x"]
    # stage totals weight each kernel by its time: (2*2e12 + 2*1e12) FLOP in 10 ms
    assert st["grouped_gemms"]["kernels"] == ["gemm_a", "gemm_b"]
    assert st["grouped_gemms"]["tflops"] == 600.0 and st["grouped_gemms"]["frac"] == 0.6
    assert st["bandwidth_kernels"] == {"kernels": ["rows"], "gbs": 5000.0, "frac": 1.0}
    assert st["metadata_us_per_step"] == 10.0


def test_recorded_traffic_only_for_the_captured_source_and_workload(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    # the committed summary gives a kernel's traffic only while the source it
    # names hashes to one of the recorded prefixes
    import hashlib
    rows = [l.split() for l in open(os.path.join(ROOT, "profiles", "ncu_traffic.txt"))
            if l.strip() and not l.startswith("#")]
    for kernel, wl, nbytes, fname, shas in rows:
        src = open(os.path.join(ROOT, "dropless_top_moe_b200", "csrc", fname), "rb").read()
        fresh = hashlib.sha256(src).hexdigest()[:16] in shas.split(",")
        assert bench.recorded_traffic(kernel, wl) == (float(nbytes) if fresh else None), kernel
    assert bench.recorded_traffic("gemm1_swiglu", "mixtral") is None
    assert bench.recorded_traffic("permute", "train_step") is None
    # a summary whose source hash is stale gives no traffic
    prof = tmp_path / "profiles"
    prof.mkdir()
    csrc = tmp_path / "dropless_top_moe_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel\n")
    import hashlib
    sha = hashlib.sha256(b"// kernel\n").hexdigest()[:16]
    (prof / "ncu_traffic.txt").write_text(f"# header\nk_new train_step 1e9 k.cu {sha}\n"
                                          f"k_old train_step 2e9 k.cu 0123456789abcdef\n"
                                          f"k_list train_step 3e9 k.cu 0123456789abcdef,{sha}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k_new", "train_step") == 1e9
    assert bench.recorded_traffic("k_old", "train_step") is None
    assert bench.recorded_traffic("k_list", "train_step") == 3e9


def test_split_gemm_launches_fold_into_their_kernel():
    sys.path.insert(0, ROOT)
    import bench
    per = {"gemm1_swiglu": (10.0, 5), "gemm1_swiglu_single": (2.5, 5), "gemm2": (4.0, 5),
           "dgrad_w2_swiglu_bwd_single": (1.0, 5)}
    out = bench.fold_split_launches(dict(per))
    # time summed, launches of the main kernel kept (its work model is per step)
    assert out["gemm1_swiglu"] == (12.5, 5)
    assert "gemm1_swiglu_single" not in out
    assert out["gemm2"] == (4.0, 5)
    # a second launch without its main kernel is left alone
    assert out["dgrad_w2_swiglu_bwd_single"] == (1.0, 5)
