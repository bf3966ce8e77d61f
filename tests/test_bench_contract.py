"""bench.py's JSON line (reference arm, CPU): one line with the contract's keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                       cwd=ROOT, timeout=600, env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--config", "tiny_decode_f32", "--steps", "2", "--warmup", "3")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"] == "tiny_decode_f32"


def test_reference_arm_multi_token_line():
    d = run_bench("--impl", "reference", "--config", "multi_token_decode_bf16", "--steps", "1", "--warmup", "3")
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert "draft tokens" in d["cpu_baseline"]["sample"]


def test_copy_blocks_measurement_pairs_are_disjoint():
    """The standalone copy_blocks figure copies distinct blocks onto distinct, unsourced blocks (the kernel's
    precondition), about 0.5 GB of each pool per launch, at most half the pool."""
    import importlib.util
    import numpy as np
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for nb, bb in ((4188, 16 * 32 * 128 * 2), (100, 1 << 20), (3, 10), (1 << 16, 4096)):
        p = bench.disjoint_block_pairs(nb, bb)
        src, dst = set(p[:, 0].tolist()), set(p[:, 1].tolist())
        assert len(src) == len(dst) == len(p) and not (src & dst)
        assert p.min() >= 0 and p.max() < nb and p.dtype == np.int64
        assert len(p) == min(nb // 2, max(1, (512 << 20) // bb))


def test_traffic_ratios_are_the_captured_dram_bytes_over_algorithmic_bytes():
    """roofline.traffic scales one ncu capture per workload: the ratio is DRAM read + written over the
    captured launch's algorithmic bytes, a little above 1 for a kernel that reads each K/V byte once."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_module2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for cfg, cap in bench.TRAFFIC_CAPTURES.items():
        ratio = bench.traffic_ratio(cfg)
        assert ratio == (cap["read_mb"] + cap["write_mb"]) / cap["algorithmic_mb"]
        assert cap["case"] and "profiles" not in cap["case"]
        if cap.get("whole"):  # shared blocks: DRAM sees the distinct bytes once, far below the logical bytes
            assert ratio < 0.1, cfg
        else:
            assert 1.0 <= ratio < 1.1, cfg


def test_reference_arm_loads_only_the_oracle():
    """The reference arm builds the workload with torch and times the oracle: the CUDA library is never
    loaded into its process."""
    code = ("import runpy, sys, json\n"
            f"sys.argv = ['bench.py', '--impl', 'reference', '--config', 'llama7b_decode_f16', '--steps', '1',"
            f" '--warmup', '3']\n"
            f"runpy.run_path({os.path.join(ROOT, 'bench.py')!r}, run_name='__main__')\n"
            "maps = open('/proc/self/maps').read()\n"
            "print('LIBS', 'libpagedkv' in maps, 'liboracle' in maps)\n")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=900,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    assert "LIBS False True" in r.stdout, r.stdout[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["cpu_baseline"]["cores"] >= 1 and d["config"]["sample"] == 64


def test_mixed_step_chunks_do_not_depend_on_the_decode_count():
    """A smaller decode batch of the mixed step (a profiling case) keeps the full step's prefill chunks."""
    from paged_kv_cache_409_b200 import workloads
    full = workloads._mixed_lengths(1005, 192, 4, 256, 32768, 8192)
    for n in (1, 8, 64):
        dl, c0 = workloads._mixed_lengths(1005, n, 4, 256, 32768, 8192)
        assert c0.tolist() == full[1].tolist() and dl.tolist() == full[0][:n].tolist()
