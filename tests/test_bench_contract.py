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


def test_traffic_ratios_match_the_committed_profiles():
    """roofline.traffic scales a committed ncu capture: each ratio's DRAM and algorithmic megabytes are the
    ones its profile summary prints (to the summary's rounding), and the profile file exists."""
    import importlib.util
    import re
    spec = importlib.util.spec_from_file_location("bench_module2", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for cfg, (ratio, source) in bench.TRAFFIC_PER_ALGORITHMIC_BYTE.items():
        path = os.path.join(ROOT, source.split(" ")[0])
        assert os.path.exists(path), (cfg, source)
        text = open(path).read()
        mbs = [float(x) for x in re.findall(r"(\d+\.\d+) MB", text)]
        assert 1.0 <= ratio < 1.1, cfg
        # some read + write (+ merge) combination of the printed figures over a printed algorithmic figure
        assert any(abs(ratio - t / a) < 2e-3 for a in mbs for t in mbs + [x + y for x in mbs for y in mbs]
                   + [x + y + z for x in mbs for y in mbs for z in mbs] if a > 0), (cfg, ratio)
