"""The oracle's C code under the address and undefined-behaviour sanitizers: every pin runs against an
instrumented build in a child process (no GPU), so an out-of-bounds read that happened to give
plausible numbers would still fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle
from oracle_pins import ALL_PINS
orc = oracle.Oracle({lib!r})
for pin in ALL_PINS:
    pin(orc)
print("pins", len(ALL_PINS))
"""


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


def test_pins_pass_on_a_sanitized_oracle(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not installed")
    lib = str(tmp_path / "liboracle_asan.so")
    subprocess.check_call(["gcc", "-O1", "-g", "-std=c11", "-fPIC", "-shared", "-fsanitize=address,undefined",
                           "-fno-sanitize-recover=all", "-o", lib, os.path.join(ROOT, "oracle", "pagedkv_oracle.c"),
                           "-lm"])
    env = {**os.environ, "LD_PRELOAD": f"{asan}:{ubsan}", "ASAN_OPTIONS": "detect_leaks=0:verify_asan_link_order=0",
           "UBSAN_OPTIONS": "print_stacktrace=1", "CUDA_VISIBLE_DEVICES": ""}
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, timeout=900)
    assert r.returncode == 0, (r.stdout[-1000:], r.stderr[-4000:])
    assert r.stdout.strip().startswith("pins ")
