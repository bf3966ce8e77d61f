"""The host block manager under the address and undefined-behaviour sanitizers: a C++ driver
(tests/bm_fuzz.cpp) runs thousands of random valid and invalid calls and checks the pool's conservation
laws after each (no GPU)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fuzz(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("bm") / "bm_fuzz")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
                           "-fno-sanitize-recover=all", "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "bm_fuzz.cpp"),
                           os.path.join(ROOT, "paged_kv_cache_409_b200", "csrc", "block_manager.cpp"), "-o", exe])
    return exe


@pytest.mark.parametrize("seed", range(1, 9))
def test_random_calls_keep_the_pool_consistent(fuzz, seed):
    r = subprocess.run([fuzz, str(seed)], capture_output=True, text=True, timeout=300,
                       env={**os.environ, "ASAN_OPTIONS": "detect_leaks=1:abort_on_error=0"})
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.strip() == f"ok {seed}"
