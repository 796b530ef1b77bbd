"""The library's host code (allocator, group tables, planner, placement) built with
AddressSanitizer and UndefinedBehaviorSanitizer and driven on seeded random inputs
(tests/native/host_fuzz.cpp), then with allocation failures injected into every allocation of
every call in turn: each such call returns TG_ENOMEM (or falls back to the same result), leaves
the allocator unchanged, hands back no object and leaks nothing. No GPU involved."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_host_code_is_clean_under_asan_and_ubsan():
    out_dir = os.path.join(ROOT, "tests", "native", "_build")   # git-ignored
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "host_fuzz")
    cmd = ["g++", "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=undefined", "-fno-omit-frame-pointer",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc"),
           os.path.join(ROOT, "tests", "native", "host_fuzz.cpp"),
           os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc", "tg_host.cpp"),
           "-o", str(exe)]
    subprocess.check_call(cmd)
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([str(exe), "200", "20261202", "20"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "200 rounds clean" in r.stdout
    assert "allocation failures: 20 rounds" in r.stdout


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_oracle_is_clean_under_asan_and_ubsan():
    """The CPU oracle's C code (oracle/tg_oracle.c) under the same sanitizers, every exported
    function on seeded random cases (tests/native/oracle_fuzz.c; OpenMP off, so one thread)."""
    out_dir = os.path.join(ROOT, "tests", "native", "_build")   # git-ignored
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "oracle_fuzz")
    cmd = ["gcc", "-std=c11", "-O1", "-g", "-fsanitize=address,undefined,float-cast-overflow",
           "-fno-sanitize-recover=all", "-fno-omit-frame-pointer", "-Wno-unknown-pragmas",
           os.path.join(ROOT, "tests", "native", "oracle_fuzz.c"),
           os.path.join(ROOT, "oracle", "tg_oracle.c"), "-lm", "-o", str(exe)]
    subprocess.check_call(cmd)
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([str(exe), "300", "20261202"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "300 rounds clean" in r.stdout


CUDA_INCLUDE = "/usr/local/cuda/include"


@pytest.mark.skipif(shutil.which("g++") is None or not os.path.exists(
    os.path.join(CUDA_INCLUDE, "cuda_runtime.h")), reason="needs g++ and the CUDA headers")
def test_host_pipe_failure_paths_with_a_fake_runtime():
    """The host-buffer pipe (csrc/tg_pipe.cpp) against stubs of the CUDA runtime calls it makes
    (tests/native/pipe_faults.cpp): each runtime call failing in turn is reported, creation
    hands back nothing and leaks nothing, the pipe serves the next call; under ASan/UBSan."""
    out_dir = os.path.join(ROOT, "tests", "native", "_build")   # git-ignored
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "pipe_faults")
    cmd = ["g++", "-std=c++17", "-O1", "-g", "-fsanitize=address,undefined",
           "-fno-sanitize-recover=undefined", "-fno-omit-frame-pointer",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc"), "-I", CUDA_INCLUDE,
           os.path.join(ROOT, "tests", "native", "pipe_faults.cpp"),
           os.path.join(ROOT, "non_uniform_paged_flash_b200", "csrc", "tg_pipe.cpp"),
           "-o", str(exe)]
    subprocess.check_call(cmd)
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0",
               UBSAN_OPTIONS="print_stacktrace=1")
    r = subprocess.run([str(exe)], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, (r.stdout + r.stderr)[-4000:]
    assert "every one reported, nothing leaked" in r.stdout
