"""AddressSanitizer + UndefinedBehaviorSanitizer builds of the CPU oracle
and of librtv's host code, each driven through its entry points on small
inputs (tests/sanitize/*.c).  The sanitizers abort on an out-of-bounds
access, a use of freed memory, a leak or an undefined operation; no GPU is
touched (the library driver calls only host-side paths)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SAN = os.path.join(ROOT, "tests", "sanitize")
SAN_FLAGS = ["-fsanitize=address", "-fsanitize=undefined", "-fno-omit-frame-pointer",
             "-fno-sanitize-recover=all", "-g", "-O1"]


def _run(exe, env_extra):
    env = dict(os.environ, **env_extra)
    out = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "runtime error" not in out.stderr and "AddressSanitizer" not in out.stderr, out.stderr
    return out.stdout


def test_oracle_under_asan_and_ubsan(tmp_path):
    exe = str(tmp_path / "oracle_driver")
    subprocess.check_call(["gcc", *SAN_FLAGS, "-ffp-contract=off", "-fopenmp", "-o", exe,
                           os.path.join(SAN, "oracle_driver.c"),
                           os.path.join(ROOT, "oracle", "rtv_oracle.c"), "-lm"])
    assert "oracle driver ok" in _run(exe, {"OMP_NUM_THREADS": "2", "ASAN_OPTIONS": "detect_leaks=1"})


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="needs nvcc to compile the library's host code")
def test_library_host_paths_under_asan_and_ubsan(tmp_path):
    from kv_cache_serving_append_b200 import build
    nvcc = build._nvcc()
    csrc = os.path.join(ROOT, "kv_cache_serving_append_b200", "csrc")
    xflags = [a for f in SAN_FLAGS for a in ("-Xcompiler", f)]
    arch = ["-gencode", "arch=compute_100a,code=sm_100a"]
    objs = []
    for src in build.SOURCES:
        obj = str(tmp_path / src.replace(".cu", ".o"))
        subprocess.check_call([nvcc, *arch, "-std=c++17", "--expt-relaxed-constexpr", *xflags,
                               "-c", os.path.join(csrc, src), "-o", obj])
        objs.append(obj)
    exe = str(tmp_path / "rtv_host_driver")
    subprocess.check_call([nvcc, *arch, *xflags, "-o", exe, os.path.join(SAN, "rtv_host_driver.c"), *objs,
                           "-lcudart"])
    # the CUDA runtime maps memory where ASan's shadow gap would sit
    assert "host driver ok" in _run(exe, {"ASAN_OPTIONS": "protect_shadow_gap=0:detect_leaks=1"})
