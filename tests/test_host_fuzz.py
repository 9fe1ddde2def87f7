"""Memory-safety fuzz of libdws's plan and argument-checking host code (no GPU).

Builds every csrc/*.cu source (host code under AddressSanitizer and
UndefinedBehaviorSanitizer) with tests/native/plan_fuzz.cu and runs it: random
plans (up to 20,000 tensors, empty, ragged and maximum sizes, invalid sizes),
their queries against the tiling rule, the delta-file header, and the entry
points' host-side refusals.  No call reaches the GPU.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def plan_fuzzer(tmp_path_factory):
    from tests._dev import build_module
    nvcc = build_module().nvcc()
    if (shutil.which(nvcc) is None and not os.path.exists(nvcc)) or shutil.which("g++") is None:
        pytest.skip("nvcc and g++ are needed to build the fuzzer")
    d = tmp_path_factory.mktemp("plan_fuzz")
    csrc = os.path.join(ROOT, "sparse_bf16_delta_b200", "csrc")
    flags = ["-O1", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
             "-Xcompiler=-fsanitize=address", "-Xcompiler=-fsanitize=undefined",
             "-Xcompiler=-fno-omit-frame-pointer", "-I", os.path.join(ROOT, "include"), "-I", csrc]
    srcs = sorted(glob.glob(os.path.join(csrc, "*.cu"))) + [
        os.path.join(ROOT, "tests", "native", "plan_fuzz.cu")]
    objs = []
    for src in srcs:
        o = str(d / (os.path.basename(src) + ".o"))
        subprocess.run([nvcc, *flags, "-c", src, "-o", o], check=True, capture_output=True)
        objs.append(o)
    cuda_lib = os.path.join(os.path.dirname(os.path.dirname(nvcc)), "lib64")
    exe = str(d / "plan_fuzz")
    subprocess.run(["g++", "-fsanitize=address", "-fsanitize=undefined", "-o", exe, *objs,
                    "-L", cuda_lib, "-lcudart_static", "-ldl", "-lpthread", "-lrt"],
                   check=True, capture_output=True)
    return exe


@pytest.mark.parametrize("seed", [1, 2])
def test_plans_and_host_refusals_under_sanitizers(plan_fuzzer, seed):
    env = dict(os.environ, UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1",
               ASAN_OPTIONS="detect_leaks=1")
    r = subprocess.run([plan_fuzzer, str(seed), "1500"], capture_output=True, text=True, env=env,
                       timeout=900)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "runtime error" not in r.stderr and "AddressSanitizer" not in r.stderr, r.stderr[-4000:]
    assert r.stdout.startswith("plans "), r.stdout
