"""Memory-safety fuzz and a CPU round trip of the delta file's host code (no GPU).

Builds csrc/st_file.cu with tests/native/st_file_fuzz.cu under AddressSanitizer
and UndefinedBehaviorSanitizer (nvcc for the host code, g++ to link) and runs
the fuzzer on mutated delta files: any out-of-bounds access, overflow or
undefined behaviour aborts it with a sanitizer report.  Accept/refuse parity
with the oracle is checked separately (tests/test_st_file_host.py).
"""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fuzzer(tmp_path_factory):
    from tests._dev import build_module
    nvcc = build_module().nvcc()
    if (shutil.which(nvcc) is None and not os.path.exists(nvcc)) or shutil.which("g++") is None:
        pytest.skip("nvcc and g++ are needed to build the fuzzer")
    d = tmp_path_factory.mktemp("fuzz")
    flags = ["-g", "-O1", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
             "-Xcompiler=-fsanitize=address", "-Xcompiler=-fsanitize=undefined",
             "-Xcompiler=-fno-omit-frame-pointer", "-I", os.path.join(ROOT, "include"),
             "-I", os.path.join(ROOT, "sparse_bf16_delta_b200", "csrc")]
    objs = []
    for src in (os.path.join(ROOT, "sparse_bf16_delta_b200", "csrc", "st_file.cu"),
                os.path.join(ROOT, "tests", "native", "st_file_fuzz.cu")):
        o = str(d / (os.path.basename(src) + ".o"))
        subprocess.run([nvcc, *flags, "-c", src, "-o", o], check=True, capture_output=True)
        objs.append(o)
    cuda_lib = os.path.join(os.path.dirname(os.path.dirname(nvcc)), "lib64")
    exe = str(d / "st_file_fuzz")
    subprocess.run(["g++", "-fsanitize=address", "-fsanitize=undefined", "-o", exe, *objs,
                    "-L", cuda_lib, "-lcudart_static", "-ldl", "-lpthread", "-lrt"],
                   check=True, capture_output=True)
    return exe


@pytest.mark.parametrize("seed", [1, 2])
def test_header_parser_survives_mutated_files(fuzzer, seed):
    env = dict(os.environ, UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1",
               ASAN_OPTIONS="detect_leaks=1")
    r = subprocess.run([fuzzer, str(seed), "60000"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "runtime error" not in r.stderr and "AddressSanitizer" not in r.stderr, r.stderr[-4000:]
    acc, ref = (int(x) for x in r.stdout.split()[1:4:2])
    assert acc > 100 and ref > 10000, r.stdout


@pytest.fixture(scope="module")
def roundtrip(tmp_path_factory):
    """csrc/st_file.cu with tests/native/st_file_roundtrip.cu, which supplies
    cudaMemcpyAsync as a host memcpy: the delta file's whole read and write
    path, copies included, runs on the CPU (under ASan and UBSan)."""
    from tests._dev import build_module
    nvcc = build_module().nvcc()
    if (shutil.which(nvcc) is None and not os.path.exists(nvcc)) or shutil.which("g++") is None:
        pytest.skip("nvcc and g++ are needed to build the round-trip test")
    d = tmp_path_factory.mktemp("st_roundtrip")
    san = ["-fsanitize=address", "-fsanitize=undefined"]
    obj = str(d / "st_file.o")
    subprocess.run([nvcc, "-O1", "-g", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    *[f"-Xcompiler={f}" for f in san], "-I", os.path.join(ROOT, "include"),
                    "-c", os.path.join(ROOT, "sparse_bf16_delta_b200", "csrc", "st_file.cu"),
                    "-o", obj], check=True, capture_output=True)
    rt = str(d / "roundtrip.o")
    subprocess.run(["g++", "-O1", "-g", "-std=c++17", *san, "-x", "c++", "-I",
                    os.path.join(ROOT, "include"), "-c",
                    os.path.join(ROOT, "tests", "native", "st_file_roundtrip.cu"), "-o", rt],
                   check=True, capture_output=True)
    exe = str(d / "st_file_roundtrip")
    subprocess.run(["g++", *san, "-o", exe, rt, obj], check=True, capture_output=True)
    return exe


@pytest.mark.parametrize("seed", [1, 2])
def test_delta_file_round_trip_with_copies_on_the_cpu(roundtrip, seed):
    # Written by dws_st_delta_write and read back by dws_st_delta_read, and
    # read from files laid out per parameter in shuffled order: offsets,
    # indices and values come back exactly (300 random deltas per seed).
    env = dict(os.environ, UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([roundtrip, str(seed)], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, (r.stdout[-2000:], r.stderr[-4000:])
    assert "runtime error" not in r.stderr and "AddressSanitizer" not in r.stderr, r.stderr[-4000:]
    assert r.stdout.strip() == "round trips 600", r.stdout
