"""The wire form of a delta on the GPU (positions byte block with per-tensor
pos_width, and the XOR-hash checksum) against the CPU oracle, byte by byte."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._dev import dev_bits, host_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _host_delta(rng, sizes, rate):
    offs, idx, val = [0], [], []
    for n in sizes:
        c = 0 if n == 0 else int(rng.binomial(n, rate))
        pos = np.sort(rng.choice(n, c, replace=False)) if c else np.zeros(0, dtype=np.int64)
        idx.append(pos.astype(np.int32))
        val.append(rng.integers(0, 1 << 16, c, dtype=np.uint16))
        offs.append(offs[-1] + c)
    return (np.array(offs, dtype=np.int64), np.concatenate(idx) if idx else np.zeros(0, np.int32),
            np.concatenate(val) if val else np.zeros(0, np.uint16))


def _dev_delta(dws, o, i, v):
    return dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                     torch.from_numpy(v.view(np.int16)).cuda())


@pytest.mark.parametrize("seed", [0, 1])
def test_pack_positions_matches_oracle_across_the_width_boundary(dws, seed):
    rng = np.random.default_rng(300 + seed)
    sizes = [0, 1, 65535, 65536, 65537, 8192 * 20 + 3, 5, 300_000, 0, 65536]
    o, i, v = _host_delta(rng, sizes, 0.05)
    plan = dws.DeltaPlan(sizes)
    assert [plan.pos_width(t) for t in range(len(sizes))] == [oracle.pos_width(n) for n in sizes]
    blob, po = plan.pack_positions(_dev_delta(dws, o, i, v))
    want_blob, want_po = oracle.pack_positions(sizes, o, i)
    np.testing.assert_array_equal(po.cpu().numpy(), want_po)
    np.testing.assert_array_equal(host_bytes(blob), want_blob)


def test_pack_positions_of_an_encoded_step(dws):
    # A scaled Qwen3-shaped step: norms (<= 65536 elements) get 2-byte
    # positions, the matrices 4-byte ones.
    s = W.SEEDS["qwen3_0p6b"]
    shapes = W.scaled_shapes(W.qwen3_0p6b_shapes(), 8)
    w0 = W.init_set(shapes, s, "cuda", 0.02)
    w1 = W.step_set(w0, s, 1, 3e-6, "cuda")
    plan = dws.DeltaPlan.for_tensors(w0.tensors)
    d = plan.encode_exact(dws.ptr_table(w0.tensors), dws.ptr_table(w1.tensors))
    sizes = [t.numel() for t in w0.tensors]
    assert {plan.pos_width(t) for t in range(len(sizes))} == {2, 4}
    blob, po = plan.pack_positions(d)
    want_blob, want_po = oracle.pack_positions(sizes, d.offsets.cpu().numpy(), d.indices.cpu().numpy())
    np.testing.assert_array_equal(po.cpu().numpy(), want_po)
    np.testing.assert_array_equal(host_bytes(blob), want_blob)
    # and the checksum of the flush
    vals = d.values.cpu().numpy().view(np.uint16)
    assert dws.checksum(blob, blob.numel(), d.values) == oracle.checksum(want_blob, vals)


def test_pack_positions_empty_delta_and_capacity(dws):
    sizes = [100, 70_000, 3]
    plan = dws.DeltaPlan(sizes)
    o = np.zeros(4, dtype=np.int64)
    blob, po = plan.pack_positions(_dev_delta(dws, o, np.zeros(0, np.int32), np.zeros(0, np.uint16)))
    assert blob.numel() == 0 and po.cpu().tolist() == [0, 0, 0, 0]
    # a block larger than the capacity given: reported with the size needed
    rng = np.random.default_rng(311)
    o, i, v = _host_delta(rng, sizes, 0.3)
    want_blob, want_po = oracle.pack_positions(sizes, o, i)
    d = _dev_delta(dws, o, i, v)
    cap = int(want_po[-1]) // 2
    positions = torch.zeros(cap, dtype=torch.uint8, device="cuda")
    pos_offsets = torch.empty(len(sizes) + 1, dtype=torch.int64, device="cuda")
    oo, ii, _, c = d.as_ref()
    code = dws.dws_pack_positions(plan.handle, oo, ii, c, positions.data_ptr(), cap,
                                  pos_offsets.data_ptr(), plan.workspace.data_ptr(),
                                  plan.workspace_bytes, torch.cuda.current_stream().cuda_stream)
    assert code == dws.DWS_OK
    st, detail = plan.status()
    assert st == dws.DWS_ERR_CAPACITY and detail == int(want_po[-1])
    np.testing.assert_array_equal(pos_offsets.cpu().numpy(), want_po)
    got = host_bytes(positions)
    np.testing.assert_array_equal(got[:cap - 4], want_blob[:cap - 4])


def test_pack_positions_flags_an_index_outside_its_tensor(dws):
    plan = dws.DeltaPlan([10, 20])
    d = _dev_delta(dws, np.array([0, 2, 3]), np.array([1, 12, 5], dtype=np.int32),
                   np.array([1, 2, 3], dtype=np.uint16))
    with pytest.raises(dws.DwsError):
        plan.pack_positions(d)


@pytest.mark.parametrize("pshift,vshift", [(0, 0), (1, 1), (7, 3), (13, 0), (0, 5)])
def test_checksum_matches_oracle_on_unaligned_views(dws, pshift, vshift):
    rng = np.random.default_rng(320 + pshift + 17 * vshift)
    nb, nv = 1_000_003, 250_001
    blob = rng.integers(0, 256, nb, dtype=np.uint8)
    vals = rng.integers(0, 1 << 16, nv, dtype=np.uint16)
    pb = torch.zeros(nb + 32, dtype=torch.uint8, device="cuda")
    pb[pshift:pshift + nb] = torch.from_numpy(blob).cuda()
    vb = torch.zeros(nv + 16, dtype=torch.bfloat16, device="cuda")
    vb[vshift:vshift + nv] = dev_bits(vals)
    got = dws.checksum(pb[pshift:pshift + nb], nb, vb[vshift:vshift + nv])
    assert got == oracle.checksum(blob, vals)


def test_checksum_every_bf16_pattern(dws):
    # All 65536 patterns (zeros, subnormals, normals, infinities, NaNs); the
    # hash of the whole set and of the 16 halves split by one index bit, so
    # that a single pattern widened differently would show.
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    empty = torch.zeros(2, dtype=torch.uint8, device="cuda")
    assert dws.checksum(empty, 0, dev_bits(pats)) == oracle.checksum(np.zeros(0, np.uint8), pats)
    for bit in range(16):
        sub = pats[(pats >> bit) & 1 == 1]
        assert dws.checksum(empty, 0, dev_bits(sub)) == oracle.checksum(np.zeros(0, np.uint8), sub), bit


def test_checksum_empty(dws):
    empty = torch.zeros(2, dtype=torch.uint8, device="cuda")
    assert dws.checksum(empty, 0, torch.zeros(0, dtype=torch.bfloat16, device="cuda")) == 0


@pytest.mark.parametrize("rate", [0.02, 0.4])
def test_encode_checksum_fused_equals_pack_then_checksum(dws, rate):
    # The checksum the encode computes on the fly equals the one of the
    # packed block (and the oracle's), over tensors of both widths, dense runs
    # and a ragged tail.
    rng = np.random.default_rng(330 + int(rate * 10))
    sizes = [100, 65536, 65537, 8192 * 5 + 11, 0, 3]
    olds, news = [], []
    for n in sizes:
        a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
        b = a.copy()
        if n:
            m = rng.random(n) < rate
            b[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
            if n > 9000:
                b[1024:9216] ^= np.uint16(0x0001)
        olds.append(a)
        news.append(b)
    plan = dws.DeltaPlan(sizes)
    ot = dws.ptr_table([dev_bits(a) for a in olds])
    nt = dws.ptr_table([dev_bits(b) for b in news])
    d, fused = plan.encode_checksum(ot, nt)
    o, i, v = oracle.encode(olds, news)
    np.testing.assert_array_equal(d.indices.cpu().numpy(), i)
    blob, _ = oracle.pack_positions(sizes, o, i)
    assert fused == oracle.checksum(blob, v)
    gblob, _ = plan.pack_positions(d)
    assert fused == dws.checksum(gblob, gblob.numel(), d.values)


def test_checksum_bit_64_comes_from_the_library(dws):
    # A negative value widens to a double with bit 63 set, so hash(values)
    # << 1 reaches bit 64: the 65-bit checksum is read back as written by
    # libdws (a 128-bit little-endian integer), nothing combined in Python.
    empty = torch.zeros(2, dtype=torch.uint8, device="cuda")
    for pats in ([0xBF80], [0xBF80, 0x3F80], [0xFFC1, 0x0001, 0x8000]):
        v = np.array(pats, dtype=np.uint16)
        want = oracle.checksum(np.zeros(0, np.uint8), v)
        got = dws.checksum(empty, 0, dev_bits(v))
        assert got == want and (got >> 64) == (oracle.checksum_parts(np.zeros(0, np.uint8), v)[1] >> 63)
    assert dws.checksum(empty, 0, dev_bits(np.array([0xBF80], np.uint16))) >> 64 == 1


def test_checksum_through_the_c_abi_from_c(dws, tmp_path):
    # tests/native/checksum_abi.c calls dws_checksum from C and prints the
    # hashes and the checksum words; they must equal the oracle's.
    import shutil
    import subprocess
    from tests._dev import ROOT
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("a C compiler is needed")
    cuda = os.path.dirname(os.path.dirname(os.path.realpath(shutil.which("nvcc") or
                                                            "/usr/local/cuda/bin/nvcc")))
    libdir = os.path.dirname(dws.LIB_PATH)
    exe = str(tmp_path / "checksum_abi")
    subprocess.run([cc, "-O2", "-o", exe, os.path.join(ROOT, "tests", "native", "checksum_abi.c"),
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    "-L", libdir, "-l:libdws.so", f"-Wl,-rpath,{libdir}",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{cuda}/lib64"],
                   check=True, capture_output=True)
    rng = np.random.default_rng(340)
    for nb, nv in ((0, 0), (13, 7), (100_003, 40_001)):
        blob = rng.integers(0, 256, nb, dtype=np.uint8)
        vals = rng.integers(0, 1 << 16, nv, dtype=np.uint16)
        vals[:min(nv, 3)] |= np.uint16(0x8000)
        inp = tmp_path / f"in_{nb}_{nv}.bin"
        inp.write_bytes(np.array([nb, nv], np.int64).tobytes() + blob.tobytes() + vals.tobytes())
        r = subprocess.run([exe, str(inp)], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stderr
        h0, h1, c0, c1 = (int(x, 16) for x in r.stdout.split())
        hp, hv = oracle.checksum_parts(blob, vals)
        assert (h0, h1) == (hp, hv)
        assert c0 | (c1 << 64) == oracle.checksum(blob, vals)
        assert c1 in (0, 1)
