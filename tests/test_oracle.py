"""Pins for the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: values the
pages fix in a worked example (tests/golden/), a library routine (numpy,
torch's float->bf16 cast), a closed form the input generator knows (the
positions it changed), brute force on tiny inputs, or invariants of the
method.  The comment on each test names the kind of mistake it would catch.
"""
from __future__ import annotations

import ctypes
import itertools
import math
import struct

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import _golden as G


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy bits (host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)


# ---------------------------------------------------------------- encode


def test_encode_golden_worked_example():
    # Off-by-one or 1-based indices, values taken from old instead of new,
    # float instead of bit compare (+0/-0, NaN), wrong offsets with empty
    # tensors: each changes the expected lists.
    olds, news, offsets, indices, values = G.encode_example()
    o, i, v = oracle.encode(olds, news)
    np.testing.assert_array_equal(o, offsets)
    np.testing.assert_array_equal(i, indices)
    np.testing.assert_array_equal(v, values)


def test_encode_matches_numpy_flatnonzero():
    # Library pin: numpy's flatnonzero over the integer views, the same
    # compare the verl snippet writes with torch (view(int) != view(int),
    # nonzero).  Catches dropped tails, skipped elements, unstable order.
    rng = np.random.default_rng(7)
    sizes = [0, 1, 7, 8, 9, 4095, 4096, 4097, 100_003, 0, 65_536]
    olds, news = [], []
    for n in sizes:
        a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
        b = a.copy()
        flip = rng.random(n) < rng.choice([0.0, 0.01, 0.3, 1.0])
        b[flip] ^= rng.integers(1, 1 << 16, int(flip.sum()), dtype=np.uint16)
        olds.append(a)
        news.append(b)
    o, i, v = oracle.encode(olds, news)
    exp_i, exp_v, exp_o = [], [], [0]
    for a, b in zip(olds, news):
        nz = np.flatnonzero(a != b)
        exp_i.append(nz.astype(np.int32))
        exp_v.append(b[nz])
        exp_o.append(exp_o[-1] + nz.size)
    np.testing.assert_array_equal(o, np.array(exp_o, dtype=np.int64))
    np.testing.assert_array_equal(i, np.concatenate(exp_i))
    np.testing.assert_array_equal(v, np.concatenate(exp_v))


SPECIALS = [0x0000, 0x8000, 0x0001, 0x8001, 0x3F80, 0xBF80, 0x7F80, 0xFF80,
            0x7FC0, 0x7FC1, 0x3F81, 0xBF81]


def test_encode_bruteforce_tiny():
    # Brute force over every pair of length-2 tensors drawn from 12 special
    # bf16 patterns (signed zeros, subnormals, +-1, +-inf, two NaN payloads),
    # against the set definition {i : old[i] != new[i]} on bits.
    pairs = list(itertools.product(SPECIALS, repeat=2))
    for a in pairs:
        for b in pairs[::7]:
            old = np.array(a, dtype=np.uint16)
            new = np.array(b, dtype=np.uint16)
            o, i, v = oracle.encode([old], [new])
            want = [k for k in range(2) if a[k] != b[k]]
            assert list(i) == want
            assert list(v) == [b[k] for k in want]
            assert list(o) == [0, len(want)]


def test_encode_invariants_and_roundtrip():
    # nnz equals the popcount of the change mask; indices strictly ascend in
    # each segment; every value differs from old at its index; applying the
    # delta to old gives new bit for bit; old == new gives an empty delta.
    rng = np.random.default_rng(11)
    olds = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in (3000, 1, 0, 12345)]
    news = []
    for a in olds:
        b = a.copy()
        m = rng.random(a.size) < 0.05
        b[m] = rng.integers(0, 1 << 16, int(m.sum()), dtype=np.uint16)
        news.append(b)
    o, i, v = oracle.encode(olds, news)
    assert o[-1] == sum(int((a != b).sum()) for a, b in zip(olds, news))
    for t, (a, b) in enumerate(zip(olds, news)):
        seg = i[o[t]:o[t + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all(a[seg] != v[o[t]:o[t + 1]])
    snaps = [a.copy() for a in olds]
    oracle.apply(snaps, o, i, v)
    for s, b in zip(snaps, news):
        np.testing.assert_array_equal(s, b)
    o2, i2, v2 = oracle.encode(olds, [a.copy() for a in olds])
    assert o2.tolist() == [0] * (len(olds) + 1) and i2.size == 0 and v2.size == 0


def test_encode_capacity_counts_but_does_not_store():
    olds, news, offsets, indices, values = G.encode_example()
    o, i, v = oracle.encode(olds, news, capacity=2)
    np.testing.assert_array_equal(o, offsets)          # still the full count
    np.testing.assert_array_equal(i, indices[:2])
    np.testing.assert_array_equal(v, values[:2])


def test_encode_rejects_numel_at_int32_bound():
    # int32 indices cannot address element 2^31 (the verl review lists the
    # silent wrap-around of int32 positions as a risk): the oracle refuses.
    lib = oracle._load()
    numels = np.array([1 << 31], dtype=np.int64)
    ptrs = (ctypes.c_void_p * 1)()
    offs = np.zeros(2, dtype=np.int64)
    rc = lib.ref_encode(1, numels.ctypes.data, ptrs, ptrs, offs.ctypes.data, None, None, 0)
    assert rc == -1


# ---------------------------------------------------------------- apply / chain


def test_apply_leaves_unchanged_positions_and_empty_is_identity():
    rng = np.random.default_rng(3)
    old = rng.integers(0, 1 << 16, 5000, dtype=np.uint16)
    new = old.copy()
    pos = np.sort(rng.choice(5000, 40, replace=False))
    new[pos] ^= 0x0101
    o, i, v = oracle.encode([old], [new])
    snap = old.copy()
    oracle.apply([snap], o, i, v)
    untouched = np.ones(5000, bool)
    untouched[pos] = False
    np.testing.assert_array_equal(snap[untouched], old[untouched])
    np.testing.assert_array_equal(snap, new)
    snap2 = old.copy()
    oracle.apply([snap2], np.zeros(2, np.int64), np.zeros(0, np.int32), np.zeros(0, np.uint16))
    np.testing.assert_array_equal(snap2, old)


def test_apply_rejects_out_of_range_index():
    snap = np.zeros(4, dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.apply([snap], np.array([0, 1], np.int64), np.array([4], np.int32),
                     np.array([1], np.uint16))


def test_chain_golden_later_delta_wins():
    anchor, deltas, final = G.chain_example()
    snaps = [a.copy() for a in anchor]
    oracle.apply_chain(snaps, deltas)
    for s, f in zip(snaps, final):
        np.testing.assert_array_equal(s, f)


def test_chain_replays_qwen_shaped_steps():
    # Anchor + 10 deltas == the 10th step's weights, on the Qwen3-0.6B
    # parameter list scaled down 32x (same 310 tensors).  Equal to applying
    # the deltas one by one.
    shapes = W.scaled_shapes(W.qwen3_0p6b_shapes(), 32)
    s = W.SEEDS["qwen3_0p6b"]
    w = W.init_set(shapes, s, "cpu", 0.02)
    anchor = [bits(t) for t in w.tensors]
    deltas = []
    prev = anchor
    for k in range(1, 11):
        w = W.step_set(w, s, k, 3e-6, "cpu")
        cur = [bits(t) for t in w.tensors]
        deltas.append(oracle.encode(prev, cur))
        prev = cur
    snaps = [a.copy() for a in anchor]
    oracle.apply_chain(snaps, deltas)
    for a, b in zip(snaps, prev):
        np.testing.assert_array_equal(a, b)
    seq = [a.copy() for a in anchor]
    for d in deltas:
        oracle.apply(seq, *d)
    for a, b in zip(seq, snaps):
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("seed", [5, 6, 7])
def test_apply_and_chain_match_numpy_assignment(seed):
    # Arbitrary deltas (not from an encode): K of them over T tensors, each an
    # ascending random subset with random values, overlapping across deltas
    # with different values.  The oracle's apply and chain must equal numpy's
    # own indexed assignment `snap[t][idx] = val`, delta after delta (a
    # transposed offset, a wrong tensor, or an order reversal fails this).
    rng = np.random.default_rng(seed)
    numels = [int(x) for x in rng.choice([0, 1, 17, 1000, 8193], 6)]
    anchor = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in numels]
    deltas = []
    for _ in range(int(rng.integers(1, 9))):
        offs, idx, val = [0], [], []
        for n in numels:
            c = int(rng.integers(0, n + 1)) if n else 0
            pick = np.sort(rng.choice(n, c, replace=False)) if c else np.zeros(0, np.int64)
            idx.append(pick.astype(np.int32))
            val.append(rng.integers(0, 1 << 16, c, dtype=np.uint16))
            offs.append(offs[-1] + c)
        deltas.append((np.array(offs, np.int64), np.concatenate(idx), np.concatenate(val)))
    want = [a.copy() for a in anchor]
    for o, i, v in deltas:
        for t in range(len(numels)):
            want[t][i[o[t]:o[t + 1]]] = v[o[t]:o[t + 1]]
    got = [a.copy() for a in anchor]
    oracle.apply_chain(got, deltas)
    for g, w in zip(got, want):
        np.testing.assert_array_equal(g, w)
    one = [a.copy() for a in anchor]
    oracle.apply(one, *deltas[0])
    first = [a.copy() for a in anchor]
    for t in range(len(numels)):
        o, i, v = deltas[0]
        first[t][i[o[t]:o[t + 1]]] = v[o[t]:o[t + 1]]
    for g, w in zip(one, first):
        np.testing.assert_array_equal(g, w)


# ---------------------------------------------------------------- XOR


def test_xor_golden():
    old, new, mask = G.xor_example()
    np.testing.assert_array_equal(oracle.xor_encode(old, new), mask)
    buf = old.copy()
    oracle.xor_apply(buf, mask)
    np.testing.assert_array_equal(buf, new)


def test_xor_closed_form_on_byte_layers():
    # Closed form: the generator knows exactly which bytes it changed, so the
    # mask's nonzero bytes must be exactly those positions; numpy's
    # bitwise_xor gives the same mask (library pin); apply restores new.
    old, new, pos = W.xor_layer(0, "cpu", nbytes=2_000_003, flips=1_700)
    old, new, pos = old.numpy(), new.numpy(), pos.numpy()
    mask = oracle.xor_encode(old, new)
    np.testing.assert_array_equal(np.flatnonzero(mask), pos)
    np.testing.assert_array_equal(mask, np.bitwise_xor(old, new))
    buf = old.copy()
    oracle.xor_apply(buf, mask)
    np.testing.assert_array_equal(buf, new)
    assert not oracle.xor_encode(old, old).any()


def test_xor_agrees_with_sparse_encode_on_bf16():
    # On bf16 data the byte mask is nonzero exactly at the bytes of the
    # elements the sparse encode lists.
    old, new = W.single("cpu")
    a, b = bits(old.tensors[0]), bits(new.tensors[0])
    mask = oracle.xor_encode(a.view(np.uint8), b.view(np.uint8)).view(np.uint16)
    o, i, v = oracle.encode([a], [b])
    np.testing.assert_array_equal(np.flatnonzero(mask), i)


# ---------------------------------------------------------------- workload 5


def test_stress_closed_form_positions():
    # Closed form: every element the stress generator picks gets different
    # low mantissa bits, so the encode lists exactly the picked positions.
    sizes = W.stress_sizes(count=40, lo=16, hi=70_000)
    clustered = W.stress_clustered(count=40)
    w = W.stress_init(sizes, "cpu")
    new, picks = W.stress_step(w, clustered, 1, "cpu")
    o, i, v = oracle.encode([bits(t) for t in w.tensors], [bits(t) for t in new.tensors])
    for t, p in enumerate(picks):
        np.testing.assert_array_equal(i[o[t]:o[t + 1]], np.flatnonzero(p.numpy()))


# ---------------------------------------------------------------- bf16 rounding


def test_bf16_rne_golden_cases():
    for f32, b16 in G.rounding_cases():
        x = np.array([f32], dtype=np.uint32).view(np.float32)
        assert int(oracle.bf16_rne(x)[0]) == b16, hex(f32)


def test_bf16_rne_matches_torch_cast():
    # Library pin: torch's float32 -> bfloat16 conversion rounds to nearest
    # even.  Random bit patterns (no NaN) plus every tie pattern near 1.
    rng = np.random.default_rng(5)
    u = rng.integers(0, 1 << 32, 20000, dtype=np.uint64).astype(np.uint32)
    u = u[(u & 0x7FFFFFFF) <= 0x7F800000]
    ties = np.uint32(0x3F800000) + (np.arange(256, dtype=np.uint32) << 16) + np.uint32(0x8000)
    u = np.concatenate([u, ties.astype(np.uint32)])
    x = u.view(np.float32)
    want = bits(torch.from_numpy(x.copy()).to(torch.bfloat16))
    np.testing.assert_array_equal(oracle.bf16_rne(x), want)


def test_update_step_matches_numpy_fp32():
    # Library pin for the update model: numpy float32 ops (each rounded),
    # then torch's cast.
    rng = np.random.default_rng(9)
    w = bits(torch.from_numpy(rng.normal(0, 0.03, 50000).astype(np.float32)).to(torch.bfloat16))
    u = np.clip(rng.normal(0, 1, 50000).astype(np.float32), -10, 10)
    lr = np.float32(3e-6)
    x = w.astype(np.uint32) << 16
    x = x.view(np.float32) - (lr * u)
    want = bits(torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16))
    np.testing.assert_array_equal(oracle.update_step(w, u, 3e-6), want)


# ---------------------------------------------------------------- absorption


def _neighbours(wbits):
    """fp32 values at and around the two rounding midpoints of w."""
    lib = oracle._load()
    w = lib.ref_bf16_to_float(wbits)
    out = []
    for nb in ((wbits - 1) & 0xFFFF, (wbits + 1) & 0xFFFF):
        m = (float(w) + float(lib.ref_bf16_to_float(nb))) / 2.0
        m32 = np.float32(m)
        out += [m32, np.nextafter(m32, np.float32(np.inf)), np.nextafter(m32, np.float32(-np.inf))]
    return out


def test_absorption_predictor_matches_integer_rounding():
    # Two independent routes to "does the cast keep w's bits": exact
    # midpoints in double vs the integer rounding of ref_bf16_rne (itself
    # pinned to torch above).  Probes every midpoint and its fp32
    # neighbours, so a tie rule or a power-of-two mistake shows up.
    rng = np.random.default_rng(13)
    ws = list(rng.integers(0x0080, 0x7F7F, 300)) + [0x3F80, 0x4000, 0x3C00, 0x0080, 0x0081,
                                                   0x0001, 0x007F, 0x7F7E]
    for wb in ws:
        for sign in (0, 0x8000):
            wbits = int(wb) | sign
            for x in _neighbours(wbits):
                want = int(oracle.bf16_rne(np.array([x], np.float32))[0] != wbits)
                assert oracle.absorption_changed(wbits, x) == want, (hex(wbits), float(x))


def test_absorption_power_of_two_is_asymmetric():
    # At w = 1.0 the neighbour below is 2^-8 away and the one above 2^-7:
    # a decrease of 0.75 * 2^-8 leaves the interval, an increase of the same
    # size stays inside.
    w = 0x3F80
    assert oracle.absorption_changed(w, 1.0 - 0.75 * 2 ** -8) == 1
    assert oracle.absorption_changed(w, 1.0 + 0.75 * 2 ** -8) == 0


def _min_visible_step(wbits):
    """Smallest |dw| (downwards) that changes w's bits, by bisection."""
    w = float(oracle.bf16_to_float([wbits])[0])
    lo, hi = 0.0, abs(w)
    for _ in range(80):
        mid = (lo + hi) / 2
        x = np.float32(w - math.copysign(mid, w))
        if oracle.absorption_changed(wbits, x):
            hi = mid
        else:
            lo = mid
    return hi


def test_absorption_thresholds_from_the_pages():
    # The pages' rule: an update below about |w|/256 is absorbed; at lr 3e-6
    # and |w| in [1e-2, 1e-1] the update is always absorbed, and |w|/256 is
    # about 4e-5 .. 4e-4.  The exact threshold lies within a factor of 2 of
    # |w|/256 (the spacing is |w|*2^-7 only up to the position inside the
    # binade).
    d = G.keyed("absorption_thresholds.txt")
    lr = float(d["lr"][0])
    for wv in map(float, d["w"]):
        wbits = int(oracle.bf16_rne(np.array([wv], np.float32))[0])
        w = float(oracle.bf16_to_float([wbits])[0])
        assert oracle.absorption_changed(wbits, np.float32(w) - np.float32(lr)) == 0
        assert oracle.absorption_changed(wbits, np.float32(w) + np.float32(lr)) == 0
        thr = _min_visible_step(wbits)
        assert abs(w) / 512 <= thr <= abs(w) / 128 * 1.0001, (wv, thr)
    assert round(0.01 / 256, 5) == float(d["threshold_at_1e-2"][0])
    assert round(0.1 / 256, 4) == float(d["threshold_at_1e-1"][0])


def test_workload1_absorption_predicts_encode_mask():
    # Every element of workload 1: the generator's new weights equal the
    # oracle's recomputation of the update, and the elements the absorption
    # rule says change are exactly those the encode lists.
    old, new = W.single("cpu")
    a, b = bits(old.tensors[0]), bits(new.tensors[0])
    u = W.update_noise(a.size, W.step_seed(W.SEEDS["single"], 1, 0), "cpu").numpy()
    np.testing.assert_array_equal(oracle.update_step(a, u, 3e-6), b)
    changed, count = oracle.absorption_predict(a, u, 3e-6)
    o, i, v = oracle.encode([a], [b])
    assert count == o[-1]
    np.testing.assert_array_equal(np.flatnonzero(changed), i)
    # The change rate the workload definition expects is "about 1%"; the
    # stated update model gives about 2.3%.  Both are far from dense.
    assert 0.005 < count / a.size < 0.05


# ---------------------------------------------------------------- shapes and reported numbers


def test_model_shapes_match_the_pages_sizes():
    d = G.keyed("model_sizes.txt")
    q = W.qwen3_0p6b_shapes()
    nq = sum(W.numel(s) for _, s in q)
    assert len(q) == 310 and nq == 596_049_920
    assert round(nq * int(d["bytes_per_bf16"][0]) / 1e9, 1) == float(d["qwen3_0p6b_full_GB"][0])
    assert 7e9 * 2 / 1e9 == float(d["seven_b_full_GB"][0])
    ll = W.llama3_8b_shapes()
    assert len(ll) == 291 and sum(W.numel(s) for _, s in ll) == 8_030_261_248
    assert max(W.numel(s) for _, s in ll) < 2 ** 31


def test_stress_sizes_are_log_uniform():
    sizes = W.stress_sizes()
    assert len(sizes) == 12000 and min(sizes) >= 256 and max(sizes) <= 4194304
    expected = 12000 * (4194304 - 256) / math.log(4194304 / 256)
    assert abs(sum(sizes) / expected - 1) < 0.05


def test_sparsity_formula_reproduces_the_log_line():
    d = G.keyed("sync_log.txt")
    changed, total = int(d["changed"][0]), int(d["total"][0])
    sparsity = 1 - changed / total
    assert round(100 * sparsity, 2) == float(d["sparsity_percent"][0])
    assert round(sparsity, 4) == float(d["sparsity_metadata"][0])


# ---------------------------------------------------------------- wire positions and checksum


def test_wire_checksum_golden_worked_example():
    d = G.keyed("wire_checksum.txt")
    numels = [int(x) for x in d["numels"]]
    offsets = np.array([int(x) for x in d["offsets"]], dtype=np.int64)
    indices = np.array([int(x) for x in d["indices"]], dtype=np.int32)
    blob, po = oracle.pack_positions(numels, offsets, indices)
    np.testing.assert_array_equal(blob, G.hex8(d["positions"]))
    np.testing.assert_array_equal(po, [int(x) for x in d["pos_offsets"]])
    values = G.hex16(d["values"])
    hp, hv = oracle.checksum_parts(blob, values)
    assert hp == int(d["hash_positions"][0], 16)
    assert hv == int(d["hash_values"][0], 16)
    assert oracle.checksum(blob, values) == int(d["checksum"][0], 16)


def test_pack_positions_brute_force_and_width_rule():
    rng = np.random.default_rng(91)
    for _ in range(20):
        numels = [int(x) for x in rng.choice([0, 1, 100, 65535, 65536, 65537, 10 ** 6], 6)]
        counts = [0 if n == 0 else int(rng.integers(0, min(n, 50) + 1)) for n in numels]
        idx, offs = [], [0]
        for n, c in zip(numels, counts):
            idx.extend(sorted(rng.choice(n, c, replace=False).tolist()) if c else [])
            offs.append(offs[-1] + c)
        blob, po = oracle.pack_positions(numels, np.array(offs), np.array(idx, dtype=np.int32))
        want, wpo = b"", [0]
        for t, n in enumerate(numels):
            fmt = "<H" if n <= 65536 else "<I"
            for j in range(offs[t], offs[t + 1]):
                want += struct.pack(fmt, idx[j])
            wpo.append(len(want))
        assert blob.tobytes() == want
        assert po.tolist() == wpo


def test_bf16_to_double_bits_all_finite_patterns():
    # Exact widening: every finite bf16 value is a double; numpy's float32 ->
    # float64 conversion of the same bits gives the pattern independently.
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):  # NaN patterns are compared apart below
        f64 = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64).view(np.uint64)
    got = np.array([oracle.bf16_to_f64_bits(int(x)) for x in b], dtype=np.uint64)
    finite = ((b >> 7) & 0xFF) != 0xFF
    np.testing.assert_array_equal(got[finite], f64[finite])
    # infinities keep their sign, NaNs stay NaN (quiet) with their sign
    assert oracle.bf16_to_f64_bits(0x7F80) == 0x7FF0000000000000
    assert oracle.bf16_to_f64_bits(0xFF80) == 0xFFF0000000000000
    for x in (0x7FC0, 0x7F81, 0xFFC1):
        u = oracle.bf16_to_f64_bits(x)
        assert (u >> 52) & 0x7FF == 0x7FF and u & ((1 << 52) - 1) != 0 and (u >> 51) & 1 == 1
        assert (u >> 63) == (x >> 15)


def test_checksum_matches_torch_hash_tensor():
    # The library routine the pages' checksum() calls, on CPU, over bytes and
    # over bf16 values of every class (zeros, subnormals, normals, infinities,
    # NaNs with payloads).
    import torch
    rng = np.random.default_rng(92)
    blob = rng.integers(0, 256, 100_003, dtype=np.uint8)
    vals = rng.integers(0, 1 << 16, 50_001, dtype=np.uint16)
    vals[:8] = [0x0000, 0x8000, 0x0001, 0x807F, 0x7F80, 0xFF80, 0x7FC1, 0xFF81]
    hp, hv = oracle.checksum_parts(blob, vals)
    assert hp == int(torch.hash_tensor(torch.from_numpy(blob)).item())
    tv = torch.from_numpy(vals.view(np.int16).copy()).view(torch.bfloat16)
    assert hv == int(torch.hash_tensor(tv).item())
    for sub in (vals[:8], vals[8:1000]):
        t = torch.from_numpy(sub.view(np.int16).copy()).view(torch.bfloat16)
        assert oracle.checksum_parts(blob[:0], sub)[1] == int(torch.hash_tensor(t).item())


def test_encode_global_matches_the_pages_shard_routine():
    # shard_delta_indices, written with torch's own ops on CPU: integer-view
    # compare, nonzero, then + offset in int64.  Offsets past 2^32 pin the
    # width.
    rng = np.random.default_rng(95)
    sizes = [1000, 0, 70_001, 5]
    bases = [0, 123, 5_000_000_000, 2 ** 31 - 3]
    olds = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    news = []
    for a in olds:
        b = a.copy()
        if a.size:
            m = rng.random(a.size) < 0.1
            b[m] ^= np.uint16(0x0040)
        news.append(b)
    o, gi, v = oracle.encode_global(olds, news, bases)
    want_i, want_v = [], []
    for a, b, off in zip(olds, news, bases):
        ta = torch.from_numpy(a.view(np.int16).copy())
        tb = torch.from_numpy(b.view(np.int16).copy())
        local = (tb != ta).nonzero(as_tuple=False).view(-1)
        want_i.append((local.to(torch.int64) + off).numpy())
        want_v.append(tb[local].numpy().view(np.uint16))
    assert gi.dtype == np.int64
    np.testing.assert_array_equal(gi, np.concatenate(want_i))
    np.testing.assert_array_equal(v, np.concatenate(want_v))
    assert gi.max() > 2 ** 32


# ---------------------------------------------------------------- gather of shards to rank 0


def test_merge_shards_hand_worked():
    # Two ranks, two parameters: rank 0 has 2 entries of p0 and 1 of p1, rank
    # 1 one of p0 and none of p1.  Rank 0's merged delta lists p0's entries
    # rank by rank, then p1's (a dropped rank, a rank-major instead of
    # parameter-major order or wrong offsets fail it).
    o, i, v = oracle.merge_shards(
        [np.array([0, 2, 3]), np.array([0, 1, 1])],
        [np.array([1, 5, 0]), np.array([9])],
        [np.array([0xA, 0xB, 0xC], np.uint16), np.array([0xD], np.uint16)])
    assert o.tolist() == [0, 3, 4]
    assert i.tolist() == [1, 5, 9, 0]
    assert v.tolist() == [0xA, 0xB, 0xD, 0xC]


@pytest.mark.parametrize("world", [2, 3, 8])
def test_merge_shards_of_row_shards_equals_the_unsharded_encode(world):
    # FSDP Shard(0): rank r holds rows [r*c, (r+1)*c) of each parameter
    # (torch.chunk sizes, so the last ranks may hold fewer rows or none).
    # Each rank encodes its slice with global positions (offset = first row x
    # row length, [verl] shard_delta_indices); merging the ranks' deltas must
    # give the encode of the whole parameters with offset 0.
    rng = np.random.default_rng(96 + world)
    shapes = [(37, 64), (5, 3), (1, 1000), (16, 16), (0, 8)]
    olds, news = [], []
    for sh in shapes:
        a = rng.integers(0, 1 << 16, sh, dtype=np.uint16)
        b = a.copy()
        m = rng.random(sh) < 0.2
        b[m] ^= np.uint16(0x0101)
        olds.append(a)
        news.append(b)
    rank_deltas = []
    for r in range(world):
        lo, hi, base = [], [], []
        for a in olds:
            rows = a.shape[0]
            c = -(-rows // world) if rows else 0
            r0, r1 = min(rows, r * c), min(rows, (r + 1) * c)
            lo.append(a[r0:r1].reshape(-1))
            base.append(r0 * (a.shape[1] if a.ndim > 1 else 1))
        for k, b in enumerate(news):
            rows = b.shape[0]
            c = -(-rows // world) if rows else 0
            r0, r1 = min(rows, r * c), min(rows, (r + 1) * c)
            hi.append(b[r0:r1].reshape(-1))
        rank_deltas.append(oracle.encode_global(lo, hi, base))
    o, i, v = oracle.merge_shards(*zip(*rank_deltas))
    wo, wi, wv = oracle.encode_global([a.reshape(-1) for a in olds], [b.reshape(-1) for b in news],
                                      [0] * len(shapes))
    np.testing.assert_array_equal(o, wo)
    np.testing.assert_array_equal(i, wi)
    np.testing.assert_array_equal(v, wv)
    assert int(o[-1]) > 100


# ---------------------------------------------------------------- byte-granular sparse XOR


def test_xor_byte_delta_golden():
    layers, offs, pos, vals, woffs, widx = G.xor_byte_delta_example()
    o, p, v = oracle.xor_byte_delta([a for a, _ in layers], [b for _, b in layers])
    assert o.tolist() == offs and p.tolist() == pos and v.tolist() == vals
    bufs = [a.copy() for a, _ in layers]
    oracle.apply_bytes(bufs, o, p, v)
    for buf, (_, b) in zip(bufs, layers):
        np.testing.assert_array_equal(buf, b)
    # the word form of the same layers (the sparse encode on 16-bit words)
    wo, wi, _ = oracle.encode([a.view(np.uint16) for a, _ in layers], [b.view(np.uint16) for _, b in layers])
    assert wo.tolist() == woffs and wi.tolist() == widx


def test_xor_byte_delta_closed_form_on_byte_layers():
    # Closed form: the generator knows which bytes it changed; the byte delta
    # lists exactly those, with the new bytes; it equals the nonzero set of
    # the dense mask; applying it to old gives new.
    old, new, pos = W.xor_layer(1, "cpu", nbytes=3_000_000, flips=2_500)
    old, new, pos = old.numpy(), new.numpy(), pos.numpy()
    o, p, v = oracle.xor_byte_delta([old], [new])
    np.testing.assert_array_equal(p, pos)
    np.testing.assert_array_equal(v, new[pos])
    np.testing.assert_array_equal(p, np.flatnonzero(oracle.xor_encode(old, new)))
    buf = old.copy()
    oracle.apply_bytes([buf], o, p, v)
    np.testing.assert_array_equal(buf, new)
    assert oracle.xor_byte_delta([old], [old])[0].tolist() == [0, 0]


@pytest.mark.parametrize("seed", [0, 1])
def test_xor_byte_delta_from_the_word_delta(seed):
    # Each word entry of the sparse encode on 16-bit words is one or two byte
    # entries (its low byte at 2i, its high byte at 2i + 1, little-endian):
    # mapping the word delta to bytes gives the byte delta (a dropped byte, a
    # swapped half or a wrong order fails it).
    rng = np.random.default_rng(700 + seed)
    sizes = [2 * int(x) for x in rng.integers(0, 3000, 6)] + [0, 2]
    olds = [rng.integers(0, 256, n, dtype=np.uint8) for n in sizes]
    news = []
    for a in olds:
        b = a.copy()
        m = rng.random(a.size) < 0.05
        b[m] = (b[m].astype(np.int32) + rng.integers(1, 256, int(m.sum()))).astype(np.uint8)
        news.append(b)
    wo, wi, wv = oracle.encode([a.view(np.uint16) for a in olds], [b.view(np.uint16) for b in news])
    o, p, v = oracle.xor_byte_delta(olds, news)
    for t, (a, b) in enumerate(zip(olds, news)):
        want_p, want_v = [], []
        for j in range(wo[t], wo[t + 1]):
            i = int(wi[j])
            for h in (0, 1):
                if a[2 * i + h] != b[2 * i + h]:
                    want_p.append(2 * i + h)
                    want_v.append((int(wv[j]) >> (8 * h)) & 0xFF)
        assert p[o[t]:o[t + 1]].tolist() == want_p
        assert v[o[t]:o[t + 1]].tolist() == want_v
    # wire size: 5 bytes per changed byte against 6 per changed word
    assert 5 * len(p) <= 6 * len(wi) * 2 and len(wi) <= len(p) <= 2 * len(wi)


def test_apply_bytes_rejects_a_position_outside_its_layer():
    buf = np.zeros(4, np.uint8)
    with pytest.raises(ValueError):
        oracle.apply_bytes([buf], np.array([0, 1]), np.array([4], np.int32), np.array([1], np.uint8))
