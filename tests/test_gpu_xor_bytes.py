"""The byte-granular sparse XOR delta (dws_xor_bytes_from_words, dws_apply_bytes)
on the GPU against the CPU oracle, element by element: random layers of
mixed sizes and densities (both bytes of a word changed, one byte, none),
the XOR workload's layers (one at its full 0.8 GB), capacity overflow, bad
word entries, and the apply's checks."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._dev import host_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _layers(rng, sizes, rate, both=0.5):
    """Byte layers (even sizes) and their new versions: each changed byte
    gets a different value; a share of the changed words change both bytes."""
    olds, news = [], []
    for n in sizes:
        a = rng.integers(0, 256, n, dtype=np.uint8)
        b = a.copy()
        if n:
            m = rng.random(n // 2) < rate
            lo = np.flatnonzero(m) * 2
            hi = lo[rng.random(lo.size) < both] + 1
            for at in (lo, hi):
                b[at] = (a[at].astype(np.int32) + rng.integers(1, 256, at.size)).astype(np.uint8)
        olds.append(a)
        news.append(b)
    return olds, news


def _dev(arrs):
    # (an empty numpy array comes through from_numpy with stride 0, which a
    # bf16 view refuses)
    return [torch.from_numpy(a).cuda() if a.size else torch.empty(0, dtype=torch.uint8, device="cuda")
            for a in arrs]


def _byte_delta(dws, olds_d, news_d, capacity=None):
    """The word encode of the layers viewed as 16-bit words, then the byte
    delta from it."""
    ow = [o.view(torch.bfloat16) for o in olds_d]
    nw = [n.view(torch.bfloat16) for n in news_d]
    plan = dws.DeltaPlan.for_tensors(ow)
    wd = plan.encode_exact(dws.ptr_table(ow), dws.ptr_table(nw))
    o, p, v = plan.xor_bytes_from_words(dws.ptr_table(ow), wd, capacity=capacity)
    return plan, wd, o, p, v


@pytest.mark.parametrize("seed,rate,both", [(0, 0.05, 0.5), (1, 0.6, 0.9), (2, 0.001, 0.0), (3, 1.0, 1.0)])
def test_byte_delta_equals_oracle(dws, seed, rate, both):
    rng = np.random.default_rng(900 + seed)
    sizes = [0, 2, 16, 8192 * 2, 8192 * 2 + 6] + [2 * int(x) for x in rng.integers(1, 40000, 7)] + [300_000]
    olds, news = _layers(rng, sizes, rate, both)
    plan, wd, o, p, v = _byte_delta(dws, _dev(olds), _dev(news))
    plan.raise_on_error()
    wo, wp, wv = oracle.xor_byte_delta(olds, news)
    n = int(wo[-1])
    np.testing.assert_array_equal(o.cpu().numpy(), wo)
    np.testing.assert_array_equal(p[:n].cpu().numpy(), wp)
    np.testing.assert_array_equal(v[:n].cpu().numpy(), wv)
    # wire: 5 bytes per changed byte against 6 per changed word
    assert wd.count <= n <= 2 * wd.count
    # apply onto the old layers gives the new ones
    bufs = _dev(olds)
    plan.apply_bytes(dws.ptr_table(bufs), o, p, v)
    plan.raise_on_error()
    for b, want in zip(bufs, news):
        np.testing.assert_array_equal(host_bytes(b), want)


def test_byte_delta_of_the_xor_workload_layers(dws):
    # Three of the XOR workload's layers at a reduced size, and the changed
    # bytes are exactly the generator's flips.
    olds, news, poss = [], [], []
    for layer in range(3):
        o, n, pos = W.xor_layer(layer, "cuda", nbytes=2_000_000, flips=1_700)
        olds.append(o)
        news.append(n)
        poss.append(pos.cpu().numpy())
    plan, wd, o, p, v = _byte_delta(dws, olds, news)
    offs = o.cpu().numpy()
    for layer in range(3):
        np.testing.assert_array_equal(p[offs[layer]:offs[layer + 1]].cpu().numpy(), poss[layer])
        np.testing.assert_array_equal(v[offs[layer]:offs[layer + 1]].cpu().numpy(),
                                      host_bytes(news[layer])[poss[layer]])


def test_byte_delta_of_a_full_size_layer(dws):
    # One layer of the XOR workload at its full size (8e8 bytes, 680,000
    # flips), in the launch configuration bench.py times.
    o_l, n_l, pos = W.xor_layer(0, "cuda")
    plan, wd, o, p, v = _byte_delta(dws, [o_l], [n_l])
    plan.raise_on_error()
    n = int(o[-1].item())
    assert n == pos.numel() == 680_000
    assert torch.equal(p[:n].to(torch.int64), pos)
    assert torch.equal(v[:n], n_l[pos])
    buf = o_l.clone()
    plan.apply_bytes(dws.ptr_table([buf]), o, p, v)
    plan.raise_on_error()
    assert torch.equal(buf, n_l)


def test_byte_delta_capacity(dws):
    rng = np.random.default_rng(950)
    olds, news = _layers(rng, [40_000, 2, 18_000], 0.2, 0.7)
    wo, wp, wv = oracle.xor_byte_delta(olds, news)
    total = int(wo[-1])
    cap = total - 123
    plan, wd, o, p, v = _byte_delta(dws, _dev(olds), _dev(news), capacity=cap)
    st, detail = plan.status()
    assert st == dws.DWS_ERR_CAPACITY and detail == total
    np.testing.assert_array_equal(o.cpu().numpy(), wo)
    np.testing.assert_array_equal(p[:cap].cpu().numpy(), wp[:cap])
    np.testing.assert_array_equal(v[:cap].cpu().numpy(), wv[:cap])


def test_byte_delta_flags_a_descending_word_entry(dws):
    rng = np.random.default_rng(960)
    olds, news = _layers(rng, [20_000], 0.1, 0.5)
    od, nd = _dev(olds), _dev(news)
    ow = [t.view(torch.bfloat16) for t in od]
    nw = [t.view(torch.bfloat16) for t in nd]
    plan = dws.DeltaPlan.for_tensors(ow)
    wd = plan.encode_exact(dws.ptr_table(ow), dws.ptr_table(nw))
    bad = wd.indices.clone()
    bad[10], bad[11] = wd.indices[11], wd.indices[10]
    wbad = dws.Delta(wd.offsets, bad, wd.values)
    plan.xor_bytes_from_words(dws.ptr_table(ow), wbad)
    st, detail = plan.status()
    assert st == dws.DWS_ERR_BAD_DELTA and detail == 11


def test_apply_bytes_checks_positions(dws):
    # A position outside its layer and a descending pair are skipped and
    # flagged; every other entry is applied.
    buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    other = torch.zeros(8, dtype=torch.uint8, device="cuda")
    plan = dws.DeltaPlan.for_tensors([buf.view(torch.bfloat16), other.view(torch.bfloat16)])
    offs = torch.tensor([0, 4, 6], dtype=torch.int64, device="cuda")
    pos = torch.tensor([1, 9, 7, 30, 3, 8], dtype=torch.int32, device="cuda")  # 7 < 9; 8 >= 8 bytes
    val = torch.tensor([11, 22, 33, 44, 55, 66], dtype=torch.uint8, device="cuda")
    plan.apply_bytes(dws.ptr_table([buf, other]), offs, pos, val)
    st, detail = plan.status()
    assert st == dws.DWS_ERR_BAD_DELTA and detail in (2, 5)
    got = buf.cpu().numpy()
    assert got[1] == 11 and got[9] == 22 and got[7] == 0 and got[30] == 44
    assert other.cpu().numpy()[3] == 55 and other.cpu().numpy().sum() == 55
