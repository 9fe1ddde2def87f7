"""libdws on the GPU against the CPU oracle, element by element.

Sizes span several 8192-element tiles with ragged tails, empty tensors,
unaligned views, thousands of tiny tensors, capacity overflow, bad deltas and
the scan's bounded wait.  Every comparison is exact (integer work)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import _golden as G
from tests._dev import assert_delta_equal, delta_to_host, dev_bits, host_bits, host_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _random_pair(rng, n, rate):
    a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
    b = a.copy()
    if n:
        m = rng.random(n) < rate
        b[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
    return a, b


def _gpu_encode(dws, olds, news, capacity=None):
    plan = dws.DeltaPlan.for_tensors(olds)
    ot, nt = dws.ptr_table(olds), dws.ptr_table(news)
    if capacity is None:
        d = plan.encode_exact(ot, nt)
    else:
        d = plan.encode(ot, nt, capacity)
    return plan, d


# ---------------------------------------------------------------- encode


def test_encode_golden_worked_example(dws):
    olds, news, offsets, indices, values = G.encode_example()
    _, d = _gpu_encode(dws, [dev_bits(a) for a in olds], [dev_bits(b) for b in news])
    assert_delta_equal(delta_to_host(d), (offsets, indices, values))


def test_encode_workload1_matches_oracle(dws):
    old, new = W.single("cuda")
    plan, d = _gpu_encode(dws, old.tensors, new.tensors)
    want = oracle.encode([host_bits(old.tensors[0])], [host_bits(new.tensors[0])])
    assert_delta_equal(delta_to_host(d), want)
    assert 0 < want[0][-1] < old.total


@pytest.mark.parametrize("seed", [0, 1])
def test_encode_ragged_sizes_and_rates(dws, seed):
    rng = np.random.default_rng(100 + seed)
    sizes = [0, 1, 7, 8, 9, 8191, 8192, 8193, 3 * 8192 + 5, 100_003, 0, 65_536, 2, 40_000]
    rates = [0.0, 0.01, 0.3, 1.0, 0.035]
    pairs = [_random_pair(rng, n, rates[i % len(rates)]) for i, n in enumerate(sizes)]
    olds = [dev_bits(a) for a, _ in pairs]
    news = [dev_bits(b) for _, b in pairs]
    plan, d = _gpu_encode(dws, olds, news)
    want = oracle.encode([a for a, _ in pairs], [b for _, b in pairs])
    assert_delta_equal(delta_to_host(d), want)
    # dws_count alone gives the same offsets
    offs = plan.count(dws.ptr_table(olds), dws.ptr_table(news))
    plan.raise_on_error()
    np.testing.assert_array_equal(offs.cpu().numpy(), want[0])


def test_encode_unaligned_views(dws):
    # Views starting 1, 3, 5 elements into a buffer (2-byte but not 16-byte
    # aligned), with old and new misaligned differently: the plain-load path.
    rng = np.random.default_rng(5)
    olds, news, ha, hb = [], [], [], []
    for k, (n, oa, ob) in enumerate([(20_000, 1, 3), (8192 * 2 + 3, 5, 5), (17, 2, 0), (9000, 0, 7)]):
        a, b = _random_pair(rng, n, 0.05 * (k + 1))
        base_a = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
        base_b = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
        va, vb = base_a[oa:oa + n], base_b[ob:ob + n]
        va.copy_(dev_bits(a))
        vb.copy_(dev_bits(b))
        olds.append(va)
        news.append(vb)
        ha.append(a)
        hb.append(b)
    _, d = _gpu_encode(dws, olds, news)
    assert_delta_equal(delta_to_host(d), oracle.encode(ha, hb))


def test_encode_many_tiny_tensors(dws):
    # 3000 tensors, most of them a single short tile: thousands of tickets
    # and look-backs across tiles with counts of 0..40.
    rng = np.random.default_rng(17)
    sizes = rng.integers(0, 41, 3000)
    pairs = [_random_pair(rng, int(n), 0.2) for n in sizes]
    olds = [dev_bits(a) for a, _ in pairs]
    news = [dev_bits(b) for _, b in pairs]
    _, d = _gpu_encode(dws, olds, news)
    assert_delta_equal(delta_to_host(d), oracle.encode([a for a, _ in pairs], [b for _, b in pairs]))


def test_encode_capacity_overflow_reports_required_nnz(dws):
    rng = np.random.default_rng(23)
    pairs = [_random_pair(rng, n, 0.1) for n in (50_000, 30_001, 0, 8192)]
    olds = [dev_bits(a) for a, _ in pairs]
    news = [dev_bits(b) for _, b in pairs]
    want = oracle.encode([a for a, _ in pairs], [b for _, b in pairs])
    nnz = int(want[0][-1])
    cap = nnz // 2
    plan = dws.DeltaPlan.for_tensors(olds)
    offsets = torch.empty(len(olds) + 1, dtype=torch.int64, device="cuda")
    idx = torch.full((cap + 64,), -7, dtype=torch.int32, device="cuda")
    val = torch.full((cap + 64,), -7, dtype=torch.int16, device="cuda")
    # keep the pointer tables alive until the kernel has run
    ot, nt = dws.ptr_table(olds), dws.ptr_table(news)
    code = dws.dws_encode(plan.handle, ot.data_ptr(), nt.data_ptr(),
                          offsets.data_ptr(), idx.data_ptr(), val.data_ptr(), cap,
                          plan.workspace.data_ptr(), plan.workspace_bytes,
                          torch.cuda.current_stream().cuda_stream)
    assert code == dws.DWS_OK
    st, detail = plan.status()
    assert st == dws.DWS_ERR_CAPACITY and detail == nnz
    np.testing.assert_array_equal(offsets.cpu().numpy(), want[0])
    np.testing.assert_array_equal(idx[:cap].cpu().numpy(), want[1][:cap])
    np.testing.assert_array_equal(val[:cap].cpu().numpy().view(np.uint16), want[2][:cap])
    assert (idx[cap:].cpu().numpy() == -7).all() and (val[cap:].cpu().numpy() == -7).all()


@pytest.mark.parametrize("shift", [1, 2, 3])
def test_encode_into_unaligned_outputs(dws, shift):
    # indices / values views that start 1-3 entries into their buffers (not
    # 16- / 8-byte aligned): entries leave one at a time.  Clustered runs of
    # changes make some tiles dense.
    rng = np.random.default_rng(37 + shift)
    sizes = (50_000, 8192 * 3 + 5, 1, 4096)
    hs, hn = [], []
    for n in sizes:
        a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
        b = a.copy()
        m = rng.random(n) < 0.05
        if n > 5000:
            m[1000:5000] = True
        b[m] ^= np.uint16(0x0100)
        hs.append(a)
        hn.append(b)
    want = oracle.encode(hs, hn)
    nnz = int(want[0][-1])
    olds, news = [dev_bits(a) for a in hs], [dev_bits(b) for b in hn]
    plan = dws.DeltaPlan.for_tensors(olds)
    offsets = torch.empty(len(olds) + 1, dtype=torch.int64, device="cuda")
    ib = torch.full((nnz + 8,), -7, dtype=torch.int32, device="cuda")
    vb = torch.full((nnz + 8,), -7, dtype=torch.int16, device="cuda")
    idx, val = ib[shift:shift + nnz], vb[shift:shift + nnz]
    ot, nt = dws.ptr_table(olds), dws.ptr_table(news)
    plan.encode_into(ot, nt, offsets, idx, val)
    plan.raise_on_error()
    np.testing.assert_array_equal(offsets.cpu().numpy(), want[0])
    np.testing.assert_array_equal(idx.cpu().numpy(), want[1])
    np.testing.assert_array_equal(val.cpu().numpy().view(np.uint16), want[2])
    assert (ib[:shift].cpu().numpy() == -7).all() and (ib[shift + nnz:].cpu().numpy() == -7).all()


def test_encode_reports_nnz_to_device_and_pinned_host(dws):
    # The entry count arrives in a device scalar and a pinned host scalar
    # after the encode, on the encode's stream, equal to the oracle's.
    rng = np.random.default_rng(91)
    pairs = [_random_pair(rng, n, 0.05) for n in (0, 7, 8192 * 3 + 11, 70000)]
    olds = [dev_bits(a) for a, _ in pairs]
    news = [dev_bits(b) for _, b in pairs]
    want = oracle.encode([a for a, _ in pairs], [b for _, b in pairs])
    plan = dws.DeltaPlan.for_tensors(olds)
    cap = int(want[0][-1]) + 5
    offsets = torch.empty(len(pairs) + 1, dtype=torch.int64, device="cuda")
    indices = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    values = torch.full((cap,), -1, dtype=torch.int16, device="cuda")
    nnz_dev = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    nnz_host = torch.full((1,), -1, dtype=torch.int64).pin_memory()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        plan.encode_into_nnz(dws.ptr_table(olds), dws.ptr_table(news), offsets, indices, values,
                             nnz_dev=nnz_dev, nnz_host=nnz_host, stream=s)
    s.synchronize()
    plan.raise_on_error("dws_encode_nnz")
    assert int(nnz_host[0]) == int(nnz_dev.item()) == int(want[0][-1])
    nnz = int(want[0][-1])
    assert_delta_equal((offsets.cpu().numpy(), indices[:nnz].cpu().numpy(),
                        values[:nnz].cpu().numpy().view(np.uint16)), want)
    # either output may be left out
    plan.encode_into_nnz(dws.ptr_table(olds), dws.ptr_table(news), offsets, indices, values)
    torch.cuda.synchronize()
    plan.raise_on_error("dws_encode_nnz")


def test_encode_identical_and_all_changed(dws):
    rng = np.random.default_rng(29)
    a = rng.integers(0, 1 << 16, 1_000_003, dtype=np.uint16)
    t = dev_bits(a)
    _, d = _gpu_encode(dws, [t], [t.clone()])
    assert d.nnz() == 0 and d.count == 0
    b = a ^ np.uint16(0x0001)
    _, d = _gpu_encode(dws, [t], [dev_bits(b)])
    assert_delta_equal(delta_to_host(d), oracle.encode([a], [b]))
    assert d.nnz() == a.size


def test_encode_reuses_workspace_across_calls(dws):
    rng = np.random.default_rng(31)
    a1, b1 = _random_pair(rng, 70_000, 0.02)
    a2, b2 = _random_pair(rng, 70_000, 0.4)
    plan = dws.DeltaPlan([70_000])
    for a, b in ((a1, b1), (a2, b2), (a1, b1)):
        ot, nt = dws.ptr_table([dev_bits(a)]), dws.ptr_table([dev_bits(b)])
        d = plan.encode_exact(ot, nt)
        assert_delta_equal(delta_to_host(d), oracle.encode([a], [b]))


def test_encode_timeout_is_reported_and_context_survives(dws):
    # Tile 1 never publishes its count; tile 2's bounded wait runs out after
    # 50 ms, the kernel records DWS_ERR_TIMEOUT, every waiter leaves, and the
    # context stays usable for the next call.
    rng = np.random.default_rng(37)
    a, b = _random_pair(rng, 8192 * 6 + 100, 0.05)
    olds, news = [dev_bits(a)], [dev_bits(b)]
    plan = dws.DeltaPlan.for_tensors(olds)
    cap = a.size
    offsets = torch.zeros(2, dtype=torch.int64, device="cuda")
    idx = torch.empty(cap, dtype=torch.int32, device="cuda")
    val = torch.empty(cap, dtype=torch.int16, device="cuda")
    ot, nt = dws.ptr_table(olds), dws.ptr_table(news)
    code = dws.dws_encode_ex(plan.handle, ot.data_ptr(), nt.data_ptr(), offsets.data_ptr(),
                             idx.data_ptr(), val.data_ptr(), cap, plan.workspace.data_ptr(),
                             plan.workspace_bytes, torch.cuda.current_stream().cuda_stream,
                             50_000_000, 1)
    assert code == dws.DWS_OK
    st, detail = plan.status()
    assert st == dws.DWS_ERR_TIMEOUT and detail >= 2
    d = plan.encode_exact(ot, nt)
    assert_delta_equal(delta_to_host(d), oracle.encode([a], [b]))


def test_workspace_of_another_plan_is_refused(dws):
    rng = np.random.default_rng(41)
    a, b = _random_pair(rng, 1000, 0.5)
    plan_a = dws.DeltaPlan([1000])
    plan_b = dws.DeltaPlan([999, 1])
    ot, nt = dws.ptr_table([dev_bits(a)]), dws.ptr_table([dev_bits(b)])
    offsets = torch.full((2,), -3, dtype=torch.int64, device="cuda")
    idx = torch.full((1000,), -3, dtype=torch.int32, device="cuda")
    val = torch.full((1000,), -3, dtype=torch.int16, device="cuda")
    # plan_a's call with plan_b's (large enough) workspace
    assert plan_b.workspace_bytes >= plan_a.workspace_bytes
    code = dws.dws_encode(plan_a.handle, ot.data_ptr(), nt.data_ptr(), offsets.data_ptr(),
                          idx.data_ptr(), val.data_ptr(), 1000, plan_b.workspace.data_ptr(),
                          plan_b.workspace_bytes, torch.cuda.current_stream().cuda_stream)
    assert code == dws.DWS_OK
    st, _ = plan_b.status()
    assert st == dws.DWS_ERR_WORKSPACE
    assert (offsets.cpu().numpy() == -3).all() and (idx.cpu().numpy() == -3).all()


# ---------------------------------------------------------------- apply


def _guarded(a: np.ndarray, guard=64):
    """Device copy of a with guard elements (0x5a5a) on both sides."""
    base = torch.full((a.size + 2 * guard,), 0x5a5a, dtype=torch.int16, device="cuda")
    base[guard:guard + a.size] = torch.from_numpy(a.view(np.int16).copy()).cuda()
    return base, base[guard:guard + a.size].view(torch.bfloat16)


def _guards_intact(base, n, guard=64):
    h = base.cpu().numpy()
    return (h[:guard] == 0x5a5a).all() and (h[guard + n:] == 0x5a5a).all()


def test_apply_roundtrip_leaves_unchanged_positions(dws):
    rng = np.random.default_rng(43)
    sizes = [30_000, 0, 8192 * 3 + 1, 5, 100_000]
    pairs = [_random_pair(rng, n, 0.03) for n in sizes]
    olds = [dev_bits(a) for a, _ in pairs]
    news = [dev_bits(b) for _, b in pairs]
    plan, d = _gpu_encode(dws, olds, news)
    snaps = [_guarded(a) for a, _ in pairs]
    plan.apply(dws.ptr_table([s for _, s in snaps]), d)
    plan.raise_on_error("apply")
    for (base, s), (a, b) in zip(snaps, pairs):
        np.testing.assert_array_equal(host_bits(s), b)
        assert _guards_intact(base, a.size)


def test_apply_empty_delta_is_identity(dws):
    a = np.arange(5000, dtype=np.uint16)
    t = dev_bits(a)
    plan, d = _gpu_encode(dws, [t], [t.clone()])
    snap = t.clone()
    plan.apply(dws.ptr_table([snap]), d)
    plan.raise_on_error()
    np.testing.assert_array_equal(host_bits(snap), a)


def test_apply_rejects_out_of_range_and_unsorted_entries(dws):
    n = 1000
    plan = dws.DeltaPlan([n])
    base, snap = _guarded(np.zeros(n, np.uint16))
    for idx in ([5, n], [5, -1], [7, 7], [9, 3]):
        offsets = torch.tensor([0, 2], dtype=torch.int64, device="cuda")
        indices = torch.tensor(idx, dtype=torch.int32, device="cuda")
        values = torch.tensor([0x1111, 0x2222], dtype=torch.int16, device="cuda")
        plan.apply(dws.ptr_table([snap]), dws.Delta(offsets, indices, values))
        st, detail = plan.status()
        assert st == dws.DWS_ERR_BAD_DELTA and detail == 1, idx
        assert _guards_intact(base, n)


def test_apply_with_bad_offsets_writes_nothing(dws):
    n = 1000
    plan = dws.DeltaPlan([n, n])
    snaps = [dev_bits(np.zeros(n, np.uint16)) for _ in range(2)]
    for offs in ([0, 3, 2], [1, 2, 3], [0, 2, 9]):
        offsets = torch.tensor(offs, dtype=torch.int64, device="cuda")
        indices = torch.tensor([1, 2, 3], dtype=torch.int32, device="cuda")
        values = torch.tensor([1, 1, 1], dtype=torch.int16, device="cuda")
        plan.apply(dws.ptr_table(snaps), dws.Delta(offsets, indices, values))
        st, _ = plan.status()
        assert st == dws.DWS_ERR_BAD_DELTA, offs
        assert all(int(s.view(torch.int16).abs().sum()) == 0 for s in snaps)


# ---------------------------------------------------------------- chain

# Both replay modes of dws_apply_chain_ex must give the sequential replay.
CHAIN_MODES = pytest.mark.parametrize("mode", [0, 1, 2], ids=["auto", "tile_merge", "scatter"])


@CHAIN_MODES
def test_chain_golden_later_delta_wins(dws, mode):
    anchor, deltas, final = G.chain_example()
    snaps = [dev_bits(a) for a in anchor]
    plan = dws.DeltaPlan.for_tensors(snaps)
    dd = [dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                    torch.from_numpy(v.view(np.int16)).cuda()) for o, i, v in deltas]
    plan.apply_chain(dws.ptr_table(snaps), dd, mode=mode)
    plan.raise_on_error()
    for s, f in zip(snaps, final):
        np.testing.assert_array_equal(host_bits(s), f)


def _chain_case(dws, shapes_or_sizes, steps, stepper, anchor_set, modes=(1, 2)):
    """Encode `steps` steps on the GPU (each delta checked against the oracle),
    replay them in one chain launch onto a copy of the anchor."""
    prev = anchor_set
    plan = dws.DeltaPlan.for_tensors(prev.tensors)
    deltas, host_deltas = [], []
    prev_h = [host_bits(t) for t in prev.tensors]
    for k in range(1, steps + 1):
        cur = stepper(prev, k)
        d = plan.encode_exact(dws.ptr_table(prev.tensors), dws.ptr_table(cur.tensors))
        cur_h = [host_bits(t) for t in cur.tensors]
        want = oracle.encode(prev_h, cur_h)
        assert_delta_equal(delta_to_host(d), want)
        deltas.append(d)
        host_deltas.append(want)
        prev, prev_h = cur, cur_h
    ref = [host_bits(t) for t in anchor_set.tensors]
    oracle.apply_chain(ref, host_deltas)
    for mode in modes:
        snaps = [t.clone() for t in anchor_set.tensors]
        plan.apply_chain(dws.ptr_table(snaps), deltas, mode=mode)
        plan.raise_on_error("apply_chain")
        for s, r, f in zip(snaps, ref, prev_h):
            np.testing.assert_array_equal(host_bits(s), r)
            np.testing.assert_array_equal(r, f)


def test_chain_qwen_shaped_scaled_ten_steps(dws):
    s = W.SEEDS["qwen3_0p6b"]
    shapes = W.scaled_shapes(W.qwen3_0p6b_shapes(), 8)
    w0 = W.init_set(shapes, s, "cuda", 0.02)
    _chain_case(dws, shapes, 10, lambda w, k: W.step_set(w, s, k, 3e-6, "cuda"), w0)


def test_chain_stress_scaled_ten_steps(dws):
    sizes = W.stress_sizes(count=300, lo=16, hi=300_000)
    clustered = W.stress_clustered(count=300)
    w0 = W.stress_init(sizes, "cuda")
    _chain_case(dws, sizes, 10, lambda w, k: W.stress_step(w, clustered, k, "cuda")[0], w0)


@CHAIN_MODES
def test_chain_on_unaligned_snapshots(dws, mode):
    # Snapshot views that are not 16-byte aligned take the direct-store path.
    rng = np.random.default_rng(47)
    n = 8192 * 2 + 77
    anchor = rng.integers(0, 1 << 16, n, dtype=np.uint16)
    cur = anchor.copy()
    host_deltas = []
    for k in range(4):
        nxt = cur.copy()
        m = rng.random(n) < 0.2
        nxt[m] ^= np.uint16(0x0101 + k)
        host_deltas.append(oracle.encode([cur], [nxt]))
        cur = nxt
    base = torch.zeros(n + 8, dtype=torch.bfloat16, device="cuda")
    snap = base[3:3 + n]
    snap.copy_(dev_bits(anchor))
    plan = dws.DeltaPlan([n])
    dd = [dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                    torch.from_numpy(v.view(np.int16)).cuda()) for o, i, v in host_deltas]
    plan.apply_chain(dws.ptr_table([snap]), dd, mode=mode)
    plan.raise_on_error()
    np.testing.assert_array_equal(host_bits(snap), cur)


@CHAIN_MODES
def test_chain_max_length_tiny_and_empty_tensors(dws, mode):
    # 64 deltas (the maximum) of mixed densities, one of them empty, over a
    # plan of many tiny tensors, empty tensors and a few multi-tile ones, so
    # that index blocks cut through tensors and hold many of them.
    rng = np.random.default_rng(64)
    sizes = [0, 1, 5, 0, 8191, 8192, 8193, 3] + [int(x) for x in rng.integers(1, 600, 120)] + \
            [3 * 8192 + 17, 0, 300_001, 2, 70_000]
    anchor = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    cur = [a.copy() for a in anchor]
    host_deltas = []
    for k in range(64):
        rate = [0.0, 0.001, 0.02, 0.3, 0.9][k % 5]
        nxt = []
        for c in cur:
            x = c.copy()
            if c.size:
                m = rng.random(c.size) < rate
                x[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
            nxt.append(x)
        host_deltas.append(oracle.encode(cur, nxt))
        cur = nxt
    ref = [a.copy() for a in anchor]
    oracle.apply_chain(ref, host_deltas)
    for r, c in zip(ref, cur):
        np.testing.assert_array_equal(r, c)
    snaps = [dev_bits(a) for a in anchor]
    plan = dws.DeltaPlan(sizes)
    dd = [dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                    torch.from_numpy(v.view(np.int16)).cuda()) for o, i, v in host_deltas]
    plan.apply_chain(dws.ptr_table(snaps), dd, mode=mode)
    plan.raise_on_error()
    for s, c in zip(snaps, cur):
        np.testing.assert_array_equal(host_bits(s), c)


def _host_chain(rng, sizes, rates, K):
    """An anchor and K consecutive random steps (per-delta rates cycled),
    with the oracle's deltas and the final snapshot."""
    anchor = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    cur = [a.copy() for a in anchor]
    host_deltas = []
    for k in range(K):
        rate = rates[k % len(rates)]
        nxt = []
        for c in cur:
            x = c.copy()
            if c.size:
                m = rng.random(c.size) < rate
                x[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
            nxt.append(x)
        host_deltas.append(oracle.encode(cur, nxt))
        cur = nxt
    return anchor, host_deltas, cur


@CHAIN_MODES
@pytest.mark.parametrize("ishift,vshift", [(1, 3), (3, 1), (2, 0)])
def test_chain_on_unaligned_delta_arrays(dws, mode, ishift, vshift):
    # Index and value arrays that start 4/8/12 and 2/6 bytes past a 16-byte
    # boundary: the staged middles, the heads and tails read from global
    # memory, and the index pass's scalar loads.
    rng = np.random.default_rng(90 + 7 * ishift + vshift)
    sizes = [8192 * 5 + 11, 3000, 8192 * 2]
    anchor, host_deltas, final = _host_chain(rng, sizes, [0.05, 0.4, 0.01], 5)
    dd = []
    for o, i, v in host_deltas:
        ib = torch.zeros(i.size + 8, dtype=torch.int32, device="cuda")
        vb = torch.zeros(v.size + 8, dtype=torch.int16, device="cuda")
        ib[ishift:ishift + i.size] = torch.from_numpy(i).cuda()
        vb[vshift:vshift + v.size] = torch.from_numpy(v.view(np.int16)).cuda()
        dd.append(dws.Delta(torch.from_numpy(o).cuda(), ib[ishift:ishift + i.size],
                            vb[vshift:vshift + v.size]))
    plan = dws.DeltaPlan(sizes)
    snaps = [dev_bits(a) for a in anchor]
    plan.apply_chain(dws.ptr_table(snaps), dd, mode=mode)
    plan.raise_on_error()
    for s_, f in zip(snaps, final):
        np.testing.assert_array_equal(host_bits(s_), f)


@CHAIN_MODES
def test_chain_denser_than_a_stage_holds(dws, mode):
    # Every element changed by every delta: a tile's entries (8192 per delta)
    # exceed what one merge stage holds, so part of them is read straight
    # from global memory; then the same with one sparse delta in between.
    rng = np.random.default_rng(91)
    sizes = [8192 * 6 + 5, 100]
    for rates in ([1.0], [1.0, 0.001, 0.9]):
        anchor, host_deltas, final = _host_chain(rng, sizes, rates, 4)
        dd = [dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                        torch.from_numpy(v.view(np.int16)).cuda()) for o, i, v in host_deltas]
        plan = dws.DeltaPlan(sizes)
        snaps = [dev_bits(a) for a in anchor]
        plan.apply_chain(dws.ptr_table(snaps), dd, mode=mode)
        plan.raise_on_error()
        for s_, f in zip(snaps, final):
            np.testing.assert_array_equal(host_bits(s_), f)


@CHAIN_MODES
def test_chain_of_single_entries_over_many_tiles(dws, mode):
    # Deltas of one entry each in a plan of thousands of tiles: the tile
    # index's long runs of rows pointing at the same entry.
    sizes = [8192 * 3000 + 1, 5, 8192 * 10]
    rng = np.random.default_rng(92)
    anchor = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    host_deltas, cur = [], [a.copy() for a in anchor]
    for t, i in ((0, 8192 * 2999 + 7), (2, 3), (0, 0), (1, 4)):
        nxt = [c.copy() for c in cur]
        nxt[t][i] ^= np.uint16(0x0102)
        host_deltas.append(oracle.encode(cur, nxt))
        cur = nxt
    dd = [dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                    torch.from_numpy(v.view(np.int16)).cuda()) for o, i, v in host_deltas]
    plan = dws.DeltaPlan(sizes)
    snaps = [dev_bits(a) for a in anchor]
    plan.apply_chain(dws.ptr_table(snaps), dd, mode=mode)
    plan.raise_on_error()
    for s_, f in zip(snaps, cur):
        np.testing.assert_array_equal(host_bits(s_), f)


@CHAIN_MODES
def test_chain_single_delta_equals_apply(dws, mode):
    rng = np.random.default_rng(65)
    sizes = [40_000, 8192 * 40 + 3, 1]
    a = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    b = []
    for x in a:
        y = x.copy()
        m = rng.random(x.size) < 0.05
        y[m] ^= np.uint16(0x8001)
        b.append(y)
    o, i, v = oracle.encode(a, b)
    d = dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                  torch.from_numpy(v.view(np.int16)).cuda())
    plan = dws.DeltaPlan(sizes)
    snaps = [dev_bits(x) for x in a]
    plan.apply_chain(dws.ptr_table(snaps), [d], mode=mode)
    plan.raise_on_error()
    for s, y in zip(snaps, b):
        np.testing.assert_array_equal(host_bits(s), y)


@CHAIN_MODES
def test_chain_rejects_index_beyond_numel(dws, mode):
    n = 9000
    plan = dws.DeltaPlan([n])
    snap = dev_bits(np.zeros(n, np.uint16))
    d = dws.Delta(torch.tensor([0, 2], dtype=torch.int64, device="cuda"),
                  torch.tensor([3, n + 5], dtype=torch.int32, device="cuda"),
                  torch.tensor([7, 7], dtype=torch.int16, device="cuda"))
    plan.apply_chain(dws.ptr_table([snap]), [d], mode=mode)
    st, detail = plan.status()
    assert st == dws.DWS_ERR_BAD_DELTA and detail == 1
    assert host_bits(snap).sum() == 0  # a chain with a bad entry writes nothing


@CHAIN_MODES
def test_chain_rejects_negative_index(dws, mode):
    n = 9000
    plan = dws.DeltaPlan([n])
    snap = dev_bits(np.zeros(n, np.uint16))
    d = dws.Delta(torch.tensor([0, 2], dtype=torch.int64, device="cuda"),
                  torch.tensor([-4, 11], dtype=torch.int32, device="cuda"),
                  torch.tensor([7, 7], dtype=torch.int16, device="cuda"))
    plan.apply_chain(dws.ptr_table([snap]), [d], mode=mode)
    st, detail = plan.status()
    assert st == dws.DWS_ERR_BAD_DELTA and detail == 0
    assert host_bits(snap).sum() == 0  # a chain with a bad entry writes nothing


# ---------------------------------------------------------------- sparse delta of XOR layers


def test_sparse_delta_of_packed_byte_layers(dws):
    # Packed low-precision layers (bytes) encoded as a sparse delta of 16-bit
    # words: the changed words are exactly the words holding the generator's
    # flipped bytes, the values are the new words, and applying the delta to
    # the old layers gives the new ones.
    nb = 1_000_002
    olds, news, poss = [], [], []
    for l in range(3):
        o, n, pos = W.xor_layer(l, "cuda", nbytes=nb, flips=850)
        olds.append(o)
        news.append(n)
        poss.append(pos)
    ow = [o.view(torch.bfloat16) for o in olds]
    nw = [n.view(torch.bfloat16) for n in news]
    plan = dws.DeltaPlan.for_tensors(ow)
    d = plan.encode_exact(dws.ptr_table(ow), dws.ptr_table(nw))
    offs = d.offsets.cpu().numpy()
    for l in range(3):
        words = torch.unique(poss[l] // 2).cpu().numpy()
        np.testing.assert_array_equal(d.indices[offs[l]:offs[l + 1]].cpu().numpy(), words)
    want = oracle.encode([host_bits(t) for t in ow], [host_bits(t) for t in nw])
    assert_delta_equal(delta_to_host(d), want)
    snaps = [o.clone() for o in olds]
    plan.apply(dws.ptr_table([t.view(torch.bfloat16) for t in snaps]), d)
    plan.raise_on_error()
    for t, n in zip(snaps, news):
        assert torch.equal(t, n)


# ---------------------------------------------------------------- XOR


@pytest.mark.parametrize("n,oa,ob,oc", [(0, 0, 0, 0), (1, 0, 0, 0), (15, 3, 3, 3), (16, 0, 0, 0),
                                        (17, 1, 1, 1), (1_000_003, 5, 5, 5), (100_001, 1, 2, 3),
                                        (4096 * 64 + 9, 0, 8, 0)])
def test_xor_encode_apply_alignments(dws, n, oa, ob, oc):
    rng = np.random.default_rng(n + oa)
    a = rng.integers(0, 256, n, dtype=np.uint8)
    b = a.copy()
    if n:
        m = rng.random(n) < 0.3
        b[m] = rng.integers(0, 256, int(m.sum()), dtype=np.uint8)
    ba = torch.zeros(n + 32, dtype=torch.uint8, device="cuda")
    bb = torch.zeros(n + 32, dtype=torch.uint8, device="cuda")
    bc = torch.full((n + 32,), 0xAB, dtype=torch.uint8, device="cuda")
    va, vb, vc = ba[oa:oa + n], bb[ob:ob + n], bc[oc:oc + n]
    va.copy_(torch.from_numpy(a))
    vb.copy_(torch.from_numpy(b))
    dws.xor_encode(va, vb, vc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bytes(vc), oracle.xor_encode(a, b))
    h = bc.cpu().numpy()
    assert (h[:oc] == 0xAB).all() and (h[oc + n:] == 0xAB).all()
    dws.xor_apply(va, vc)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bytes(va), b)


def test_xor_layer_closed_form(dws):
    old, new, pos = W.xor_layer(2, "cuda", nbytes=3_000_017, flips=2_550)
    mask = dws.xor_encode(old, new)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(np.flatnonzero(host_bytes(mask)), pos.cpu().numpy())
    buf = old.clone()
    dws.xor_apply(buf, mask)
    torch.cuda.synchronize()
    assert torch.equal(buf, new)


@pytest.mark.parametrize("pinned_masks", [False, True])
def test_xor_apply_layers_double_buffered(dws, pinned_masks):
    sizes = [1_000_000, 333_333, 2_500_001, 16, 0, 777_777]
    olds, news, masks = [], [], []
    for l, n in enumerate(sizes):
        o, nw, _ = W.xor_layer(l, "cuda", nbytes=max(n, 1), flips=max(1, n // 1000))
        o, nw = o[:n], nw[:n]
        olds.append(o.clone())
        news.append(nw)
        m = dws.xor_encode(o, nw) if n else torch.empty(0, dtype=torch.uint8, device="cuda")
        masks.append(m.cpu().pin_memory() if pinned_masks else m)
    torch.cuda.synchronize()
    staging = [torch.empty(600_000, dtype=torch.uint8, device="cuda") for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    dws.xor_apply_layers(olds, masks, staging[0], staging[1],
                         apply_stream=torch.cuda.current_stream(), copy_stream=copy_stream)
    torch.cuda.current_stream().synchronize()
    for o, nw in zip(olds, news):
        assert torch.equal(o, nw)


# ---------------------------------------------------------------- malformed deltas


def _malformed_chain(rng, sizes):
    """Three deltas over `sizes` (dws layout, host arrays) and, for each, the
    mask of its entries that the pairwise rule flags: delta 0 holds descending
    pairs (one inside a tile, one across adjacent tiles, one across distant tiles),
    delta 1 repeated indices, delta 2 is well formed.  Each flagged entry is
    followed by one above the entry before it, so no later entry of the
    segment lies at or below an earlier one except the flagged ones."""
    deltas, flags = [], []
    for k in range(3):
        offs, idx, val, bad = [0], [], [], []
        for t, n in enumerate(sizes):
            pos = np.sort(rng.choice(n, min(n, max(1, n // 40)), replace=False)).astype(np.int64)
            pos = list(pos)
            b = [False] * len(pos)
            if k == 0 and t == 1:
                # insert b < a right after a, then continue above a
                # the third pair reaches two tiles back (tensor 1's local
                # tiles 25 and 23)
                for a_at in (8195, 9000, 25 * 8192 + 10):
                    a_i = next(i for i, x in enumerate(pos) if x >= a_at)
                    below = pos[a_i] - (7 if a_at == 8195 else (5000 if a_at == 9000 else 8192 * 2))
                    if a_i + 1 < len(pos) and pos[a_i + 1] > pos[a_i] + 1:
                        pos.insert(a_i + 1, below)
                        b.insert(a_i + 1, True)
            if k == 1 and len(pos) > 4:
                for dup_at in (1, len(pos) // 2, len(pos) - 2):
                    pos.insert(dup_at + 1, pos[dup_at])
                    b.insert(dup_at + 1, True)
            idx += pos
            bad += b
            val += list(rng.integers(0, 1 << 16, len(pos), dtype=np.uint16))
            offs.append(offs[-1] + len(pos))
        deltas.append((np.array(offs, np.int64), np.array(idx, np.int32), np.array(val, np.uint16)))
        flags.append(np.array(bad, bool))
    return deltas, flags


def test_chain_with_unordered_or_repeated_entries_writes_nothing_in_every_mode(dws):
    # Descending pairs (inside a tile, across adjacent tiles, across distant tiles)
    # and repeated indices: every mode records DWS_ERR_BAD_DELTA and leaves
    # the snapshot exactly as it was; dws_apply, one delta at a time, skips
    # the flagged entries and applies the rest; without the malformed deltas
    # the chain is applied.
    rng = np.random.default_rng(77)
    sizes = [50_000, 8192 * 40 + 3, 7, 20_000]
    deltas, flags = _malformed_chain(rng, sizes)
    assert flags[0].sum() >= 3 and flags[1].sum() >= 3 and not flags[2].any()
    anchor = [rng.integers(0, 1 << 16, n, dtype=np.uint16) for n in sizes]
    valid = []
    for (o, i, v), f in zip(deltas, flags):
        keep = ~f
        t_of = np.repeat(np.arange(len(sizes)), np.diff(o))
        vo = np.concatenate([[0], np.cumsum(np.bincount(t_of[keep], minlength=len(sizes)))])
        valid.append((vo.astype(np.int64), i[keep], v[keep]))
    ref = [a.copy() for a in anchor]
    oracle.apply_chain(ref, valid)

    def dev(o, i, v):
        return dws.Delta(torch.from_numpy(o).cuda(), torch.from_numpy(i).cuda(),
                         torch.from_numpy(v.view(np.int16)).cuda())

    plan = dws.DeltaPlan(sizes)
    dd = [dev(*d) for d in deltas]
    for mode in (0, 1, 2):
        for chain in (dd, [dd[2], dd[0]], [dd[1]], dd * 6):  # 18 deltas: two passes
            snaps = [dev_bits(a) for a in anchor]
            plan.apply_chain(dws.ptr_table(snaps), chain, mode=mode)
            st, _ = plan.status()
            assert st == dws.DWS_ERR_BAD_DELTA, (mode, len(chain))
            for s, a in zip(snaps, anchor):
                np.testing.assert_array_equal(host_bits(s), a)
    # three sequential dws_apply calls skip the flagged entries
    snaps = [dev_bits(a) for a in anchor]
    for d in dd:
        plan.apply(dws.ptr_table(snaps), d)
    st, _ = plan.status()
    assert st == dws.DWS_ERR_BAD_DELTA
    for s, r in zip(snaps, ref):
        np.testing.assert_array_equal(host_bits(s), r)
    # the well-formed parts replay as the oracle says, in every mode
    vd = [dev(*v) for v in valid]
    for mode in (0, 1, 2):
        snaps = [dev_bits(a) for a in anchor]
        plan.apply_chain(dws.ptr_table(snaps), vd, mode=mode)
        assert plan.status()[0] == dws.DWS_OK
        for s, r in zip(snaps, ref):
            np.testing.assert_array_equal(host_bits(s), r)
