"""dws_merge_shards (rank 0's split-and-concatenate of gathered shard deltas)
on the GPU against the CPU oracle, element by element.  The ranks are
simulated on one GPU: each shard is encoded with dws_encode_global, the
buffers are padded and stacked as the gather leaves them on rank 0."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests._dev import dev_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _params(rng, shapes, rate):
    olds, news = [], []
    for sh in shapes:
        a = rng.integers(0, 1 << 16, sh, dtype=np.uint16)
        b = a.copy()
        m = rng.random(sh) < rate
        b[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
        if sh[0] > 40:
            b[3:7] ^= np.uint16(1)  # a dense run of rows inside rank 0's slice
        olds.append(a)
        news.append(b)
    return olds, news


def _shard_deltas(dws, olds, news, world):
    """Each simulated rank encodes its Shard(0) rows with global positions on
    the GPU; returns the stacked gathered buffers (offsets, padded indices,
    padded values) and the ranks' host deltas."""
    deltas = []
    for r in range(world):
        lo, hi, base = [], [], []
        for a, b in zip(olds, news):
            rows = a.shape[0]
            c = -(-rows // world) if rows else 0
            r0, r1 = min(rows, r * c), min(rows, (r + 1) * c)
            lo.append(dev_bits(a[r0:r1].reshape(-1)))
            hi.append(dev_bits(b[r0:r1].reshape(-1)))
            base.append(r0 * a.shape[1])
        plan = dws.DeltaPlan([t.numel() for t in lo])
        d = plan.encode_global(dws.ptr_table(lo), dws.ptr_table(hi),
                               torch.tensor(base, dtype=torch.int64, device="cuda"))
        deltas.append(d)
    stride = max(1, max(d.count for d in deltas))
    ro = torch.stack([d.offsets for d in deltas])
    ri = torch.zeros(world, stride, dtype=torch.int64, device="cuda")
    rv = torch.zeros(world, stride, dtype=torch.int16, device="cuda")
    for r, d in enumerate(deltas):
        ri[r, :d.count] = d.indices
        rv[r, :d.count] = d.values
    return ro, ri, rv, deltas


@pytest.mark.parametrize("world,rate", [(2, 0.05), (3, 0.3), (8, 0.01)])
def test_merge_shards_equals_the_unsharded_global_encode(dws, world, rate):
    rng = np.random.default_rng(500 + world)
    shapes = [(300, 1000), (7, 33), (1, 9000), (64, 64), (0, 16), (world * 3 + 2, 2048)]
    olds, news = _params(rng, shapes, rate)
    ro, ri, rv, deltas = _shard_deltas(dws, olds, news, world)
    plan = dws.DeltaPlan([max(1, int(np.prod(sh))) for sh in shapes])
    got = plan.merge_shards(ro, ri, rv)
    wo, wi, wv = oracle.encode_global([a.reshape(-1) for a in olds], [b.reshape(-1) for b in news],
                                      [0] * len(shapes))
    np.testing.assert_array_equal(got.offsets.cpu().numpy(), wo)
    np.testing.assert_array_equal(got.indices.cpu().numpy(), wi)
    np.testing.assert_array_equal(got.values.cpu().numpy().view(np.uint16), wv)
    # and the oracle's merge of the same gathered buffers
    mo, mi, mv = oracle.merge_shards([d.offsets.cpu().numpy() for d in deltas],
                                     [d.indices.cpu().numpy() for d in deltas],
                                     [d.values.cpu().numpy().view(np.uint16) for d in deltas])
    np.testing.assert_array_equal(got.indices.cpu().numpy(), mi)
    np.testing.assert_array_equal(got.values.cpu().numpy().view(np.uint16), mv)


def test_merge_shards_capacity_and_bad_layouts(dws):
    rng = np.random.default_rng(520)
    shapes = [(50, 500), (20, 20)]
    olds, news = _params(rng, shapes, 0.2)
    ro, ri, rv, deltas = _shard_deltas(dws, olds, news, 2)
    plan = dws.DeltaPlan([int(np.prod(sh)) for sh in shapes])
    wo, wi, wv = oracle.merge_shards([d.offsets.cpu().numpy() for d in deltas],
                                     [d.indices.cpu().numpy() for d in deltas],
                                     [d.values.cpu().numpy().view(np.uint16) for d in deltas])
    nnz = int(wo[-1])
    stream = torch.cuda.current_stream().cuda_stream
    cap = nnz - 11
    offs = torch.empty(3, dtype=torch.int64, device="cuda")
    idx = torch.full((cap + 4,), -5, dtype=torch.int64, device="cuda")
    val = torch.full((cap + 4,), -5, dtype=torch.int16, device="cuda")

    def call(o, capacity):
        return dws.dws_merge_shards(plan.handle, 2, o.data_ptr(), ri.data_ptr(), rv.data_ptr(),
                                    ri.shape[1], offs.data_ptr(), idx.data_ptr(), val.data_ptr(),
                                    capacity, plan.workspace.data_ptr(), plan.workspace_bytes, stream)

    assert call(ro, cap) == dws.DWS_OK
    st, detail = plan.status()
    assert st == dws.DWS_ERR_CAPACITY and detail == nnz
    np.testing.assert_array_equal(offs.cpu().numpy(), wo)
    np.testing.assert_array_equal(idx[:cap].cpu().numpy(), wi[:cap])
    np.testing.assert_array_equal(val[:cap].cpu().numpy().view(np.uint16), wv[:cap])
    assert (idx[cap:].cpu().numpy() == -5).all()
    # a rank layout that decreases, or ends past the padded length: nothing written
    idx.fill_(-5)
    for r, bad in ((1, lambda o: o.__setitem__(1, o[2] + 1)), (0, lambda o: o.__setitem__(-1, ri.shape[1] + 1))):
        b = ro.clone()
        bad(b[r])
        assert call(b, cap) == dws.DWS_OK
        st, detail = plan.status()
        assert st == dws.DWS_ERR_BAD_DELTA and detail == -1 - r
        assert (idx.cpu().numpy() == -5).all()
    # host-side refusals
    assert dws.dws_merge_shards(plan.handle, 0, ro.data_ptr(), ri.data_ptr(), rv.data_ptr(), 1,
                                offs.data_ptr(), idx.data_ptr(), val.data_ptr(), cap,
                                plan.workspace.data_ptr(), plan.workspace_bytes, stream) \
        == dws.DWS_ERR_INVALID
    assert dws.dws_merge_shards(plan.handle, 2, ro.data_ptr(), ri.data_ptr() + 4, rv.data_ptr(), 1,
                                offs.data_ptr(), idx.data_ptr(), val.data_ptr(), cap,
                                plan.workspace.data_ptr(), plan.workspace_bytes, stream) \
        == dws.DWS_ERR_INVALID
