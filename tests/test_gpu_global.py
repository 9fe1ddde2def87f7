"""dws_encode_global (int64 global positions, index_base[t] + local index) on
the GPU against the CPU oracle, element by element."""
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


def _pairs(rng, sizes, rate):
    olds, news = [], []
    for n in sizes:
        a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
        b = a.copy()
        if n:
            m = rng.random(n) < rate
            b[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
            if n > 9000:
                b[2000:6100] ^= np.uint16(0x0001)  # a dense run
        olds.append(a)
        news.append(b)
    return olds, news


@pytest.mark.parametrize("rate", [0.01, 0.3])
def test_encode_global_matches_oracle(dws, rate):
    rng = np.random.default_rng(401 + int(rate * 100))
    sizes = [8192 * 3 + 7, 0, 1, 100_000, 5, 8192]
    bases = [0, 7, 5_000_000_000, 2 ** 31 - 1, 2 ** 40 + 3, 12345]
    olds, news = _pairs(rng, sizes, rate)
    plan = dws.DeltaPlan(sizes)
    ot = dws.ptr_table([dev_bits(a) for a in olds])
    nt = dws.ptr_table([dev_bits(b) for b in news])
    base_t = torch.tensor(bases, dtype=torch.int64, device="cuda")
    d = plan.encode_global(ot, nt, base_t)
    o, gi, v = oracle.encode_global(olds, news, bases)
    np.testing.assert_array_equal(d.offsets.cpu().numpy(), o)
    assert d.indices.dtype == torch.int64
    np.testing.assert_array_equal(d.indices.cpu().numpy(), gi)
    np.testing.assert_array_equal(d.values.cpu().numpy().view(np.uint16), v)
    # the same local positions as the 32-bit encode
    d32 = plan.encode_exact(ot, nt)
    counts = np.diff(o)
    np.testing.assert_array_equal(d32.indices.cpu().numpy().astype(np.int64) + np.repeat(bases, counts), gi)


@pytest.mark.parametrize("shift", [1, 3])
def test_encode_global_unaligned_outputs_and_capacity(dws, shift):
    rng = np.random.default_rng(410 + shift)
    sizes = [50_000, 8192 * 2 + 1]
    bases = [3_000_000_000, 17]
    olds, news = _pairs(rng, sizes, 0.05)
    o, gi, v = oracle.encode_global(olds, news, bases)
    nnz = int(o[-1])
    cap = nnz - 37
    plan = dws.DeltaPlan(sizes)
    ot = dws.ptr_table([dev_bits(a) for a in olds])
    nt = dws.ptr_table([dev_bits(b) for b in news])
    base_t = torch.tensor(bases, dtype=torch.int64, device="cuda")
    offsets = torch.empty(len(sizes) + 1, dtype=torch.int64, device="cuda")
    ib = torch.full((cap + 8,), -9, dtype=torch.int64, device="cuda")
    vb = torch.full((cap + 8,), -9, dtype=torch.int16, device="cuda")
    idx, val = ib[shift:shift + cap], vb[shift:shift + cap]
    code = dws.dws_encode_global(plan.handle, ot.data_ptr(), nt.data_ptr(), base_t.data_ptr(),
                                 offsets.data_ptr(), idx.data_ptr(), val.data_ptr(), cap,
                                 plan.workspace.data_ptr(), plan.workspace_bytes,
                                 torch.cuda.current_stream().cuda_stream)
    assert code == dws.DWS_OK
    st, detail = plan.status()
    assert st == dws.DWS_ERR_CAPACITY and detail == nnz
    np.testing.assert_array_equal(offsets.cpu().numpy(), o)
    np.testing.assert_array_equal(idx.cpu().numpy(), gi[:cap])
    np.testing.assert_array_equal(val.cpu().numpy().view(np.uint16), v[:cap])
    assert (ib[:shift].cpu().numpy() == -9).all() and (ib[shift + cap:].cpu().numpy() == -9).all()
