"""dws_encode_noalloc: the encode for callers that cannot allocate device memory
(code running inside another framework's memory pool, where every device
allocation goes through an allocator the caller does not control or is not
allowed, and latency-critical paths that cannot afford a cudaMalloc and the
synchronisation it implies).  Its scratch is a fixed array inside libdws, so
the caller passes only inputs and outputs.

Its output must equal the CPU oracle's and the workspace-based dws_encode's,
exactly (integer work), on calls in a row: each call runs on whatever the one
before left in the shared array (a smaller layout after a larger one
included).  This file is collected last on purpose."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 8191, 8192, 8193, 100_003, 3 * 8192 + 5, 65_536]


def _pair(rng, n, rate):
    a = rng.integers(0, 1 << 16, n, dtype=np.uint16)
    b = a.copy()
    if n:
        m = rng.random(n) < rate
        b[m] ^= rng.integers(1, 1 << 16, int(m.sum()), dtype=np.uint16)
    return a, b


def _dev(a):
    return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.bfloat16)


def _noalloc(dws, sizes, ot, nt, cap):
    stream = torch.cuda.current_stream().cuda_stream
    offsets = torch.full((len(sizes) + 1,), -1, dtype=torch.int64, device="cuda")
    indices = torch.full((max(cap, 1),), -1, dtype=torch.int32, device="cuda")
    values = torch.full((max(cap, 1),), -1, dtype=torch.int16, device="cuda")
    status = torch.full((2,), -1, dtype=torch.int64, device="cuda")
    code = dws.dws_encode_noalloc(sizes, ot.data_ptr(), nt.data_ptr(), offsets.data_ptr(),
                                  indices.data_ptr(), values.data_ptr(), cap, status.data_ptr(),
                                  stream)
    torch.cuda.synchronize()
    return code, offsets.cpu().numpy(), indices.cpu().numpy(), \
        values.cpu().numpy().view(np.uint16), status.tolist()


def test_noalloc_encode_matches_oracle_and_workspace_encode_on_calls_in_a_row():
    import sparse_bf16_delta_b200 as dws
    # two calls of the full layout, then a smaller one (fewer tensors, fewer
    # tiles) on top of what the larger calls left behind
    cases = [(SIZES, 201, 0.03), (SIZES, 202, 0.3), (SIZES[2:6], 203, 0.1)]
    for call, (sizes, seed, rate) in enumerate(cases):
        rng = np.random.default_rng(seed)
        pairs = [_pair(rng, n, rate) for n in sizes]
        olds = [_dev(a) for a, _ in pairs]
        news = [_dev(b) for _, b in pairs]
        ot, nt = dws.ptr_table(olds), dws.ptr_table(news)
        want_o, want_i, want_v = oracle.encode([a for a, _ in pairs], [b for _, b in pairs])
        nnz = int(want_o[-1])

        # the existing entry point, with a torch-allocated workspace
        plan = dws.DeltaPlan.for_tensors(olds)
        ws = plan.encode_exact(ot, nt)
        np.testing.assert_array_equal(ws.offsets.cpu().numpy(), want_o)

        # the allocation-free entry point, into caller-owned outputs
        cap = sum(sizes)
        code, offs, idx, val, status = _noalloc(dws, sizes, ot, nt, cap)
        assert code == dws.DWS_OK, call
        assert status == [dws.DWS_OK, 0], call
        np.testing.assert_array_equal(offs, want_o)
        np.testing.assert_array_equal(idx[:nnz], want_i)
        np.testing.assert_array_equal(val[:nnz], want_v)
        np.testing.assert_array_equal(idx[:nnz], ws.indices.cpu().numpy())
        np.testing.assert_array_equal(val[:nnz], ws.values.cpu().numpy().view(np.uint16))
        assert (idx[nnz:cap] == -1).all()


def test_noalloc_reports_capacity_overflow_in_status_out():
    import sparse_bf16_delta_b200 as dws
    rng = np.random.default_rng(204)
    pairs = [_pair(rng, n, 0.2) for n in SIZES]
    ot = dws.ptr_table([_dev(a) for a, _ in pairs])
    nt = dws.ptr_table([_dev(b) for _, b in pairs])
    want_o, want_i, want_v = oracle.encode([a for a, _ in pairs], [b for _, b in pairs])
    nnz = int(want_o[-1])
    cap = nnz // 3
    code, offs, idx, val, status = _noalloc(dws, SIZES, ot, nt, cap)
    assert code == dws.DWS_OK
    assert status == [dws.DWS_ERR_CAPACITY, nnz]
    np.testing.assert_array_equal(offs, want_o)  # complete even when the entries are not
    np.testing.assert_array_equal(idx[:cap], want_i[:cap])
    np.testing.assert_array_equal(val[:cap], want_v[:cap])


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # Refused on the host before anything is enqueued: real (tiny) device
    # buffers are passed, so nothing could fault even if a check regressed,
    # and the outputs must come back untouched.
    import sparse_bf16_delta_b200 as dws
    stream = torch.cuda.current_stream().cuda_stream
    a = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    table = dws.ptr_table([a] * 300)
    offsets = torch.full((300,), -7, dtype=torch.int64, device="cuda")
    idx = torch.full((16,), -7, dtype=torch.int32, device="cuda")
    val = torch.full((16,), -7, dtype=torch.int16, device="cuda")
    status = torch.full((2,), -7, dtype=torch.int64, device="cuda")
    args = (table.data_ptr(), table.data_ptr(), offsets.data_ptr(), idx.data_ptr(), val.data_ptr(),
            16, status.data_ptr(), stream)
    assert dws.dws_encode_noalloc([16] * 257, *args) == dws.DWS_ERR_WORKSPACE
    assert dws.dws_encode_noalloc([(1 << 31) - 1], *args) == dws.DWS_ERR_WORKSPACE
    assert dws.dws_encode_noalloc([8192 * 257] * 256, *args) == dws.DWS_ERR_WORKSPACE  # 65,792 tiles
    assert dws.dws_encode_noalloc([1 << 31], *args) == dws.DWS_ERR_INVALID
    torch.cuda.synchronize()
    for t in (offsets, idx, val, status):
        assert (t.cpu() == -7).all()
