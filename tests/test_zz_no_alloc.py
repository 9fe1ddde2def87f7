"""dws_encode_noalloc: the encode for callers that cannot allocate device memory
(code running inside another framework's memory pool, where every device
allocation goes through an allocator the caller does not control or is not
allowed, and latency-critical paths that cannot afford a cudaMalloc and the
synchronisation it implies).  Its scratch is a fixed array inside libdws, so
the caller passes only inputs and outputs.

Its output must equal the workspace-based dws_encode's, exactly (integer
work), on two calls in a row -- the second call runs on whatever the first
left in the shared array.  This file is collected last on purpose."""
from __future__ import annotations

import numpy as np
import pytest
import torch

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


@pytest.mark.gpu
def test_noalloc_encode_matches_workspace_encode_on_two_calls():
    import sparse_bf16_delta_b200 as dws
    stream = torch.cuda.current_stream().cuda_stream
    for call, (seed, rate) in enumerate([(201, 0.03), (202, 0.3)]):
        rng = np.random.default_rng(seed)
        pairs = [_pair(rng, n, rate) for n in SIZES]
        olds = [_dev(a) for a, _ in pairs]
        news = [_dev(b) for _, b in pairs]
        ot, nt = dws.ptr_table(olds), dws.ptr_table(news)

        # the existing entry point, with a torch-allocated workspace
        plan = dws.DeltaPlan.for_tensors(olds)
        want = plan.encode_exact(ot, nt)
        nnz = want.nnz()

        # the allocation-free entry point, into caller-owned outputs
        cap = sum(SIZES)
        offsets = torch.full((len(SIZES) + 1,), -1, dtype=torch.int64, device="cuda")
        indices = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
        values = torch.full((cap,), -1, dtype=torch.int16, device="cuda")
        status = torch.full((2,), -1, dtype=torch.int64, device="cuda")
        code = dws.dws_encode_noalloc(SIZES, ot.data_ptr(), nt.data_ptr(), offsets.data_ptr(),
                                      indices.data_ptr(), values.data_ptr(), cap, status.data_ptr(),
                                      stream)
        assert code == dws.DWS_OK, call
        torch.cuda.synchronize()
        assert status.tolist() == [dws.DWS_OK, 0], call
        np.testing.assert_array_equal(offsets.cpu().numpy(), want.offsets.cpu().numpy())
        np.testing.assert_array_equal(indices[:nnz].cpu().numpy(), want.indices.cpu().numpy())
        np.testing.assert_array_equal(values[:nnz].cpu().numpy(), want.values.cpu().numpy())
        assert (indices[nnz:].cpu().numpy() == -1).all()


def test_noalloc_refuses_sizes_beyond_its_scratch():
    # Refused on the host before anything is enqueued (no GPU needed).
    import sparse_bf16_delta_b200 as dws
    fake = 0x1000
    assert dws.dws_encode_noalloc([16] * 257, fake, fake, fake, fake, fake, 16, 0, None) \
        == dws.DWS_ERR_WORKSPACE
    assert dws.dws_encode_noalloc([(1 << 31) - 1], fake, fake, fake, fake, fake, 16, 0, None) \
        == dws.DWS_ERR_WORKSPACE
    assert dws.dws_encode_noalloc([8192 * 257] * 256, fake, fake, fake, fake, fake, 16, 0, None) \
        == dws.DWS_ERR_WORKSPACE  # 65,792 tiles
    assert dws.dws_encode_noalloc([1 << 31], fake, fake, fake, fake, fake, 16, 0, None) \
        == dws.DWS_ERR_INVALID
