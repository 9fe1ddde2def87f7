"""The delta file on the GPU: dws_st_delta_write from the encode's device arrays
and dws_st_delta_read into device arrays, through the C ABI.

Small cases: the written file equals the oracle's byte for byte, and reading
the oracle's file, or one the safetensors library wrote in its own layout,
gives the oracle's delta; the applied snapshot is the new one.  Full size
(Qwen3-0.6B-shaped set, 596 M elements): properties that hold at any size --
the safetensors library reads the file back to the device arrays, reading
returns the same arrays, and applying the read delta gives the new snapshot.
"""
from __future__ import annotations

import json

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import st_file
from tests._dev import assert_delta_equal, delta_to_host, host_bits

pytestmark = pytest.mark.gpu
pytest.importorskip("safetensors")
from safetensors.torch import load as st_load  # noqa: E402
from safetensors.torch import save as st_save  # noqa: E402


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _pair(div, s, lr):
    shapes = W.scaled_shapes(W.qwen3_0p6b_shapes(), div)
    w0 = W.init_set(shapes, s, "cuda", 0.02)
    w1 = W.step_set(w0, s, 1, lr, "cuda")
    return w0, w1


def _check_apply(dws, plan, w0, delta, h1):
    snap = [t.clone() for t in w0.tensors]
    plan.apply(dws.ptr_table(snap), delta)
    plan.raise_on_error("dws_apply")
    for x, y in zip(snap, h1):
        np.testing.assert_array_equal(host_bits(x), y)


@pytest.mark.parametrize("div,lr,version", [(16, 3e-6, 123), (64, 1e-4, -7), (256, 0.0, 0)])
def test_written_file_equals_oracle_and_reads_back(dws, div, lr, version):
    # lr 0: nothing changes, a file of metadata only.
    w0, w1 = _pair(div, 31 + div, lr)
    plan = dws.DeltaPlan.for_tensors(w0.tensors)
    d = plan.encode_exact(dws.ptr_table(w0.tensors), dws.ptr_table(w1.tensors))
    h0 = [host_bits(t) for t in w0.tensors]
    h1 = [host_bits(t) for t in w1.tensors]
    o, i, v = oracle.encode(h0, h1)
    want = st_file.write_delta(w0.names, w0.numels, o, i, v, version)
    got = plan.write_delta_file(d, w0.names, version)
    assert got.is_pinned()
    assert bytes(got.numpy()) == want
    for src in (got, want):  # pinned tensor (writer's layout); bytes (pageable)
        d2, ver = plan.read_delta_file(src, w0.names)
        assert ver == version
        assert_delta_equal(delta_to_host(d2), (o, i, v))
    _check_apply(dws, plan, w0, plan.read_delta_file(got, w0.names)[0], h1)


@pytest.mark.parametrize("seed", [0, 1])
def test_reads_a_file_in_the_library_layout(dws, seed):
    # safetensors orders the data by dtype and name, so every parameter is a
    # separate range: the reader copies per parameter, not two blocks.
    w0, w1 = _pair(32, 50 + seed, 1e-4)
    plan = dws.DeltaPlan.for_tensors(w0.tensors)
    h0 = [host_bits(t) for t in w0.tensors]
    h1 = [host_bits(t) for t in w1.tensors]
    o, i, v = oracle.encode(h0, h1)
    rng = np.random.default_rng(seed)
    tensors, changed = {}, []
    for t in rng.permutation(len(h0)):
        a, b = int(o[t]), int(o[t + 1])
        if a < b:
            name = w0.names[t]
            tensors[name + ".indices"] = torch.from_numpy(i[a:b].copy())
            tensors[name + ".values"] = torch.from_numpy(v[a:b].view(np.int16).copy()).view(
                torch.bfloat16)
            changed.append(name)
    assert len(changed) > 10
    blob = st_save(tensors, metadata={"sparse": "True", "model_version": "5",
                                      "changed_params": json.dumps(changed)})
    pinned = torch.empty(len(blob), dtype=torch.uint8, pin_memory=True)
    pinned.copy_(torch.frombuffer(bytearray(blob), dtype=torch.uint8))
    d, ver = plan.read_delta_file(pinned, w0.names, capacity=int(o[-1]))
    assert ver == 5
    assert_delta_equal(delta_to_host(d), (o, i, v))
    _check_apply(dws, plan, w0, d, h1)


def test_capacity_and_refusal_are_reported(dws):
    w0, w1 = _pair(64, 60, 1e-4)
    plan = dws.DeltaPlan.for_tensors(w0.tensors)
    d = plan.encode_exact(dws.ptr_table(w0.tensors), dws.ptr_table(w1.tensors))
    f = plan.write_delta_file(d, w0.names, 1)
    with pytest.raises(dws.DwsError) as e:
        plan.read_delta_file(f, w0.names, capacity=d.count - 1)
    assert e.value.code == dws.DWS_ERR_CAPACITY and e.value.detail == d.count
    offs = d.offsets.cpu().numpy()
    first = next(t for t in range(len(w0.names)) if offs[t + 1] > offs[t])
    other = list(w0.names)
    other[first] = other[first] + ".renamed"  # the file names a parameter outside the table
    with pytest.raises(dws.DwsError) as e:
        plan.read_delta_file(f, other)
    assert e.value.code == dws.DWS_ERR_BAD_DELTA
    with pytest.raises(dws.DwsError) as e:
        plan.read_delta_file(bytes(f.numpy())[:100], w0.names)
    assert e.value.code == dws.DWS_ERR_BAD_DELTA


def test_full_size_qwen3_round_trip(dws):
    s = W.SEEDS["qwen3_0p6b"]
    w0 = W.init_set(W.qwen3_0p6b_shapes(), s, "cuda", 0.02)
    w1 = W.step_set(w0, s, 1, 3e-6, "cuda")
    plan = dws.DeltaPlan.for_tensors(w0.tensors)
    d = plan.encode_exact(dws.ptr_table(w0.tensors), dws.ptr_table(w1.tensors))
    nnz = d.count
    f = plan.write_delta_file(d, w0.names, 42)
    assert f.numel() == len(plan.delta_file_header(w0.names, d.offsets, 42)) + 6 * nnz
    # the safetensors library reads every entry back to the device arrays
    lib = st_load(bytes(f.numpy()))
    offs = d.offsets.cpu().numpy()
    idx_h, val_h = d.indices.cpu(), d.values.cpu()
    changed = [w0.names[t] for t in range(len(w0.names)) if offs[t + 1] > offs[t]]
    assert sorted(lib) == sorted(n + s for n in changed for s in (".indices", ".values"))
    for t, name in enumerate(w0.names):
        a, b = int(offs[t]), int(offs[t + 1])
        if a < b:
            assert torch.equal(lib[name + ".indices"], idx_h[a:b])
            assert torch.equal(lib[name + ".values"].view(torch.int16), val_h[a:b])
    del lib
    d2, ver = plan.read_delta_file(f, w0.names, capacity=nnz)
    assert ver == 42
    assert torch.equal(d2.offsets, d.offsets)
    assert torch.equal(d2.indices, d.indices) and torch.equal(d2.values, d.values)
    snap = [t.clone() for t in w0.tensors]
    plan.apply(dws.ptr_table(snap), d2)
    plan.raise_on_error("dws_apply")
    assert all(torch.equal(x.view(torch.int16), y.view(torch.int16))
               for x, y in zip(snap, w1.tensors))
