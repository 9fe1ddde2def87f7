"""libdws at the workloads' full sizes, in the launch configuration the
benchmark times.

Element-by-element comparison with the CPU oracle runs on sampled tensors
(every tensor the oracle can finish in seconds is taken whole); properties
that hold at any size cover everything else: per-tensor change counts equal
torch's count of differing 16-bit patterns, applying a delta gives the new
snapshot bit for bit, chain replay gives the final weights, and the
generators' known change positions (XOR and stress workloads) are exactly the
encoded ones."""
from __future__ import annotations

import gc

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests._dev import host_bits, host_bytes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dws():
    import sparse_bf16_delta_b200 as m
    return m


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _std(name):
    return (0.01, 1.0) if W.is_norm(name) else (0.02, 0.0)


def _counts_by_torch(olds, news):
    """Per-tensor number of differing 16-bit patterns (torch library compare)."""
    return [int(torch.count_nonzero(a.view(torch.int16) != b.view(torch.int16))) for a, b in zip(olds, news)]


def _check_segments(delta, olds, news, tensors):
    """Oracle comparison of the delta's segments of the given tensors."""
    offs = delta.offsets.cpu().numpy()
    for t in tensors:
        a, b = host_bits(olds[t]), host_bits(news[t])
        o, i, v = oracle.encode([a], [b])
        lo, hi = offs[t], offs[t + 1]
        assert hi - lo == o[-1], t
        np.testing.assert_array_equal(delta.indices[lo:hi].cpu().numpy(), i)
        np.testing.assert_array_equal(delta.values[lo:hi].cpu().numpy().view(np.uint16), v)


def _check_absorption(delta, olds, s, k, lr, tensors):
    """The absorption rule, evaluated independently from the old weights and
    the step's noise (exact midpoints in double precision), predicts exactly
    the positions the encode listed, tensor by tensor."""
    offs = delta.offsets.cpu().numpy()
    for t in tensors:
        u = W.update_noise(olds[t].numel(), W.step_seed(s, k, t), "cuda").cpu().numpy()
        changed, cnt = oracle.absorption_predict(host_bits(olds[t]), u, lr)
        assert cnt == offs[t + 1] - offs[t], t
        np.testing.assert_array_equal(np.flatnonzero(changed),
                                      delta.indices[offs[t]:offs[t + 1]].cpu().numpy())
        del u, changed


_LAYER0 = ["self_attn.q_proj", "self_attn.k_proj", "self_attn.v_proj", "self_attn.o_proj",
           "mlp.gate_proj", "mlp.up_proj", "mlp.down_proj", "input_layernorm",
           "post_attention_layernorm"]


@pytest.mark.parametrize("lr", [3e-6, 1e-5])
def test_llama3_8b_encode_apply_full(dws, lr):
    s = W.SEEDS["llama3_8b"]
    shapes = W.llama3_8b_shapes()
    sizes = [W.numel(sh) for _, sh in shapes]
    std = [_std(nm) for nm, _ in shapes]
    dev = torch.device("cuda")
    old_flat, old = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, *std[t]), dev)
    new_flat, new = W.pack_flat(
        sizes, lambda t, n: W.optimizer_step(old[t], W.update_noise(n, W.step_seed(s, 1, t), dev), lr), dev)
    plan = dws.DeltaPlan.for_tensors(old)
    d = plan.encode_exact(dws.ptr_table(old), dws.ptr_table(new))
    # every tensor's count equals torch's count of differing bit patterns
    counts = np.diff(d.offsets.cpu().numpy())
    assert list(counts) == _counts_by_torch(old, new)
    # oracle, element by element: embedding, all of layer 0, norms, lm_head
    names = [nm for nm, _ in shapes]
    sample = [0] + [t for t, nm in enumerate(names) if nm.startswith("model.layers.0.")] + \
             [names.index("model.layers.31.input_layernorm.weight"), names.index("model.norm.weight"),
              names.index("lm_head.weight")]
    _check_segments(d, old, new, sample)
    # the absorption rule predicts exactly the encoded positions: the embedding,
    # every weight and norm of layer 0, the final norm (12 tensors)
    _check_absorption(d, old, s, 1, lr,
                      [names.index("model.embed_tokens.weight"), names.index("model.norm.weight")] +
                      [names.index(f"model.layers.0.{m}.weight") for m in _LAYER0])
    # apply onto a copy of old gives new, bit for bit, everywhere
    snap_flat = old_flat.clone()
    snap = [snap_flat[v.storage_offset():][:v.numel()] for v in old]
    plan.apply(dws.ptr_table(snap), d)
    plan.raise_on_error("apply")
    assert torch.equal(snap_flat, new_flat)
    del old_flat, new_flat, snap_flat, old, new, snap, d, plan
    _free()


def test_qwen3_0p6b_chain_full(dws):
    s = W.SEEDS["qwen3_0p6b"]
    shapes = W.qwen3_0p6b_shapes()
    sizes = [W.numel(sh) for _, sh in shapes]
    std = [_std(nm) for nm, _ in shapes]
    dev = torch.device("cuda")
    anchor_flat, anchor = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, *std[t]), dev)
    plan = dws.DeltaPlan.for_tensors(anchor)
    prev_flat, prev = W.pack_flat(sizes, lambda t, n: anchor[t], dev)
    cur_flat, cur = W.pack_flat(sizes, lambda t, n: None, dev)
    deltas = []
    for k in range(1, 11):
        for t in range(len(sizes)):
            cur[t].copy_(W.optimizer_step(prev[t], W.update_noise(sizes[t], W.step_seed(s, k, t), dev), 3e-6))
        d = plan.encode_exact(dws.ptr_table(prev), dws.ptr_table(cur))
        assert list(np.diff(d.offsets.cpu().numpy())) == _counts_by_torch(prev, cur)
        if k == 1:
            _check_segments(d, prev, cur, range(len(sizes)))  # the whole step, every tensor
            names = [nm for nm, _ in shapes]
            _check_absorption(d, prev, s, 1, 3e-6,
                              [names.index("model.embed_tokens.weight")] +
                              [names.index(f"model.layers.0.{m}.weight")
                               for m in _LAYER0 + ["self_attn.q_norm", "self_attn.k_norm"]])
        elif k == 10:
            _check_segments(d, prev, cur, [0, 1, 5, 6, 7, 10, 309])
        deltas.append(d)
        prev_flat, cur_flat = cur_flat, prev_flat
        prev, cur = cur, prev
    # the fused 10-delta replay, in both modes
    for mode in (dws.DWS_CHAIN_TILE_MERGE, dws.DWS_CHAIN_SCATTER):
        snap_flat = anchor_flat.clone()
        snap = [snap_flat[v.storage_offset():][:v.numel()] for v in anchor]
        plan.apply_chain(dws.ptr_table(snap), deltas, mode=mode)
        plan.raise_on_error("apply_chain")
        assert torch.equal(snap_flat, prev_flat), mode
        del snap_flat, snap
    del anchor_flat, prev_flat, cur_flat, deltas, plan
    _free()


def test_xor_nvfp4_full(dws):
    dev = torch.device("cuda")
    L, B = 40, 800_000_000
    olds, news, masks = [], [], []
    for l in range(L):
        o, n, pos = W.xor_layer(l, dev, nbytes=B)
        m = dws.xor_encode(o, n)
        # closed form: the mask is nonzero exactly at the generator's positions
        assert torch.equal(torch.nonzero(m).flatten(), pos)
        olds.append(o)
        news.append(n)
        masks.append(m)
        del pos
    # oracle, byte by byte, on the first and last layer
    for l in (0, L - 1):
        np.testing.assert_array_equal(host_bytes(masks[l]),
                                      oracle.xor_encode(host_bytes(olds[l]), host_bytes(news[l])))
    staging = [torch.empty(B, dtype=torch.uint8, device=dev) for _ in range(2)]
    dws.xor_apply_layers(olds, masks, staging[0], staging[1], copy_stream=torch.cuda.Stream())
    torch.cuda.current_stream().synchronize()
    for o, n in zip(olds, news):
        assert torch.equal(o, n)
    del olds, news, masks, staging
    _free()


def test_stress_12000_tensors_chain_full(dws):
    s = W.SEEDS["stress"]
    sizes = W.stress_sizes()
    clustered = W.stress_clustered()
    dev = torch.device("cuda")
    anchor_flat, anchor = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, 0.02), dev)
    plan = dws.DeltaPlan.for_tensors(anchor)
    prev_flat, prev = W.pack_flat(sizes, lambda t, n: anchor[t], dev)
    cur_flat, cur = W.pack_flat(sizes, lambda t, n: None, dev)
    rng = np.random.default_rng(4)
    sample = sorted(set(rng.choice(len(sizes), 40, replace=False).tolist()))
    deltas = []
    for k in range(1, 11):
        picked_counts = []
        for t in range(len(sizes)):
            nw, pk = W.stress_change(prev[t], clustered[t], W.step_seed(s, k, t), dev)
            cur[t].copy_(nw)
            picked_counts.append(pk)
        d = plan.encode_exact(dws.ptr_table(prev), dws.ptr_table(cur))
        offs = d.offsets.cpu().numpy()
        # closed form: exactly the generator's picked positions, every tensor
        counts = torch.stack([pk.sum() for pk in picked_counts]).cpu().numpy()
        np.testing.assert_array_equal(np.diff(offs), counts)
        for t in sample[:8]:
            np.testing.assert_array_equal(d.indices[offs[t]:offs[t + 1]].cpu().numpy(),
                                          torch.nonzero(picked_counts[t]).flatten().cpu().numpy())
        if k in (1, 10):
            _check_segments(d, prev, cur, sample)
        del picked_counts
        deltas.append(d)
        prev_flat, cur_flat = cur_flat, prev_flat
        prev, cur = cur, prev
    for mode in (dws.DWS_CHAIN_TILE_MERGE, dws.DWS_CHAIN_SCATTER):
        snap_flat = anchor_flat.clone()
        snap = [snap_flat[v.storage_offset() - anchor_flat.storage_offset():][:v.numel()] for v in anchor]
        plan.apply_chain(dws.ptr_table(snap), deltas, mode=mode)
        plan.raise_on_error("apply_chain")
        assert torch.equal(snap_flat, prev_flat), mode
        del snap_flat, snap
    del anchor_flat, prev_flat, cur_flat, deltas, plan
    _free()


def test_largest_tensor_int32_index_bound(dws):
    # One tensor of 2^31 - 1 elements: the largest int32 indices, tiles up to
    # the very last element, a ragged last tile.
    n = (1 << 31) - 1
    dev = torch.device("cuda")
    old = torch.zeros(n, dtype=torch.int16, device=dev)
    new = old.clone()
    te = dws.dws_tile_elems()
    pos = np.array(sorted({0, 1, te - 1, te, te + 1, 12345678, (n // te) * te - 1, (n // te) * te,
                           n - 9, n - 2, n - 1}), dtype=np.int64)
    new[torch.from_numpy(pos).to(dev)] = torch.arange(1, pos.size + 1, dtype=torch.int16, device=dev)
    o16, n16 = old.view(torch.bfloat16), new.view(torch.bfloat16)
    plan = dws.DeltaPlan([n])
    d = plan.encode_exact(dws.ptr_table([o16]), dws.ptr_table([n16]))
    assert d.nnz() == pos.size
    np.testing.assert_array_equal(d.indices.cpu().numpy().astype(np.int64), pos)
    np.testing.assert_array_equal(d.values.cpu().numpy(), np.arange(1, pos.size + 1, dtype=np.int16))
    snap = old.clone().view(torch.bfloat16)
    plan.apply(dws.ptr_table([snap]), d)
    plan.raise_on_error()
    assert torch.equal(snap.view(torch.int16), new)
    del old, new, snap, d, plan
    _free()
