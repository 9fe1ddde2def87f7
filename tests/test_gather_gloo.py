"""The gather of shard deltas to rank 0 (sparse_bf16_delta_b200.gather) as
separate `gloo` processes on CPU, one per rank, the way torchrun starts them.

Each rank diffs its FSDP Shard(0) slice of every parameter with global
positions (the oracle's encode_global, [verl] shard_delta_indices) and takes
part in the protocol: all_gather of the offsets, padded gathers of positions
and values.  On rank 0 the merge step is the oracle's (CPU tensors; the libdws
merge kernel is tested on the GPU), and the result must equal the oracle's
encode of the unsharded parameters.  No GPU."""
from __future__ import annotations

import json
import os
import sys

import pytest

from tests.test_replicas_gloo import ROOT, _launch

_RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch, torch.distributed as dist
import oracle
import sparse_bf16_delta_b200 as dws
from sparse_bf16_delta_b200.gather import gather_to_rank0

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rng = np.random.default_rng(int(sys.argv[2]))
shapes = [(37, 64), (5, 3), (1, 1000), (16, 16), (world * 2 + 1, 8), (0, 4)]
olds, news = [], []
for sh in shapes:
    a = rng.integers(0, 1 << 16, sh, dtype=np.uint16)
    b = a.copy()
    m = rng.random(sh) < float(sys.argv[3])
    b[m] ^= np.uint16(0x8001)
    olds.append(a); news.append(b)
lo, hi, base = [], [], []
for a, b in zip(olds, news):
    rows = a.shape[0]
    c = -(-rows // world) if rows else 0
    r0, r1 = min(rows, rank * c), min(rows, (rank + 1) * c)
    lo.append(a[r0:r1].reshape(-1)); hi.append(b[r0:r1].reshape(-1))
    base.append(r0 * a.shape[1])
o, i, v = oracle.encode_global(lo, hi, base)
mine = dws.Delta(torch.from_numpy(o), torch.from_numpy(i), torch.from_numpy(v.view(np.int16)))

def oracle_merge(ro, ri, rv):
    R = ro.shape[0]
    mo, mi, mv = oracle.merge_shards([ro[r].numpy() for r in range(R)],
                                     [ri[r].numpy() for r in range(R)],
                                     [rv[r].numpy().view(np.uint16) for r in range(R)])
    return dws.Delta(torch.from_numpy(mo), torch.from_numpy(mi), torch.from_numpy(mv.view(np.int16)))

got = gather_to_rank0(mine, merge=oracle_merge)
out = {"rank": rank, "none": got is None, "mine": int(o[-1])}
if rank == 0:
    wo, wi, wv = oracle.encode_global([a.reshape(-1) for a in olds], [b.reshape(-1) for b in news],
                                      [0] * len(shapes))
    out["equal"] = (np.array_equal(got.offsets.numpy(), wo) and np.array_equal(got.indices.numpy(), wi)
                    and np.array_equal(got.values.numpy().view(np.uint16), wv))
    out["nnz"] = int(wo[-1])
dist.barrier()
dist.destroy_process_group()
print(json.dumps(out))
"""


@pytest.mark.parametrize("world,seed,rate", [(2, 1, 0.1), (2, 2, 0.0), (3, 3, 0.5)])
def test_gather_to_rank0_equals_the_unsharded_encode(tmp_path, world, seed, rate):
    script = tmp_path / "rank.py"
    script.write_text(_RANK_SCRIPT)
    outs = [json.loads(o.strip().splitlines()[-1])
            for o in _launch([str(script), ROOT, str(seed), str(rate)], world)]
    by_rank = {o["rank"]: o for o in outs}
    assert set(by_rank) == set(range(world))
    assert by_rank[0]["equal"] and not by_rank[0]["none"]
    assert all(by_rank[r]["none"] for r in range(1, world))
    assert by_rank[0]["nnz"] == sum(o["mine"] for o in outs)
    if rate > 0:
        assert by_rank[0]["nnz"] > 0
