"""bench.py's multi-process path on CPU: two `gloo` ranks (one process per
rank, as torchrun starts them) agree on the slowest rank's time, the
whole-job value counts every replica, and the reference arm runs on rank 0
only.  No GPU: the replicas share nothing but the barrier and the max."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, sys.argv[1])
import torch, torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
ms = 10.0 + 7.5 * rank                       # rank 1 is the slow one
got = bench.max_over_ranks(ms, world, torch.device("cpu"))
dist.barrier()
dist.destroy_process_group()
print(json.dumps({"rank": rank, "max": got,
                  "value": bench.replicas_value(world, 2e9, got)}))
"""


def _launch(script_args, world, extra_env=None, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(world),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, *script_args], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    try:
        for p in procs:
            out, err = p.communicate(timeout=timeout)
            assert p.returncode == 0, err[-2000:]
            outs.append(out)
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    return outs


def test_two_gloo_ranks_take_the_slowest_time():
    outs = _launch(["-c", _RANK_SCRIPT, ROOT], 2)
    res = sorted((json.loads(o.strip().splitlines()[-1]) for o in outs), key=lambda d: d["rank"])
    assert [d["max"] for d in res] == [17.5, 17.5]
    # 2 replicas x 2 GB in 17.5 ms
    assert res[0]["value"] == pytest.approx(2 * 2e9 / 17.5e-3 / 1e9)
    assert res[0]["value"] == res[1]["value"]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, None) == 3.25
    assert bench.replicas_value(1, 1e9, 1.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only():
    # Rank 1 of the reference arm exits 0 at once, printing nothing.
    outs = _launch(["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                    "--warmup", "0", "--layers", "0"], 2, timeout=600)
    lines = [o.strip().splitlines() for o in outs]
    assert lines[1] == []
    line = json.loads(lines[0][-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def test_theoretical_hbm_peak_from_device_attributes():
    # The two device attributes libdws reports (memory clock in kHz, bus
    # width in bits) give clock x 2 (double data rate) x width / 8: an H100
    # SXM's 2,619 MHz x 5120 bits is its 3.35 TB/s; 3,996 MHz x 7680 bits is
    # 7.67 TB/s.  A failed query or a zero attribute gives no peak.
    import types

    import bench

    def fake(khz, bits):
        return types.SimpleNamespace(dws_device_memory=lambda dev: (khz, bits))

    peak, khz, bits = bench.theoretical_hbm_gbs(fake(2_619_000, 5120), 0)
    assert abs(peak - 3352.3) < 0.1 and (khz, bits) == (2_619_000, 5120)
    assert abs(bench.theoretical_hbm_gbs(fake(3_996_000, 7680), 0)[0] - 7672.3) < 0.1
    assert bench.theoretical_hbm_gbs(fake(0, 8), 0)[0] is None

    def broken(dev):
        raise RuntimeError("no device")

    assert bench.theoretical_hbm_gbs(types.SimpleNamespace(dws_device_memory=broken), 0) == (None, None, None)
