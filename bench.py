#!/usr/bin/env python
"""Delta encode+apply throughput of bf16 weights on B200 (libdws).

One step = dws_encode(old, new -> sparse delta) + dws_apply(delta -> snapshot)
on the Llama-3-8B-shaped parameter set (291 tensors, 8,030,261,248 bf16
elements, 16.06 GB per snapshot) after one simulated optimizer step at
lr 3e-6.  Inputs (32 GB) are much larger than the 126 MB L2, so no flush is
needed between steps.  value = weight bytes (2 B x elements, summed over
ranks) / device time per step, max over ranks.

Also reported on the same JSON line:
  roofline      encode kernel: algorithmic bytes (4N + 6 nnz) / CUDA-event
                time vs the measured HBM copy bandwidth;
  cpu_baseline  the single-threaded CPU oracle on a bounded sample (rank 0, N=1);
  e2e           the same metric with the new snapshot coming from pinned host
                memory and the delta going device->host->device, copies timed;
  rows          the other hot-path rows: encode at lr 1e-5, count-only,
                XOR encode/apply and the double-buffered layer pipeline on 40
                x 0.8 GB byte layers, chain replay of 10 deltas on the
                Qwen3-0.6B-shaped set and on the 12000-tensor stress set.

Multi-GPU: replicas only -- every rank runs the same workload on its own GPU
(no data-path collective); NCCL is used for the barrier and the max-over-ranks
timing reduction.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import contextlib
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "delta encode+apply GB/s of bf16 weights (1 B200) and % of HBM peak"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--lr", type=float, default=3e-6)
    ap.add_argument("--layers", type=int, default=None,
                    help="only the first LAYERS decoder layers (a small case for profiling)")
    ap.add_argument("--no-rows", action="store_true", help="skip the other hot-path rows")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--rows-reps", type=int, default=5)
    ap.add_argument("--xor-layers", type=int, default=40,
                    help="layers of 0.8 GB in the XOR rows (fewer: a small case for profiling)")
    ap.add_argument("--stress-tensors", type=int, default=12000,
                    help="tensors of the stress set (fewer: a small case for profiling)")
    ap.add_argument("--rows-only", default=None,
                    help="comma list of single, qwen_chain, xor, stress_chain: time only these rows "
                         "(no Llama-3-8B step; a small case for profiling)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# plumbing
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def max_over_ranks(ms, world, device):
    """The slowest rank's time (all ranks take part; world 1: ms itself)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replicas_value(world, bytes_per_rank, ms_per_step):
    """Whole-job GB/s: every replica moves bytes_per_rank per step, the step
    taking the slowest rank's time."""
    return world * bytes_per_rank / (ms_per_step / 1e3) / 1e9


def theoretical_hbm_gbs(dws, device_index):
    """HBM peak from the device attributes libdws reads from the CUDA runtime
    (dws_device_memory): memory clock (kHz) x 2 (double data rate) x bus width
    (bits) / 8, in GB/s, with its two inputs; (None, None, None) if unknown."""
    try:
        khz, bits = dws.dws_device_memory(device_index)
    except Exception:
        return None, None, None
    if khz <= 0 or bits <= 0:
        return None, khz, bits
    return khz * 1e3 * 2 * bits / 8 / 1e9, khz, bits


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def llama_shapes(layers):
    import workloads as W
    shapes = W.llama3_8b_shapes()
    if layers is None:
        return shapes
    keep = [s for s in shapes if not s[0].startswith("model.layers.")]
    lay = [s for s in shapes if s[0].startswith("model.layers.")
           and int(s[0].split(".")[2]) < layers]
    # a small case: decoder layers only (no embedding / lm_head)
    return lay if layers > 0 else keep


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int, uuid: str | None):
        self.dev = device_index
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        target = f"GPU-{self.uuid}" if self.uuid else str(self.dev)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", target, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 10:  # wait for the first sample
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        with open(self.path) as f:
            self.skip = len(f.read().splitlines())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.read().splitlines()[self.skip:]
        os.unlink(self.path)
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < len(self.FIELDS):
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


def encode_traffic_per_elem():
    """DRAM bytes per element of the encode kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    summ = os.path.join(ROOT, "profiles", "encode_kernel_llama3_8b.md")
    src = os.path.join(ROOT, "sparse_bf16_delta_b200", "csrc", "encode.cu")
    if not os.path.exists(summ):
        return None, None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for ln in open(summ):
        if ln.startswith("- ") and ":" in ln:
            k, _, v = ln[2:].rpartition(": ")
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("encode.cu sha256[:16]") != h:
        return None, None
    try:
        return float(vals["dram bytes per element"]), float(vals["nnz fraction"])
    except (KeyError, ValueError):
        return None, None


# ---------------------------------------------------------------------------
# ncu DRAM figures for the rows, from the committed summaries under profiles/
# ---------------------------------------------------------------------------

def ncu_dram_GBps(profile):
    """DRAM GB/s (read + write bytes / duration) of the launch captured in a
    committed ncu summary, or None if the file or its figures are missing.
    ncu serialises launches and starts them with a cold cache."""
    path = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    dur = re.search(r"^\| duration[^|]*\| ([\d.,]+) us", txt, re.M)
    tot = re.search(r"dram__bytes_read\.sum \+ dram__bytes_write\.sum \| [\d.]+ \+ [\d.]+ = ([\d.]+) GB", txt)
    if tot:
        nbytes = float(tot.group(1)) * 1e9
    else:
        parts = [re.search(r"^\| dram__bytes_%s\.sum \| ([\d.]+) (GB|MB)" % k, txt, re.M) for k in ("read", "write")]
        if not all(parts):
            return None
        nbytes = sum(float(m.group(1)) * (1e9 if m.group(2) == "GB" else 1e6) for m in parts)
    if not dur:
        return None
    us = float(dur.group(1).replace(",", ""))
    return round(nbytes / (us * 1e-6) / 1e9, 1) if us > 0 else None


# Per bench row (first match wins): the committed captures of the kernels
# that carry it, with what differs between the captured case and the row,
# or why no DRAM figure applies.
_L2_RESIDENT = ("2 MB per snapshot stays in the 126 MB L2: a latency row, "
                "which the DRAM counters do not measure")
_HOST_LINK = "bound by the host link (copy engine transfers to or from pinned host memory), not by a kernel's DRAM traffic"
NCU_ROWS = [
    (r"^count_", [("encode_kernel_count_llama3_8b_2layers.md", "encode_kernel<0,0,0>", None)], None),
    (r"^encode_global_int64_", [("encode_kernel_global_llama3_8b_2layers.md", "encode_kernel<1,1,0>", None)], None),
    (r"^encode_checksum_", [("encode_kernel_checksum_llama3_8b_2layers.md", "encode_kernel<1,0,1>", None)], None),
    (r"^delta_file_", [], _HOST_LINK),
    (r"^encode_llama3_8b_lr1e-5", [("encode_kernel_llama3_8b_2layers_lr1e-5.md", "encode_kernel<1,0,0>", None)], None),
    (r"^apply_llama3_8b_lr1e-5", [("apply_kernel_llama3_8b_2layers_lr1e-5.md", "apply_kernel", None)], None),
    (r"^encode_llama3_8b", [("encode_kernel_llama3_8b.md", "encode_kernel<1,0,0>", None)], None),
    (r"^apply_llama3_8b", [("apply_kernel_llama3_8b.md", "apply_kernel", None)], None),
    (r"^pack_positions_", [("pack_positions_kernel_llama3_8b_2layers.md", "pack_positions_kernel", None)], None),
    (r"^checksum_", [("checksum_kernel_llama3_8b_2layers.md", "checksum_kernel", None)], None),
    (r"_single_1024x1024$", [], _L2_RESIDENT),
    (r"^apply_chain_qwen3_0p6b_k10_tile_merge$", [("chain_index_kernel_qwen3_0p6b_k10.md", "chain_index_kernel", None),
                                                  ("chain_tile_kernel_merge_qwen3_0p6b_k10.md", "chain_tile_kernel<merge>", None)], None),
    (r"^apply_chain_qwen3_0p6b_k10", [("chain_index_kernel_qwen3_0p6b_k10.md", "chain_index_kernel", None),
                                      ("chain_tile_kernel_scatter_qwen3_0p6b_k10.md", "chain_tile_kernel<scatter>", None)], None),
    (r"^merge_shards_", [("merge_copy_kernel_qwen3_0p6b_8ranks.md", "merge_copy_kernel", None)], None),
    (r"^encode_qwen3_0p6b", [("encode_kernel_qwen3_0p6b.md", "encode_kernel<1,0,0>", None)], None),
    (r"^xor_apply_layers_pinned_host", [], _HOST_LINK),
    (r"^xor_apply_layers_double_buffered", [("xor_vec_kernel_2x0.8GB.md", "xor_vec_kernel",
                                            "the apply kernel; the next layer's mask copy runs beside it on a copy engine")], None),
    (r"^xor_(encode|apply)_", [("xor_vec_kernel_2x0.8GB.md", "xor_vec_kernel", None)], None),
    (r"^encode_sparse_bytes_", [("encode_kernel_words_xor_2x0.8GB.md", "encode_kernel<1,0,0>", None),
                                ("bytes_write_kernel_xor_2x0.8GB.md", "bytes_write_kernel", None)], None),
    (r"^encode_sparse_", [("encode_kernel_words_xor_2x0.8GB.md", "encode_kernel<1,0,0>", None)], None),
    (r"^bytes_from_words_", [("bytes_write_kernel_xor_2x0.8GB.md", "bytes_write_kernel", None)], None),
    (r"^apply_bytes_", [("apply_bytes_kernel_xor_2x0.8GB.md", "apply_bytes_kernel", None)], None),
    (r"^apply_sparse_from_pinned_host", [], _HOST_LINK),
    (r"^apply_sparse_", [("apply_kernel_words_xor_2x0.8GB.md", "apply_kernel", None)], None),
    (r"^apply_chain_stress_.*_tile_merge$", [("chain_index_kernel_stress_1200t_k10.md", "chain_index_kernel",
                                              "captured on the 1200-tensor stress chain"),
                                             ("chain_tile_kernel_merge_stress_1200t_k10.md", "chain_tile_kernel<merge>",
                                              "captured on the 1200-tensor stress chain")], None),
    (r"^apply_chain_stress_", [("chain_index_kernel_stress_1200t_k10.md", "chain_index_kernel",
                                "captured on the 1200-tensor stress chain"),
                               ("chain_tile_kernel_scatter_stress_1200t_k10.md", "chain_tile_kernel<scatter>",
                                "captured on the 1200-tensor stress chain")], None),
    (r"^encode_stress_", [("encode_kernel_stress_1200t.md", "encode_kernel<1,0,0>",
                           "captured on the 1200-tensor stress set")], None),
]


def ncu_for_row(name):
    """The `ncu` entry of a bench row: per captured kernel its profile, its
    DRAM GB/s in the captured launch, and what differs from the row; or the
    reason there is none."""
    for pat, caps, reason in NCU_ROWS:
        if re.search(pat, name):
            if reason is not None:
                return {"dram_GBps": None, "reason": reason}
            out = []
            for prof, kernel, note in caps:
                e = {"kernel": kernel, "profile": "profiles/" + prof, "dram_GBps": ncu_dram_GBps(prof)}
                if note:
                    e["note"] = note
                out.append(e)
            return {"captures": out, "case": "ncu: one launch, cold cache, serialised"}
    return {"dram_GBps": None, "reason": "no committed capture for this row"}


def attach_ncu(rows):
    for name, row in rows.items():
        row["ncu"] = ncu_for_row(name)
    return rows


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def host_tensor(shapes, s, lr, device, t):
    """Tensor t of the workload (old and new bits on the host)."""
    import numpy as np
    import torch

    import workloads as W

    def bits(x):
        return x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    name, shape = shapes[t]
    n = W.numel(shape)
    std_mean = (0.01, 1.0) if W.is_norm(name) else (0.02, 0.0)
    w = W.init_tensor(n, W.weight_seed(s, t), device, *std_mean)
    u = W.update_noise(n, W.step_seed(s, 1, t), device)
    new = W.optimizer_step(w, u, lr)
    return bits(w), bits(new)


def layer_order(shapes):
    order = [i for i, (nm, _) in enumerate(shapes) if nm.startswith("model.layers.")]
    return order or list(range(len(shapes)))


PINNED_CORE = {"core": None}


@contextlib.contextmanager
def one_core():
    """Run the calling thread on one of its allowed cores (the lowest) and put
    its affinity back afterwards; without affinity support it runs unpinned."""
    try:
        allowed = os.sched_getaffinity(0)
        core = min(allowed)
        os.sched_setaffinity(0, {core})
    except (AttributeError, OSError, ValueError):
        yield None
        return
    try:
        PINNED_CORE["core"] = core
        yield core
    finally:
        os.sched_setaffinity(0, allowed)


def time_oracle(pairs):
    """Seconds the oracle spends on encode + apply over the (old, new) pairs,
    on one pinned core (the oracle is single-threaded)."""
    import oracle
    tot = 0.0
    with one_core():
        for a, b in pairs:
            snap = a.copy()
            t0 = time.perf_counter()
            o, i, v = oracle.encode([a], [b])
            oracle.apply([snap], o, i, v)
            tot += time.perf_counter() - t0
    return tot


def oracle_sample(shapes, s, lr, device, seconds):
    """Time the oracle's encode + apply tensor by tensor (decoder layers in
    order) until `seconds` of CPU time are spent.  Returns (bytes, secs,
    elements, tensors)."""
    tot_t, tot_n, count = 0.0, 0, 0
    for t in layer_order(shapes):
        a, b = host_tensor(shapes, s, lr, device, t)
        tot_t += time_oracle([(a, b)])
        tot_n += a.size
        count += 1
        if tot_t >= seconds:
            break
    return 2 * tot_n, tot_t, tot_n, count


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------------------
# --impl reference: the oracle as it stands on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    import torch
    import workloads as W
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    shapes = llama_shapes(args.layers)
    s = W.SEEDS["llama3_8b"]
    # Each step is a bounded sample of the workload, sized so that the whole
    # run stays within about two minutes of oracle time.
    per_step = min(5.0, max(0.3, 120.0 / max(1, args.steps + args.warmup)))
    order = layer_order(shapes)
    first = host_tensor(shapes, s, args.lr, dev, order[0])
    rate = first[0].size / max(1e-6, time_oracle([first]))
    pairs, n = [first], first[0].size
    for t in order[1:]:
        if n >= rate * per_step:
            break
        pairs.append(host_tensor(shapes, s, args.lr, dev, t))
        n += pairs[-1][0].size
    for _ in range(args.warmup):
        time_oracle(pairs)
    secs = [time_oracle(pairs) for _ in range(args.steps)]
    tt = sum(secs)
    value = 2 * n * args.steps / tt / 1e9
    sample = (f"per step: the first {len(pairs)} decoder-layer tensors of the Llama-3-8B-shaped "
              f"set ({n} bf16 elements, {2 * n / 1e9:.3f} GB of weights), oracle encode + apply, "
              f"one thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tt / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": "llama3_8b-shaped bf16 parameter set (bounded sample per step)",
                   "lr": args.lr, "parallelism": "replicas"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model(), "pinned_core": PINNED_CORE["core"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# --impl ours
# ---------------------------------------------------------------------------

def events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def time_reps(fn, reps, warm=1):
    """Median and min device time (ms) of fn() over reps, CUDA events."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = events(2)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts), min(ts)


def touched_sectors(offsets, indices):
    """Distinct 32-byte sectors (16 bf16 elements) a delta writes, counted
    on the device; every tensor starts on a 256-byte boundary in the bench's
    packed buffers, so sector k of a tensor is its elements [16k, 16k+16)."""
    import torch
    T = offsets.numel() - 1
    counts = offsets[1:] - offsets[:-1]
    if int(offsets[-1].item()) == 0:
        return 0
    tid = torch.repeat_interleave(torch.arange(T, device=offsets.device, dtype=torch.int64), counts)
    key = (tid << 40) | (indices.to(torch.int64) >> 4)  # ascending: tensor order, then index
    n = 1 + int((key[1:] != key[:-1]).sum().item())
    del tid, key
    return n


def clean_bytes(nnz, dev):
    """What dws_apply reads before its scatter: the delta arrays' first bytes,
    twice the L2 size at most (indices, then values)."""
    import torch
    budget = 2 * torch.cuda.get_device_properties(dev).L2_cache_size
    ib = min(4 * nnz, budget)
    return ib + min(2 * nnz, budget - ib)


def sector_model(nnz, sectors, ms, peak, pre=0):
    """The apply's DRAM traffic model: 6 bytes read per entry, every touched
    32-byte sector read and written back whole by L2 (HBM has no byte-masked
    writes), and the `pre` bytes read before the scatter: 6 nnz + 64 S + pre."""
    b = 6 * nnz + 64 * sectors + pre
    return {"sectors": sectors, "traffic_model_bytes": b, "traffic_model_pre_read_bytes": pre,
            "traffic_model_GBps": round(b / ms / 1e6, 1), "traffic_model_frac": round(b / ms / 1e6 / peak, 4)}


def row(name, ms, alg_bytes, weight_bytes, peak, extra=None, elems=None):
    """A bench row: time, algorithmic and weight GB/s, the fraction of the HBM
    peak and elements per second (elems: the row's elements, default the bf16
    elements of weight_bytes)."""
    elems = weight_bytes // 2 if elems is None else elems
    d = {"ms": round(ms, 4), "alg_GBps": round(alg_bytes / ms / 1e6, 1),
         "weight_GBps": round(weight_bytes / ms / 1e6, 1),
         "elems_per_s": round(elems / ms * 1e3, 1),
         "hbm_frac": round(alg_bytes / ms / 1e6 / peak, 4)}
    if extra:
        d.update(extra)
    return name, d


ROW_GROUPS = ("single", "qwen_chain", "xor", "stress_chain")
# (dws_apply_chain_ex mode, row-name suffix); 0 = the library's default
CHAIN_MODES = ((0, ""), (1, "_tile_merge"), (2, "_scatter"))


def rows_single(args, dev, peak):
    """Workload 1 (one 1024x1024 bf16 tensor, one step at lr 3e-6): latency of
    encode, apply, XOR encode and XOR apply, median of 50 launches.  4 MB in
    all: it lives in L2, so these rows measure latency, not HBM bandwidth."""
    import torch

    import sparse_bf16_delta_b200 as dws
    import workloads as W
    old, new = W.single(dev)
    a, b = old.tensors[0], new.tensors[0]
    N = a.numel()
    plan = dws.DeltaPlan.for_tensors([a])
    ot, nt = dws.ptr_table([a]), dws.ptr_table([b])
    d = plan.encode_exact(ot, nt)
    nnz = d.nnz()
    snap = a.clone()
    st = dws.ptr_table([snap])
    mask = torch.empty(2 * N, dtype=torch.uint8, device=dev)
    buf = a.clone()
    reps = max(50, args.rows_reps)
    ms_e, mn_e = time_reps(lambda: plan.encode_into(ot, nt, d.offsets, d.indices, d.values), reps, warm=5)
    ms_a, mn_a = time_reps(lambda: plan.apply(st, d), reps, warm=5)
    ok = bool(torch.equal(snap, b)) and plan.status()[0] == dws.DWS_OK
    ms_x, mn_x = time_reps(lambda: dws.xor_encode(a, b, mask), reps, warm=5)
    ms_y, mn_y = time_reps(lambda: (dws.xor_apply(buf, mask), dws.xor_apply(buf, mask)), reps, warm=5)
    ok_x = bool(torch.equal(buf, a))
    lat = {"latency_row": True, "l2_resident": True, "reps": reps}
    out = {}
    out.update([row("encode_single_1024x1024", ms_e, 4 * N + 6 * nnz, 2 * N, peak,
                    {**lat, "min_ms": round(mn_e, 4), "nnz": nnz})])
    out.update([row("apply_single_1024x1024", ms_a, 8 * nnz, 2 * N, peak,
                    {**lat, "min_ms": round(mn_a, 4), "exact": ok})])
    out.update([row("xor_encode_single_1024x1024", ms_x, 6 * N, 2 * N, peak,
                    {**lat, "min_ms": round(mn_x, 4)}, elems=2 * N)])
    out.update([row("xor_apply_single_1024x1024", ms_y / 2, 6 * N, 2 * N, peak,
                    {**lat, "min_ms": round(mn_y / 2, 4), "exact": ok_x}, elems=2 * N)])
    return out


def run_rows(args, dev, peak, groups=ROW_GROUPS):
    """The other hot-path rows, each on its own workload, timed with events."""
    out = {}
    if "single" in groups:
        out.update(rows_single(args, dev, peak))
    if "qwen_chain" in groups:
        out.update(rows_qwen_chain(args, dev, peak))
    if "xor" in groups:
        out.update(rows_xor(args, dev, peak))
    if "stress_chain" in groups:
        out.update(rows_stress_chain(args, dev, peak))
    return out


def rows_qwen_chain(args, dev, peak):
    """Qwen3-0.6B-shaped chain of 10 deltas: replay, and encode of each step."""
    import gc

    import torch

    import sparse_bf16_delta_b200 as dws
    import workloads as W
    out = {}
    t0 = time.time()
    s = W.SEEDS["qwen3_0p6b"]
    shapes = W.qwen3_0p6b_shapes()
    sizes = [W.numel(sh) for _, sh in shapes]
    std = [(0.01, 1.0) if W.is_norm(nm) else (0.02, 0.0) for nm, _ in shapes]
    anchor_flat, anchor = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, *std[t]), dev)
    plan = dws.DeltaPlan.for_tensors(anchor)
    prev_flat, prev = W.pack_flat(sizes, lambda t, n: anchor[t], dev)
    cur_flat, cur = W.pack_flat(sizes, lambda t, n: None, dev)
    deltas, enc_ms, nnzs = [], [], []
    for k in range(1, 11):
        for t in range(len(sizes)):
            u = W.update_noise(sizes[t], W.step_seed(s, k, t), dev)
            cur[t].copy_(W.optimizer_step(prev[t], u, 3e-6))
        ot, nt = dws.ptr_table(prev), dws.ptr_table(cur)
        d = plan.encode_exact(ot, nt)
        ms, _ = time_reps(lambda: plan.encode_into(ot, nt, d.offsets, d.indices, d.values), 3)
        enc_ms.append(ms)
        nnzs.append(d.nnz())
        deltas.append(d)
        prev_flat, cur_flat = cur_flat, prev_flat
        prev, cur = cur, prev
    N = sum(sizes)
    tot = sum(nnzs)
    for mode, suffix in CHAIN_MODES:
        snap_flat = anchor_flat.clone()
        snap = [snap_flat[v.storage_offset() - anchor_flat.storage_offset():][:v.numel()] for v in anchor]
        st = dws.ptr_table(snap)
        # every rep replays onto the result of the previous one: the same
        # writes, and the snapshot stays the final one
        ms, mn = time_reps(lambda: plan.apply_chain(st, deltas, mode=mode), args.rows_reps)
        plan.raise_on_error("qwen chain")
        ok = torch.equal(snap_flat, prev_flat)
        out.update([row("apply_chain_qwen3_0p6b_k10" + suffix, ms, 4 * N + 6 * tot, 2 * N, peak,
                        {"min_ms": round(mn, 4), "nnz_total": tot, "exact": ok})])
        del snap_flat, snap, st
    out.update(merge_shards_row(args, dev, peak, plan, shapes, deltas[0]))
    mean_enc = statistics.mean(enc_ms)
    out.update([row("encode_qwen3_0p6b", mean_enc, 4 * N + 6 * tot / 10, 2 * N, peak,
                    {"nnz_mean": tot // 10, "sparsity_mean": round(1 - tot / 10 / N, 5)})])
    del deltas, anchor_flat, prev_flat, cur_flat, anchor, prev, cur, plan
    gc.collect()
    torch.cuda.empty_cache()
    log(f"rows: qwen chain done in {time.time() - t0:.1f}s")
    return out


def merge_shards_row(args, dev, peak, plan, shapes, d, R=8):
    """Rank 0's merge of sharded deltas (dws_merge_shards): step 1 of the
    Qwen3-0.6B chain split among R simulated ranks as FSDP Shard(0) would
    (rank r holds rows [r c, (r+1) c) of every parameter, c = ceil(rows / R)),
    each rank's delta in global int64 positions, padded and stacked as the
    gather leaves them on rank 0; then merged back.  Reads and writes 10
    bytes per entry."""
    import torch

    import sparse_bf16_delta_b200 as dws
    T = len(shapes)
    counts = d.offsets[1:] - d.offsets[:-1]
    tid = torch.repeat_interleave(torch.arange(T, device=dev), counts)
    rows = torch.tensor([sh[0] for _, sh in shapes], dtype=torch.int64, device=dev)
    numel = torch.tensor([math.prod(sh) for _, sh in shapes], dtype=torch.int64, device=dev)
    rowlen = numel // rows
    chunk = (rows + R - 1) // R * rowlen
    gidx = d.indices.to(torch.int64)
    rank = torch.clamp(gidx // chunk[tid], max=R - 1)
    per = []
    for r in range(R):
        m = rank == r
        c = torch.bincount(tid[m], minlength=T)
        o = torch.zeros(T + 1, dtype=torch.int64, device=dev)
        o[1:] = torch.cumsum(c, 0)
        per.append((o, gidx[m], d.values[m]))
    stride = max(int(x[1].numel()) for x in per)
    ro = torch.stack([x[0] for x in per])
    ri = torch.zeros(R, stride, dtype=torch.int64, device=dev)
    rv = torch.zeros(R, stride, dtype=torch.int16, device=dev)
    for r, (_, i, v) in enumerate(per):
        ri[r, :i.numel()] = i
        rv[r, :v.numel()] = v
    nnz = int(gidx.numel())
    offs = torch.empty(T + 1, dtype=torch.int64, device=dev)
    oidx = torch.empty(nnz, dtype=torch.int64, device=dev)
    oval = torch.empty(nnz, dtype=torch.int16, device=dev)
    cs = torch.cuda.current_stream().cuda_stream

    def merge():
        dws.dws_merge_shards(plan.handle, R, ro.data_ptr(), ri.data_ptr(), rv.data_ptr(), stride,
                             offs.data_ptr(), oidx.data_ptr(), oval.data_ptr(), nnz,
                             plan.workspace.data_ptr(), plan.workspace_bytes, cs)

    ms, mn = time_reps(merge, args.rows_reps)
    ok = (plan.status()[0] == dws.DWS_OK and torch.equal(offs, d.offsets) and torch.equal(oidx, gidx)
          and torch.equal(oval, d.values))
    out = [row(f"merge_shards_qwen3_0p6b_{R}ranks", ms, 20 * nnz + 8 * (T + 1) * (R + 1), 0, peak,
               {"min_ms": round(mn, 4), "entries": nnz, "entries_per_s": round(nnz / ms * 1e3, 1),
                "exact": ok}, elems=nnz)]
    del ro, ri, rv, offs, oidx, oval, per
    return out


def rows_xor(args, dev, peak):
    """XOR path: 40 layers x 0.8 GB, encode, apply, double-buffered apply."""
    import gc

    import torch

    import sparse_bf16_delta_b200 as dws
    import workloads as W
    out = {}
    t0 = time.time()
    L, B = args.xor_layers, 800_000_000
    tag = f"{L}x0.8GB"
    olds, news, masks = [], [], []
    for l in range(L):
        o, n, _ = W.xor_layer(l, dev, nbytes=B)
        olds.append(o)
        news.append(n)
        masks.append(torch.empty(B, dtype=torch.uint8, device=dev))
    torch.cuda.synchronize()

    def xor_enc():
        for l in range(L):
            dws.xor_encode(olds[l], news[l], masks[l])

    ms, mn = time_reps(xor_enc, args.rows_reps)
    ok = all(int(torch.count_nonzero(masks[l])) == 680_000 for l in (0, L - 1))
    out.update([row("xor_encode_nvfp4_" + tag, ms, 3 * L * B, L * B, peak,
                    {"min_ms": round(mn, 4), "launches": L, "exact_flip_count": ok}, elems=L * B)])
    # apply twice per rep so the buffers end where they started
    bufs = olds

    def xor_app2():
        for l in range(L):
            dws.xor_apply(bufs[l], masks[l])
        for l in range(L):
            dws.xor_apply(bufs[l], masks[l])

    ms2, mn2 = time_reps(xor_app2, args.rows_reps)
    out.update([row("xor_apply_nvfp4_" + tag, ms2 / 2, 3 * L * B, L * B, peak,
                    {"min_ms": round(mn2 / 2, 4)}, elems=L * B)])
    # double-buffered layer pipeline, masks staged D2D (stand-in for the DE)
    staging = [torch.empty(B, dtype=torch.uint8, device=dev) for _ in range(2)]
    cs = torch.cuda.Stream()

    def pipe2():
        dws.xor_apply_layers(bufs, masks, staging[0], staging[1], copy_stream=cs)
        dws.xor_apply_layers(bufs, masks, staging[0], staging[1], copy_stream=cs)

    msp, mnp = time_reps(pipe2, max(2, args.rows_reps // 2))
    dws.xor_apply(bufs[0], masks[0])
    dws.xor_apply(bufs[L - 1], masks[L - 1])
    torch.cuda.synchronize()
    ok = torch.equal(bufs[0], news[0]) and torch.equal(bufs[L - 1], news[L - 1])
    dws.xor_apply(bufs[0], masks[0])
    dws.xor_apply(bufs[L - 1], masks[L - 1])
    out.update([row("xor_apply_layers_double_buffered_" + tag, msp / 2, 5 * L * B, L * B, peak,
                    {"min_ms": round(mnp / 2, 4), "staging": "2 x 0.8 GB, D2D copy stream",
                     "exact": ok}, elems=L * B)])
    # the same pipeline with the masks in pinned host memory (the host link
    # bounds it): 4 layers, against a plain pinned H2D copy of one layer
    LH = min(4, L)
    hmasks = [torch.empty(B, dtype=torch.uint8, pin_memory=True) for _ in range(LH)]
    for l in range(LH):
        hmasks[l].copy_(masks[l])
    ms_h2d, _ = time_reps(lambda: staging[0].copy_(hmasks[0], non_blocking=True), args.rows_reps)

    def pipe_host2():
        dws.xor_apply_layers(bufs[:LH], hmasks, staging[0], staging[1], copy_stream=cs)
        dws.xor_apply_layers(bufs[:LH], hmasks, staging[0], staging[1], copy_stream=cs)

    msh, mnh = time_reps(pipe_host2, max(2, args.rows_reps // 2))
    dws.xor_apply(bufs[0], masks[0])
    torch.cuda.synchronize()
    ok_h = torch.equal(bufs[0], news[0])
    dws.xor_apply(bufs[0], masks[0])
    link = LH * B / (msh / 2) / 1e6
    out[f"xor_apply_layers_pinned_host_{LH}x0.8GB"] = {
        "ms": round(msh / 2, 3), "min_ms": round(mnh / 2, 3), "link_GBps": round(link, 1),
        "h2d_copy_GBps": round(B / ms_h2d / 1e6, 1), "link_frac": round(link / (B / ms_h2d / 1e6), 4),
        "bound": "host link (plain pinned H2D copy of 0.8 GB timed in the same run)", "exact": ok_h}
    del hmasks
    # the same layers as a sparse delta of 16-bit words (indices + values):
    # 680,000 changed bytes per layer travel as about 4 MB instead of 0.8 GB
    ow = [o.view(torch.bfloat16) for o in olds]
    nw = [n.view(torch.bfloat16) for n in news]
    splan = dws.DeltaPlan.for_tensors(ow)
    sot, snt = dws.ptr_table(ow), dws.ptr_table(nw)
    sd = splan.encode_exact(sot, snt)
    snnz = sd.nnz()
    ms_e, mn_e = time_reps(lambda: splan.encode_into(sot, snt, sd.offsets, sd.indices, sd.values),
                           args.rows_reps)
    out.update([row("encode_sparse_nvfp4_" + tag, ms_e, 2 * L * B + 6 * snnz, L * B, peak,
                    {"min_ms": round(mn_e, 4), "nnz": snnz, "delta_bytes": 6 * snnz + 8 * (L + 1)},
                    elems=L * B)])
    # the same delta at byte granularity: one entry per changed byte (int32
    # position + the new byte, 5 bytes) made from the word delta
    bo, bp, bv = splan.xor_bytes_from_words(sot, sd)
    bn = int(bo[-1].item())
    st_ = torch.cuda.current_stream().cuda_stream
    so_, si_, sv_, sc_ = sd.as_ref()

    def to_bytes():
        dws.dws_xor_bytes_from_words(splan.handle, sot.data_ptr(), so_, si_, sv_, sc_, bo.data_ptr(),
                                     bp.data_ptr(), bv.data_ptr(), bp.numel(), splan.workspace.data_ptr(),
                                     splan.workspace_bytes, st_)

    ms_b, mn_b = time_reps(to_bytes, args.rows_reps)
    splan.raise_on_error("xor bytes from words")
    conv_bytes = 8 * snnz + 5 * bn  # word entries + the old words gathered, byte entries written
    out.update([row("bytes_from_words_nvfp4_" + tag, ms_b, conv_bytes, L * B, peak,
                    {"min_ms": round(mn_b, 4), "byte_entries": bn, "word_entries": snnz,
                     "delta_bytes": 5 * bn + 8 * (L + 1), "word_delta_bytes": 6 * snnz + 8 * (L + 1)},
                    elems=L * B)])

    def enc_bytes():
        splan.encode_into(sot, snt, sd.offsets, sd.indices, sd.values)
        to_bytes()

    ms_eb, mn_eb = time_reps(enc_bytes, args.rows_reps)
    out.update([row("encode_sparse_bytes_nvfp4_" + tag, ms_eb, 2 * L * B + 6 * snnz + conv_bytes, L * B, peak,
                    {"min_ms": round(mn_eb, 4), "byte_entries": bn, "delta_bytes": 5 * bn + 8 * (L + 1)},
                    elems=L * B)])
    bst = dws.ptr_table(olds)
    ms_ab, mn_ab = time_reps(lambda: splan.apply_bytes(bst, bo, bp, bv, count=bn), args.rows_reps)
    splan.raise_on_error("byte xor apply")
    ok_b = all(torch.equal(olds[l], news[l]) for l in (0, L - 1))
    out.update([row("apply_bytes_nvfp4_" + tag, ms_ab, 6 * bn, L * B, peak,
                    {"min_ms": round(mn_ab, 4), "exact": ok_b,
                     "entries_per_s": round(bn / ms_ab * 1e3, 1)}, elems=L * B)])
    del bo, bp, bv, bst
    sst = dws.ptr_table(ow)
    ms_a, mn_a = time_reps(lambda: splan.apply(sst, sd), args.rows_reps)
    splan.raise_on_error("sparse xor apply")
    ok = all(torch.equal(olds[l], news[l]) for l in (0, L - 1))
    out.update([row("apply_sparse_nvfp4_" + tag, ms_a, 8 * snnz, L * B, peak,
                    {"min_ms": round(mn_a, 4), "exact": ok,
                     "entries_per_s": round(snnz / ms_a * 1e3, 1)}, elems=L * B)])
    # that delta arriving from pinned host memory: H2D of its 6 bytes per
    # entry, then the apply (the dense masks would move all 32 GB)
    hd = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in
          (sd.offsets, sd.indices, sd.values)]
    for h, x in zip(hd, (sd.offsets, sd.indices, sd.values)):
        h.copy_(x)
    rd = dws.Delta(torch.empty_like(sd.offsets), torch.empty_like(sd.indices),
                   torch.empty_like(sd.values))

    def host_apply():
        for x, h in zip((rd.offsets, rd.indices, rd.values), hd):
            x.copy_(h, non_blocking=True)
        splan.apply(sst, rd)

    ms_ha, mn_ha = time_reps(host_apply, args.rows_reps)
    splan.raise_on_error("sparse xor apply from host")
    hbytes = sum(h.numel() * h.element_size() for h in hd)
    out["apply_sparse_from_pinned_host_nvfp4_" + tag] = {
        "ms": round(ms_ha, 3), "min_ms": round(mn_ha, 3), "h2d_bytes": hbytes,
        "link_GBps": round(hbytes / ms_ha / 1e6, 1),
        "exact": all(torch.equal(olds[l], news[l]) for l in (0, L - 1))}
    del hd, rd
    del ow, nw, splan, sot, snt, sd, sst
    del olds, news, masks, bufs, staging
    gc.collect()
    torch.cuda.empty_cache()
    log(f"rows: xor done in {time.time() - t0:.1f}s")
    return out


def rows_stress_chain(args, dev, peak):
    """12000 log-uniform tensors, half with clustered changes: chain of 10."""
    import gc

    import torch

    import sparse_bf16_delta_b200 as dws
    import workloads as W
    out = {}
    t0 = time.time()
    s = W.SEEDS["stress"]
    sizes = W.stress_sizes(count=args.stress_tensors)
    clustered = W.stress_clustered(count=args.stress_tensors)
    stag = f"{args.stress_tensors}t"
    anchor_flat, anchor = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, 0.02), dev)
    plan = dws.DeltaPlan.for_tensors(anchor)
    prev_flat, prev = W.pack_flat(sizes, lambda t, n: anchor[t], dev)
    cur_flat, cur = W.pack_flat(sizes, lambda t, n: None, dev)
    deltas, nnzs, enc_ms, exp_nnz = [], [], [], []
    for k in range(1, 11):
        picked_total = 0
        for t in range(len(sizes)):
            nw, pk = W.stress_change(prev[t], clustered[t], W.step_seed(s, k, t), dev)
            cur[t].copy_(nw)
            picked_total += int(pk.sum())
        ot, nt = dws.ptr_table(prev), dws.ptr_table(cur)
        d = plan.encode_exact(ot, nt)
        ms, _ = time_reps(lambda: plan.encode_into(ot, nt, d.offsets, d.indices, d.values), 3)
        enc_ms.append(ms)
        nnzs.append(d.nnz())
        exp_nnz.append(picked_total)
        deltas.append(d)
        prev_flat, cur_flat = cur_flat, prev_flat
        prev, cur = cur, prev
    N = sum(sizes)
    tot = sum(nnzs)
    for mode, suffix in CHAIN_MODES:
        snap_flat = anchor_flat.clone()
        snap = [snap_flat[v.storage_offset() - anchor_flat.storage_offset():][:v.numel()] for v in anchor]
        st = dws.ptr_table(snap)
        ms, mn = time_reps(lambda: plan.apply_chain(st, deltas, mode=mode), args.rows_reps)
        plan.raise_on_error("stress chain")
        ok = torch.equal(snap_flat, prev_flat) and nnzs == exp_nnz
        out.update([row("apply_chain_stress_" + stag + "_k10" + suffix, ms, 4 * N + 6 * tot, 2 * N, peak,
                        {"min_ms": round(mn, 4), "elements": N, "nnz_total": tot, "exact": ok})])
        del snap_flat, snap, st
    out.update([row("encode_stress_" + stag, statistics.mean(enc_ms), 4 * N + 6 * tot / 10, 2 * N, peak,
                    {"nnz_mean": tot // 10})])
    del deltas, anchor_flat, prev_flat, cur_flat, anchor, prev, cur, plan
    gc.collect()
    torch.cuda.empty_cache()
    log(f"rows: stress chain done in {time.time() - t0:.1f}s")
    return out


def delta_file_rows(dws, plan, names, delta, args):
    """The delta as a safetensors file: device arrays -> pinned host file
    (header on the host + two D2H copies) and back (parse + H2D copies),
    against plain pinned copies of the same bytes timed in the same run."""
    import numpy as np
    import torch
    out = {}
    T = len(names)
    nnz = delta.count
    arr = dws.make_name_array(names)
    oh = delta.offsets.cpu().numpy()
    cs = torch.cuda.current_stream().cuda_stream
    st, fbytes = dws.dws_st_delta_write(plan.handle, arr, oh.ctypes.data, 1, delta.indices.data_ptr(),
                                        delta.values.data_ptr(), None, 0, cs)
    fbuf = torch.empty(fbytes, dtype=torch.uint8, pin_memory=True)

    def write():
        dws.dws_st_delta_write(plan.handle, arr, oh.ctypes.data, 1, delta.indices.data_ptr(),
                               delta.values.data_ptr(), fbuf.data_ptr(), fbytes, cs)

    ms_w, mn_w = time_reps(write, args.rows_reps)
    hb = fbytes - 6 * nnz
    body = fbuf[hb:]

    def plain_d2h():
        body[:4 * nnz].copy_(delta.indices.view(torch.uint8), non_blocking=True)
        body[4 * nnz:].copy_(delta.values.view(torch.uint8), non_blocking=True)

    ms_pd, _ = time_reps(plain_d2h, args.rows_reps)
    out["delta_file_write_llama3_8b"] = {
        "ms": round(ms_w, 3), "min_ms": round(mn_w, 3), "file_bytes": fbytes, "header_bytes": hb,
        "GBps": round(fbytes / ms_w / 1e6, 1), "plain_d2h_ms": round(ms_pd, 3),
        "link_frac": round(ms_pd / ms_w, 4),
        "bound": "host link (plain pinned D2H copies of the same bytes timed in the same run)"}
    oh2 = np.zeros(T + 1, dtype=np.int64)
    r_off = torch.empty_like(delta.offsets)
    r_idx = torch.empty_like(delta.indices)
    r_val = torch.empty_like(delta.values)

    def read():
        dws.dws_st_delta_read(plan.handle, arr, fbuf.data_ptr(), fbytes, oh2.ctypes.data,
                              r_off.data_ptr(), r_idx.data_ptr(), r_val.data_ptr(), nnz, cs)

    ms_r, mn_r = time_reps(read, args.rows_reps)
    torch.cuda.synchronize()
    ok = (torch.equal(r_off, delta.offsets) and torch.equal(r_idx, delta.indices)
          and torch.equal(r_val, delta.values))

    def plain_h2d():
        r_idx.view(torch.uint8).copy_(body[:4 * nnz], non_blocking=True)
        r_val.view(torch.uint8).copy_(body[4 * nnz:], non_blocking=True)

    ms_ph, _ = time_reps(plain_h2d, args.rows_reps)
    out["delta_file_read_llama3_8b"] = {
        "ms": round(ms_r, 3), "min_ms": round(mn_r, 3), "GBps": round(fbytes / ms_r / 1e6, 1),
        "plain_h2d_ms": round(ms_ph, 3), "link_frac": round(ms_ph / ms_r, 4), "exact": ok,
        "bound": "host link (plain pinned H2D copies of the same bytes timed in the same run)"}
    del fbuf, body, r_off, r_idx, r_val
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import sparse_bf16_delta_b200 as dws
    import workloads as W

    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    peak, peak_kind = measured_peaks()

    if args.rows_only:
        groups = [g.strip() for g in args.rows_only.split(",") if g.strip()]
        bad = [g for g in groups if g not in ROW_GROUPS]
        if bad:
            raise SystemExit(f"unknown row group(s) {bad}; choose from {ROW_GROUPS}")
        rows = run_rows(args, dev, peak, groups)
        exact = all(v.get("exact", True) and v.get("exact_flip_count", True) for v in rows.values())
        if rank == 0:
            print(json.dumps({"rows": attach_ncu(rows), "rows_only": groups}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0 if exact else 3

    # ---- workload: Llama-3-8B-shaped set, one step -------------------------
    t0 = time.time()
    s = W.SEEDS["llama3_8b"]
    shapes = llama_shapes(args.layers)
    sizes = [W.numel(sh) for _, sh in shapes]
    std = [(0.01, 1.0) if W.is_norm(nm) else (0.02, 0.0) for nm, _ in shapes]
    T, N = len(sizes), sum(sizes)
    old_flat, old = W.pack_flat(sizes, lambda t, n: W.init_tensor(n, W.weight_seed(s, t), dev, *std[t]), dev)

    def make_new(lr):
        def mk(t, n):
            u = W.update_noise(n, W.step_seed(s, 1, t), dev)
            return W.optimizer_step(old[t], u, lr)
        return mk

    new_flat, new = W.pack_flat(sizes, make_new(args.lr), dev)
    torch.cuda.synchronize()
    log(f"[rank {rank}] generated {T} tensors, {N} elements in {time.time() - t0:.1f}s")

    plan = dws.DeltaPlan.for_tensors(old)
    ot, nt = dws.ptr_table(old), dws.ptr_table(new)
    offsets = plan.count(ot, nt)
    plan.raise_on_error("dws_count")
    nnz = int(offsets[-1].item())
    indices = torch.empty(nnz, dtype=torch.int32, device=dev)
    values = torch.empty(nnz, dtype=torch.int16, device=dev)
    delta = dws.Delta(offsets, indices, values)
    snap_flat = old_flat.clone()
    snap = [snap_flat[v.storage_offset():][:v.numel()] for v in old]
    st = dws.ptr_table(snap)

    def encode():
        plan.encode_into(ot, nt, offsets, indices, values)

    def apply():
        plan.apply(st, delta)

    for _ in range(args.warmup):
        encode()
        apply()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    K = args.steps
    e_enc0, e_enc1, e_app1 = events(K), events(K), events(K)
    start, end = events(2)
    props = torch.cuda.get_device_properties(dev)
    theo, mem_khz, bus_bits = theoretical_hbm_gbs(dws, dev.index if dev.index is not None else 0)
    clocks = Clocks(local, str(getattr(props, "uuid", "")) or None)
    clocks.start()
    launches0 = dws.dws_launch_count()
    start.record()
    for k in range(K):
        e_enc0[k].record()
        encode()
        e_enc1[k].record()
        apply()
        e_app1[k].record()
    end.record()
    torch.cuda.synchronize()
    launches = dws.dws_launch_count() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    total_ms = start.elapsed_time(end)
    enc_ms = statistics.mean(e_enc0[k].elapsed_time(e_enc1[k]) for k in range(K))
    app_ms = statistics.mean(e_enc1[k].elapsed_time(e_app1[k]) for k in range(K))
    total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / K

    # correctness of what was timed: the applied snapshot is the new snapshot
    st_code, st_detail = plan.status()
    exact = bool(torch.equal(snap_flat, new_flat)) and st_code == dws.DWS_OK
    if not exact:
        log(f"[rank {rank}] RESULT MISMATCH (status {st_code}, detail {st_detail})")

    weight_bytes = 2 * N
    value = replicas_value(world, weight_bytes, ms_per_step)
    enc_alg = 4 * N + 6 * nnz + 8 * (T + 1)
    achieved = enc_alg / (enc_ms / 1e3) / 1e9
    tpe, nnz_frac_prof = encode_traffic_per_elem()
    traffic = None
    if tpe is not None:
        traffic = int(tpe * N)
    app_alg = 8 * nnz
    app_sectors = touched_sectors(offsets, indices)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
        "data": "synthetic (seeded random bf16 weights of the model's shapes; no trained weights)",
        "config": {
            "workload": (f"llama3_8b-shaped bf16 parameter set: {T} tensors, {N} elements "
                         f"({weight_bytes / 1e9:.2f} GB per snapshot), one simulated optimizer step at lr {args.lr}"),
            "step": "dws_encode(old,new -> delta) + dws_apply(delta -> snapshot), one launch each over all tensors",
            "lr": args.lr, "nnz": nnz, "sparsity": round(1 - nnz / N, 6),
            "delta_bytes": 6 * nnz + 8 * (T + 1),
            "l2": "inputs (2 x 16 GB) >> 126 MB L2; no flush needed",
            "parallelism": f"replicas x{world}",
        },
        "hbm_frac_step": round((enc_alg + app_alg) / (ms_per_step / 1e3) / 1e9 / peak, 4),
        "kernels": {
            "encode": {"ms": round(enc_ms, 4), "alg_bytes": enc_alg,
                       "alg_GBps": round(achieved, 1), "weight_GBps": round(weight_bytes / enc_ms / 1e6, 1),
                       "elems_per_s": round(N / enc_ms * 1e3, 1),
                       "ncu": ncu_for_row("encode_llama3_8b")},
            "apply": {"ms": round(app_ms, 4), "alg_bytes": app_alg,
                      "alg_GBps": round(app_alg / app_ms / 1e6, 1),
                      "weight_GBps": round(weight_bytes / app_ms / 1e6, 1),
                      "elems_per_s": round(N / app_ms * 1e3, 1),
                      "entries_per_s": round(nnz / app_ms * 1e3, 1),
                      **sector_model(nnz, app_sectors, app_ms, peak, clean_bytes(nnz, dev)),
                      "ncu": ncu_for_row("apply_llama3_8b")},
        },
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": "encode (dws_encode: workspace reset + fused detect/scan/compact)",
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "theoretical_peak": round(theo, 1) if theo else None,
                     "theoretical_inputs": {"memory_clock_khz": mem_khz, "bus_width_bits": bus_bits,
                                            "formula": "khz x 1e3 x 2 x bits / 8"},
                     "frac_of_theoretical": round(achieved / theo, 4) if theo else None},
        "gpu_launches": int(launches),
        "clocks": clk,
        "exact": exact,
    }

    # ---- e2e: new snapshot from pinned host memory, delta through the host --
    # as the delta file of the pages' wire format: the trainer side writes it
    # into pinned host memory, the receiver side reads it back and applies it.
    if not args.no_e2e:
        import numpy as np
        host_new = torch.empty_like(new_flat, device="cpu").pin_memory()
        host_new.copy_(new_flat)
        names_arr = dws.make_name_array([nm for nm, _ in shapes])
        h_off = torch.empty_like(offsets, device="cpu").pin_memory()
        h_off_np = h_off.numpy()
        h_off.copy_(offsets)
        st_, fcap = dws.dws_st_delta_write(plan.handle, names_arr, h_off_np.ctypes.data, 1, 0, 0,
                                           None, 0, 0)
        fbuf = torch.empty(fcap, dtype=torch.uint8, pin_memory=True)
        oh2 = np.zeros(T + 1, dtype=np.int64)
        r_off, r_idx, r_val = torch.empty_like(offsets), torch.empty_like(indices), torch.empty_like(values)
        rdelta = dws.Delta(r_off, r_idx, r_val)
        cs_e = torch.cuda.current_stream()
        codes = []

        def e2e_step():
            new_flat.copy_(host_new, non_blocking=True)
            plan.encode_into(ot, nt, offsets, indices, values)
            h_off.copy_(offsets, non_blocking=True)
            cs_e.synchronize()  # the file's header needs the counts
            cw, fb = dws.dws_st_delta_write(plan.handle, names_arr, h_off_np.ctypes.data, 1,
                                            indices.data_ptr(), values.data_ptr(), fbuf.data_ptr(),
                                            fcap, cs_e.cuda_stream)
            cr, _, _ = dws.dws_st_delta_read(plan.handle, names_arr, fbuf.data_ptr(), fb,
                                             oh2.ctypes.data, r_off.data_ptr(), r_idx.data_ptr(),
                                             r_val.data_ptr(), r_idx.numel(), cs_e.cuda_stream)
            codes.append((cw, cr))
            plan.apply(st, rdelta)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = events(2)
        a.record()
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), world, dev) / args.e2e_steps
        ok = (bool(torch.equal(snap_flat, new_flat)) and plan.status()[0] == dws.DWS_OK
              and all(c == (dws.DWS_OK, dws.DWS_OK) for c in codes))
        line["e2e"] = {"value": round(replicas_value(world, weight_bytes, e_ms), 2), "unit": "GB/s",
                       "h2d_bytes_per_step": 2 * new_flat.numel() + 6 * nnz + 8 * (T + 1),
                       "d2h_bytes_per_step": 8 * (T + 1) + 6 * nnz, "ms_per_step": round(e_ms, 3),
                       "steps": args.e2e_steps, "exact": ok, "delta_file_bytes": fcap,
                       "path": ("pinned host new snapshot -> H2D -> dws_encode -> offsets D2H -> "
                                "dws_st_delta_write (delta file into pinned host memory) -> "
                                "dws_st_delta_read (back into device arrays) -> dws_apply")}
        del host_new, h_off, fbuf, r_off, r_idx, r_val, rdelta

    # ---- encode / apply at lr 1e-5 and count-only ----------------------------
    if not args.no_rows:
        ms_c, _ = time_reps(lambda: plan.count(ot, nt, offsets), args.rows_reps)
        rows = {}
        rows.update([row("count_llama3_8b_lr%g" % args.lr, ms_c, 4 * N, weight_bytes, peak)])
        # the same step with int64 global positions (shard offset per tensor)
        bases = torch.tensor([(t + 1) * (1 << 33) for t in range(T)], dtype=torch.int64, device=dev)
        gidx = torch.empty(nnz, dtype=torch.int64, device=dev)
        gval = torch.empty(nnz, dtype=torch.int16, device=dev)
        goffs = torch.empty(T + 1, dtype=torch.int64, device=dev)
        cs0 = torch.cuda.current_stream().cuda_stream

        def enc_global():
            dws.dws_encode_global(plan.handle, ot.data_ptr(), nt.data_ptr(), bases.data_ptr(),
                                  goffs.data_ptr(), gidx.data_ptr(), gval.data_ptr(), nnz,
                                  plan.workspace.data_ptr(), plan.workspace_bytes, cs0)

        ms_g, mn_g = time_reps(enc_global, args.rows_reps)
        ok_g = plan.status()[0] == dws.DWS_OK and bool(torch.equal(goffs, offsets))
        rows.update([row("encode_global_int64_llama3_8b_lr%g" % args.lr, ms_g, 4 * N + 10 * nnz,
                         weight_bytes, peak, {"min_ms": round(mn_g, 4), "offsets_equal": ok_g})])
        del gidx, gval, goffs, bases
        # the same step with the wire checksum computed on the fly
        hashes = torch.empty(2, dtype=torch.int64, device=dev)
        wire = torch.empty(2, dtype=torch.int64, device=dev)
        coffs = torch.empty(T + 1, dtype=torch.int64, device=dev)
        cidx = torch.empty(nnz, dtype=torch.int32, device=dev)
        cval = torch.empty(nnz, dtype=torch.int16, device=dev)

        def enc_checksum():
            dws.dws_encode_checksum(plan.handle, ot.data_ptr(), nt.data_ptr(), coffs.data_ptr(),
                                    cidx.data_ptr(), cval.data_ptr(), nnz, hashes.data_ptr(),
                                    wire.data_ptr(), plan.workspace.data_ptr(), plan.workspace_bytes,
                                    cs0)

        ms_s, mn_s = time_reps(enc_checksum, args.rows_reps)
        ok_s = plan.status()[0] == dws.DWS_OK and bool(torch.equal(cidx, indices))
        rows.update([row("encode_checksum_llama3_8b_lr%g" % args.lr, ms_s, 4 * N + 6 * nnz,
                         weight_bytes, peak, {"min_ms": round(mn_s, 4), "indices_equal": ok_s})])
        del hashes, wire, coffs, cidx, cval
        rows.update(delta_file_rows(dws, plan, [nm for nm, _ in shapes], delta, args))
        lr2 = 1e-5
        for t in range(T):
            new[t].copy_(make_new(lr2)(t, sizes[t]))
        offs2 = plan.count(ot, nt)
        nnz2 = int(offs2[-1].item())
        del indices, values, delta
        idx2 = torch.empty(nnz2, dtype=torch.int32, device=dev)
        val2 = torch.empty(nnz2, dtype=torch.int16, device=dev)
        d2 = dws.Delta(offs2, idx2, val2)
        ms_e, mn_e = time_reps(lambda: plan.encode_into(ot, nt, offs2, idx2, val2), args.rows_reps)
        snap_flat.copy_(old_flat)
        ms_a, mn_a = time_reps(lambda: plan.apply(st, d2), args.rows_reps)
        ok = bool(torch.equal(snap_flat, new_flat)) and plan.status()[0] == dws.DWS_OK
        rows.update([row("encode_llama3_8b_lr1e-5", ms_e, 4 * N + 6 * nnz2, weight_bytes, peak,
                         {"min_ms": round(mn_e, 4), "nnz": nnz2, "sparsity": round(1 - nnz2 / N, 6)})])
        rows.update([row("apply_llama3_8b_lr1e-5", ms_a, 8 * nnz2, weight_bytes, peak,
                         {"min_ms": round(mn_a, 4), "exact": ok, "entries_per_s": round(nnz2 / ms_a * 1e3, 1),
                          **sector_model(nnz2, touched_sectors(offs2, idx2), ms_a, peak, clean_bytes(nnz2, dev))})])
        # wire form of the same delta: positions block (2 or 4 bytes each) and checksum
        pcap = 4 * nnz2
        positions = torch.empty(max(2, pcap), dtype=torch.uint8, device=dev)
        pos_offsets = torch.empty(T + 1, dtype=torch.int64, device=dev)
        hashes = torch.empty(2, dtype=torch.int64, device=dev)
        wire = torch.empty(2, dtype=torch.int64, device=dev)
        cs = torch.cuda.current_stream().cuda_stream

        def pack():
            dws.dws_pack_positions(plan.handle, offs2.data_ptr(), idx2.data_ptr(), nnz2,
                                   positions.data_ptr(), pcap, pos_offsets.data_ptr(),
                                   plan.workspace.data_ptr(), plan.workspace_bytes, cs)

        ms_p, mn_p = time_reps(pack, args.rows_reps)
        pbytes = int(pos_offsets[-1].item())
        offs_h = offs2.cpu().numpy()
        ok_p = plan.status()[0] == dws.DWS_OK and pbytes == 4 * nnz2 - 2 * sum(
            int(offs_h[t + 1] - offs_h[t]) for t in range(T) if sizes[t] <= 65536)
        rows.update([row("pack_positions_llama3_8b_lr1e-5", ms_p, 4 * nnz2 + pbytes + 8 * (T + 1),
                         weight_bytes, peak, {"min_ms": round(mn_p, 4), "block_bytes": pbytes,
                                              "sizes_ok": ok_p})])

        def csum():
            dws.dws_checksum(positions.data_ptr(), pbytes, val2.data_ptr(), nnz2, hashes.data_ptr(),
                             wire.data_ptr(), cs)

        ms_k, mn_k = time_reps(csum, args.rows_reps)
        rows.update([row("checksum_llama3_8b_lr1e-5", ms_k, pbytes + 2 * nnz2, weight_bytes, peak,
                         {"min_ms": round(mn_k, 4)})])
        del positions, pos_offsets, hashes, wire
        del old_flat, new_flat, snap_flat, old, new, snap, idx2, val2, d2, offs2
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        if args.layers is None:
            rows.update(run_rows(args, dev, peak))
        line["rows"] = attach_ncu(rows)

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N=1) ---------
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b, sec, n, c = oracle_sample(llama_shapes(args.layers), s, args.lr, dev, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": round(b / sec / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": (f"the first {c} decoder-layer tensors of the same Llama-3-8B-shaped set "
                       f"({n} elements, {2 * n / 1e9:.2f} GB of weights), oracle encode + apply "
                       f"in {sec:.1f} s on one thread"),
            "cpu": cpu_model(), "host_threads": os.cpu_count(), "pinned_core": PINNED_CORE["core"]}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if exact else 3


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
