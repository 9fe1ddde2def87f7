"""Seeded synthetic workloads for the delta weight sync hot path.

This module only DRAWS inputs: weight snapshots, simulated optimizer steps and
the flip patterns of the XOR and stress workloads.  It holds none of the
method's own arithmetic (no bit compare, compaction, scatter or XOR), so both
the CUDA library's tests and the CPU oracle can be fed from it without sharing
any of the code under test.  Every draw is made with an explicitly seeded
``torch.Generator`` on the device given; the same seed on the same device type
gives the same bits.

Workloads (shapes follow the model architectures; no trained weights exist
here, values are random):

1. ``single``  -- one 1024x1024 bf16 tensor, w ~ N(0, 0.03), one step at
   lr 3e-6.
2. ``qwen3_0p6b`` -- the Qwen3-0.6B parameter list (310 tensors,
   596,049,920 elements, tied embedding), w ~ N(0, 0.02), norm weights
   ~ N(1, 0.01); a chain of 10 steps at lr 3e-6.
3. ``llama3_8b`` -- the Llama-3-8B parameter list (291 tensors,
   8,030,261,248 elements, untied lm_head), same value model, one step at
   lr 3e-6 or 1e-5.
4. ``xor_nvfp4`` -- 40 uint8 layers of 8e8 random bytes; 680,000 distinct
   positions per layer get a different random byte.
5. ``stress`` -- 12000 bf16 tensors, sizes log-uniform in [256, 4194304];
   2% of elements change per step, in whole 4096-element runs for tensors
   whose coin says "clustered", element by element otherwise; 10 steps.

The simulated optimizer step (workloads 1-3) is the one the workload
definition fixes: in fp32, x = float(w) - lr * u with u ~ N(0, 1) clipped to
[-10, 10], then a round-to-nearest-even cast back to bf16.  lr is rounded to
fp32 first and the product and the difference are separate fp32 operations
(separate kernels, so nothing is fused into a multiply-add).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

# Seeds of the five workloads.
SEEDS = {"single": 0, "qwen3_0p6b": 1, "llama3_8b": 2, "xor_nvfp4": 3, "stress": 4}

_PRIME = 1_000_003


def weight_seed(s: int, t: int) -> int:
    """Seed of tensor t's initial weights in a workload with seed s."""
    return s * _PRIME + t


def step_seed(s: int, k: int, t: int) -> int:
    """Seed of tensor t's draws for step k (k = 1, 2, ...) of workload s."""
    return (s * 1000 + k) * _PRIME + t


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


# --------------------------------------------------------------------------
# Parameter lists (name, shape)
# --------------------------------------------------------------------------

def qwen3_0p6b_shapes():
    """Qwen3-0.6B: vocab 151936, hidden 1024, 28 layers, 16 q heads and 8 kv
    heads of dim 128, MLP 3072, tied embedding."""
    h, v, layers, mlp = 1024, 151936, 28, 3072
    q, kv = 16 * 128, 8 * 128
    out = [("model.embed_tokens.weight", (v, h))]
    for i in range(layers):
        p = f"model.layers.{i}."
        out += [
            (p + "self_attn.q_proj.weight", (q, h)),
            (p + "self_attn.k_proj.weight", (kv, h)),
            (p + "self_attn.v_proj.weight", (kv, h)),
            (p + "self_attn.o_proj.weight", (h, q)),
            (p + "self_attn.q_norm.weight", (128,)),
            (p + "self_attn.k_norm.weight", (128,)),
            (p + "mlp.gate_proj.weight", (mlp, h)),
            (p + "mlp.up_proj.weight", (mlp, h)),
            (p + "mlp.down_proj.weight", (h, mlp)),
            (p + "input_layernorm.weight", (h,)),
            (p + "post_attention_layernorm.weight", (h,)),
        ]
    out.append(("model.norm.weight", (h,)))
    return out


def llama3_8b_shapes():
    """Llama-3-8B: vocab 128256, hidden 4096, 32 layers, 32 q heads and 8 kv
    heads of dim 128, MLP 14336, untied lm_head."""
    h, v, layers, mlp = 4096, 128256, 32, 14336
    q, kv = 32 * 128, 8 * 128
    out = [("model.embed_tokens.weight", (v, h))]
    for i in range(layers):
        p = f"model.layers.{i}."
        out += [
            (p + "self_attn.q_proj.weight", (q, h)),
            (p + "self_attn.k_proj.weight", (kv, h)),
            (p + "self_attn.v_proj.weight", (kv, h)),
            (p + "self_attn.o_proj.weight", (h, q)),
            (p + "mlp.gate_proj.weight", (mlp, h)),
            (p + "mlp.up_proj.weight", (mlp, h)),
            (p + "mlp.down_proj.weight", (h, mlp)),
            (p + "input_layernorm.weight", (h,)),
            (p + "post_attention_layernorm.weight", (h,)),
        ]
    out.append(("model.norm.weight", (h,)))
    out.append(("lm_head.weight", (v, h)))
    return out


def scaled_shapes(shapes, div: int):
    """The same parameter list with every dimension divided by ``div``
    (at least 1): a small stand-in with the same tensor count and mix."""
    return [(n, tuple(max(1, d // div) for d in s)) for n, s in shapes]


def stress_sizes(s: int = SEEDS["stress"], count: int = 12000, lo: int = 256,
                 hi: int = 4194304):
    """Tensor sizes floor(exp(U[ln lo, ln hi])), drawn on the CPU generator so
    they do not depend on the device."""
    g = _gen(s * _PRIME + 999_983, "cpu")
    u = torch.rand(count, generator=g, dtype=torch.float64)
    a, b = math.log(lo), math.log(hi)
    return [int(math.floor(math.exp(a + float(x) * (b - a)))) for x in u]


def stress_clustered(s: int = SEEDS["stress"], count: int = 12000):
    """Per-tensor coin: True means changes come in whole 4096-element runs."""
    g = _gen(s * _PRIME + 999_979, "cpu")
    return [bool(x) for x in (torch.rand(count, generator=g) < 0.5)]


def numel(shape) -> int:
    n = 1
    for d in shape:
        n *= int(d)
    return n


# --------------------------------------------------------------------------
# bf16 weights and the simulated optimizer step
# --------------------------------------------------------------------------

def is_norm(name: str) -> bool:
    return "norm" in name


def init_tensor(n: int, seed: int, device, std: float, mean: float = 0.0) -> torch.Tensor:
    """bf16 weights: fp32 N(mean, std) draw, cast with round-to-nearest-even."""
    g = _gen(seed, device)
    w = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    w = w * std
    if mean != 0.0:
        w = w + mean
    return w.to(torch.bfloat16)


def update_noise(n: int, seed: int, device) -> torch.Tensor:
    """u ~ N(0, 1) clipped to [-10, 10], fp32."""
    g = _gen(seed, device)
    u = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    return u.clamp_(-10.0, 10.0)


def optimizer_step(w: torch.Tensor, u: torch.Tensor, lr: float) -> torch.Tensor:
    """new = bf16_rne(fl32(float(w) - fl32(lr * u)))."""
    lr32 = torch.tensor(lr, dtype=torch.float32)
    step = u * lr32
    x = w.float() - step
    return x.to(torch.bfloat16)


@dataclass
class BF16Set:
    """A list of bf16 tensors (flat) with their names."""
    names: list
    tensors: list

    @property
    def numels(self):
        return [t.numel() for t in self.tensors]

    @property
    def total(self) -> int:
        return sum(self.numels)


def pack_flat(sizes, make, device, align: int = 128):
    """Lay tensors out back to back in one zero-filled bf16 buffer, each
    starting on a multiple of ``align`` elements (as separate allocations
    would be aligned).  ``make(t, n)`` returns tensor t's values (or None to
    leave zeros).  Returns (flat buffer, list of views)."""
    offs, off = [], 0
    for n in sizes:
        offs.append(off)
        off += (int(n) + align - 1) // align * align
    flat = torch.zeros(max(off, 1), dtype=torch.bfloat16, device=device)
    views = []
    for t, (o, n) in enumerate(zip(offs, sizes)):
        v = flat[o:o + int(n)]
        x = make(t, int(n))
        if x is not None:
            v.copy_(x)
            del x
        views.append(v)
    return flat, views


def init_set(shapes, s: int, device, std: float) -> BF16Set:
    names, ts = [], []
    for t, (name, shape) in enumerate(shapes):
        n = numel(shape)
        if is_norm(name):
            ts.append(init_tensor(n, weight_seed(s, t), device, 0.01, 1.0))
        else:
            ts.append(init_tensor(n, weight_seed(s, t), device, std))
        names.append(name)
    return BF16Set(names, ts)


def step_set(ws: BF16Set, s: int, k: int, lr: float, device) -> BF16Set:
    """Step k of the simulated optimizer applied to every tensor of ws."""
    out = []
    for t, w in enumerate(ws.tensors):
        u = update_noise(w.numel(), step_seed(s, k, t), device)
        out.append(optimizer_step(w, u, lr))
        del u
    return BF16Set(list(ws.names), out)


def single(device, lr: float = 3e-6):
    """Workload 1: (old, new) one-tensor sets and the noise u of the step."""
    s = SEEDS["single"]
    old = init_set([("w", (1024, 1024))], s, device, 0.03)
    new = step_set(old, s, 1, lr, device)
    return old, new


# --------------------------------------------------------------------------
# Workload 4: byte layers with a few random byte changes
# --------------------------------------------------------------------------

def xor_layer(layer: int, device, nbytes: int = 800_000_000, flips: int = 680_000,
              s: int = SEEDS["xor_nvfp4"]):
    """One layer of the XOR workload.

    old: uniform random bytes.  ``flips`` distinct positions are drawn
    uniformly (draw with repeats, drop repeats, keep a random subset of
    exactly ``flips``); at each the new byte is old + r (mod 256) with r
    uniform in [1, 255], i.e. a uniformly random byte different from old.
    Returns (old, new, positions sorted int64).
    """
    g = _gen(weight_seed(s, layer), device)
    old = torch.randint(0, 256, (nbytes,), generator=g, device=device, dtype=torch.uint8)
    flips = min(flips, nbytes)
    gp = _gen(step_seed(s, 1, layer), device)
    pos = torch.empty(0, dtype=torch.int64, device=device)
    extra = max(64, flips // 64)
    while pos.numel() < flips:
        draw = torch.randint(0, nbytes, (flips + extra,), generator=gp, device=device)
        pos = torch.unique(torch.cat([pos, draw]))
        extra *= 2
    keep = torch.randperm(pos.numel(), generator=gp, device=device)[:flips]
    pos = torch.sort(pos[keep]).values
    r = torch.randint(1, 256, (flips,), generator=gp, device=device, dtype=torch.int32)
    new = old.clone()
    new[pos] = ((old[pos].to(torch.int32) + r) % 256).to(torch.uint8)
    return old, new, pos


# --------------------------------------------------------------------------
# Workload 5: many tensors, 2% changes, clustered or uniform
# --------------------------------------------------------------------------

RUN = 4096


def stress_init(sizes, device, s: int = SEEDS["stress"]) -> BF16Set:
    return BF16Set([f"t{t}" for t in range(len(sizes))],
                   [init_tensor(n, weight_seed(s, t), device, 0.02) for t, n in enumerate(sizes)])


def stress_change(w: torch.Tensor, clustered: bool, seed: int, device, p: float = 0.02,
                  run: int = RUN):
    """Change a fraction p of w's elements.

    Clustered: the tensor is cut into consecutive runs of ``run`` elements
    (the last one partial); each run is picked with probability p and every
    element in it changes.  Uniform: each element is picked with
    probability p.  A picked element gets new low 7 mantissa bits
    (old + r) mod 128 with r uniform in [1, 127], so it stays finite and
    always differs.  Returns (new, picked bool mask).
    """
    n = w.numel()
    g = _gen(seed, device)
    if clustered:
        runs = (n + run - 1) // run
        pick_runs = torch.rand(runs, generator=g, device=device) < p
        picked = pick_runs.repeat_interleave(run)[:n]
    else:
        picked = torch.rand(n, generator=g, device=device) < p
    r = torch.randint(1, 128, (n,), generator=g, device=device, dtype=torch.int32)
    bits = w.view(torch.int16).to(torch.int32) & 0xFFFF
    low = (bits + r) & 0x7F
    changed_bits = (bits & 0xFF80) | low
    out_bits = torch.where(picked, changed_bits, bits)
    out_bits = torch.where(out_bits >= 0x8000, out_bits - 0x10000, out_bits)
    new = out_bits.to(torch.int16).view(torch.bfloat16)
    return new, picked


def stress_step(ws: BF16Set, clustered, k: int, device, s: int = SEEDS["stress"]):
    """Step k of workload 5 on every tensor; returns (new set, picked masks)."""
    outs, picks = [], []
    for t, w in enumerate(ws.tensors):
        new, picked = stress_change(w, clustered[t], step_seed(s, k, t), device)
        outs.append(new)
        picks.append(picked)
    return BF16Set(list(ws.names), outs), picks
