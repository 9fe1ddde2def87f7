"""Plain single-threaded CPU oracle for the delta weight sync hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the ``sparse_bf16_delta_b200`` package and its CUDA library) never imports,
links or executes anything here, and nothing here imports the product path.

The arithmetic lives in ``oracle.c`` (plain C, one loop per definition); this
module compiles it with gcc on first use and wraps it with ctypes so the
tests can hand it numpy arrays.  Sources, by page title and section:

* "Shipping a Trillion Parameters With a Hub Bucket: Delta Weight Sync in TRL"
  §2 (why bf16 RL updates are sparse), §4.1 (safetensors wire format: int32
  indices + bf16 values per changed parameter; anchors and delta chains),
  §4.3 (receiver: ``snap.flatten()[indices] = values``).
* verl PR #6974 review, key source snippets, ``sparse_gather.py``
  (``shard_delta_indices``: integer-view compare, ``nonzero``, gather).
* humans& weight-sync summary, first paragraph (XOR mask delta).

``st_file.py`` (plain Python, json + struct) writes and reads a delta in the
safetensors format of the TRL page's §4.1.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``_build/liboracle.so`` (atomic replace)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= newest_src:
        return _LIB_PATH
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=_BUILD_DIR)
    os.close(fd)
    try:
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    vp, vpp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p)
    lib.ref_encode.restype = i64
    lib.ref_encode.argtypes = [i32, vp, vpp, vpp, vp, vp, vp, i64]
    lib.ref_apply.restype = i32
    lib.ref_apply.argtypes = [i32, vp, vpp, vp, vp, vp]
    lib.ref_apply_chain.restype = i32
    lib.ref_apply_chain.argtypes = [i32, vp, vpp, i32, vpp, vpp, vpp]
    lib.ref_xor_encode.restype = None
    lib.ref_xor_encode.argtypes = [vp, vp, vp, i64]
    lib.ref_xor_apply.restype = None
    lib.ref_xor_apply.argtypes = [vp, vp, i64]
    lib.ref_xor_byte_delta.restype = i64
    lib.ref_xor_byte_delta.argtypes = [i32, vp, vpp, vpp, vp, vp, vp, i64]
    lib.ref_apply_bytes.restype = i32
    lib.ref_apply_bytes.argtypes = [i32, vp, vpp, vp, vp, vp]
    lib.ref_bf16_rne.restype = ctypes.c_uint16
    lib.ref_bf16_rne.argtypes = [f32]
    lib.ref_bf16_to_float.restype = f32
    lib.ref_bf16_to_float.argtypes = [ctypes.c_uint16]
    lib.ref_update_step.restype = None
    lib.ref_update_step.argtypes = [vp, vp, f32, vp, i64]
    lib.ref_absorption_changed.restype = i32
    lib.ref_absorption_changed.argtypes = [ctypes.c_uint16, f32]
    lib.ref_absorption_predict.restype = i64
    lib.ref_absorption_predict.argtypes = [vp, vp, f32, vp, i64]
    lib.ref_pack_positions.restype = i64
    lib.ref_pack_positions.argtypes = [i32, vp, vp, vp, vp, vp]
    lib.ref_hash_bytes.restype = ctypes.c_uint64
    lib.ref_hash_bytes.argtypes = [vp, i64]
    lib.ref_hash_bf16.restype = ctypes.c_uint64
    lib.ref_hash_bf16.argtypes = [vp, i64]
    lib.ref_bf16_to_f64_bits.restype = ctypes.c_uint64
    lib.ref_bf16_to_f64_bits.argtypes = [ctypes.c_uint16]
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a).reshape(-1)


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _ptr_array(arrays) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(arrays)))()
    for i, a in enumerate(arrays):
        arr[i] = _ptr(a)
    return arr


def encode(olds, news, capacity: int | None = None):
    """Sparse delta of ``news`` against ``olds`` (lists of uint16 arrays).

    Returns ``(offsets int64[T+1], indices int32[nnz], values uint16[nnz])``.
    With a ``capacity`` below nnz only the first ``capacity`` entries are
    kept and the arrays are that long; offsets still describe all of nnz.
    """
    lib = _load()
    olds = [_c(a, np.uint16) for a in olds]
    news = [_c(a, np.uint16) for a in news]
    if len(olds) != len(news):
        raise ValueError("old/new tensor counts differ")
    for a, b in zip(olds, news):
        if a.size != b.size:
            raise ValueError("old/new sizes differ")
    T = len(olds)
    numels = np.array([a.size for a in olds] or [0], dtype=np.int64)
    offsets = np.zeros(T + 1, dtype=np.int64)
    if capacity is None:
        capacity = int(sum(a.size for a in olds))
    indices = np.empty(max(1, capacity), dtype=np.int32)
    values = np.empty(max(1, capacity), dtype=np.uint16)
    nnz = lib.ref_encode(T, _ptr(numels), _ptr_array(olds), _ptr_array(news),
                         _ptr(offsets), _ptr(indices), _ptr(values), capacity)
    if nnz < 0:
        raise ValueError("invalid tensor size (numel must be in [0, 2^31))")
    kept = min(nnz, capacity)
    return offsets, indices[:kept].copy(), values[:kept].copy()


def apply(snaps, offsets, indices, values) -> None:
    """Scatter one delta into ``snaps`` (list of uint16 arrays) in place."""
    lib = _load()
    for s in snaps:
        if s.dtype != np.uint16 or not s.flags.c_contiguous:
            raise TypeError("snapshots must be contiguous uint16 arrays")
    numels = np.array([s.size for s in snaps] or [0], dtype=np.int64)
    offsets = _c(offsets, np.int64)
    indices = _c(indices, np.int32) if len(indices) else np.zeros(1, np.int32)
    values = _c(values, np.uint16) if len(values) else np.zeros(1, np.uint16)
    rc = lib.ref_apply(len(snaps), _ptr(numels), _ptr_array(snaps), _ptr(offsets),
                       _ptr(indices), _ptr(values))
    if rc != 0:
        raise ValueError("bad delta (index out of range or offsets not monotone)")


def apply_chain(snaps, deltas) -> None:
    """Replay ``deltas`` (list of (offsets, indices, values)) in order."""
    lib = _load()
    for s in snaps:
        if s.dtype != np.uint16 or not s.flags.c_contiguous:
            raise TypeError("snapshots must be contiguous uint16 arrays")
    numels = np.array([s.size for s in snaps] or [0], dtype=np.int64)
    keep = []
    offs, idxs, vals = [], [], []
    for o, i, v in deltas:
        o = _c(o, np.int64)
        i = _c(i, np.int32) if len(i) else np.zeros(1, np.int32)
        v = _c(v, np.uint16) if len(v) else np.zeros(1, np.uint16)
        keep += [o, i, v]
        offs.append(o)
        idxs.append(i)
        vals.append(v)
    rc = lib.ref_apply_chain(len(snaps), _ptr(numels), _ptr_array(snaps), len(deltas),
                             _ptr_array(offs), _ptr_array(idxs), _ptr_array(vals))
    if rc != 0:
        raise ValueError("bad delta in chain")


def xor_encode(old_b, new_b) -> np.ndarray:
    lib = _load()
    a = _c(old_b, np.uint8)
    b = _c(new_b, np.uint8)
    if a.size != b.size:
        raise ValueError("size mismatch")
    mask = np.empty(a.size, dtype=np.uint8)
    lib.ref_xor_encode(_ptr(a), _ptr(b), _ptr(mask), a.size)
    return mask


def xor_apply(buf: np.ndarray, mask) -> None:
    lib = _load()
    if buf.dtype != np.uint8 or not buf.flags.c_contiguous:
        raise TypeError("buf must be a contiguous uint8 array")
    m = _c(mask, np.uint8)
    if m.size != buf.size:
        raise ValueError("size mismatch")
    lib.ref_xor_apply(_ptr(buf), _ptr(m), buf.size)


def xor_byte_delta(olds, news, capacity: int | None = None):
    """The sparse XOR delta at byte granularity of ``news`` against ``olds``
    (lists of uint8 arrays, one per layer): per layer the ascending int32
    positions of the bytes that differ and the new bytes there ("humans&
    weight sync" summary, first paragraph: the XOR mask is nonzero exactly at
    those bytes).  Returns ``(offsets int64[T+1], positions int32[n],
    values uint8[n])``; capacity as in ``encode``."""
    lib = _load()
    olds = [_c(a, np.uint8) for a in olds]
    news = [_c(a, np.uint8) for a in news]
    if len(olds) != len(news) or any(a.size != b.size for a, b in zip(olds, news)):
        raise ValueError("old/new layers differ in number or size")
    T = len(olds)
    nbytes = np.array([a.size for a in olds] or [0], dtype=np.int64)
    offsets = np.zeros(T + 1, dtype=np.int64)
    if capacity is None:
        capacity = int(sum(a.size for a in olds))
    positions = np.empty(max(1, capacity), dtype=np.int32)
    values = np.empty(max(1, capacity), dtype=np.uint8)
    n = lib.ref_xor_byte_delta(T, _ptr(nbytes), _ptr_array(olds), _ptr_array(news),
                               _ptr(offsets), _ptr(positions), _ptr(values), capacity)
    if n < 0:
        raise ValueError("invalid layer size (must be below 2^31 bytes)")
    kept = min(n, capacity)
    return offsets, positions[:kept].copy(), values[:kept].copy()


def apply_bytes(bufs, offsets, positions, values) -> None:
    """Scatter a byte-granular delta into ``bufs`` (uint8 arrays) in place."""
    lib = _load()
    for b in bufs:
        if b.dtype != np.uint8 or not b.flags.c_contiguous:
            raise TypeError("layers must be contiguous uint8 arrays")
    nbytes = np.array([b.size for b in bufs] or [0], dtype=np.int64)
    offsets = _c(offsets, np.int64)
    positions = _c(positions, np.int32) if len(positions) else np.zeros(1, np.int32)
    values = _c(values, np.uint8) if len(values) else np.zeros(1, np.uint8)
    rc = lib.ref_apply_bytes(len(bufs), _ptr(nbytes), _ptr_array(bufs), _ptr(offsets),
                             _ptr(positions), _ptr(values))
    if rc != 0:
        raise ValueError("bad byte delta (position out of range or offsets not monotone)")


def bf16_rne(x) -> np.ndarray:
    """Elementwise fp32 -> bf16 bits (round to nearest even)."""
    lib = _load()
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    return np.array([lib.ref_bf16_rne(float(v)) for v in x], dtype=np.uint16)


def bf16_to_float(b) -> np.ndarray:
    lib = _load()
    b = np.asarray(b, dtype=np.uint16).reshape(-1)
    return np.array([lib.ref_bf16_to_float(int(v)) for v in b], dtype=np.float32)


def update_step(w, u, lr: float) -> np.ndarray:
    """The synthetic optimizer step, recomputed: bf16_rne(fl32(w) - fl32(lr*u))."""
    lib = _load()
    w = _c(w, np.uint16)
    u = _c(u, np.float32)
    if w.size != u.size:
        raise ValueError("size mismatch")
    out = np.empty(w.size, dtype=np.uint16)
    lib.ref_update_step(_ptr(w), _ptr(u), float(np.float32(lr)), _ptr(out), w.size)
    return out


def absorption_changed(w_bits: int, x: float) -> int:
    return int(_load().ref_absorption_changed(int(w_bits) & 0xFFFF, float(np.float32(x))))


def absorption_predict(w, u, lr: float):
    """Per-element prediction of which bf16 weights change under the update."""
    lib = _load()
    w = _c(w, np.uint16)
    u = _c(u, np.float32)
    if w.size != u.size:
        raise ValueError("size mismatch")
    changed = np.empty(w.size, dtype=np.uint8)
    n = lib.ref_absorption_predict(_ptr(w), _ptr(u), float(np.float32(lr)), _ptr(changed), w.size)
    if n < 0:
        raise ValueError("non-finite weight")
    return changed, int(n)


def pos_width(numel: int) -> int:
    """Bytes per position of a parameter of `numel` elements (2 or 4)."""
    return 2 if numel <= 65536 else 4


def pack_positions(numels, offsets, indices):
    """Wire positions: (byte block uint8[total], pos_offsets int64[T+1])."""
    lib = _load()
    n = _c(numels, np.int64)
    o = _c(offsets, np.int64)
    i = _c(indices, np.int32)
    T = n.size
    if o.size != T + 1:
        raise ValueError("offsets must have T+1 entries")
    total = int(sum(pos_width(int(n[t])) * int(o[t + 1] - o[t]) for t in range(T)))
    out = np.zeros(max(1, total), dtype=np.uint8)
    po = np.zeros(T + 1, dtype=np.int64)
    got = lib.ref_pack_positions(T, _ptr(n), _ptr(o), _ptr(i), _ptr(out), _ptr(po))
    if got < 0:
        raise ValueError("invalid sizes or offsets")
    return out[:got], po


def checksum_parts(positions, values):
    """(hash of the position bytes, hash of the bf16 values), both uint64."""
    lib = _load()
    p = _c(positions, np.uint8)
    v = _c(np.asarray(values).view(np.uint16), np.uint16)
    return int(lib.ref_hash_bytes(_ptr(p), p.size)), int(lib.ref_hash_bf16(_ptr(v), v.size))


def checksum(positions, values) -> int:
    """The wire checksum: hash(positions) ^ (hash(values) << 1) (65 bits)."""
    hp, hv = checksum_parts(positions, values)
    return hp ^ (hv << 1)


def bf16_to_f64_bits(b: int) -> int:
    return int(_load().ref_bf16_to_f64_bits(b))


def encode_global(olds, news, index_base):
    """Encode with global int64 positions ([verl] review, key source snippets,
    sparse_gather.py shard_delta_indices: global_idx = local_idx + offset):
    (offsets, int64 positions, values), entry j of tensor t at
    index_base[t] + its local index."""
    offsets, indices, values = encode(olds, news)
    counts = np.diff(offsets)
    base = np.repeat(np.asarray(index_base, dtype=np.int64), counts)
    return offsets, indices.astype(np.int64) + base, values


def merge_shards(rank_offsets, rank_indices, rank_values):
    """One delta from the ranks' deltas of their shards, as the page's
    gather_v_batched_to_rank0 leaves it on rank 0 ([verl] review, key source
    snippets, sparse_gather.py: after the gather, rank 0 splits each rank's
    buffer by that rank's per-parameter counts and concatenates, per
    parameter, the ranks' pieces in rank order).
    rank_offsets: R arrays int64[T+1] (each rank's delta layout);
    rank_indices, rank_values: R arrays holding at least rank_offsets[r][T]
    entries (global int64 positions, bf16 bits).
    Returns (offsets int64[T+1], indices int64[n], values uint16[n])."""
    R = len(rank_offsets)
    T = len(rank_offsets[0]) - 1
    offsets = [0]
    idx, val = [], []
    for t in range(T):
        n = 0
        for r in range(R):
            a, b = int(rank_offsets[r][t]), int(rank_offsets[r][t + 1])
            idx.append(np.asarray(rank_indices[r][a:b], dtype=np.int64))
            val.append(np.asarray(rank_values[r][a:b]).view(np.uint16))
            n += b - a
        offsets.append(offsets[-1] + n)
    idx.append(np.zeros(0, np.int64))
    val.append(np.zeros(0, np.uint16))
    return np.array(offsets, dtype=np.int64), np.concatenate(idx), np.concatenate(val)
