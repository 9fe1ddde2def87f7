"""Python binding of libdws, the B200 (sm_100a) delta weight sync library.

Two layers, both argument marshalling only -- every step of the hot path runs
in libdws's CUDA kernels:

* ``dws_*`` functions with the C ABI's names and arguments (pointers as
  Python ints, streams as ``torch.cuda.Stream.cuda_stream`` ints).
* ``DeltaPlan`` and a few helpers that take torch CUDA tensors, allocate
  outputs / workspace with torch and call the ``dws_*`` functions.

Importing this package loads ``libdws.so`` from the package directory and
raises ``ImportError`` if it is missing: there is no CPU fallback.  Build it
with ``python sparse_bf16_delta_b200/_build.py`` (or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdws.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libdws.so not found at {LIB_PATH}; build it with "
        "`python sparse_bf16_delta_b200/_build.py` (needs nvcc for sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

# Status codes (include/dws.h)
DWS_OK = 0
DWS_ERR_INVALID = 1
DWS_ERR_UNSUPPORTED = 2
DWS_ERR_CAPACITY = 3
DWS_ERR_BAD_DELTA = 4
DWS_ERR_TIMEOUT = 5
DWS_ERR_CUDA = 6
DWS_ERR_WORKSPACE = 7
DWS_MAX_CHAIN = 64
DWS_CHAIN_AUTO = 0
DWS_CHAIN_TILE_MERGE = 1
DWS_CHAIN_SCATTER = 2

_i32, _i64, _sz, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p


class dws_delta_t(ctypes.Structure):
    _fields_ = [("offsets", _vp), ("indices", _vp), ("values", _vp), ("count", _i64)]


def _sig(name, restype, argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_sig("dws_plan_create", _i32, [_vp, _i32, _i32, ctypes.POINTER(_vp)])
_sig("dws_plan_destroy", None, [_vp])
_sig("dws_plan_num_tensors", _i32, [_vp])
_sig("dws_plan_num_elements", _i64, [_vp])
_sig("dws_plan_num_tiles", _i64, [_vp])
_sig("dws_tile_elems", _i64, [])
_sig("dws_plan_workspace_bytes", _sz, [_vp])
_sig("dws_plan_upload", _i32, [_vp, _vp, _sz, _vp])
_sig("dws_encode", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_encode_nnz", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _vp])
_sig("dws_encode_ex", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp, _i64, _i64])
_sig("dws_count", _i32, [_vp, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("dws_encode_noalloc", _i32, [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp])
_sig("dws_apply", _i32, [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_apply_chain", _i32, [_vp, _vp, ctypes.POINTER(dws_delta_t), _i32, _vp, _sz, _vp])
_sig("dws_apply_chain_ex", _i32, [_vp, _vp, ctypes.POINTER(dws_delta_t), _i32, _i32, _vp, _sz, _vp])
_sig("dws_pos_width", _i32, [_vp, _i32])
_sig("dws_merge_shards", _i32, [_vp, _i32, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_xor_bytes_from_words", _i32, [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_apply_bytes", _i32, [_vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_encode_global", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _sz, _vp])
_sig("dws_encode_checksum", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _sz, _vp])
_sig("dws_pack_positions", _i32, [_vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _sz, _vp])
_sig("dws_checksum", _i32, [_vp, _i64, _vp, _i64, _vp, _vp, _vp])
_sig("dws_st_delta_header", _i32, [_vp, _vp, _vp, _i64, _vp, _i64, ctypes.POINTER(_i64)])
_sig("dws_st_delta_write", _i32,
     [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, ctypes.POINTER(_i64), _vp])
_sig("dws_st_delta_read", _i32, [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _i64,
                                 ctypes.POINTER(_i64), ctypes.POINTER(_i64), _vp])
_sig("dws_xor_encode", _i32, [_vp, _vp, _vp, _i64, _vp])
_sig("dws_xor_apply", _i32, [_vp, _vp, _i64, _vp])
_sig("dws_xor_apply_layers", _i32, [_vp, _vp, _vp, _i32, _vp, _vp, _i64, _vp, _vp])
_sig("dws_status", _i32, [_vp, ctypes.POINTER(_i64), _vp])
_sig("dws_strerror", ctypes.c_char_p, [_i32])
_sig("dws_version", ctypes.c_char_p, [])
_sig("dws_launch_count", ctypes.c_uint64, [])
_sig("dws_device_memory", _i32, [_i32, ctypes.POINTER(_i32), ctypes.POINTER(_i32)])


class DwsError(RuntimeError):
    def __init__(self, code: int, where: str, detail: int | None = None):
        self.code = int(code)
        self.detail = detail
        msg = f"{where}: {dws_strerror(code)} (status {code})"
        if detail is not None:
            msg += f", detail {detail}"
        super().__init__(msg)


def _check(code: int, where: str) -> None:
    if code != DWS_OK:
        raise DwsError(code, where)


# ---------------------------------------------------------------------------
# C-ABI names (pointers and streams as ints)
# ---------------------------------------------------------------------------

def dws_plan_create(numels, elem_size: int = 2) -> int:
    arr = (ctypes.c_int64 * max(1, len(numels)))(*[int(n) for n in numels])
    out = _vp()
    _check(_lib.dws_plan_create(arr, len(numels), int(elem_size), ctypes.byref(out)),
           "dws_plan_create")
    return out.value


def dws_plan_destroy(plan: int) -> None:
    _lib.dws_plan_destroy(plan)


def dws_plan_num_tensors(plan: int) -> int:
    return _lib.dws_plan_num_tensors(plan)


def dws_plan_num_elements(plan: int) -> int:
    return _lib.dws_plan_num_elements(plan)


def dws_plan_num_tiles(plan: int) -> int:
    return _lib.dws_plan_num_tiles(plan)


def dws_tile_elems() -> int:
    return _lib.dws_tile_elems()


def dws_plan_workspace_bytes(plan: int) -> int:
    return _lib.dws_plan_workspace_bytes(plan)


def dws_plan_upload(plan, workspace, workspace_bytes, stream) -> int:
    return _lib.dws_plan_upload(plan, workspace, workspace_bytes, stream)


def dws_encode(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, workspace,
               workspace_bytes, stream) -> int:
    return _lib.dws_encode(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                           workspace, workspace_bytes, stream)


def dws_encode_nnz(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, nnz_dev,
                   nnz_host, workspace, workspace_bytes, stream) -> int:
    return _lib.dws_encode_nnz(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                               nnz_dev, nnz_host, workspace, workspace_bytes, stream)


def dws_encode_ex(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, workspace,
                  workspace_bytes, stream, wait_limit_ns, debug_withhold_tile) -> int:
    return _lib.dws_encode_ex(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                              workspace, workspace_bytes, stream, wait_limit_ns,
                              debug_withhold_tile)


def dws_encode_noalloc(numels, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                       status_out, stream) -> int:
    """Encode without a caller-provided workspace (see include/dws.h): the
    scratch is a fixed device array inside libdws.  ``numels`` is a list."""
    arr = (ctypes.c_int64 * max(1, len(numels)))(*[int(n) for n in numels])
    return _lib.dws_encode_noalloc(arr, len(numels), old_ptrs, new_ptrs, offsets, indices, values,
                                   capacity, status_out, stream)


def dws_count(plan, old_ptrs, new_ptrs, offsets, workspace, workspace_bytes, stream) -> int:
    return _lib.dws_count(plan, old_ptrs, new_ptrs, offsets, workspace, workspace_bytes, stream)


def dws_apply(plan, snap_ptrs, offsets, indices, values, count, workspace, workspace_bytes,
              stream) -> int:
    return _lib.dws_apply(plan, snap_ptrs, offsets, indices, values, count, workspace,
                          workspace_bytes, stream)


def dws_apply_chain(plan, snap_ptrs, deltas, K, workspace, workspace_bytes, stream) -> int:
    """``deltas``: a ctypes array of dws_delta_t (see ``make_delta_array``)."""
    return _lib.dws_apply_chain(plan, snap_ptrs, deltas, K, workspace, workspace_bytes, stream)


def dws_apply_chain_ex(plan, snap_ptrs, deltas, K, mode, workspace, workspace_bytes,
                       stream) -> int:
    """dws_apply_chain with an explicit replay mode (DWS_CHAIN_*)."""
    return _lib.dws_apply_chain_ex(plan, snap_ptrs, deltas, K, mode, workspace, workspace_bytes,
                                   stream)


def dws_encode_global(plan, old_ptrs, new_ptrs, index_base, offsets, indices, values, capacity,
                      workspace, workspace_bytes, stream) -> int:
    return _lib.dws_encode_global(plan, old_ptrs, new_ptrs, index_base, offsets, indices, values,
                                  capacity, workspace, workspace_bytes, stream)


def dws_encode_checksum(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity, hashes,
                        checksum, workspace, workspace_bytes, stream) -> int:
    return _lib.dws_encode_checksum(plan, old_ptrs, new_ptrs, offsets, indices, values, capacity,
                                    hashes, checksum, workspace, workspace_bytes, stream)


def dws_xor_bytes_from_words(plan, old_ptrs, word_offsets, word_indices, word_values, word_count,
                             byte_offsets, byte_positions, byte_values, capacity, workspace,
                             workspace_bytes, stream):
    return _lib.dws_xor_bytes_from_words(plan, old_ptrs, word_offsets, word_indices, word_values,
                                         word_count, byte_offsets, byte_positions, byte_values, capacity,
                                         workspace, workspace_bytes, stream)


def dws_apply_bytes(plan, buf_ptrs, offsets, positions, values, count, workspace, workspace_bytes, stream):
    return _lib.dws_apply_bytes(plan, buf_ptrs, offsets, positions, values, count, workspace,
                                workspace_bytes, stream)


def dws_merge_shards(plan, num_ranks, rank_offsets, rank_indices, rank_values, stride, offsets,
                     indices, values, capacity, workspace, workspace_bytes, stream) -> int:
    return _lib.dws_merge_shards(plan, num_ranks, rank_offsets, rank_indices, rank_values, stride,
                                 offsets, indices, values, capacity, workspace, workspace_bytes,
                                 stream)


def dws_pos_width(plan, t) -> int:
    return _lib.dws_pos_width(plan, t)


def dws_pack_positions(plan, offsets, indices, count, positions, pos_capacity, pos_offsets,
                       workspace, workspace_bytes, stream) -> int:
    return _lib.dws_pack_positions(plan, offsets, indices, count, positions, pos_capacity,
                                   pos_offsets, workspace, workspace_bytes, stream)


def dws_checksum(positions, pos_bytes, values, nnz, hashes, checksum, stream) -> int:
    return _lib.dws_checksum(positions, pos_bytes, values, nnz, hashes, checksum, stream)


def dws_st_delta_header(plan, names, offsets, model_version, out, capacity):
    """Returns (status, header_bytes).  ``names``: see ``make_name_array``;
    ``offsets``, ``out``: host pointers."""
    n = ctypes.c_int64(0)
    st = _lib.dws_st_delta_header(plan, names, offsets, model_version, out, capacity,
                                  ctypes.byref(n))
    return int(st), int(n.value)


def dws_st_delta_write(plan, names, offsets, model_version, indices, values, file, capacity,
                       stream):
    """Returns (status, file_bytes)."""
    n = ctypes.c_int64(0)
    st = _lib.dws_st_delta_write(plan, names, offsets, model_version, indices, values, file,
                                 capacity, ctypes.byref(n), stream)
    return int(st), int(n.value)


def dws_st_delta_read(plan, names, file, file_size, offsets_host, offsets, indices, values,
                      capacity, stream):
    """Returns (status, nnz, model_version)."""
    nnz, ver = ctypes.c_int64(0), ctypes.c_int64(0)
    st = _lib.dws_st_delta_read(plan, names, file, file_size, offsets_host, offsets, indices,
                                values, capacity, ctypes.byref(nnz), ctypes.byref(ver), stream)
    return int(st), int(nnz.value), int(ver.value)


def dws_xor_encode(old_bytes, new_bytes, mask, nbytes, stream) -> int:
    return _lib.dws_xor_encode(old_bytes, new_bytes, mask, nbytes, stream)


def dws_xor_apply(buf, mask, nbytes, stream) -> int:
    return _lib.dws_xor_apply(buf, mask, nbytes, stream)


def dws_xor_apply_layers(bufs, masks, nbytes, L, staging0, staging1, staging_bytes,
                         apply_stream, copy_stream) -> int:
    """``bufs``, ``masks``: ctypes void* arrays; ``nbytes``: ctypes int64 array."""
    return _lib.dws_xor_apply_layers(bufs, masks, nbytes, L, staging0, staging1, staging_bytes,
                                     apply_stream, copy_stream)


def dws_status(workspace, stream):
    """Returns (status, detail) and clears the workspace's status word."""
    detail = ctypes.c_int64(0)
    st = _lib.dws_status(workspace, ctypes.byref(detail), stream)
    return int(st), int(detail.value)


def dws_strerror(code: int) -> str:
    return _lib.dws_strerror(int(code)).decode()


def dws_version() -> str:
    return _lib.dws_version().decode()


def dws_launch_count() -> int:
    return int(_lib.dws_launch_count())


def dws_device_memory(device: int = 0):
    """(memory clock kHz, bus width bits) of a device, from the CUDA runtime."""
    khz, bits = _i32(0), _i32(0)
    _check(_lib.dws_device_memory(int(device), ctypes.byref(khz), ctypes.byref(bits)),
           "dws_device_memory")
    return int(khz.value), int(bits.value)


def make_delta_array(deltas):
    """[(offsets_ptr, indices_ptr, values_ptr, count), ...] -> ctypes array."""
    arr = (dws_delta_t * max(1, len(deltas)))()
    for k, (o, i, v, c) in enumerate(deltas):
        arr[k] = dws_delta_t(o, i, v, c)
    return arr


def make_name_array(names):
    """Tensor names (str) -> ctypes array of NUL-terminated UTF-8 strings."""
    arr = (ctypes.c_char_p * max(1, len(names)))()
    for k, n in enumerate(names):
        arr[k] = n.encode("utf-8")
    return arr


def make_ptr_array(ptrs):
    arr = (ctypes.c_void_p * max(1, len(ptrs)))()
    for k, p in enumerate(ptrs):
        arr[k] = p
    return arr


# ---------------------------------------------------------------------------
# torch convenience layer (allocation + marshalling)
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream_handle(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def ptr_table(tensors, device=None):
    """Device int64 array of the tensors' data pointers (the per-call
    pointer arrays the C ABI takes)."""
    torch = _torch()
    dev = device if device is not None else tensors[0].device
    ptrs = [int(t.data_ptr()) if t.numel() > 0 else 0 for t in tensors]
    table = torch.tensor(ptrs, dtype=torch.int64).to(dev, non_blocking=False)
    # The table holds references to its tensors, so their memory cannot be
    # freed (and reused) while a kernel may still read through the table.
    table._dws_tensors = list(tensors)
    return table


class Delta:
    """One sparse delta on the device: offsets int64[T+1], indices int32[n],
    values as bf16 bits (int16 storage) [n]."""

    def __init__(self, offsets, indices, values):
        self.offsets = offsets
        self.indices = indices
        self.values = values

    @property
    def count(self) -> int:
        return int(self.indices.numel())

    def nnz(self) -> int:
        return int(self.offsets[-1].item())

    def as_ref(self):
        return (self.offsets.data_ptr(), self.indices.data_ptr() if self.count else 0,
                self.values.data_ptr() if self.count else 0, self.count)


class DeltaPlan:
    """A plan (multi-tensor descriptor table) for a list of bf16 tensors with a
    torch-allocated, uploaded workspace."""

    def __init__(self, numels, device="cuda", elem_size: int = 2, stream=None):
        torch = _torch()
        self.numels = [int(n) for n in numels]
        self.handle = dws_plan_create(self.numels, elem_size)
        self.device = torch.device(device)
        self.workspace_bytes = dws_plan_workspace_bytes(self.handle)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=self.device)
        _check(dws_plan_upload(self.handle, self.workspace.data_ptr(), self.workspace_bytes,
                               _stream_handle(stream)), "dws_plan_upload")

    @classmethod
    def for_tensors(cls, tensors, **kw):
        return cls([t.numel() for t in tensors], device=tensors[0].device, **kw)

    @property
    def num_tensors(self) -> int:
        return len(self.numels)

    @property
    def num_elements(self) -> int:
        return dws_plan_num_elements(self.handle)

    @property
    def num_tiles(self) -> int:
        return dws_plan_num_tiles(self.handle)

    def close(self):
        if getattr(self, "handle", None):
            dws_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- status --
    def status(self, stream=None):
        return dws_status(self.workspace.data_ptr(), _stream_handle(stream))

    def raise_on_error(self, where="libdws", stream=None):
        st, detail = self.status(stream)
        if st != DWS_OK:
            raise DwsError(st, where, detail)

    # -- encode --
    def count(self, old_table, new_table, offsets=None, stream=None):
        torch = _torch()
        if offsets is None:
            offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        _check(dws_count(self.handle, old_table.data_ptr(), new_table.data_ptr(),
                         offsets.data_ptr(), self.workspace.data_ptr(), self.workspace_bytes,
                         _stream_handle(stream)), "dws_count")
        return offsets

    def encode_into(self, old_table, new_table, offsets, indices, values, stream=None):
        _check(dws_encode(self.handle, old_table.data_ptr(), new_table.data_ptr(),
                          offsets.data_ptr(), indices.data_ptr() if indices.numel() else 0,
                          values.data_ptr() if values.numel() else 0, int(indices.numel()),
                          self.workspace.data_ptr(), self.workspace_bytes,
                          _stream_handle(stream)), "dws_encode")

    def encode(self, old_table, new_table, capacity: int, stream=None) -> Delta:
        """One-pass encode into buffers of `capacity` entries (trimmed to nnz;
        raises DwsError(DWS_ERR_CAPACITY) if nnz > capacity)."""
        torch = _torch()
        offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        indices = torch.empty(max(0, capacity), dtype=torch.int32, device=self.device)
        values = torch.empty(max(0, capacity), dtype=torch.int16, device=self.device)
        self.encode_into(old_table, new_table, offsets, indices, values, stream)
        self.raise_on_error("dws_encode", stream)
        nnz = int(offsets[-1].item())
        return Delta(offsets, indices[:nnz], values[:nnz])

    def encode_into_nnz(self, old_table, new_table, offsets, indices, values, nnz_dev=None,
                        nnz_host=None, stream=None):
        """encode_into that also copies the entry count to a device int64
        tensor and/or a pinned host int64 tensor after the encode (valid once
        the stream has reached the copies)."""
        _check(dws_encode_nnz(self.handle, old_table.data_ptr(), new_table.data_ptr(),
                              offsets.data_ptr(), indices.data_ptr() if indices.numel() else 0,
                              values.data_ptr() if values.numel() else 0, int(indices.numel()),
                              nnz_dev.data_ptr() if nnz_dev is not None else 0,
                              nnz_host.data_ptr() if nnz_host is not None else 0,
                              self.workspace.data_ptr(), self.workspace_bytes,
                              _stream_handle(stream)), "dws_encode_nnz")

    def encode_exact(self, old_table, new_table, stream=None) -> Delta:
        """Count first, then encode into exactly-sized buffers (two passes)."""
        offsets = self.count(old_table, new_table, stream=stream)
        self.raise_on_error("dws_count", stream)
        return self.encode(old_table, new_table, int(offsets[-1].item()), stream)

    # -- apply --
    def apply(self, snap_table, delta: Delta, stream=None):
        o, i, v, c = delta.as_ref()
        _check(dws_apply(self.handle, snap_table.data_ptr(), o, i, v, c,
                         self.workspace.data_ptr(), self.workspace_bytes,
                         _stream_handle(stream)), "dws_apply")

    def encode_global(self, old_table, new_table, index_base, stream=None) -> Delta:
        """Encode with int64 global positions (index_base[t] + local index);
        index_base: device int64 tensor [T].  Sized exactly (count first)."""
        torch = _torch()
        offsets = self.count(old_table, new_table, stream=stream)
        nnz = int(offsets[-1].item())
        indices = torch.empty(nnz, dtype=torch.int64, device=self.device)
        values = torch.empty(nnz, dtype=torch.int16, device=self.device)
        _check(dws_encode_global(self.handle, old_table.data_ptr(), new_table.data_ptr(),
                                 index_base.data_ptr(), offsets.data_ptr(),
                                 indices.data_ptr() if nnz else 0, values.data_ptr() if nnz else 0,
                                 nnz, self.workspace.data_ptr(), self.workspace_bytes,
                                 _stream_handle(stream)), "dws_encode_global")
        self.raise_on_error("dws_encode_global", stream)
        return Delta(offsets, indices, values)

    def encode_checksum(self, old_table, new_table, stream=None):
        """(Delta, checksum): the exact encode and the 65-bit wire checksum
        that libdws computed for the delta it wrote (dws_encode_checksum)."""
        torch = _torch()
        offsets = self.count(old_table, new_table, stream=stream)
        nnz = int(offsets[-1].item())
        indices = torch.empty(nnz, dtype=torch.int32, device=self.device)
        values = torch.empty(nnz, dtype=torch.int16, device=self.device)
        hashes = torch.empty(2, dtype=torch.int64, device=self.device)
        wire = torch.empty(2, dtype=torch.int64, device=self.device)
        _check(dws_encode_checksum(self.handle, old_table.data_ptr(), new_table.data_ptr(),
                                   offsets.data_ptr(), indices.data_ptr() if nnz else 0,
                                   values.data_ptr() if nnz else 0, nnz, hashes.data_ptr(),
                                   wire.data_ptr(), self.workspace.data_ptr(),
                                   self.workspace_bytes, _stream_handle(stream)),
               "dws_encode_checksum")
        self.raise_on_error("dws_encode_checksum", stream)
        return Delta(offsets, indices, values), _wire_int(wire)

    def merge_shards(self, rank_offsets, rank_indices, rank_values, stream=None) -> Delta:
        """One delta (int64 global positions) from R ranks' gathered deltas:
        rank_offsets int64 [R, T+1], rank_indices int64 [R, stride],
        rank_values int16 [R, stride] (device tensors, row r = rank r's
        padded buffer).  Per tensor, the ranks' entries in rank order."""
        torch = _torch()
        R, stride = int(rank_indices.shape[0]), int(rank_indices.shape[1])
        nnz = int(rank_offsets[:, -1].sum().item())
        offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        indices = torch.empty(nnz, dtype=torch.int64, device=self.device)
        values = torch.empty(nnz, dtype=torch.int16, device=self.device)
        ro, ri, rv = (x.contiguous() for x in (rank_offsets, rank_indices, rank_values))
        _check(dws_merge_shards(self.handle, R, ro.data_ptr(), ri.data_ptr() if stride else 0,
                                rv.data_ptr() if stride else 0, stride, offsets.data_ptr(),
                                indices.data_ptr() if nnz else 0, values.data_ptr() if nnz else 0,
                                nnz, self.workspace.data_ptr(), self.workspace_bytes,
                                _stream_handle(stream)), "dws_merge_shards")
        self.raise_on_error("dws_merge_shards", stream)
        return Delta(offsets, indices, values)

    # -- byte-granular sparse XOR (the plan: packed layers as 16-bit words) --
    def xor_bytes_from_words(self, old_table, word_delta: Delta, capacity=None, stream=None):
        """(offsets int64[T+1], positions int32[n], values uint8[n]) of the
        byte-granular XOR delta made from a word delta of the same layers;
        capacity defaults to twice the word entries (every byte changed)."""
        torch = _torch()
        cap = 2 * word_delta.count if capacity is None else int(capacity)
        offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        positions = torch.empty(max(1, cap), dtype=torch.int32, device=self.device)
        values = torch.empty(max(1, cap), dtype=torch.uint8, device=self.device)
        o, i, v, c = word_delta.as_ref()
        _check(dws_xor_bytes_from_words(self.handle, old_table.data_ptr(), o, i, v, c, offsets.data_ptr(),
                                        positions.data_ptr(), values.data_ptr(), cap,
                                        self.workspace.data_ptr(), self.workspace_bytes,
                                        _stream_handle(stream)), "dws_xor_bytes_from_words")
        return offsets, positions, values

    def apply_bytes(self, buf_table, offsets, positions, values, count=None, stream=None):
        n = int(offsets[-1].item()) if count is None else int(count)
        _check(dws_apply_bytes(self.handle, buf_table.data_ptr(), offsets.data_ptr(),
                               positions.data_ptr() if n else 0, values.data_ptr() if n else 0, n,
                               self.workspace.data_ptr(), self.workspace_bytes, _stream_handle(stream)),
               "dws_apply_bytes")

    # -- wire form --
    def pos_width(self, t: int) -> int:
        return dws_pos_width(self.handle, t)

    def pack_positions(self, delta: Delta, stream=None):
        """(positions uint8[block size], pos_offsets int64[T+1]) of a delta."""
        torch = _torch()
        cap = 4 * delta.count
        positions = torch.empty(max(2, cap), dtype=torch.uint8, device=self.device)
        pos_offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        o, i, _, c = delta.as_ref()
        _check(dws_pack_positions(self.handle, o, i, c, positions.data_ptr(), cap,
                                  pos_offsets.data_ptr(), self.workspace.data_ptr(),
                                  self.workspace_bytes, _stream_handle(stream)), "dws_pack_positions")
        self.raise_on_error("dws_pack_positions", stream)
        return positions[:int(pos_offsets[-1].item())], pos_offsets

    # -- delta file (safetensors) --
    @staticmethod
    def _host_bytes(buf, what):
        """The file buffer is read and written by host code: a contiguous
        uint8 tensor in CPU memory."""
        if buf.device.type != "cpu" or buf.dtype != _torch().uint8 or not buf.is_contiguous():
            raise ValueError(f"{what} must be a contiguous uint8 tensor in host memory")
        return buf

    def _host_offsets(self, offsets):
        import numpy as np
        if hasattr(offsets, "detach"):
            offsets = offsets.detach().cpu().numpy()
        o = np.ascontiguousarray(offsets, dtype=np.int64)
        if o.size != self.num_tensors + 1:
            raise ValueError("offsets must have T+1 entries")
        return o

    def delta_file_header(self, names, offsets, model_version: int) -> bytes:
        """The delta file's header (length prefix + JSON) for these offsets."""
        o = self._host_offsets(offsets)
        arr = make_name_array(names)
        st, n = dws_st_delta_header(self.handle, arr, o.ctypes.data, int(model_version), None, 0)
        _check(st, "dws_st_delta_header")
        buf = ctypes.create_string_buffer(max(1, n))
        st, n = dws_st_delta_header(self.handle, arr, o.ctypes.data, int(model_version),
                                    ctypes.addressof(buf), n)
        _check(st, "dws_st_delta_header")
        return buf.raw[:n]

    def write_delta_file(self, delta: Delta, names, model_version: int, out=None, stream=None):
        """The delta file of `delta` in a host uint8 tensor (pinned when this
        call allocates it; `out` may pass a big enough one).  Reads the
        offsets to the host and waits for the stream: the bytes are there on
        return."""
        torch = _torch()
        o = self._host_offsets(delta.offsets)
        arr = make_name_array(names)
        _, i, v, _ = delta.as_ref()
        st, need = dws_st_delta_write(self.handle, arr, o.ctypes.data, int(model_version), i, v,
                                      None, 0, 0)
        _check(st, "dws_st_delta_write")
        if out is not None:
            self._host_bytes(out, "out")
        if out is None or out.numel() < need:
            out = torch.empty(max(1, need), dtype=torch.uint8, pin_memory=True)
        sh = _stream_handle(stream)
        st, need = dws_st_delta_write(self.handle, arr, o.ctypes.data, int(model_version), i, v,
                                      out.data_ptr(), int(out.numel()), sh)
        _check(st, "dws_st_delta_write")
        (stream or torch.cuda.current_stream()).synchronize()
        return out[:need]

    def read_delta_file(self, file, names, capacity=None, stream=None):
        """(Delta on the device, model_version) from a delta file held in a
        host uint8 tensor or a bytes-like object.  Without `capacity` the
        header is parsed twice (size, then copies).  Waits for the stream."""
        import numpy as np
        torch = _torch()
        if not hasattr(file, "data_ptr"):
            file = torch.frombuffer(bytearray(file), dtype=torch.uint8) if len(file) else \
                torch.empty(0, dtype=torch.uint8)
        self._host_bytes(file, "file")
        arr = make_name_array(names)
        oh = np.zeros(self.num_tensors + 1, dtype=np.int64)
        offsets = torch.empty(self.num_tensors + 1, dtype=torch.int64, device=self.device)
        fp, fs = (file.data_ptr() if file.numel() else 0), int(file.numel())
        sh = _stream_handle(stream)
        if capacity is None:
            st, capacity, _ = dws_st_delta_read(self.handle, arr, fp, fs, oh.ctypes.data,
                                                offsets.data_ptr(), 0, 0, 0, sh)
            if st not in (DWS_OK, DWS_ERR_CAPACITY):
                raise DwsError(st, "dws_st_delta_read")
        indices = torch.empty(capacity, dtype=torch.int32, device=self.device)
        values = torch.empty(capacity, dtype=torch.int16, device=self.device)
        st, nnz, ver = dws_st_delta_read(self.handle, arr, fp, fs, oh.ctypes.data,
                                         offsets.data_ptr(), indices.data_ptr() if capacity else 0,
                                         values.data_ptr() if capacity else 0, capacity, sh)
        if st != DWS_OK:
            raise DwsError(st, "dws_st_delta_read", nnz if st == DWS_ERR_CAPACITY else None)
        (stream or torch.cuda.current_stream()).synchronize()
        return Delta(offsets, indices[:nnz], values[:nnz]), ver

    def apply_chain(self, snap_table, deltas, stream=None, mode=DWS_CHAIN_AUTO):
        arr = make_delta_array([d.as_ref() for d in deltas])
        if mode == DWS_CHAIN_AUTO:
            _check(dws_apply_chain(self.handle, snap_table.data_ptr(), arr, len(deltas),
                                   self.workspace.data_ptr(), self.workspace_bytes,
                                   _stream_handle(stream)), "dws_apply_chain")
        else:
            _check(dws_apply_chain_ex(self.handle, snap_table.data_ptr(), arr, len(deltas), mode,
                                      self.workspace.data_ptr(), self.workspace_bytes,
                                      _stream_handle(stream)), "dws_apply_chain_ex")


def _wire_int(wire) -> int:
    """The 128-bit little-endian integer libdws wrote into a 2-word device
    tensor, as a Python int (reading only: libdws computed it)."""
    return int.from_bytes(wire.cpu().numpy().tobytes(), "little")


def checksum(positions, pos_bytes: int, values, stream=None) -> int:
    """The wire checksum of a byte block and bf16 values (device tensors), as
    libdws computes it (dws_checksum); synchronises to read it."""
    torch = _torch()
    dev = values.device if values.numel() else positions.device
    hashes = torch.empty(2, dtype=torch.int64, device=dev)
    wire = torch.empty(2, dtype=torch.int64, device=dev)
    nnz = int(values.numel())
    _check(dws_checksum(positions.data_ptr() if pos_bytes else 0, int(pos_bytes),
                        values.data_ptr() if nnz else 0, nnz, hashes.data_ptr(), wire.data_ptr(),
                        _stream_handle(stream)), "dws_checksum")
    return _wire_int(wire)


def xor_encode(old, new, mask=None, stream=None):
    """mask = old ^ new over the tensors' bytes (device tensors)."""
    torch = _torch()
    nbytes = old.numel() * old.element_size()
    if new.numel() * new.element_size() != nbytes:
        raise ValueError("size mismatch")
    if mask is None:
        mask = torch.empty(nbytes, dtype=torch.uint8, device=old.device)
    _check(dws_xor_encode(old.data_ptr(), new.data_ptr(), mask.data_ptr(), nbytes,
                          _stream_handle(stream)), "dws_xor_encode")
    return mask


def xor_apply(buf, mask, stream=None):
    """buf ^= mask in place over buf's bytes."""
    nbytes = buf.numel() * buf.element_size()
    if mask.numel() * mask.element_size() != nbytes:
        raise ValueError("size mismatch")
    _check(dws_xor_apply(buf.data_ptr(), mask.data_ptr(), nbytes, _stream_handle(stream)),
           "dws_xor_apply")


def xor_apply_layers(bufs, masks, staging0, staging1, apply_stream=None, copy_stream=None):
    """Double-buffered per-layer XOR apply (see dws_xor_apply_layers)."""
    L = len(bufs)
    nb = (ctypes.c_int64 * max(1, L))(*[b.numel() * b.element_size() for b in bufs])
    sb = min(staging0.numel() * staging0.element_size(),
             staging1.numel() * staging1.element_size())
    _check(dws_xor_apply_layers(make_ptr_array([b.data_ptr() for b in bufs]),
                                make_ptr_array([m.data_ptr() for m in masks]), nb, L,
                                staging0.data_ptr(), staging1.data_ptr(), sb,
                                _stream_handle(apply_stream), _stream_handle(copy_stream)),
           "dws_xor_apply_layers")
