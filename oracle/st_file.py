"""Plain CPU oracle for the delta file: a delta in the safetensors format.

TEST INFRASTRUCTURE ONLY (the same rule as the rest of ``oracle/``: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it).

Source: "Shipping a Trillion Parameters With a Hub Bucket: Delta Weight Sync in
TRL", §4.1 (safetensors as the wire format): a delta file holds, for every
parameter that changed, two entries, ``{name}.indices`` (int32, flat element
indices, shape [num_changed]) and ``{name}.values`` (bf16, shape
[num_changed]), and string metadata ``sparse``, ``model_version``,
``sparsity`` and ``changed_params``; §4.3 (the receiver reads the metadata,
takes the parameters that ``changed_params`` lists, and writes
``values`` at ``indices`` into the flattened snapshot).

The safetensors container itself: an 8-byte little-endian header length H,
H bytes of a UTF-8 JSON object (each tensor name -> {dtype, shape,
data_offsets [begin, end) into the data that follows}, plus "__metadata__",
a map of strings to strings), then the data.

Readings taken where the page leaves the bytes open (the same in the CUDA
library, which shares no code with this file):
* metadata values: ``sparse`` "True"; ``model_version`` the decimal integer;
  ``sparsity`` = 1 - nnz / (total elements), printed with 6 decimals ("%.6f";
  1.000000 when there are no elements); ``changed_params`` the JSON list of
  the names of the parameters with at least one change, in table order;
* JSON: no spaces, ``__metadata__`` first, then ``{name}.indices`` and
  ``{name}.values`` for each changed parameter in table order; strings
  escaped as Python's ``json.dumps(..., ensure_ascii=False)`` does; the
  header padded with spaces to a multiple of 8 bytes;
* data: all parameters' indices (table order), then all their values, so
  the data is the encode's two arrays as they stand.
A reader takes any key order and any data layout; the parameters applied are
exactly those that ``changed_params`` lists (§4.3), and a file whose tensor
entries disagree with that list is refused.  It takes the JSON grammar
strictly: a repeated key in an object, NaN/Infinity, a count or offset that
is not a plain non-negative integer (``true``, ``1.0``), or a model_version
that is not a decimal integer of 64 bits is refused.
"""
from __future__ import annotations

import json
import re
import struct

import numpy as np

DTYPE_BYTES = {"I32": 4, "BF16": 2}


class DeltaFileError(ValueError):
    """The bytes are not a delta file this reader accepts."""


def _dumps(obj) -> str:
    return json.dumps(obj, ensure_ascii=False, separators=(",", ":"))


def _no_repeats(pairs):
    keys = [k for k, _ in pairs]
    if len(set(keys)) != len(keys):
        raise DeltaFileError("a JSON object repeats a key")
    return dict(pairs)


def _no_constants(name):
    raise DeltaFileError(f"non-standard JSON constant {name}")


def _loads(text: str):
    return json.loads(text, object_pairs_hook=_no_repeats, parse_constant=_no_constants)


def _count(x) -> bool:
    return type(x) is int and x >= 0


def sparsity(nnz: int, total: int) -> str:
    return "%.6f" % ((1.0 - nnz / total) if total > 0 else 1.0)


def write_delta(names, numels, offsets, indices, values, model_version: int) -> bytes:
    """The delta file of one encode (offsets int64[T+1], indices int32[nnz],
    values as uint16 bf16 bits [nnz])."""
    offsets = np.asarray(offsets, dtype=np.int64)
    indices = np.asarray(indices, dtype=np.int32)
    values = np.asarray(values).view(np.uint16)
    T = len(names)
    if offsets.size != T + 1 or len(numels) != T:
        raise ValueError("names, numels and offsets disagree on T")
    nnz = int(offsets[T])
    changed = [names[t] for t in range(T) if offsets[t + 1] > offsets[t]]
    header = {"__metadata__": {
        "sparse": "True",
        "model_version": str(int(model_version)),
        "sparsity": sparsity(nnz, int(sum(int(n) for n in numels))),
        "changed_params": _dumps(changed),
    }}
    for t in range(T):
        a, b = int(offsets[t]), int(offsets[t + 1])
        if b == a:
            continue
        header[names[t] + ".indices"] = {"dtype": "I32", "shape": [b - a],
                                         "data_offsets": [4 * a, 4 * b]}
        header[names[t] + ".values"] = {"dtype": "BF16", "shape": [b - a],
                                        "data_offsets": [4 * nnz + 2 * a, 4 * nnz + 2 * b]}
    text = _dumps(header).encode("utf-8")
    text += b" " * (-len(text) % 8)
    body = indices[:nnz].astype("<i4").tobytes() + values[:nnz].astype("<u2").tobytes()
    return struct.pack("<Q", len(text)) + text + body


def read_delta(blob: bytes, names, numels=None):
    """Parse a delta file into the encode layout of the table `names`:
    (offsets int64[T+1], indices int32[nnz], values uint16[nnz], model_version).
    With `numels` (the table's element counts), a parameter listing more
    entries than it has elements is refused: a delta names each changed
    element of a parameter once ([TRL] §4.1), so it has at most numel of them,
    the bound the writer keeps too."""
    if len(blob) < 8:
        raise DeltaFileError("shorter than the length prefix")
    (hlen,) = struct.unpack_from("<Q", blob, 0)
    if hlen > len(blob) - 8:
        raise DeltaFileError("header runs past the end")
    try:
        header = _loads(blob[8:8 + hlen].decode("utf-8"))
    except (UnicodeDecodeError, json.JSONDecodeError) as e:
        raise DeltaFileError(f"header is not UTF-8 JSON: {e}") from None
    if not isinstance(header, dict):
        raise DeltaFileError("header is not an object")
    data = memoryview(blob)[8 + hlen:]
    meta = header.pop("__metadata__", None)
    if not isinstance(meta, dict) or meta.get("sparse") != "True":
        raise DeltaFileError("not a delta (metadata sparse != True)")
    version, changed = meta.get("model_version"), meta.get("changed_params")
    if not isinstance(version, str) or not re.fullmatch(r"-?[0-9]+", version):
        raise DeltaFileError("model_version is not a decimal integer")
    version = int(version)
    if not -(1 << 63) <= version < (1 << 63):
        raise DeltaFileError("model_version does not fit 64 bits")
    if not isinstance(changed, str):
        raise DeltaFileError("changed_params missing")
    try:
        changed = _loads(changed)
    except json.JSONDecodeError as e:
        raise DeltaFileError(f"changed_params is not JSON: {e}") from None
    if not isinstance(changed, list) or not all(isinstance(n, str) for n in changed):
        raise DeltaFileError("changed_params is not a list of names")
    if len(set(changed)) != len(changed):
        raise DeltaFileError("changed_params repeats a name")
    slot = {n: t for t, n in enumerate(names)}
    if len(slot) != len(names):
        raise ValueError("the table repeats a name")
    listed = set(changed)
    for key in header:
        base = key.rsplit(".", 1)[0] if key.endswith((".indices", ".values")) else None
        if base is None or base not in listed:
            raise DeltaFileError(f"tensor {key!r} is not a listed parameter's")

    def entry(key, dtype):
        e = header.get(key)
        if not isinstance(e, dict) or e.get("dtype") != dtype:
            raise DeltaFileError(f"{key!r}: missing or not {dtype}")
        shape, span = e.get("shape"), e.get("data_offsets")
        if not (isinstance(shape, list) and len(shape) == 1 and _count(shape[0])
                and isinstance(span, list) and len(span) == 2 and all(map(_count, span))):
            raise DeltaFileError(f"{key!r}: shape or data_offsets malformed")
        a, b = span
        if not a <= b <= len(data) or b - a != shape[0] * DTYPE_BYTES[dtype]:
            raise DeltaFileError(f"{key!r}: shape and data offsets disagree")
        return shape[0], bytes(data[a:b])

    T = len(names)
    parts = [None] * T
    for n in changed:
        if n not in slot:
            raise DeltaFileError(f"{n!r} is not a parameter of the table")
        ni, ib = entry(n + ".indices", "I32")
        nv, vb = entry(n + ".values", "BF16")
        if ni != nv:
            raise DeltaFileError(f"{n!r}: indices and values differ in length")
        if numels is not None and ni > numels[slot[n]]:
            raise DeltaFileError(f"{n!r}: more entries than the parameter has elements")
        parts[slot[n]] = (np.frombuffer(ib, dtype="<i4"), np.frombuffer(vb, dtype="<u2"))
    offsets = np.zeros(T + 1, dtype=np.int64)
    for t in range(T):
        offsets[t + 1] = offsets[t] + (0 if parts[t] is None else parts[t][0].size)
    empty = (np.zeros(0, np.int32), np.zeros(0, np.uint16))
    idx = np.concatenate([p[0] if p is not None else empty[0] for p in parts] + [empty[0]])
    val = np.concatenate([p[1] if p is not None else empty[1] for p in parts] + [empty[1]])
    return offsets, idx.astype(np.int32), val.astype(np.uint16), version
