"""Pins for the delta-file oracle (oracle/st_file.py), no GPU.

The oracle writes and reads a delta in the safetensors format.  It is pinned
to two things other than itself: the hand-written files under tests/golden/
(the format definition written out byte by byte), and the `safetensors`
library, which reads what the oracle writes and writes files (in its own key
order and data layout) that the oracle must read back to the same delta.
"""
from __future__ import annotations

import json
import struct

import numpy as np
import pytest
import torch

safetensors = pytest.importorskip("safetensors")
from safetensors import safe_open  # noqa: E402
from safetensors.torch import load as st_load  # noqa: E402
from safetensors.torch import save as st_save  # noqa: E402

from oracle import st_file  # noqa: E402
from tests import _golden as G  # noqa: E402


def _case(d, k):
    names = d[f"{k} names"]
    numels = [int(x) for x in d[f"{k} numels"]]
    offsets = np.array([int(x) for x in d[f"{k} offsets"]], dtype=np.int64)
    indices = np.array([int(x) for x in d[f"{k} indices"]], dtype=np.int32)
    values = G.hex16(d[f"{k} values"])
    return names, numels, offsets, indices, values, int(d[f"{k} model_version"][0])


@pytest.mark.parametrize("k", ["1", "2"])
def test_delta_file_golden_bytes(k):
    # A wrong length prefix, missing padding, a key out of order, a quote
    # escaped once instead of twice inside changed_params, ASCII-escaped
    # UTF-8, values before indices, or big-endian data: each changes a byte.
    d = G.keyed("st_delta_files.txt")
    names, numels, offsets, indices, values, version = _case(d, k)
    blob = st_file.write_delta(names, numels, offsets, indices, values, version)
    text = d[f"{k} header"][0].encode("utf-8")
    hb = int(d[f"{k} header_bytes"][0])
    assert hb % 8 == 0 and len(text) <= hb < len(text) + 8
    want = struct.pack("<Q", hb) + text + b" " * (hb - len(text)) + bytes(G.hex8(d[f"{k} body"]))
    assert blob == want
    o, i, v, ver = st_file.read_delta(blob, names)
    np.testing.assert_array_equal(o, offsets)
    np.testing.assert_array_equal(i, indices)
    np.testing.assert_array_equal(v, values)
    assert ver == version


def _random_delta(rng, T, weird=False):
    alphabet = list("abcdefgh_.0123456789") + (['"', "\\", "\n", "\t", "\x01", "é", "文", "\x7f"]
                                               if weird else [])
    names = []
    while len(names) < T:
        n = "".join(rng.choice(alphabet, int(rng.integers(1, 12))))
        if n not in names:
            names.append(n)
    numels = [int(x) for x in rng.choice([0, 1, 7, 300, 5000], T)]
    offs, idx, val = [0], [], []
    for n in numels:
        c = int(rng.integers(0, n + 1)) if n and rng.random() < 0.7 else 0
        idx.extend(sorted(rng.choice(n, c, replace=False).tolist()) if c else [])
        val.extend(rng.integers(0, 1 << 16, c).tolist())
        offs.append(offs[-1] + c)
    return (names, numels, np.array(offs, dtype=np.int64), np.array(idx, dtype=np.int32),
            np.array(val, dtype=np.uint16))


@pytest.mark.parametrize("seed,weird", [(1, False), (2, True), (3, True)])
def test_library_reads_the_oracle_file(tmp_path, seed, weird):
    # The safetensors library parses the oracle's header and data: a wrong
    # offset, dtype, shape, escape or length prefix makes it fail or give
    # other tensors.
    rng = np.random.default_rng(seed)
    names, numels, offsets, indices, values = _random_delta(rng, 12, weird)
    blob = st_file.write_delta(names, numels, offsets, indices, values, 41)
    path = tmp_path / "d.safetensors"
    path.write_bytes(blob)
    changed = [names[t] for t in range(12) if offsets[t + 1] > offsets[t]]
    with safe_open(str(path), framework="pt") as f:
        meta = f.metadata()
        assert meta["sparse"] == "True" and meta["model_version"] == "41"
        assert json.loads(meta["changed_params"]) == changed
        nnz = int(offsets[-1])
        assert meta["sparsity"] == "%.6f" % (1 - nnz / sum(numels))
        assert sorted(f.keys()) == sorted([n + s for n in changed for s in (".indices", ".values")])
    tensors = st_load(blob)
    for t, n in enumerate(names):
        a, b = int(offsets[t]), int(offsets[t + 1])
        if a == b:
            continue
        got_i = tensors[n + ".indices"]
        got_v = tensors[n + ".values"]
        assert got_i.dtype == torch.int32 and got_v.dtype == torch.bfloat16
        np.testing.assert_array_equal(got_i.numpy(), indices[a:b])
        np.testing.assert_array_equal(got_v.view(torch.int16).numpy().view(np.uint16), values[a:b])


@pytest.mark.parametrize("seed", [4, 5])
def test_oracle_reads_the_library_file(seed):
    # The library writes its own key order and data layout (sorted by dtype
    # and name), so the reader must follow data_offsets rather than assume
    # the oracle's layout.
    rng = np.random.default_rng(seed)
    names, numels, offsets, indices, values = _random_delta(rng, 15, weird=seed == 5)
    changed = [names[t] for t in range(15) if offsets[t + 1] > offsets[t]]
    tensors = {}
    for t in rng.permutation(15):
        a, b = int(offsets[t]), int(offsets[t + 1])
        if a < b:
            tensors[names[t] + ".values"] = torch.from_numpy(
                values[a:b].view(np.int16).copy()).view(torch.bfloat16)
            tensors[names[t] + ".indices"] = torch.from_numpy(indices[a:b].copy())
    meta = {"changed_params": json.dumps(changed), "model_version": "7", "sparse": "True",
            "sparsity": "0.5"}
    o, i, v, ver = st_file.read_delta(st_save(tensors, metadata=meta), names)
    np.testing.assert_array_equal(o, offsets)
    np.testing.assert_array_equal(i, indices)
    np.testing.assert_array_equal(v, values)
    assert ver == 7


def test_reader_refuses_inconsistent_files():
    # sec 4.3: the receiver applies what changed_params lists; a file whose
    # entries disagree with it, an anchor (sparse False), a truncated
    # header or a length mismatch is refused, not half-applied.
    names = ["a", "b"]
    ok = {"a.indices": torch.tensor([1], dtype=torch.int32),
          "a.values": torch.tensor([1.0], dtype=torch.bfloat16)}
    meta = {"sparse": "True", "model_version": "1", "changed_params": '["a"]'}
    st_file.read_delta(st_save(ok, metadata=meta), names)
    bad = [
        (ok, {**meta, "sparse": "False"}),
        (ok, {**meta, "changed_params": '["a","b"]'}),
        (ok, {**meta, "changed_params": '["a","a"]'}),
        (ok, {**meta, "changed_params": '["c"]'}),
        (ok, {**meta, "changed_params": "[]"}),
        ({**ok, "b.values": torch.tensor([1.0], dtype=torch.bfloat16)}, meta),
        ({**ok, "a.values": torch.tensor([1.0, 2.0], dtype=torch.bfloat16)}, meta),
        ({**ok, "a.indices": torch.tensor([1], dtype=torch.int64)}, meta),
        (ok, {k: v for k, v in meta.items() if k != "changed_params"}),
    ]
    for tensors, m in bad:
        with pytest.raises(st_file.DeltaFileError):
            st_file.read_delta(st_save(tensors, metadata=m), names)
    blob = st_save(ok, metadata=meta)
    for cut in (0, 7, 20):
        with pytest.raises(st_file.DeltaFileError):
            st_file.read_delta(blob[:cut], names)


def test_empty_delta_and_sparsity_edges():
    # nnz = 0: metadata only, no tensors, no data; the library accepts it.
    blob = st_file.write_delta(["x"], [10], [0, 0], [], [], 3)
    meta = json.loads(blob[8:8 + struct.unpack_from("<Q", blob)[0]])
    assert meta == {"__metadata__": {"sparse": "True", "model_version": "3",
                                     "sparsity": "1.000000", "changed_params": "[]"}}
    assert st_load(blob) == {}
    o, i, v, _ = st_file.read_delta(blob, ["x"])
    assert o.tolist() == [0, 0] and i.size == 0 and v.size == 0
    # no elements at all: sparsity 1; every element changed: 0
    assert st_file.sparsity(0, 0) == "1.000000"
    assert st_file.sparsity(5, 5) == "0.000000"


def _raw(header_text: str, data: bytes = b"") -> bytes:
    t = header_text.encode("utf-8")
    return struct.pack("<Q", len(t)) + t + data


def test_reader_takes_the_json_grammar_strictly():
    # What Python's json module would let through but a safetensors header
    # may not hold: repeated keys, NaN, true or 1.0 as a count, a padded or
    # signed-plus model_version.  Each is refused; the well-formed variant
    # of the same file (first line) is read.
    md = '"__metadata__":{"sparse":"True","model_version":"%s","changed_params":"[\\"a\\"]"}'
    good_entries = ('"a.indices":{"dtype":"I32","shape":[%s],"data_offsets":[0,4]},'
                    '"a.values":{"dtype":"BF16","shape":[1],"data_offsets":[4,6]}')
    data = struct.pack("<iH", 3, 0x3F80)
    ok = _raw("{" + md % "5" + "," + good_entries % "1" + "}", data)
    o, i, v, ver = st_file.read_delta(ok, ["a"])
    assert o.tolist() == [0, 1] and i.tolist() == [3] and v.tolist() == [0x3F80] and ver == 5
    assert st_file.read_delta(_raw(" {" + md % "-0" + "," + good_entries % "1" + "}  ", data),
                              ["a"])[3] == 0
    bad = [
        "{" + md % "5" + "," + good_entries % "true" + "}",
        "{" + md % "5" + "," + good_entries % "1.0" + "}",
        "{" + md % "5" + "," + good_entries % "NaN" + "}",
        "{" + md % " 5" + "," + good_entries % "1" + "}",
        "{" + md % "+5" + "," + good_entries % "1" + "}",
        "{" + md % "9223372036854775808" + "," + good_entries % "1" + "}",
        "{" + md % "5" + "," + good_entries % "1" + "," + good_entries % "1" + "}",
        "{" + md % "5" + "," + good_entries % "1" + "} x",
        "[" + md % "5" + "]",
    ]
    for text in bad:
        with pytest.raises(st_file.DeltaFileError):
            st_file.read_delta(_raw(text, data), ["a"])
    with pytest.raises(ValueError):
        st_file.read_delta(ok, ["a", "a"])


def test_reader_refuses_more_entries_than_elements_when_given_the_sizes():
    # [TRL] §4.1: a delta names each changed element of a parameter once, so
    # a parameter with n elements has at most n entries.  A hand-written file
    # listing 3 entries for "a": read without sizes, refused for a 2-element
    # "a", read for a 3-element one.
    md = '"__metadata__":{"sparse":"True","model_version":"1","changed_params":"[\\"a\\"]"}'
    ent = ('"a.indices":{"dtype":"I32","shape":[3],"data_offsets":[0,12]},'
           '"a.values":{"dtype":"BF16","shape":[3],"data_offsets":[12,18]}')
    blob = _raw("{" + md + "," + ent + "}", struct.pack("<3i3H", 0, 1, 2, 1, 2, 3))
    assert st_file.read_delta(blob, ["a"])[0].tolist() == [0, 3]
    assert st_file.read_delta(blob, ["a"], [3])[1].tolist() == [0, 1, 2]
    with pytest.raises(st_file.DeltaFileError):
        st_file.read_delta(blob, ["a"], [2])
