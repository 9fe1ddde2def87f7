"""The delta file's host code in libdws, checked against the oracle without a GPU.

dws_st_delta_header builds the header on the host (no CUDA call), so its bytes
are compared with the oracle's file here.  dws_st_delta_read parses and
validates on the host before it copies anything; called with capacity 0 it
stops there for any delta with entries (DWS_ERR_CAPACITY, offsets and nnz
filled in).  Its only possible copy then is the offsets array, and the tests
point that at host memory (a numpy array), so no call here touches device
memory.  Every accept/refuse decision must match the oracle's, on crafted
files and on thousands of byte-level mutations of valid ones.
"""
from __future__ import annotations

import json
import struct

import numpy as np
import pytest

pytest.importorskip("safetensors")
from safetensors.torch import save as st_save  # noqa: E402

from oracle import st_file  # noqa: E402
from tests import _golden as G  # noqa: E402
from tests.test_oracle_st_file import _random_delta  # noqa: E402


@pytest.fixture(scope="module")
def dws():
    from tests._dev import build_module
    build_module().build()
    import sparse_bf16_delta_b200 as m
    return m


class _Plan:
    def __init__(self, dws, numels):
        self.dws = dws
        self.h = dws.dws_plan_create(numels)

    def __del__(self):
        self.dws.dws_plan_destroy(self.h)


def c_header(dws, numels, names, offsets, version):
    p = _Plan(dws, numels)
    arr = dws.make_name_array(names)
    o = np.ascontiguousarray(offsets, dtype=np.int64)
    st, n = dws.dws_st_delta_header(p.h, arr, o.ctypes.data, version, None, 0)
    assert st == dws.DWS_OK
    buf = np.zeros(n, dtype=np.uint8)
    st, n2 = dws.dws_st_delta_header(p.h, arr, o.ctypes.data, version, buf.ctypes.data, n)
    assert st == dws.DWS_OK and n2 == n
    # the size a full write would need, asked without a buffer (no copy)
    st, need = dws.dws_st_delta_write(p.h, arr, o.ctypes.data, version, 0, 0, None, 0, 0)
    assert st == dws.DWS_OK
    return buf.tobytes(), need


def c_read(dws, numels, names, blob):
    """('refused' | 'accepted', offsets or None, version or None) from libdws,
    parsing only (capacity 0; the offsets copy goes to host memory)."""
    p = _Plan(dws, numels)
    arr = dws.make_name_array(names)
    T = len(names)
    f = np.frombuffer(blob, dtype=np.uint8).copy() if blob else np.zeros(1, np.uint8)
    oh = np.zeros(T + 1, dtype=np.int64)
    sink = np.zeros(T + 1, dtype=np.int64)   # host memory standing in for the device offsets
    st, nnz, ver = dws.dws_st_delta_read(p.h, arr, f.ctypes.data, len(blob), oh.ctypes.data,
                                         sink.ctypes.data, 0, 0, 0, 0)
    if st == dws.DWS_ERR_BAD_DELTA:
        return "refused", None, None
    assert st in (dws.DWS_ERR_CAPACITY, dws.DWS_OK, dws.DWS_ERR_CUDA), st
    assert nnz == oh[-1]
    return "accepted", oh, ver


def o_read(names, blob, numels=None):
    try:
        o, _, _, ver = st_file.read_delta(blob, names, numels)
    except st_file.DeltaFileError:
        return "refused", None, None
    return "accepted", o, ver


@pytest.mark.parametrize("k", ["1", "2"])
def test_header_golden(dws, k):
    d = G.keyed("st_delta_files.txt")
    names = d[f"{k} names"]
    numels = [int(x) for x in d[f"{k} numels"]]
    offsets = [int(x) for x in d[f"{k} offsets"]]
    hb = int(d[f"{k} header_bytes"][0])
    text = d[f"{k} header"][0].encode("utf-8")
    got, need = c_header(dws, numels, names, offsets, int(d[f"{k} model_version"][0]))
    assert got == struct.pack("<Q", hb) + text + b" " * (hb - len(text))
    assert need == 8 + hb + 6 * offsets[-1]


@pytest.mark.parametrize("seed,weird", [(11, False), (12, True), (13, True), (14, True)])
def test_header_matches_oracle(dws, seed, weird):
    rng = np.random.default_rng(seed)
    for trial in range(8):
        names, numels, offsets, indices, values = _random_delta(rng, 1 + 7 * trial, weird)
        version = int(rng.integers(-(1 << 62), 1 << 62))
        want = st_file.write_delta(names, numels, offsets, indices, values, version)
        got, need = c_header(dws, numels, names, offsets, version)
        assert want[:len(got)] == got
        assert len(want) == len(got) + 6 * int(offsets[-1]) == need


def test_writer_host_errors(dws):
    p = _Plan(dws, [4, 4])
    o = np.array([0, 1, 2], dtype=np.int64)
    ok = dws.make_name_array(["a", "b"])
    buf = np.zeros(4096, dtype=np.uint8)
    hdr = dws.dws_st_delta_header
    assert hdr(p.h, ok, o.ctypes.data, 0, None, 0)[0] == dws.DWS_OK
    assert hdr(p.h, dws.make_name_array(["a", "a"]), o.ctypes.data, 0, None, 0)[0] == \
        dws.DWS_ERR_INVALID
    bad_utf8 = (dws.ctypes.c_char_p * 2)(b"a", b"\xff")
    assert hdr(p.h, bad_utf8, o.ctypes.data, 0, None, 0)[0] == dws.DWS_ERR_INVALID
    assert hdr(p.h, None, o.ctypes.data, 0, None, 0)[0] == dws.DWS_ERR_INVALID
    assert hdr(0, ok, o.ctypes.data, 0, None, 0)[0] == dws.DWS_ERR_INVALID
    for bad in ([1, 1, 2], [0, 2, 1], [0, 5, 5], [0, 1, 6]):
        b = np.array(bad, dtype=np.int64)
        assert hdr(p.h, ok, b.ctypes.data, 0, None, 0)[0] == dws.DWS_ERR_BAD_DELTA, bad
    st, n = hdr(p.h, ok, o.ctypes.data, 0, buf.ctypes.data, 8)
    assert st == dws.DWS_ERR_CAPACITY and n > 8 and not buf[:8].any()
    # the full write refuses a small buffer before it copies anything
    st, need = dws.dws_st_delta_write(p.h, ok, o.ctypes.data, 0, 8, 8, buf.ctypes.data, 16, 0)
    assert st == dws.DWS_ERR_CAPACITY and need == n + 12
    assert dws.dws_st_delta_write(p.h, ok, o.ctypes.data, 0, 0, 0, buf.ctypes.data, 4096,
                                  0)[0] == dws.DWS_ERR_INVALID  # entries but no arrays


def _crafted_files():
    """(names, numels, blob) cases around the reader's rules."""
    out = []
    names, numels = ["a", "b.c", 'q"x'], [4, 5, 6]
    good = st_file.write_delta(names, numels, [0, 2, 2, 3], [1, 3, 5], [1, 2, 3], 9)
    out.append((names, numels, good))
    # library-written files: other key order and data layout
    import torch
    t = {"b.c.values": torch.tensor([1.0, 2.0], dtype=torch.bfloat16),
         "b.c.indices": torch.tensor([0, 4], dtype=torch.int32),
         'q"x.indices': torch.tensor([5], dtype=torch.int32),
         'q"x.values': torch.tensor([3.0], dtype=torch.bfloat16)}
    meta = {"sparse": "True", "model_version": "-3", "changed_params": json.dumps(["b.c", 'q"x'])}
    out.append((names, numels, st_save(t, metadata=meta)))
    for m in ({**meta, "sparse": "False"}, {**meta, "changed_params": '["b.c"]'},
              {**meta, "changed_params": '["b.c","q\\"x","a"]'},
              {**meta, "changed_params": '["b.c","b.c"]'}, {**meta, "model_version": "1.5"},
              {**meta, "model_version": ""}, {**meta, "changed_params": '{"b.c":1}'},
              {k: v for k, v in meta.items() if k != "sparse"}):
        out.append((names, numels, st_save(t, metadata=m)))
    out.append((names, numels, st_save({**t, "a.extra": torch.zeros(1)}, metadata=meta)))

    def raw(text, data=b""):
        b = text.encode("utf-8", "surrogatepass")
        return struct.pack("<Q", len(b)) + b + data

    md = '"__metadata__":{"sparse":"True","model_version":"1","changed_params":"[\\"a\\"]"%s}'
    ent = ('"a.indices":{"dtype":"I32","shape":[1],"data_offsets":[0,4]},'
           '"a.values":{"dtype":"BF16","shape":[1],"data_offsets":[4,6]}')
    data = struct.pack("<iH", 2, 0x4000)
    for extra in ("", ',"deep":' + "[" * 100 + "]" * 100, ',"big":1e400', ',"s":"\\ud800"',
                  ',"u":"\\ud83d\\ude00"', ',"n":null,"t":true,"f":false', ',"x":-0.5e-3'):
        out.append((["a"], [4], raw("{" + md % extra + "," + ent + "}", data)))
    for bad in ('{' + md % "" + ',' + ent + ',}', '﻿{' + md % "" + ',' + ent + '}',
                '{' + md % ',"v":NaN' + ',' + ent + '}', '{' + md % ',"v":01' + ',' + ent + '}',
                '{' + md % ',"v":"\\x"' + ',' + ent + '}', '{' + md % ',"v":"a\tb"' + ',' + ent + '}',
                '{' + md % ',"v":"\\ud800\\uzzzz"' + ',' + ent + '}'):
        out.append((["a"], [4], raw(bad, data)))
    # more entries than the parameter has elements (5 for a 4-element "a")
    ent5 = ('"a.indices":{"dtype":"I32","shape":[5],"data_offsets":[0,20]},'
            '"a.values":{"dtype":"BF16","shape":[5],"data_offsets":[20,30]}')
    data5 = struct.pack("<5i5H", 0, 1, 2, 3, 4, *([0x4000] * 5))
    out.append((["a"], [4], raw("{" + md % "" + "," + ent5 + "}", data5)))
    out.append((["a"], [5], raw("{" + md % "" + "," + ent5 + "}", data5)))
    b = bytearray(raw("{" + md % ',"v":"é"' + "," + ent + "}", data))
    out.append((["a"], [4], bytes(b)))
    b[b.index(b"\xc3")] = 0xC0  # overlong / invalid UTF-8
    out.append((["a"], [4], bytes(b)))
    out.append((["a"], [4], struct.pack("<Q", 1 << 63) + b"{}"))
    out.append((["a"], [4], b"\x02\x00\x00\x00\x00\x00\x00\x00{}"))
    out.append((["a"], [4], b""))
    return out


def test_reader_matches_oracle_on_crafted_files(dws):
    seen = set()
    for names, numels, blob in _crafted_files():
        want = o_read(names, blob, numels)
        got = c_read(dws, numels, names, blob)
        assert got[0] == want[0], (blob[:200], want[0])
        if want[0] == "accepted":
            np.testing.assert_array_equal(got[1], want[1])
            assert got[2] == want[2]
        seen.add(want[0])
    assert seen == {"accepted", "refused"}


@pytest.mark.parametrize("seed", [21, 22, 23])
def test_reader_matches_oracle_on_mutated_files(dws, seed):
    # Flip, insert or delete bytes of valid files (the oracle's layout and
    # the library's): the two parsers must take the same decision on every
    # mutant, and the same offsets when they accept.
    rng = np.random.default_rng(seed)
    decisions = {"accepted": 0, "refused": 0}
    for base in range(6):
        names, numels, offsets, indices, values = _random_delta(rng, 5, weird=base % 2 == 1)
        blob = st_file.write_delta(names, numels, offsets, indices, values, base)
        hl = struct.unpack_from("<Q", blob)[0]
        for trial in range(150):
            b = bytearray(blob)
            for _ in range(int(rng.integers(1, 3))):
                pos = int(rng.integers(8, 8 + hl))  # inside the header
                r = rng.random()
                if r < 0.15:  # whitespace after a separator keeps the file valid
                    seps = [i for i in range(8, 8 + hl) if b[i] in b",:"]
                    b.insert(int(rng.choice(seps)) + 1, int(rng.choice([0x20, 0x09, 0x0A, 0x0D])))
                elif r < 0.6:
                    b[pos] = int(rng.choice([ord(c) for c in '{}[]":,\\0123456789-.eE tu"a']
                                            + [0, 0x80, 0xC3, 0xFF]))
                elif r < 0.8:
                    b.insert(pos, int(rng.integers(0x20, 0x7F)))
                else:
                    del b[pos]
                hl2 = len(b) - 8 - (len(blob) - 8 - hl)  # the data keeps its length
                b[:8] = struct.pack("<Q", max(0, hl2))
            blob2 = bytes(b)
            want = o_read(names, blob2, numels)
            got = c_read(dws, numels, names, blob2)
            assert got[0] == want[0], (blob2[8:8 + hl + 2], want[0])
            if want[0] == "accepted":
                np.testing.assert_array_equal(got[1], want[1])
                assert got[2] == want[2]
            decisions[want[0]] += 1
    assert decisions["accepted"] > 40 and decisions["refused"] > 200, decisions


def test_binding_refuses_file_buffers_outside_host_memory(dws):
    # The header is written and parsed by host code, so a device (here a
    # meta-device) or non-byte buffer is refused before libdws sees it.
    import types

    import torch
    fake = types.SimpleNamespace(num_tensors=1, handle=0, _host_bytes=dws.DeltaPlan._host_bytes)
    with pytest.raises(ValueError):
        dws.DeltaPlan.read_delta_file(fake, torch.empty(16, dtype=torch.uint8, device="meta"), ["a"])
    with pytest.raises(ValueError):
        dws.DeltaPlan.read_delta_file(fake, torch.empty(4, dtype=torch.int32), ["a"])
    with pytest.raises(ValueError):
        dws.DeltaPlan.read_delta_file(fake, torch.empty(32, dtype=torch.uint8)[::2], ["a"])
    dws.DeltaPlan._host_bytes(torch.empty(8, dtype=torch.uint8), "file")  # accepted
