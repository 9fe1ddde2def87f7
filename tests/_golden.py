"""Readers for the small text fixtures under tests/golden/ (each cites its source)."""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if line:
                yield line


def keyed(name) -> dict:
    """'key: v1 v2 ...' lines -> {key: [tokens]}."""
    out = {}
    for line in _lines(name):
        key, _, rest = line.partition(":")
        out[key.strip()] = rest.split()
    return out


def hex16(tokens) -> np.ndarray:
    if tokens == ["-"]:
        return np.zeros(0, dtype=np.uint16)
    return np.array([int(t, 16) for t in tokens], dtype=np.uint16)


def hex8(tokens) -> np.ndarray:
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def encode_example():
    d = keyed("encode_two_tensors.txt")
    T = sum(1 for k in d if k.startswith("old "))
    olds = [hex16(d[f"old {t}"]) for t in range(T)]
    news = [hex16(d[f"new {t}"]) for t in range(T)]
    offsets = np.array([int(x) for x in d["offsets"]], dtype=np.int64)
    indices = np.array([int(x) for x in d["indices"]], dtype=np.int32)
    values = hex16(d["values"])
    return olds, news, offsets, indices, values


def chain_example():
    d = keyed("chain_later_wins.txt")
    T = sum(1 for k in d if k.startswith("anchor "))
    anchor = [hex16(d[f"anchor {t}"]) for t in range(T)]
    final = [hex16(d[f"final {t}"]) for t in range(T)]
    deltas = []
    k = 1
    while f"delta {k} offsets" in d:
        deltas.append((np.array([int(x) for x in d[f"delta {k} offsets"]], dtype=np.int64),
                       np.array([int(x) for x in d[f"delta {k} indices"]], dtype=np.int32),
                       hex16(d[f"delta {k} values"])))
        k += 1
    return anchor, deltas, final


def xor_example():
    d = keyed("xor_bytes.txt")
    return hex8(d["old"]), hex8(d["new"]), hex8(d["mask"])


def xor_byte_delta_example():
    d = keyed("xor_byte_delta.txt")
    layers = [(hex8(d[f"layer{t}_old"]), hex8(d[f"layer{t}_new"])) for t in range(4)]
    ints = lambda k: [int(x) for x in d[k]]
    return (layers, ints("offsets"), ints("positions"), [int(x, 16) for x in d["values"]],
            ints("word_offsets"), ints("word_indices"))


def rounding_cases():
    out = []
    for line in _lines("bf16_rounding.txt"):
        f32, b16, *_ = line.split()
        out.append((int(f32, 16), int(b16, 16)))
    return out
