"""Helpers shared by the GPU tests: moving bits between torch and numpy and
comparing libdws outputs with the CPU oracle."""
from __future__ import annotations

import importlib.util
import os

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def build_module():
    """sparse_bf16_delta_b200/_build.py, loaded by path (importing the package
    would need the library it builds)."""
    path = os.path.join(ROOT, "sparse_bf16_delta_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("dws_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Any 2-byte tensor -> its uint16 bits on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)


def host_bytes(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.uint8).cpu().numpy().reshape(-1)


def dev_bits(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 numpy -> bf16 device tensor with those bits."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16).copy()).to(device).view(torch.bfloat16)


def delta_to_host(delta):
    return (delta.offsets.cpu().numpy(), delta.indices.cpu().numpy(),
            delta.values.cpu().numpy().view(np.uint16))


def assert_delta_equal(got, want):
    go, gi, gv = got
    wo, wi, wv = want
    np.testing.assert_array_equal(go, wo)
    np.testing.assert_array_equal(gi, wi)
    np.testing.assert_array_equal(gv, wv)
