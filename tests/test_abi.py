"""The C-ABI library without a GPU: it builds, loads, exports every symbol
include/dws.h declares, and its host-side validation answers as documented.
No call here launches or touches device memory."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "dws.h")).read()
    return sorted(set(re.findall(r"^DWS_API[^(]*?\b(dws_\w+)\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    from tests._dev import build_module
    path = build_module().build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for name in ["dws_plan_create", "dws_plan_upload", "dws_encode", "dws_count", "dws_apply",
                 "dws_apply_chain", "dws_apply_chain_ex", "dws_xor_encode", "dws_xor_apply", "dws_xor_apply_layers",
                 "dws_status", "dws_strerror"]:
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    from tests._dev import build_module
    out = subprocess.run(["nm", "-D", "--defined-only", build_module().LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [s for s in _declared_symbols() if s not in exported]
    assert not missing, missing
    for s in _declared_symbols():
        getattr(lib, s)  # resolvable through the dynamic loader


def test_plan_validation_on_the_host():
    import sparse_bf16_delta_b200 as dws
    with pytest.raises(dws.DwsError) as e:
        dws.dws_plan_create([10, 1 << 31])
    assert e.value.code == dws.DWS_ERR_INVALID
    with pytest.raises(dws.DwsError) as e:
        dws.dws_plan_create([10, -1])
    assert e.value.code == dws.DWS_ERR_INVALID
    with pytest.raises(dws.DwsError) as e:
        dws.dws_plan_create([])
    assert e.value.code == dws.DWS_ERR_INVALID
    with pytest.raises(dws.DwsError) as e:
        dws.dws_plan_create([10], elem_size=4)
    assert e.value.code == dws.DWS_ERR_UNSUPPORTED


def test_plan_tiling_and_workspace_size():
    import sparse_bf16_delta_b200 as dws
    te = dws.dws_tile_elems()
    numels = [0, 1, te, te + 1, 3 * te, (1 << 31) - 1]
    p = dws.dws_plan_create(numels)
    try:
        assert dws.dws_plan_num_tensors(p) == len(numels)
        assert dws.dws_plan_num_elements(p) == sum(numels)
        want_tiles = sum(max(1, -(-n // te)) for n in numels)
        assert dws.dws_plan_num_tiles(p) == want_tiles
        ws = dws.dws_plan_workspace_bytes(p)
        assert ws % 256 == 0
        # header + tensor table + 68 bytes per tile (map 4, scan state 8 in
        # a 32-byte slot, descriptor 32), each region 256-aligned
        lo = 256 + 16 * len(numels) + 8 + 68 * want_tiles
        assert lo <= ws <= lo + 256 * 6
    finally:
        dws.dws_plan_destroy(p)


def test_host_side_argument_errors_need_no_device():
    import sparse_bf16_delta_b200 as dws
    p = dws.dws_plan_create([100])
    try:
        # null workspace / misaligned workspace / too small: refused on the host
        assert dws.dws_encode(p, 1, 1, 1, 1, 1, 10, None, 0, None) == dws.DWS_ERR_INVALID
        assert dws.dws_encode(p, 1, 1, 1, 1, 1, 10, 0x1000 + 8, 1 << 20, None) == dws.DWS_ERR_WORKSPACE
        assert dws.dws_encode(p, 1, 1, 1, 1, 1, 10, 0x1000, 16, None) == dws.DWS_ERR_WORKSPACE
        assert dws.dws_encode(p, 1, 1, 1, 1, 1, -1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_apply(p, 1, 1, 1, 1, -5, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        arr = dws.make_delta_array([(1, 1, 1, 0)])
        assert dws.dws_apply_chain(p, 1, arr, 0, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_chain(p, 1, arr, 65, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_encode_global(p, 1, 1, None, 1, 1, 1, 10, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_encode_checksum(p, 1, 1, 1, 1, 1, 10, None, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_encode_nnz(p, 1, 1, 1, 1, 1, 10, 1, 1, None, 0, None) == dws.DWS_ERR_INVALID
        assert dws.dws_encode_nnz(p, 1, 1, 1, 1, 1, -1, 1, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_pack_positions(p, 1, 1, 4, 0x1001, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_checksum(1, -1, 1, 1, 0x1000, 0x2000, None) == dws.DWS_ERR_INVALID
        assert dws.dws_checksum(1, 4, 1, 1, None, 0x2000, None) == dws.DWS_ERR_INVALID
        assert dws.dws_pos_width(p, 0) == 2 and dws.dws_pos_width(p, 1) == 0
        # dws_merge_shards: ranks out of range, null or misaligned arrays, negative sizes
        assert dws.dws_merge_shards(p, 0, 8, 8, 8, 1, 8, 8, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_merge_shards(p, 1, None, 8, 8, 1, 8, 8, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_merge_shards(p, 1, 8, 12, 8, 1, 8, 8, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_merge_shards(p, 1, 8, 8, 9, 1, 8, 8, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_merge_shards(p, 1, 8, 8, 8, -1, 8, 8, 8, 1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_merge_shards(p, 1, 8, 8, 8, 1, 8, 8, 8, 1, 0x1000, 16, None) == dws.DWS_ERR_WORKSPACE
        # byte-granular XOR delta: null or misaligned arrays, negative sizes
        ws = (0x1000, 1 << 20, None)
        assert dws.dws_xor_bytes_from_words(p, None, 8, 8, 8, 1, 8, 8, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_xor_bytes_from_words(p, 8, 8, 0x1001, 8, 1, 8, 8, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_xor_bytes_from_words(p, 8, 8, 8, 9, 1, 8, 8, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_xor_bytes_from_words(p, 8, 8, 8, 8, -1, 8, 8, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_xor_bytes_from_words(p, 8, 8, 8, 8, 1, 8, 8, 8, -1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_xor_bytes_from_words(p, 8, 8, 8, 8, 1, 8, 0x1002, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_bytes(p, None, 8, 8, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_bytes(p, 8, 8, 0x1002, 8, 1, *ws) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_bytes(p, 8, 8, 8, 8, -1, *ws) == dws.DWS_ERR_INVALID
        big = dws.dws_plan_create([1 << 30])  # 2^31 bytes: byte positions would not fit int32
        try:
            assert dws.dws_xor_bytes_from_words(big, 8, 8, 8, 8, 1, 8, 8, 8, 1, 0x1000, 1 << 26, None) \
                == dws.DWS_ERR_INVALID
            assert dws.dws_apply_bytes(big, 8, 8, 8, 8, 1, 0x1000, 1 << 26, None) == dws.DWS_ERR_INVALID
        finally:
            dws.dws_plan_destroy(big)
        assert dws.dws_apply_chain_ex(p, 1, arr, 1, 3, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_chain_ex(p, 1, arr, 1, -1, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
        assert dws.dws_apply_chain_ex(p, 1, arr, 0, 2, 0x1000, 1 << 20, None) == dws.DWS_ERR_INVALID
    finally:
        dws.dws_plan_destroy(p)
    assert dws.dws_xor_encode(1, 1, 1, -1, None) == dws.DWS_ERR_INVALID
    assert dws.dws_xor_encode(0, 0, 0, 0, None) == dws.DWS_OK  # empty: nothing to do
    assert dws.dws_strerror(dws.DWS_ERR_CAPACITY) == "output capacity exceeded"
    assert "sm_100a" in dws.dws_version()


def test_product_path_does_not_reach_the_oracle():
    pkg = os.path.join(ROOT, "sparse_bf16_delta_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "oracle.h" not in text and "liboracle" not in text, f
    # and the other way: the oracle reaches neither the package nor libdws
    for dirpath, _, files in os.walk(os.path.join(ROOT, "oracle")):
        for f in files:
            if f.endswith((".py", ".c", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                for ref in ("import sparse_bf16_delta_b200", "from sparse_bf16_delta_b200",
                            "libdws.so", '#include "dws', "dws_internal"):
                    assert ref not in text, (f, ref)
