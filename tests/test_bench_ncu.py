"""bench.py's per-row ncu figures, on CPU: every committed capture it cites
exists and yields a DRAM rate equal to its own table's bytes over its
duration, and every row the bench prints maps to captures or to a stated
reason."""
from __future__ import annotations

import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# The rows of the default bench line (their names as bench.py builds them).
ROWS = [
    "count_llama3_8b_lr3e-06", "encode_global_int64_llama3_8b_lr3e-06", "encode_checksum_llama3_8b_lr3e-06",
    "delta_file_write_llama3_8b", "delta_file_read_llama3_8b", "encode_llama3_8b_lr1e-5",
    "apply_llama3_8b_lr1e-5", "pack_positions_llama3_8b_lr1e-5", "checksum_llama3_8b_lr1e-5",
    "encode_single_1024x1024", "apply_single_1024x1024", "xor_encode_single_1024x1024",
    "xor_apply_single_1024x1024", "apply_chain_qwen3_0p6b_k10", "apply_chain_qwen3_0p6b_k10_tile_merge",
    "apply_chain_qwen3_0p6b_k10_scatter", "merge_shards_qwen3_0p6b_8ranks", "encode_qwen3_0p6b",
    "xor_encode_nvfp4_40x0.8GB", "xor_apply_nvfp4_40x0.8GB", "xor_apply_layers_double_buffered_40x0.8GB",
    "xor_apply_layers_pinned_host_4x0.8GB", "encode_sparse_nvfp4_40x0.8GB", "bytes_from_words_nvfp4_40x0.8GB",
    "encode_sparse_bytes_nvfp4_40x0.8GB", "apply_bytes_nvfp4_40x0.8GB", "apply_sparse_nvfp4_40x0.8GB",
    "apply_sparse_from_pinned_host_nvfp4_40x0.8GB", "apply_chain_stress_12000t_k10",
    "apply_chain_stress_12000t_k10_tile_merge", "apply_chain_stress_12000t_k10_scatter", "encode_stress_12000t",
    # kernels.encode / kernels.apply
    "encode_llama3_8b", "apply_llama3_8b",
]


def test_every_cited_capture_exists_and_parses():
    for _, caps, _ in bench.NCU_ROWS:
        for prof, _, _ in caps:
            assert os.path.exists(os.path.join(ROOT, "profiles", prof)), prof
            v = bench.ncu_dram_GBps(prof)
            assert v is not None and 100 < v < 8000, (prof, v)


def test_dram_rate_is_the_tables_bytes_over_duration():
    # chain_index_kernel_qwen3_0p6b_k10.md: 0.864 GB in 189.3 us
    assert bench.ncu_dram_GBps("chain_index_kernel_qwen3_0p6b_k10.md") == pytest.approx(0.864e9 / 189.3e-6 / 1e9, abs=0.1)
    # encode_kernel_llama3_8b.md lists read and write bytes on separate rows
    txt = open(os.path.join(ROOT, "profiles", "encode_kernel_llama3_8b.md")).read()
    rd = float(re.search(r"dram__bytes_read\.sum \| ([\d.]+) GB", txt).group(1)) * 1e9
    wr = float(re.search(r"dram__bytes_write\.sum \| ([\d.]+) MB", txt).group(1)) * 1e6
    us = float(re.search(r"\| duration[^|]*\| ([\d.]+) us", txt).group(1))
    assert bench.ncu_dram_GBps("encode_kernel_llama3_8b.md") == pytest.approx((rd + wr) / (us * 1e-6) / 1e9, abs=0.1)
    assert bench.ncu_dram_GBps("no_such_capture.md") is None


@pytest.mark.parametrize("name", ROWS)
def test_every_row_has_an_ncu_figure_or_a_reason(name):
    e = bench.ncu_for_row(name)
    if "captures" in e:
        assert e["captures"] and all(c["dram_GBps"] for c in e["captures"])
    else:
        assert e["dram_GBps"] is None and e["reason"] != "no committed capture for this row"


def test_rows_get_the_capture_of_their_own_kernel():
    assert [c["kernel"] for c in bench.ncu_for_row("apply_chain_qwen3_0p6b_k10_tile_merge")["captures"]] == \
        ["chain_index_kernel", "chain_tile_kernel<merge>"]
    assert [c["kernel"] for c in bench.ncu_for_row("apply_chain_qwen3_0p6b_k10_scatter")["captures"]] == \
        ["chain_index_kernel", "chain_tile_kernel<scatter>"]
    assert bench.ncu_for_row("encode_sparse_bytes_nvfp4_40x0.8GB")["captures"][1]["kernel"] == "bytes_write_kernel"
    assert "reason" in bench.ncu_for_row("xor_apply_layers_pinned_host_4x0.8GB")
    assert bench.ncu_for_row("something_new")["reason"] == "no committed capture for this row"


def _fake_tree(tmp_path, src, sha_line):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "sparse_bf16_delta_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "encode.cu").write_bytes(src)
    (tmp_path / "profiles" / "encode_kernel_llama3_8b.md").write_text(
        "# encode capture\n\n"
        f"- encode.cu sha256[:16]: `{sha_line}`\n"
        "- dram bytes per element: 4.25\n"
        "- nnz fraction: 0.035\n")


def test_encode_traffic_needs_the_capture_of_the_current_source(tmp_path, monkeypatch):
    # roofline.traffic comes from the committed capture only while the
    # kernel source is the one that was captured; any change makes it null.
    import hashlib
    src = b"// some kernel source\n"
    _fake_tree(tmp_path, src, hashlib.sha256(src).hexdigest()[:16])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.encode_traffic_per_elem() == (4.25, 0.035)
    (tmp_path / "sparse_bf16_delta_b200" / "csrc" / "encode.cu").write_bytes(src + b"// changed\n")
    assert bench.encode_traffic_per_elem() == (None, None)
    (tmp_path / "profiles" / "encode_kernel_llama3_8b.md").unlink()
    assert bench.encode_traffic_per_elem() == (None, None)


def test_committed_encode_capture_is_of_the_committed_kernel():
    per_elem, frac = bench.encode_traffic_per_elem()
    assert per_elem is not None and 4.0 < per_elem < 4.4
    assert 0.03 < frac < 0.04
