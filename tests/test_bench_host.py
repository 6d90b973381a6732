"""Host arithmetic of bench.py that the reported numbers rest on (CPU only).

kept_flops: the effective FLOPs of the kept blocks (the metric's numerator). Pinned by two facts
that do not restate its formula: with every causal block kept it equals the dense causal count
2 * d * L^2 per head and sequence for any L (ragged last block included, since
L = (nb - 1) * B + n_last), and dropping one off-diagonal block of query block i removes exactly
one QK^T and one PV product of n_i rows by B keys, 4 * d * n_i * B.

measured_traffic: the committed DRAM-traffic record is reported only while the kernel sources hash
to the value recorded with it.
"""
import hashlib
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _full_counts(lens, B, hq):
    cols = []
    for L in lens:
        nb = (L + B - 1) // B
        cols.append(np.tile(np.arange(1, nb + 1, dtype=np.int32), (hq, 1)))
    return np.concatenate(cols, axis=1)


@pytest.mark.parametrize("lens,B", [([4096], 128), ([3000], 128), ([1, 129, 640, 77], 64), ([0, 300, 0, 5], 128)])
def test_kept_flops_with_every_block_kept_equals_dense(lens, B):
    hq, d = 3, 128
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    counts = _full_counts(lens, B, hq)
    eff, dense = bench.kept_flops(counts, cu, B, d)
    assert dense == pytest.approx(2.0 * d * hq * sum(float(L) ** 2 for L in lens), rel=0, abs=0)
    assert eff == pytest.approx(dense, rel=1e-12)


def test_kept_flops_dropping_one_block_removes_its_two_products():
    B, d, hq = 128, 128, 2
    lens = [1000]  # 8 blocks, the last of 1000 - 7 * 128 = 104 rows
    cu = np.array([0, 1000], np.int64)
    counts = _full_counts(lens, B, hq)
    eff0, _ = bench.kept_flops(counts, cu, B, d)
    for h, i in [(0, 3), (1, 7)]:
        c = counts.copy()
        c[h, i] -= 1  # one off-diagonal block of (head h, query block i) no longer kept
        n_i = min(B, 1000 - i * B)
        eff1, _ = bench.kept_flops(c, cu, B, d)
        assert eff0 - eff1 == pytest.approx(4.0 * d * n_i * B, rel=1e-12)


def _write_record(root, kernel, workload, sources, read, write):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(root, rel), "rb") as f:
            h.update(f.read())
    rec = {"kernel": kernel, "workload": workload, "dram_bytes_read": read, "dram_bytes_write": write,
           "sources": sources, "sources_sha256": h.hexdigest()}
    with open(os.path.join(root, "profiles", "attn_kernel_traffic.json"), "w") as f:
        json.dump(rec, f)


def test_measured_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    root = str(tmp_path)
    for name, text in [("a.cu", "kernel a"), ("b.cuh", "header b")]:
        (tmp_path / name).write_text(text)
    _write_record(root, "attn_kernel<128>", "w128k", ["a.cu", "b.cuh"], 3.0e9, 1.0e9)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.measured_traffic("attn_kernel<128>", "w128k") == 4.0e9
    assert bench.measured_traffic("attn_kernel<64>", "w128k") is None      # another kernel
    assert bench.measured_traffic("attn_kernel<128>", "w32k") is None      # another workload
    (tmp_path / "b.cuh").write_text("header b, changed")
    assert bench.measured_traffic("attn_kernel<128>", "w128k") is None      # sources changed
    os.remove(tmp_path / "a.cu")
    assert bench.measured_traffic("attn_kernel<128>", "w128k") is None      # a source is missing
