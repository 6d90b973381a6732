"""GPU parity at the full workload sizes, in the launch configuration the benchmark times.

Index lists: the whole list set against the oracle's full search (bit-exact outside the tie band).
Attention: sampled (token, head) rows recomputed one by one by the oracle on the GPU's own lists
(first and last token of every sequence plus seeded random rows).
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import compare_attention, compare_lists, gpu_prefill, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run(w, tau, nrows=96, seed=0):
    x = synth.make_inputs(w)
    res = gpu_prefill(x, w.hq, w.hkv, w.block, tau, with_lse=True)
    cu = x["cu_seqlens"]
    qb, kb = oracle.pool(x["q"], cu, w.block), oracle.pool(x["k"], cu, w.block)
    np.testing.assert_allclose(res["k_pool"], kb, rtol=0, atol=5e-5)
    oc, oi, band = oracle.search(qb, kb, cu, w.block, tau)
    nband, nkept = compare_lists(res["counts"], res["indices"], oc, oi, band, cu, w.block, w.hq)
    rows = sample_rows(cu, w.hq, nrows, seed)
    st = compare_attention(x, res, w.hq, w.block, *rows)
    assert st["rel"] <= 2e-2, st
    return st, nkept


@pytest.mark.parametrize("name", ["llama3-8b-L131072", "llama3-8b-L262144", "llama3-8b-varlen8-T264192"])
def test_full_workload(name):
    w = synth.WORKLOADS[name]
    _run(w, w.tau)


def test_full_128k_supplementary_sparse_tau():
    """Same 128K workload at tau = 0.95 (a labelled supplementary setting with real sparsity)."""
    w = synth.WORKLOADS["llama3-8b-L131072"]
    st, nkept = _run(w, 0.95, nrows=64, seed=3)
    causal = w.hq * (1024 * 1025 // 2)
    assert nkept < 0.9 * causal
