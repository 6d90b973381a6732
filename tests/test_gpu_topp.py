"""The cumulative top-p comparison selector on the GPU (fp_block_search_topp) against the oracle's
top-p selection: lists bit-exact outside the tie band (the decision mass within 1e-4 of gamma, or a
near-tie at the cut), on the same pooled tensors."""
import numpy as np
import pytest

import oracle
import synth
from helpers import check_lists_valid, keep_mask, to_dev

pytestmark = pytest.mark.gpu


def gpu_topp(x, hq, hkv, B, gamma):
    import torch
    import block_sparse_long_causal_b200 as fp
    p = fp.problem(x["cu_seqlens"], hq, hkv, 128, B)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    nb = max(p.total_blocks, 1)
    q_pool = torch.empty((nb, hq, 128), dtype=torch.float32, device="cuda")
    k_pool = torch.empty((nb, hkv, 128), dtype=torch.float32, device="cuda")
    scores = torch.empty(max(p.index_elems, 1), dtype=torch.float32, device="cuda")
    counts = torch.zeros((hq, nb), dtype=torch.int32, device="cuda")
    indices = torch.full((max(p.index_elems, 1),), -3, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp.block_pool(p, q, k, q_pool, k_pool)
    fp.block_search_topp(p, q_pool, k_pool, gamma, scores, counts, indices, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return counts[:, : p.total_blocks].cpu().numpy(), indices[: p.index_elems].cpu().numpy()


def check(x, hq, hkv, B, gamma):
    cu = x["cu_seqlens"]
    g_counts, g_idx = gpu_topp(x, hq, hkv, B, gamma)
    check_lists_valid(g_counts, g_idx, cu, B, hq)
    qbar, kbar = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    o_counts, o_idx, o_band = oracle.search_topp(qbar, kbar, cu, B, gamma)
    mg = keep_mask(g_counts, g_idx, cu, B, hq)
    mo = keep_mask(o_counts, o_idx, cu, B, hq)
    outside = (mg != mo) & (o_band == 0)
    assert not outside.any(), f"{int(outside.sum())} entries differ outside the tie band"
    return float(mo.mean())


@pytest.mark.parametrize("lens,hq,hkv,B,gamma", [
    ((700, 300), 4, 2, 64, 0.5),
    ((700, 300), 4, 2, 128, 0.9),
    ((1500,), 6, 2, 64, 0.95),
    ((900, 1, 257), 4, 4, 64, 0.99),
])
def test_topp_matches_the_oracle(lens, hq, hkv, B, gamma):
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + hq, scale=3.0)
    density = check(x, hq, hkv, B, gamma)
    assert 0.0 < density <= 1.0


def test_topp_edges_keep_forced_or_all():
    x = synth.random_inputs((500,), 4, 2, 128, seed=9, scale=3.0)
    for gamma in (0.0, -0.5, 1.0, 3.0):
        check(x, 4, 2, 64, gamma)


def test_topp_on_the_structured_workload():
    w = synth.WORKLOADS["mha4-L2048-B64"]
    x = synth.make_inputs(w)
    check(x, w.hq, w.hkv, w.block, 0.9)


def test_topp_rows_longer_than_the_register_path():
    """Rows of more than 1024 blocks take the path that re-reads the scores from memory."""
    x = synth.random_inputs((68000,), 2, 1, 128, seed=13, scale=3.0)
    check(x, 2, 1, 64, 0.9)
