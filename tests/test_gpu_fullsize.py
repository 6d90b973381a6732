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


def test_full_128k_fp8_attention():
    """FP8 (e4m3 Q and K, per-tensor scales, bf16 V) at 128K on the GPU's own lists: sampled rows
    against the exact attention of the dequantised inputs."""
    import torch
    import block_sparse_long_causal_b200 as fp
    w = synth.WORKLOADS["llama3-8b-L131072"]
    x = synth.make_inputs(w)
    res = gpu_prefill(x, w.hq, w.hkv, w.block, w.tau, with_lse=False)
    cu = x["cu_seqlens"]
    q32, k32 = synth.bf16_bits_to_f32(x["q"]), synth.bf16_bits_to_f32(x["k"])
    qs, ks = float(np.abs(q32).max()) / 448.0, float(np.abs(k32).max()) / 448.0
    qc, kc = synth.to_e4m3_bits(q32 / qs), synth.to_e4m3_bits(k32 / ks)
    del q32, k32
    p = fp.problem(cu, w.hq, w.hkv, 128, w.block)
    out = torch.empty((p.total_tokens, w.hq, 128), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    from helpers import bf16_to_np, to_dev
    fp.block_sparse_attn_fp8(p, torch.from_numpy(qc).cuda(), torch.from_numpy(kc).cuda(), to_dev(x["v"]), qs, ks,
                             torch.from_numpy(res["counts"]).cuda().contiguous(),
                             torch.from_numpy(res["indices"]).cuda().contiguous(), 0.0, out, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got_all = bf16_to_np(out)
    rows_tok, rows_head = sample_rows(cu, w.hq, 96, 5)
    qd = synth.to_bf16_bits(synth.e4m3_bits_to_f32(qc))
    kd = synth.to_bf16_bits(synth.e4m3_bits_to_f32(kc))
    o_ref, _ = oracle.attn_rows(qd, kd, x["v"], cu, w.block, rows_tok, rows_head, res["counts"], res["indices"],
                                scale=qs * ks / np.sqrt(128.0))
    got = synth.bf16_bits_to_f32(got_all[rows_tok, rows_head]).astype(np.float64)
    err = np.abs(got - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())


def test_full_128k_topp_selector():
    """The cumulative top-p comparison selector at 128K: every list against the oracle's top-p."""
    import torch
    import block_sparse_long_causal_b200 as fp
    from helpers import keep_mask, to_dev
    w = synth.WORKLOADS["llama3-8b-L131072"]
    x = synth.make_inputs(w)
    cu = x["cu_seqlens"]
    p = fp.problem(cu, w.hq, w.hkv, 128, w.block)
    sp = fp.SparsePrefill(p)
    fp.block_pool(p, to_dev(x["q"]), to_dev(x["k"]), sp.q_pool, sp.k_pool)
    scores = torch.empty(p.index_elems, dtype=torch.float32, device="cuda")
    fp.block_search_topp(p, sp.q_pool, sp.k_pool, 0.95, scores, sp.counts, sp.indices, sp.dev_status)
    torch.cuda.synchronize()
    assert int(sp.dev_status.item()) == 0
    g_counts = sp.counts[:, : p.total_blocks].cpu().numpy()
    g_idx = sp.indices[: p.index_elems].cpu().numpy()
    qb, kb = oracle.pool(x["q"], cu, w.block), oracle.pool(x["k"], cu, w.block)
    o_counts, o_idx, o_band = oracle.search_topp(qb, kb, cu, w.block, 0.95)
    mg = keep_mask(g_counts, g_idx, cu, w.block, w.hq)
    mo = keep_mask(o_counts, o_idx, cu, w.block, w.hq)
    assert not ((mg != mo) & (o_band == 0)).any()
    assert mo.mean() < 0.99  # a real selection


def test_full_32k_chunk_after_24k_cached_prefix_in_pages():
    """Chunked prefill at the 32K workload shape: the last 8K tokens as a chunk after a 24K cached
    prefix held in randomly permuted pages; lists against the full prefill's rows (whole set),
    attention on sampled rows."""
    import torch
    import block_sparse_long_causal_b200 as fp
    from helpers import bf16_to_np, to_dev
    w = synth.WORKLOADS["llama3-8b-L32768"]
    x = synth.make_inputs(w)
    cu_full = x["cu_seqlens"]
    L, P, B, ps, hq, hkv = int(cu_full[-1]), 24576, w.block, 512, w.hq, w.hkv
    rng = np.random.default_rng(4)
    need = L // ps
    num_pages = need + 5
    perm = rng.permutation(num_pages)
    kc = np.zeros((num_pages * ps, hkv, 128), np.uint16)
    vc = np.zeros_like(kc)
    table = np.zeros((1, need), np.int32)
    for n in range(need):
        table[0, n] = perm[n]
        kc[perm[n] * ps:(perm[n] + 1) * ps] = x["k"][n * ps:(n + 1) * ps]
        vc[perm[n] * ps:(perm[n] + 1) * ps] = x["v"][n * ps:(n + 1) * ps]
    p = fp.problem(np.array([0, L - P], np.int32), hq, hkv, 128, B)
    c = fp.paged_cache(p, [P], table, ps, num_pages)
    q = to_dev(x["q"][P:])
    nb = p.total_blocks
    q_pool = torch.empty((nb, hq, 128), dtype=torch.float32, device="cuda")
    k_pool = torch.empty((c.total_kv_blocks, hkv, 128), dtype=torch.float32, device="cuda")
    counts = torch.zeros((hq, nb), dtype=torch.int32, device="cuda")
    indices = torch.zeros(c.index_elems, dtype=torch.int32, device="cuda")
    out = torch.empty((L - P, hq, 128), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kcd, vcd = to_dev(kc), to_dev(vc)
    fp.paged_block_pool(p, c, q, kcd, q_pool, k_pool)
    tau = 0.9  # a selective threshold on this workload (the list check is then non-trivial)
    fp.paged_block_search(p, c, q_pool, k_pool, tau, counts, indices, st)
    fp.paged_block_sparse_attn(p, c, q, kcd, vcd, counts, indices, 0.0, out, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g_counts, g_idx, got_all = counts.cpu().numpy(), indices.cpu().numpy(), bf16_to_np(out)
    qb, kb = oracle.pool(x["q"], cu_full, B), oracle.pool(x["k"], cu_full, B)
    o_counts, o_idx, o_band = oracle.search(qb, kb, cu_full, B, tau)
    pb, nbf = P // B, L // B
    full_counts = np.zeros_like(o_counts)
    full_idx = np.zeros_like(o_idx)
    for h in range(hq):
        for i_abs in range(nbf):
            off = oracle.row_offset(cu_full, B, hq, 0, h, i_abs)
            if i_abs < pb:
                full_counts[h, i_abs] = i_abs + 1
                full_idx[off: off + i_abs + 1] = np.arange(i_abs + 1)
                continue
            i = i_abs - pb
            n = int(g_counts[h, i])
            start = h * (nb * pb + nb * (nb + 1) // 2) + i * pb + i * (i + 1) // 2
            got = g_idx[start: start + n]
            want = set(o_idx[off: off + int(o_counts[h, i_abs])].tolist())
            for j in set(got.tolist()) ^ want:
                assert o_band[off + j], (h, i, j)
            full_counts[h, i_abs] = n
            full_idx[off: off + n] = got
    rows_tok = np.concatenate([[P, L - 1], rng.integers(P, L, 62)]).astype(np.int64)
    rows_head = rng.integers(0, hq, len(rows_tok)).astype(np.int32)
    o_ref, _ = oracle.attn_rows(x["q"], x["k"], x["v"], cu_full, B, rows_tok, rows_head, full_counts, full_idx)
    got = synth.bf16_bits_to_f32(got_all[rows_tok - P, rows_head]).astype(np.float64)
    err = np.abs(got - o_ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
