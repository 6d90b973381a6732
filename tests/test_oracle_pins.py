"""Pins for the fp64 CPU oracle: checks against what the pages and mathematics fix.

Each test ties the oracle to something other than itself: hand-worked examples of the
FlashPrefill block search (FlashPrefill skill summary page, "Stage 1: Block-Level Attention
Approximation" and "Core Concept" item 3), textbook softmax attention (numpy full-matrix form
and torch's scaled_dot_product_attention in fp64), closed forms, invariants and special cases.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _tokens(dim0, d):
    x = np.zeros((len(dim0), 1, d), np.float32)
    x[:, 0, 0] = dim0
    return synth.to_bf16_bits(x)


def _examples():
    with open(GOLD) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("ex", _examples(), ids=lambda e: e["name"][:1])
def test_worked_example_pooling_scores_ratios(ex):
    d, B = ex["d"], ex["B"]
    q, k = _tokens(ex["q_dim0"], d), _tokens(ex["k_dim0"], d)
    cu = np.array([0, len(ex["q_dim0"])], np.int32)
    qbar, kbar = oracle.pool(q, cu, B), oracle.pool(k, cu, B)
    np.testing.assert_array_equal(qbar[:, 0, 0], ex["qbar_dim0"])
    np.testing.assert_array_equal(kbar[:, 0, 0], ex["kbar_dim0"])
    assert not qbar[:, 0, 1:].any() and not kbar[:, 0, 1:].any()
    for row in ex["rows"]:
        sc, p, r = oracle.pooled_row(qbar, kbar, cu, B, 0, 0, row["i"])
        np.testing.assert_allclose(sc, row["scores"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(p, row["p"], rtol=0, atol=1e-9)
        np.testing.assert_allclose(r, [math.exp(e) for e in row["ratio_exponent"]], rtol=1e-12, atol=0)
        assert abs(p.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("ex", _examples(), ids=lambda e: e["name"][:1])
def test_worked_example_keep_sets(ex):
    d, B = ex["d"], ex["B"]
    q, k = _tokens(ex["q_dim0"], d), _tokens(ex["k_dim0"], d)
    cu = np.array([0, len(ex["q_dim0"])], np.int32)
    qbar, kbar = oracle.pool(q, cu, B), oracle.pool(k, cu, B)
    for tau, want in ex["keep"].items():
        counts, idx, _ = oracle.search(qbar, kbar, cu, B, float(tau))
        got = oracle.lists_as_sets(counts, idx, cu, B, 1)
        assert [list(got[(0, 0, i)]) for i in range(len(want))] == want, tau


def _rand(lens, hq, hkv, d=32, seed=0, scale=1.0):
    return synth.random_inputs(lens, hq, hkv, d, seed, scale)


def _all_rows(T, hq):
    tok = np.repeat(np.arange(T, dtype=np.int64), hq)
    head = np.tile(np.arange(hq, dtype=np.int32), T)
    return tok, head


def _numpy_textbook_attention(q, k, v, cu, scale):
    """Full-matrix causal softmax attention per sequence and head, fp64 (textbook form)."""
    qf, kf, vf = (synth.bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v))
    T, hq, d = qf.shape
    G = hq // kf.shape[1]
    out = np.zeros((T, hq, d))
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        L = b - a
        if L == 0:
            continue
        mask = np.tril(np.ones((L, L), bool))
        for h in range(hq):
            logits = qf[a:b, h] @ kf[a:b, h // G].T * scale
            logits = np.where(mask, logits, -np.inf)
            w = np.exp(logits - logits.max(1, keepdims=True))
            w /= w.sum(1, keepdims=True)
            out[a:b, h] = w @ vf[a:b, h // G]
    return out


@pytest.mark.parametrize("lens,hq,hkv,B", [((37,), 2, 2, 8), ((64, 1, 29), 4, 2, 16), ((130,), 4, 1, 64)])
def test_tau0_sparse_equals_textbook_dense(lens, hq, hkv, B):
    x = _rand(lens, hq, hkv)
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    d = q.shape[2]
    counts, idx, _ = oracle.search(oracle.pool(q, cu, B), oracle.pool(k, cu, B), cu, B, 0.0)
    # tau = 0 keeps every causal block
    for (s, h, i), blocks in oracle.lists_as_sets(counts, idx, cu, B, hq).items():
        assert blocks == tuple(range(i + 1))
    tok, head = _all_rows(int(cu[-1]), hq)
    o_sparse, lse = oracle.attn_rows(q, k, v, cu, B, tok, head, counts, idx)
    o_dense, _ = oracle.attn_rows(q, k, v, cu, B, tok, head)
    ref = _numpy_textbook_attention(q, k, v, cu, 1 / math.sqrt(d))
    np.testing.assert_allclose(o_sparse.reshape(ref.shape), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_dense.reshape(ref.shape), ref, rtol=0, atol=1e-12)


def test_dense_matches_torch_sdpa_fp64():
    x = _rand((96,), 4, 2, d=64, seed=3)
    q, k, v, cu = x["q"], x["k"], x["v"], x["cu_seqlens"]
    tok, head = _all_rows(96, 4)
    o, lse = oracle.attn_rows(q, k, v, cu, 32, tok, head)
    tq, tk, tv = (torch.from_numpy(synth.bf16_bits_to_f32(a).astype(np.float64)).permute(1, 0, 2) for a in (q, k, v))
    tk, tv = tk.repeat_interleave(2, 0), tv.repeat_interleave(2, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(o.reshape(ref.shape), ref, rtol=0, atol=1e-12)
    # log-sum-exp against torch.logsumexp of the masked logits
    logits = torch.einsum("htd,hsd->hts", tq, tk) / math.sqrt(64)
    logits = logits.masked_fill(~torch.ones(96, 96, dtype=torch.bool).tril(), float("-inf"))
    ref_lse = torch.logsumexp(logits, -1).permute(1, 0).numpy()
    np.testing.assert_allclose(lse.reshape(ref_lse.shape), ref_lse, rtol=0, atol=1e-12)


def test_pooled_rows_sum_to_one_and_ratio_max_is_one():
    x = synth.make_inputs(synth.WORKLOADS["mha4-L2048-B64"].with_lens([700]))
    cu, B = x["cu_seqlens"], 64
    qbar, kbar = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    for h in range(4):
        for i in (0, 1, 5, 10):
            _, p, r = oracle.pooled_row(qbar, kbar, cu, B, 0, h, i)
            assert abs(p.sum() - 1) < 1e-12 and (p >= 0).all()
            assert abs(r.max() - 1) < 1e-15


@pytest.mark.parametrize("tau", [1e-3, 0.1, 0.5, 0.99, 1.0, 5.0])
def test_sink_and_diagonal_always_kept(tau):
    x = _rand((300, 77), 4, 2, d=16, seed=5, scale=3.0)  # large scale -> peaked block softmax
    cu, B = x["cu_seqlens"], 16
    counts, idx, _ = oracle.search(oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B), cu, B, tau)
    for (s, h, i), blocks in oracle.lists_as_sets(counts, idx, cu, B, 4).items():
        assert blocks[0] == 0 and blocks[-1] == i
        assert list(blocks) == sorted(set(blocks)) and len(blocks) <= i + 1


def test_keep_sets_shrink_monotonically_with_tau():
    x = _rand((400,), 2, 1, d=16, seed=7, scale=3.0)
    cu, B = x["cu_seqlens"], 16
    qbar, kbar = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    prev = None
    for tau in (0.0, 0.01, 0.1, 0.3, 0.6, 0.9, 1.0):
        c, idx, _ = oracle.search(qbar, kbar, cu, B, tau)
        sets = {key: set(v) for key, v in oracle.lists_as_sets(c, idx, cu, B, 2).items()}
        if prev is not None:
            assert all(sets[key] <= prev[key] for key in sets)
        prev = sets
    assert sum(len(v) for v in prev.values()) < sum(i + 1 for (_, _, i) in prev)  # something dropped


def test_block_size_one_reduces_to_token_softmax_threshold():
    """B = 1: pooling is the identity, so the keep rule is the textbook token softmax test."""
    x = _rand((50,), 2, 2, d=16, seed=11, scale=2.0)
    q, k, cu = x["q"], x["k"], x["cu_seqlens"]
    tau = 0.2
    counts, idx, _ = oracle.search(oracle.pool(q, cu, 1), oracle.pool(k, cu, 1), cu, 1, tau)
    sets = oracle.lists_as_sets(counts, idx, cu, 1, 2)
    tq = torch.from_numpy(synth.bf16_bits_to_f32(q).astype(np.float64))
    tk = torch.from_numpy(synth.bf16_bits_to_f32(k).astype(np.float64))
    for h in range(2):
        logits = tq[:, h] @ tk[:, h].T / 4.0
        logits = logits.masked_fill(~torch.ones(50, 50, dtype=torch.bool).tril(), float("-inf"))
        p = torch.softmax(logits, -1)
        for i in range(50):
            want = {j for j in range(i + 1) if p[i, j] >= tau * p[i].max()} | {0, i}
            assert set(sets[(0, h, i)]) == want


def test_pool_closed_forms():
    """Mean of tokens 1..n is (n+1)/2 in every block, partial last block included."""
    L, B = 23, 8
    vals = np.concatenate([np.arange(1, 9), np.arange(1, 9), np.arange(1, 8)]).astype(np.float32)
    x = np.repeat(vals[:, None, None], 3, axis=2)  # [L, 1, 3]
    qbar = oracle.pool(synth.to_bf16_bits(x), np.array([0, L], np.int32), B)
    np.testing.assert_array_equal(qbar[:, 0, 0], [4.5, 4.5, 4.0])


def test_all_equal_keys_give_prefix_mean_of_values():
    """Equal keys -> uniform weights over visible keys -> O_t = mean of V over kept keys <= t."""
    L, d, B = 40, 8, 8
    x = _rand((L,), 1, 1, d=d, seed=13)
    k = np.tile(x["k"][:1], (L, 1, 1))
    cu = x["cu_seqlens"]
    tok, head = _all_rows(L, 1)
    o, lse = oracle.attn_rows(x["q"], k, x["v"], cu, B, tok, head)
    vf = synth.bf16_bits_to_f32(x["v"])[:, 0].astype(np.float64)
    want = np.cumsum(vf, 0) / np.arange(1, L + 1)[:, None]
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    # LSE closed form: logit + ln(t + 1)
    qf = synth.bf16_bits_to_f32(x["q"])[:, 0].astype(np.float64)
    kf = synth.bf16_bits_to_f32(k)[0, 0].astype(np.float64)
    np.testing.assert_allclose(lse, qf @ kf / math.sqrt(d) + np.log(np.arange(1, L + 1)), rtol=0, atol=1e-12)


def test_diagonal_only_mask_with_block_size_one_is_identity():
    L = 17
    x = _rand((L,), 2, 1, d=8, seed=17)
    cu = x["cu_seqlens"]
    counts = np.ones((2, L), np.int32)
    n = oracle.index_elems(cu, 1, 2)
    idx = np.zeros(n, np.int32)
    for h in range(2):
        for i in range(L):
            idx[oracle.row_offset(cu, 1, 2, 0, h, i)] = i
    tok, head = _all_rows(L, 2)
    o, lse = oracle.attn_rows(x["q"], x["k"], x["v"], cu, 1, tok, head, counts, idx)
    vf = synth.bf16_bits_to_f32(x["v"])[:, 0].astype(np.float64)
    np.testing.assert_array_equal(o.reshape(L, 2, 8), np.repeat(vf[:, None], 2, 1))


def test_lse_at_least_max_logit():
    x = _rand((70,), 2, 2, d=16, seed=19)
    cu = x["cu_seqlens"]
    tok, head = _all_rows(70, 2)
    _, lse = oracle.attn_rows(x["q"], x["k"], x["v"], cu, 16, tok, head)
    qf, kf = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in (x["q"], x["k"]))
    for r, (t, h) in enumerate(zip(tok, head)):
        assert lse[r] >= (kf[: t + 1, h] @ qf[t, h]).max() / 4.0 - 1e-12


def test_varlen_packing_equals_separate_sequences():
    lens = (45, 1, 100, 16)
    x = _rand(lens, 4, 2, d=16, seed=23, scale=2.0)
    cu, B, tau = x["cu_seqlens"], 16, 0.3
    qbar, kbar = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    counts, idx, _ = oracle.search(qbar, kbar, cu, B, tau)
    packed = oracle.lists_as_sets(counts, idx, cu, B, 4)
    tok, head = _all_rows(int(cu[-1]), 4)
    o_packed, _ = oracle.attn_rows(x["q"], x["k"], x["v"], cu, B, tok, head, counts, idx)
    o_packed = o_packed.reshape(int(cu[-1]), 4, 16)
    for s, L in enumerate(lens):
        a, b = cu[s], cu[s + 1]
        one = np.array([0, L], np.int32)
        q1, k1, v1 = x["q"][a:b], x["k"][a:b], x["v"][a:b]
        c1, i1, _ = oracle.search(oracle.pool(q1, one, B), oracle.pool(k1, one, B), one, B, tau)
        sep = oracle.lists_as_sets(c1, i1, one, B, 4)
        assert all(packed[(s, h, i)] == sep[(0, h, i)] for (_, h, i) in sep)
        t1, h1 = _all_rows(L, 4)
        o1, _ = oracle.attn_rows(q1, k1, v1, one, B, t1, h1, c1, i1)
        np.testing.assert_array_equal(o_packed[a:b], o1.reshape(L, 4, 16))


def test_gqa_equals_explicitly_repeated_kv_heads():
    x = _rand((90,), 4, 2, d=16, seed=29, scale=2.0)
    cu, B, tau = x["cu_seqlens"], 16, 0.2
    k_rep, v_rep = np.repeat(x["k"], 2, axis=1), np.repeat(x["v"], 2, axis=1)
    c1, i1, _ = oracle.search(oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B), cu, B, tau)
    c2, i2, _ = oracle.search(oracle.pool(x["q"], cu, B), oracle.pool(k_rep, cu, B), cu, B, tau)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(i1, i2)
    tok, head = _all_rows(90, 4)
    o1, _ = oracle.attn_rows(x["q"], x["k"], x["v"], cu, B, tok, head, c1, i1)
    o2, _ = oracle.attn_rows(x["q"], k_rep, v_rep, cu, B, tok, head, c2, i2)
    np.testing.assert_array_equal(o1, o2)


def test_tie_band_marks_only_blocks_near_the_threshold():
    ex = _examples()[0]
    q, k = _tokens(ex["q_dim0"], 4), _tokens(ex["k_dim0"], 4)
    cu = np.array([0, 8], np.int32)
    qbar, kbar = oracle.pool(q, cu, 2), oracle.pool(k, cu, 2)
    tau = math.exp(-1)  # exactly the ratio of block 3 in row 3 -> inside the band
    counts, idx, band = oracle.search(qbar, kbar, cu, 2, tau)
    row3 = oracle.row_offset(cu, 2, 1, 0, 0, 3)
    assert list(band[row3:row3 + 4]) == [0, 0, 0, 1]
    _, _, band2 = oracle.search(qbar, kbar, cu, 2, 0.25)
    assert not band2.any()


def test_index_layout_offsets():
    cu = np.array([0, 300, 301, 700], np.int32)
    B, hq = 64, 3
    nbs = [5, 1, 7]
    assert oracle.total_blocks(cu, B) == sum(nbs)
    assert oracle.index_elems(cu, B, hq) == sum(hq * n * (n + 1) // 2 for n in nbs)
    assert oracle.row_offset(cu, B, hq, 2, 1, 3) == hq * 15 + hq * 1 + 1 * 28 + 6


def test_generator_is_deterministic_and_structured():
    w = synth.WORKLOADS["mha4-L2048-B64"]
    a, b = synth.make_inputs(w), synth.make_inputs(w)
    for key in ("q", "k", "v"):
        np.testing.assert_array_equal(a[key], b[key])
    with open(os.path.join(os.path.dirname(__file__), "golden", "synth_sha256.json")) as f:
        want = json.load(f)["mha4-L2048-B64"]
    import hashlib
    for key in ("q", "k", "v"):
        assert hashlib.sha256(a[key].tobytes()).hexdigest() == want[key], key
