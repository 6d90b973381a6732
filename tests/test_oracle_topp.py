"""Pins of the oracle's cumulative top-p block selector (the comparison selector).

FlashPrefill skill summary page, "The Problem": Top-k / Top-p selection needs score computation,
sorting and cumulative sums; FlexPrefill abstract, "Cumulative-Attention Based Index Selection":
keep the indexes whose attention scores sum to a preset threshold. Reading: on the pooled causal
softmax p of a row, keep the most probable blocks until their mass reaches gamma (blocks tied at
the cut together), plus the sink block 0 and the diagonal block i as in the threshold search.
"""
import numpy as np
import pytest

import oracle
import synth

D = 128


def _row_problem(weights):
    """One sequence, B = 1, one head: q-bar of the last block and k-bars chosen so that the scores of
    the last row are log(weights) (q = sqrt(d) e_0, k_j = log(w_j) e_0); earlier rows are unused."""
    n = len(weights)
    qbar = np.zeros((n, 1, D))
    kbar = np.zeros((n, 1, D))
    qbar[:, 0, 0] = np.sqrt(D)
    kbar[:, 0, 0] = np.log(np.asarray(weights, np.float64))
    cu = np.array([0, n], np.int32)
    return qbar, kbar, cu


def _last_row(counts, indices, n):
    start = (n - 1) * n // 2
    return indices[start: start + counts[0, n - 1]].tolist()


# Hand-worked rows. p = w / sum(w); blocks ranked by p (largest first) until the mass reaches gamma.
#   w = [0.05, 0.5, 0.3, 0.1, 0.05]: ranking j1 (0.5), j2 (0.3), j3 (0.1), then j0, j4 (0.05 each)
#     gamma 0.79: j1 (D=0), j2 (D=0.5) kept; j3 has D = 0.8 >= 0.79, dropped -> {0, 1, 2, 4}
#     gamma 0.81: j3 has D = 0.8 < 0.81, kept; j0/j4 have D = 0.9 -> dropped but forced -> all
#     gamma 0.45: only j1 (D = 0) -> {0, 1, 4};  gamma 0: forced only -> {0, 4}
#   w = [0.1, 0.3, 0.3, 0.2, 0.1], gamma 0.35: j1 and j2 tie at the top (D = 0 for both) -> kept
#     together; j3 has D = 0.6 -> dropped -> {0, 1, 2, 4}
WORKED = [
    ([0.05, 0.5, 0.3, 0.1, 0.05], 0.79, [0, 1, 2, 4]),
    ([0.05, 0.5, 0.3, 0.1, 0.05], 0.81, [0, 1, 2, 3, 4]),
    ([0.05, 0.5, 0.3, 0.1, 0.05], 0.45, [0, 1, 4]),
    ([0.05, 0.5, 0.3, 0.1, 0.05], 0.0, [0, 4]),
    ([0.1, 0.3, 0.3, 0.2, 0.1], 0.35, [0, 1, 2, 4]),
    ([0.1, 0.3, 0.3, 0.2, 0.1], 1.0, [0, 1, 2, 3, 4]),
]


@pytest.mark.parametrize("w,gamma,want", WORKED)
def test_worked_rows(w, gamma, want):
    qbar, kbar, cu = _row_problem(w)
    counts, indices, _ = oracle.search_topp(qbar, kbar, cu, 1, gamma)
    assert _last_row(counts, indices, len(w)) == want


def _numpy_topp(p, gamma, i):
    """Token-level top-p by sort + cumulative sum (numpy), ties at the cut kept, plus {0, i}."""
    order = np.argsort(-p, kind="stable")
    cums = np.cumsum(p[order])
    if gamma >= 1.0:
        keep = set(range(i + 1))
    elif gamma <= 0.0:
        keep = set()
    else:
        k = int(np.searchsorted(cums, gamma, side="left"))  # first position whose cumulative >= gamma
        cut = p[order[min(k, len(p) - 1)]]
        keep = set(np.nonzero(p >= cut)[0].tolist())
    return sorted(keep | {0, i})


@pytest.mark.parametrize("gamma", [0.3, 0.7, 0.9, 0.97])
def test_block_size_one_is_token_level_top_p(gamma):
    """B = 1: pooling is the identity and the rows are token-level causal softmax rows."""
    x = synth.random_inputs((48,), 2, 1, D, seed=21, scale=2.0)
    cu = x["cu_seqlens"]
    qbar, kbar = oracle.pool(x["q"], cu, 1), oracle.pool(x["k"], cu, 1)
    counts, indices, band = oracle.search_topp(qbar, kbar, cu, 1, gamma)
    q = synth.bf16_bits_to_f32(x["q"]).astype(np.float64)
    k = synth.bf16_bits_to_f32(x["k"]).astype(np.float64)
    for h in range(2):
        for i in range(48):
            s = k[: i + 1, 0] @ q[i, h] / np.sqrt(D)
            p = np.exp(s - s.max())
            p /= p.sum()
            start = h * 48 * 49 // 2 + i * (i + 1) // 2
            got = set(indices[start: start + counts[h, i]].tolist())
            want = set(_numpy_topp(p, gamma, i))
            for j in got ^ want:
                assert band[start + j], (h, i, j)


def test_invariants_on_random_rows():
    x = synth.random_inputs((700, 300), 4, 2, D, seed=5, scale=3.0)
    cu, B = x["cu_seqlens"], 64
    qbar, kbar = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    sets = {}
    for gamma in (-1.0, 0.0, 0.5, 0.8, 0.95, 1.0, 2.0):
        c, idx, _ = oracle.search_topp(qbar, kbar, cu, B, gamma, want_band=False)
        sets[gamma] = oracle.lists_as_sets(c, idx, cu, B, 4)
    for (s, h, i), kept in sets[0.0].items():
        assert kept == tuple(sorted({0, i}))                     # gamma <= 0: forced blocks only
        assert sets[-1.0][(s, h, i)] == kept
        assert sets[1.0][(s, h, i)] == tuple(range(i + 1))       # gamma >= 1: every causal block
        assert sets[2.0][(s, h, i)] == tuple(range(i + 1))
        for a, b in ((0.5, 0.8), (0.8, 0.95), (0.95, 1.0)):      # monotone in gamma
            assert set(sets[a][(s, h, i)]) <= set(sets[b][(s, h, i)])
    # the kept mass reaches gamma, and dropping the least probable unforced kept block (when it is
    # not tied) falls below it: the set is the smallest one
    gamma = 0.8
    for (s, h, i), kept in sets[gamma].items():
        if i < 3:
            continue
        _, p, _ = oracle.pooled_row(qbar, kbar, cu, B, s, h, i)
        assert p[list(kept)].sum() >= gamma - 1e-12
        free = [j for j in kept if j not in (0, i)]
        if free:
            jmin = min(free, key=lambda j: p[j])
            ties = [j for j in range(i + 1) if j != jmin and abs(p[j] - p[jmin]) <= 1e-12]
            if not ties:
                top = sorted(range(i + 1), key=lambda j: -p[j])
                rank = top.index(jmin)
                assert p[top[:rank]].sum() < gamma
