"""Shared helpers for the parity tests: GPU runs through the C ABI and list/output comparisons
against the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle

# Tolerances of the attention output for bf16 I/O with fp32 accumulation (stated for the method's
# problem: max-abs 2e-2, mean-abs 2e-3 against the exact fp64 result on the same block mask).
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3


def to_dev(a: np.ndarray, device="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_to_np(t) -> np.ndarray:
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def row_offsets(cu, B, hq):
    """Triangular offset of every row, ordered [h, global block] like the counts tensor."""
    cu = np.asarray(cu, np.int64)
    nbs = (np.diff(cu) + B - 1) // B
    base = 0
    per_seq = []
    for s, nb in enumerate(nbs):
        i = np.arange(nb, dtype=np.int64)
        per_seq.append((base, nb, i))
        base += hq * nb * (nb + 1) // 2
    out = np.zeros((hq, int(nbs.sum())), np.int64)
    gb = 0
    for (b0, nb, i) in per_seq:
        for h in range(hq):
            out[h, gb:gb + nb] = b0 + h * nb * (nb + 1) // 2 + i * (i + 1) // 2
        gb += nb
    return out


def row_blocks(cu, B, hq):
    """Local block id i of every row, [h, global block]."""
    cu = np.asarray(cu, np.int64)
    nbs = (np.diff(cu) + B - 1) // B
    loc = np.concatenate([np.arange(n) for n in nbs]) if len(nbs) else np.zeros(0, np.int64)
    return np.tile(loc, (hq, 1))


def keep_mask(counts, indices, cu, B, hq):
    """Dense triangular keep mask (same layout as the index buffer) decoded from lists."""
    offs = row_offsets(cu, B, hq).ravel()
    c = np.asarray(counts, np.int64).ravel()
    n = int(c.sum())
    starts = np.repeat(offs, c)
    within = np.arange(n) - np.repeat(np.cumsum(c) - c, c)
    vals = np.asarray(indices)[starts + within].astype(np.int64)
    mask = np.zeros(len(indices), np.uint8)
    mask[starts + vals] = 1
    return mask


def check_lists_valid(counts, indices, cu, B, hq):
    """Every row: count in [1, i+1], ascending, in [0, i], starts with 0, ends with i."""
    offs = row_offsets(cu, B, hq).ravel()
    ib = row_blocks(cu, B, hq).ravel()
    c = np.asarray(counts, np.int64).ravel()
    assert (c >= 1).all() and (c <= ib + 1).all(), "count out of range"
    n = int(c.sum())
    starts = np.repeat(offs, c)
    within = np.arange(n) - np.repeat(np.cumsum(c) - c, c)
    vals = np.asarray(indices)[starts + within].astype(np.int64)
    rowi = np.repeat(ib, c)
    assert (vals >= 0).all() and (vals <= rowi).all(), "entry out of range"
    first = within == 0
    last = within == np.repeat(c, c) - 1
    assert (vals[first] == 0).all(), "sink block missing"
    assert (vals[last] == rowi[last]).all(), "diagonal block missing"
    asc = vals[1:] > vals[:-1]
    assert asc[~first[1:]].all(), "entries not ascending"


def compare_lists(g_counts, g_idx, o_counts, o_idx, o_band, cu, B, hq):
    """Bit-exact list parity outside the tie band. Returns (#band disagreements, #kept)."""
    check_lists_valid(g_counts, g_idx, cu, B, hq)
    mg = keep_mask(g_counts, g_idx, cu, B, hq)
    mo = keep_mask(o_counts, o_idx, cu, B, hq)
    diff = mg != mo
    outside = diff & (o_band == 0)
    if outside.any():
        where = np.nonzero(outside)[0][:10]
        raise AssertionError(f"{int(outside.sum())} list entries differ outside the tie band, e.g. at {where}")
    return int(diff.sum()), int(mo.sum())


def gpu_prefill(x, hq, hkv, B, tau, dense=False, with_lse=True, check_status=True, fused=True):
    """Run pool + search + sparse (or dense) attention through the C ABI on cuda:0.

    fused=True uses the one-call fp_block_pool_search; fused=False calls fp_block_pool and
    fp_block_search separately."""
    import torch
    import block_sparse_long_causal_b200 as fp
    cu = x["cu_seqlens"]
    p = fp.problem(cu, hq, hkv, 128, B)
    sp = fp.SparsePrefill(p, with_lse=with_lse)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sp.search(q, k, tau, fused=fused)
    if dense:
        sp.dense(q, k, v)
    else:
        sp.attend(q, k, v)
    torch.cuda.synchronize()
    res = {
        "q_pool": sp.q_pool[: p.total_blocks].cpu().numpy(),
        "k_pool": sp.k_pool[: p.total_blocks].cpu().numpy(),
        "counts": sp.counts[:, : p.total_blocks].cpu().numpy(),
        "indices": sp.indices[: p.index_elems].cpu().numpy(),
        "out": bf16_to_np(sp.out[: p.total_tokens]),
        "lse": sp.lse[:, : p.total_tokens].cpu().numpy() if with_lse else None,
        "status": int(sp.dev_status.item()),
    }
    if check_status:
        assert res["status"] == 0, f"dev_status = {res['status']}"
    return res


def sample_rows(cu, hq, n, seed):
    """Seeded (token, head) sample: first/last token of every sequence plus n random rows."""
    rng = np.random.default_rng(seed)
    cu = np.asarray(cu, np.int64)
    toks = []
    for s in range(len(cu) - 1):
        if cu[s + 1] > cu[s]:
            toks += [cu[s], cu[s + 1] - 1]
    T = int(cu[-1])
    toks += list(rng.integers(0, T, n))
    toks = np.array(toks, np.int64)
    heads = rng.integers(0, hq, len(toks)).astype(np.int32)
    return toks, heads


def compare_attention(x, res, hq, B, rows_tok=None, rows_head=None, lists=True):
    """Oracle attention on the GPU's own lists vs the GPU output (selected rows or all rows)."""
    T = x["q"].shape[0]
    if rows_tok is None:
        rows_tok = np.repeat(np.arange(T, dtype=np.int64), hq)
        rows_head = np.tile(np.arange(hq, dtype=np.int32), T)
    counts = res["counts"] if lists else None
    idx = res["indices"] if lists else None
    o_ref, lse_ref = oracle.attn_rows(x["q"], x["k"], x["v"], x["cu_seqlens"], B, rows_tok, rows_head, counts, idx)
    got = bf16_to_f32_rows(res["out"], rows_tok, rows_head)
    err = np.abs(got - o_ref)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    rel = float(np.linalg.norm(got - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
    assert max_abs <= ATOL_MAX, f"max-abs {max_abs}"
    assert mean_abs <= ATOL_MEAN, f"mean-abs {mean_abs}"
    out = {"max_abs": max_abs, "mean_abs": mean_abs, "rel": rel}
    if res.get("lse") is not None:
        lse_got = res["lse"][rows_head, rows_tok].astype(np.float64)
        out["lse_max_abs"] = float(np.abs(lse_got - lse_ref).max())
        assert out["lse_max_abs"] <= 1e-2, f"lse max-abs {out['lse_max_abs']}"
    return out


def bf16_to_f32_rows(out_bits, rows_tok, rows_head):
    from synth import bf16_bits_to_f32
    return bf16_bits_to_f32(out_bits[rows_tok, rows_head]).astype(np.float64)
