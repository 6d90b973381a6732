"""GPU attention on hand-made index lists whose item patterns drive every path of the kernel's item
pipeline: a unit pairs two rows of one kv-head, and the two rows' lists decide which items are
shared, which belong to one slot only, and how long a run of one slot's items is (the MMA issue
order differs for each). Logits that jump half-way along the key axis make the running max rise
by more than the lazy-rescale margin inside those runs, so O is rescaled between items of a run.

The lists are valid method outputs in form (ascending, sink and diagonal present) but are chosen
here, not by the search; the oracle attends exactly the same blocks. Each case runs under both
attention schedules (FP_ATTN_UNITS): tile pairs, and single tiles whose two softmax warpgroups split
every item's keys (plain B = 128; with B = 64 both runs take the pairs).
"""
import numpy as np
import pytest

import synth
from helpers import bf16_to_np, compare_attention, to_dev

pytestmark = pytest.mark.gpu


def _lists(nb, hq, B, dens_odd, dens_even, rng):
    """Triangular index lists (row (h, i) at h*nb*(nb+1)/2 + i*(i+1)/2): query blocks in odd and even
    128-row tiles get different keep densities, so adjacent rows differ in length and order."""
    per = 128 // B
    counts = np.zeros((hq, nb), np.int32)
    idx = np.zeros(hq * nb * (nb + 1) // 2, np.int32)
    for h in range(hq):
        for i in range(nb):
            dens = dens_odd if (i // per) % 2 else dens_even
            keep = [j for j in range(1, i) if rng.random() < dens]
            row = sorted(set([0, i] + keep))
            base = h * nb * (nb + 1) // 2 + i * (i + 1) // 2
            idx[base: base + len(row)] = row
            counts[h, i] = len(row)
    return counts, idx


@pytest.mark.parametrize("L,hq,hkv,B,dens_odd,dens_even,step", [
    (4096, 4, 2, 128, 0.9, 0.1, 47.0),    # long runs of the odd tile's slot, a jump in the logits
    (4096, 4, 2, 128, 0.1, 0.9, 47.0),    # the same with the slots swapped
    (3000, 2, 1, 128, 0.5, 0.5, 47.0),    # random interleavings
    (2944, 6, 2, 128, 0.7, 0.2, 0.0),     # G = 3, odd tile count: one-slot units run alone
    (2048, 4, 2, 64, 0.8, 0.15, 47.0),    # B = 64: two lists per slot
])
@pytest.mark.parametrize("units", ["pairs", "rows"])
def test_attention_on_item_patterns(L, hq, hkv, B, dens_odd, dens_even, step, units, monkeypatch):
    import torch
    import block_sparse_long_causal_b200 as fp
    monkeypatch.setenv("FP_ATTN_UNITS", units)  # rows: the single-tile schedule (B = 128 only)
    rng = np.random.default_rng(L + 7 * hq + B)
    x = synth.random_inputs((L,), hq, hkv, 128, seed=L + hq, scale=1.0)
    if step:
        # a shared direction carried by every query and, from the middle of the sequence on, by the
        # keys with weight `step`: a query's logits jump by about 2 * step / sqrt(d) = 8.3 (12 in
        # log2 units) at the middle, so rows of the second half see their running max grow by more
        # than the kernel's lazy-rescale margin (8 in log2 units) inside their lists, while their
        # softmax still spreads over hundreds of keys
        d = np.zeros(128, np.float32)
        d[:8] = 1.0 / np.sqrt(8.0)
        q32 = synth.bf16_bits_to_f32(x["q"]).copy()
        k32 = synth.bf16_bits_to_f32(x["k"]).copy()
        q32 += 2.0 * d
        k32[L // 2:] += step * d
        x = dict(x, q=synth.to_bf16_bits(q32), k=synth.to_bf16_bits(k32))
    nb = (L + B - 1) // B
    counts, idx = _lists(nb, hq, B, dens_odd, dens_even, rng)
    cu = x["cu_seqlens"]
    p = fp.problem(cu, hq, hkv, 128, B)
    out = torch.empty((L, hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((hq, L), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp.block_sparse_attn(p, to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]), to_dev(counts), to_dev(idx), 0.0,
                         out, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    res = {"counts": counts, "indices": idx, "out": bf16_to_np(out), "lse": lse.cpu().numpy()}
    compare_attention(x, res, hq, B)
