"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Index lists: bit-exact outside the tie band (|p/max p - tau| <= 1e-4 tau).
Attention: oracle on the GPU's own lists; max-abs <= 2e-2, mean-abs <= 2e-3 (bf16 I/O, fp32
accumulation), plus a relative L2 error bound of 2e-2 so that real bugs are not hidden by the small
magnitude of long-context outputs.
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
    import block_sparse_long_causal_b200  # noqa: F401  (fails loudly without libfp.so)


def _oracle_lists(x, B, tau):
    cu = x["cu_seqlens"]
    qb, kb = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    return qb, kb, oracle.search(qb, kb, cu, B, tau)


def _check_case(x, hq, hkv, B, tau, rows=None, rel_max=2e-2, fused=True):
    res = gpu_prefill(x, hq, hkv, B, tau, fused=fused)
    qb, kb, (oc, oi, band) = _oracle_lists(x, B, tau)
    np.testing.assert_allclose(res["q_pool"], qb, rtol=0, atol=5e-5)
    np.testing.assert_allclose(res["k_pool"], kb, rtol=0, atol=5e-5)
    nband, nkept = compare_lists(res["counts"], res["indices"], oc, oi, band, x["cu_seqlens"], B, hq)
    if rows is None:
        st = compare_attention(x, res, hq, B)
    else:
        st = compare_attention(x, res, hq, B, *rows)
    assert st["rel"] <= rel_max, st
    return res, st, nkept


SMALL = [
    # (lens, hq, hkv, B, tau, scale)
    ((128,), 1, 1, 128, 0.1, 1.0),
    ((300,), 2, 1, 128, 0.5, 3.0),
    ((1,), 1, 1, 128, 0.1, 1.0),
    ((1000,), 4, 2, 128, 0.9, 3.0),
    ((257, 1, 130, 640), 8, 2, 128, 0.7, 3.0),
    ((513,), 4, 4, 64, 0.5, 3.0),
    ((64, 65, 127, 191), 4, 1, 64, 0.8, 3.0),
    ((2048,), 8, 1, 128, 0.0, 1.0),
    ((900, 385), 6, 2, 128, 0.6, 3.0),      # G = 3: units pair query tiles of one head
    ((1000, 129), 3, 1, 64, 0.7, 3.0),      # G = 3 with B = 64 (four lists per unit)
    ((513,), 2, 2, 128, 0.3, 3.0),          # G = 1, odd tile count (last unit runs one slot)
    # edge cases of the method
    ((1000,), 4, 2, 128, 1.0, 3.0),         # tau = 1: argmax ties, sink and diagonal only
    ((700, 300), 4, 2, 128, 5.0, 3.0),      # tau > 1: sink and diagonal only
    ((700, 129), 4, 2, 64, -1.0, 3.0),      # tau < 0: every causal block
    ((700, 0, 500), 4, 2, 128, 0.5, 3.0),   # a zero-length sequence inside a packed batch
    ((0, 400, 0), 4, 1, 64, 0.6, 1.0),      # zero-length sequences at both ends
    ((1000, 300), 16, 2, 64, 0.7, 1.0),     # G = 8 with B = 64
    ((2000,), 16, 2, 64, 0.95, 1.0),        # G = 8 with B = 64, sparse threshold
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"L{'-'.join(map(str, c[0]))}_h{c[1]}x{c[2]}_B{c[3]}_t{c[4]}")
def test_small_ragged_cases(case):
    lens, hq, hkv, B, tau, scale = case
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + hq, scale=scale)
    _check_case(x, hq, hkv, B, tau)


@pytest.mark.parametrize("tau", [0.1, 0.95, 0.98])
def test_mha4_L2048_B64(tau):
    w = synth.WORKLOADS["mha4-L2048-B64"]
    x = synth.make_inputs(w)
    _check_case(x, w.hq, w.hkv, w.block, tau)


@pytest.mark.parametrize("case", [SMALL[1], SMALL[4], SMALL[6], SMALL[8]],
                         ids=["L300", "varlen", "B64-varlen", "G3"])
def test_unfused_pool_then_search(case):
    """fp_block_pool and fp_block_search called separately (the two steps) against the oracle."""
    lens, hq, hkv, B, tau, scale = case
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + hq, scale=scale)
    _check_case(x, hq, hkv, B, tau, fused=False)


def test_dense_matches_oracle_dense():
    w = synth.WORKLOADS["mha4-L2048-B64"]
    x = synth.make_inputs(w.with_lens([1500]))
    res = gpu_prefill(x, w.hq, w.hkv, w.block, w.tau, dense=True)
    st = compare_attention(x, res, w.hq, w.block, lists=False)
    assert st["rel"] <= 2e-2


def test_dense_equals_sparse_at_tau0_bitwise():
    w = synth.WORKLOADS["llama3-8b-L32768"]
    x = synth.make_inputs(w.with_lens([3000, 700]))
    a = gpu_prefill(x, w.hq, w.hkv, w.block, 0.0, dense=False)
    b = gpu_prefill(x, w.hq, w.hkv, w.block, 0.0, dense=True)
    np.testing.assert_array_equal(a["out"], b["out"])


@pytest.mark.parametrize("tau", [0.1, 0.95])
def test_llama3_8b_L32768(tau):
    w = synth.WORKLOADS["llama3-8b-L32768"]
    x = synth.make_inputs(w)
    rows = sample_rows(x["cu_seqlens"], w.hq, 192, seed=1)
    _check_case(x, w.hq, w.hkv, w.block, tau, rows=rows)


def test_exp2_polynomial_error_bound():
    """The FMA-pipe exp2 (degree-3 minimax, relative error 7.5e-5 by construction) against exact
    2^x in fp64 and against the hardware ex2.approx, over the softmax's input range."""
    import torch
    import block_sparse_long_causal_b200 as fp
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.arange(-126, 9), np.arange(-126, 9) + 0.5,
                        [0.0, -0.0, 1e-8, -1e-8]]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yp, ym = torch.empty_like(xd), torch.empty_like(xd)
    fp.selftest_exp2(xd, yp, ym)
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    ypn, ymn = yp.cpu().numpy().astype(np.float64), ym.cpu().numpy().astype(np.float64)
    normal = x >= -125.0  # the exponent-field add keeps full precision while the result is a normal float
    rel_poly = np.abs(ypn[normal] / exact[normal] - 1.0)
    rel_mufu = np.abs(ymn[normal] / exact[normal] - 1.0)
    assert rel_poly.max() <= 1e-4, rel_poly.max()   # 7.5e-5 minimax bound + float32 rounding
    assert rel_mufu.max() <= 1e-5, rel_mufu.max()
    assert (ypn[~normal] >= 0).all() and (ypn[~normal] <= 2.0 ** -124).all()
    # below the clamp the polynomial returns 2^-126 times its value at the clamp, never garbage
    xs = torch.tensor([-200.0, -1e30, float("-inf")], device="cuda")
    yp2, ym2 = torch.empty_like(xs), torch.empty_like(xs)
    fp.selftest_exp2(xs, yp2, ym2)
    torch.cuda.synchronize()
    v = yp2.cpu().numpy()
    assert (v >= 0).all() and (v <= 2.0 ** -125).all()


def test_one_call_sparse_prefill_matches_the_three_calls():
    import torch
    import block_sparse_long_causal_b200 as fp
    from helpers import bf16_to_np, to_dev
    w = synth.WORKLOADS["llama3-8b-L32768"]
    x = synth.make_inputs(w.with_lens([3000, 129, 1800]))
    ref = gpu_prefill(x, w.hq, w.hkv, w.block, 0.9)
    p = fp.problem(x["cu_seqlens"], w.hq, w.hkv, 128, w.block)
    ws = torch.empty(fp.sparse_prefill_workspace(p), dtype=torch.uint8, device="cuda")
    out = torch.empty((p.total_tokens, w.hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.hq, p.total_tokens), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    fp.sparse_prefill(p, q, k, v, 0.9, 0.0, ws, out, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(bf16_to_np(out), ref["out"])
    np.testing.assert_array_equal(lse.cpu().numpy(), ref["lse"])


@pytest.mark.parametrize("case", [c for c in SMALL if c[3] == 128],
                         ids=lambda c: f"L{'-'.join(map(str, c[0]))}_h{c[1]}x{c[2]}_t{c[4]}")
def test_small_cases_on_the_row_schedule(case, monkeypatch):
    """The single-tile attention schedule (chosen by the kernel for sparse lists) on every B = 128
    case, forced whatever the density. Inputs at the workloads' scale (q, k ~ N(0, 1)): at 3x the
    O bound is about one bf16 ulp of the largest outputs, where the row sum's rounding order alone
    can decide a case."""
    monkeypatch.setenv("FP_ATTN_UNITS", "rows")
    lens, hq, hkv, B, tau, _ = case
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + hq + 7, scale=1.0)
    _check_case(x, hq, hkv, B, tau)
