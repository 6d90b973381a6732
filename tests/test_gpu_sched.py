"""The attention work counter (fp_problem.sched): with it every CTA takes its next work unit when it
is free instead of a fixed share. Which CTA computes a unit does not change how it is computed, so
the outputs must equal the fixed schedule's bit for bit; every launch must leave the counter at
zero (also one whose waits ran out), so that launches in a row and CUDA graph replays share it."""
import numpy as np
import pytest

import synth
from helpers import bf16_to_np, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _attn(p, q, k, v, counts, indices, dense):
    import torch
    import block_sparse_long_causal_b200 as fp
    out = torch.empty((p.total_tokens, p.num_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((p.num_q_heads, p.total_tokens), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if dense:
        fp.dense_attn(p, q, k, v, 0.0, out, lse, st)
    else:
        fp.block_sparse_attn(p, q, k, v, counts, indices, 0.0, out, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return bf16_to_np(out), lse.cpu().numpy()


@pytest.mark.parametrize("B,units", [(64, "pairs"), (128, "pairs"), (128, "rows")])
def test_counter_and_fixed_schedule_agree_bit_for_bit(B, units, monkeypatch):
    import block_sparse_long_causal_b200 as fp
    monkeypatch.setenv("FP_ATTN_UNITS", units)
    # three sequences of uneven length and a selective threshold: lists of very different lengths
    x = synth.random_inputs((3000, 700, 5100), 8, 2, 128, seed=61, scale=2.0)
    cu = x["cu_seqlens"]
    p_dyn = fp.problem(cu, 8, 2, 128, B)
    p_fix = fp.problem(cu, 8, 2, 128, B, work_counter=False)
    assert p_dyn.sched is not None and p_fix.sched is None
    sp = fp.SparsePrefill(p_dyn)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sp.search(q, k, 0.9)
    for dense in (False, True):
        o_fix, l_fix = _attn(p_fix, q, k, v, sp.counts, sp.indices, dense)
        for _ in range(3):  # launches in a row reuse the counter
            o_dyn, l_dyn = _attn(p_dyn, q, k, v, sp.counts, sp.indices, dense)
            np.testing.assert_array_equal(o_dyn, o_fix)
            np.testing.assert_array_equal(l_dyn, l_fix)
            assert p_dyn.sched.cpu().tolist() == [0, 0]


def test_one_call_prefill_with_its_workspace_counter_matches_the_three_calls():
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs((2500, 4100), 4, 2, 128, seed=62, scale=2.0)
    cu = x["cu_seqlens"]
    p = fp.problem(cu, 4, 2, 128, 128, work_counter=False)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sp = fp.SparsePrefill(p)
    sp(q, k, v, 0.8)
    want = bf16_to_np(sp.out)
    # a workspace full of garbage: the call zeroes its counter words before the attention launch
    ws = torch.full((fp.sparse_prefill_workspace(p),), 0x5A, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(sp.out)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        fp.sparse_prefill(p, q, k, v, 0.8, 0.0, ws, out, None, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        np.testing.assert_array_equal(bf16_to_np(out), want)


def test_counter_in_a_cuda_graph_replays():
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs((4096, 1500), 8, 2, 128, seed=63, scale=2.0)
    cu = x["cu_seqlens"]
    p = fp.problem(cu, 8, 2, 128, 128)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sp = fp.SparsePrefill(p)
    sp(q, k, v, 0.9)
    torch.cuda.synchronize()
    want = bf16_to_np(sp.out)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            sp(q, k, v, 0.9, stream=s)
    torch.cuda.synchronize()
    for _ in range(3):
        sp.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bf16_to_np(sp.out), want)
        assert p.sched.cpu().tolist() == [0, 0]
    del g


@pytest.mark.parametrize("units", ["pairs", "rows"])
def test_counter_is_zero_after_a_launch_whose_waits_ran_out(monkeypatch, units):
    import torch
    import block_sparse_long_causal_b200 as fp
    monkeypatch.setenv("FP_ATTN_UNITS", units)
    x = synth.random_inputs((900, 300), 4, 2, 128, seed=64)
    p = fp.problem(x["cu_seqlens"], 4, 2, 128, 128)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    sp = fp.SparsePrefill(p)
    sp.search(q, k, 0.0)
    torch.cuda.synchronize()
    monkeypatch.setenv("FP_TEST_UNSIGNALLED_WAIT", "1")
    monkeypatch.setenv("FP_WAIT_LIMIT_MS", "50")
    sp.attend(q, k, v)
    torch.cuda.synchronize()
    assert int(sp.dev_status.item()) & fp.FP_DEV_TIMEOUT
    assert p.sched.cpu().tolist() == [0, 0]
    monkeypatch.delenv("FP_TEST_UNSIGNALLED_WAIT")
    monkeypatch.delenv("FP_WAIT_LIMIT_MS")
    sp.dev_status.zero_()
    sp.attend(q, k, v)
    torch.cuda.synchronize()
    assert int(sp.dev_status.item()) == 0
