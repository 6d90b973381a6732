"""Failure detection on the GPU without a GPU fault: bounded waits that run out return a status
bit and leave the context usable; malformed index lists are flagged and skipped, never trapped."""
import numpy as np
import pytest

import synth
from helpers import compare_attention, gpu_prefill, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.mark.parametrize("units", ["pairs", "rows"])
def test_wait_that_nothing_signals_times_out_and_context_survives(monkeypatch, units):
    import block_sparse_long_causal_b200 as fp
    monkeypatch.setenv("FP_ATTN_UNITS", units)  # both attention schedules
    x = synth.random_inputs((700, 300), 4, 2, 128, seed=41)
    good = gpu_prefill(x, 4, 2, 128, 0.0)
    monkeypatch.setenv("FP_TEST_UNSIGNALLED_WAIT", "1")
    monkeypatch.setenv("FP_WAIT_LIMIT_MS", "50")
    bad = gpu_prefill(x, 4, 2, 128, 0.0, check_status=False)
    assert bad["status"] & fp.FP_DEV_TIMEOUT
    monkeypatch.delenv("FP_TEST_UNSIGNALLED_WAIT")
    monkeypatch.delenv("FP_WAIT_LIMIT_MS")
    again = gpu_prefill(x, 4, 2, 128, 0.0)      # the context is still usable and correct
    np.testing.assert_array_equal(again["out"], good["out"])
    assert again["status"] == 0


def test_validator_flags_malformed_lists():
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs((600,), 4, 2, 128, seed=43)
    p = fp.problem(x["cu_seqlens"], 4, 2, 128, 128)
    sp = fp.SparsePrefill(p)
    q, k = to_dev(x["q"]), to_dev(x["k"])
    sp.search(q, k, 0.5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp.validate_lists(p, sp.counts, sp.indices, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for corrupt in ("count0", "count_big", "missing_sink", "out_of_range", "descending"):
        c, idx = sp.counts.clone(), sp.indices.clone()
        if corrupt == "count0":
            c[1, 3] = 0
        elif corrupt == "count_big":
            c[2, 2] = 4
        elif corrupt == "missing_sink":
            idx[3 * 15 + 10] = 1  # first entry of row (h=3, i=4) (offset h*15 + i(i+1)/2) is not 0
        elif corrupt == "out_of_range":
            c[0, 4] = 5
            idx[10:15] = torch.tensor([0, 1, 2, 9, 4], dtype=torch.int32)
        else:
            c[0, 4] = 5
            idx[10:15] = torch.tensor([0, 2, 1, 3, 4], dtype=torch.int32)
        st.zero_()
        fp.validate_lists(p, c, idx, st)
        torch.cuda.synchronize()
        assert int(st.item()) & fp.FP_DEV_BAD_LIST, corrupt


def test_out_of_range_entries_are_skipped_and_flagged():
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs((640,), 2, 1, 128, seed=47)
    res = gpu_prefill(x, 2, 1, 128, 0.0)
    p = fp.problem(x["cu_seqlens"], 2, 1, 128, 128)
    counts = torch.from_numpy(res["counts"].copy()).cuda()
    idx = torch.from_numpy(res["indices"].copy()).cuda()
    # row (h=0, i=4) at offset 10: dense list 0..4; append garbage by replacing entry 2 with -7 and
    # entry 3 with 99 (both out of range): the kernel skips them and flags FP_DEV_BAD_LIST
    idx[12] = -7
    idx[13] = 99
    out = torch.empty((640, 2, 128), dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    fp.block_sparse_attn(p, q, k, v, counts, idx, 0.0, out, None, st)
    torch.cuda.synchronize()
    assert int(st.item()) & fp.FP_DEV_BAD_LIST
    # rows of that tile equal the oracle on the lists with the bad entries removed
    res2 = dict(res, counts=res["counts"].copy(), indices=res["indices"].copy(),
                out=out.view(torch.int16).cpu().numpy().view(np.uint16), lse=None)
    res2["indices"][10:13] = [0, 1, 4]
    res2["counts"][0, 4] = 3
    rows_tok = np.arange(512, 640, dtype=np.int64)
    rows_head = np.zeros(128, np.int32)
    compare_attention(x, res2, 2, 128, rows_tok, rows_head)
