"""fp_sparse_prefill_noalloc: the one-call sparse prefill for callers that cannot allocate device
memory (serving loops with a fixed memory plan, plugin hosts without a workspace, code that cannot
take cudaMalloc's implicit synchronisation). Its intermediates live in a fixed array inside the
library, so it must give the same output as fp_sparse_prefill with a caller workspace.

This file is collected last, so a run that stops at the first failure has run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import synth
from helpers import bf16_to_np, to_dev


def test_rejects_problems_beyond_the_static_array():
    """Too-large problems fail on the host with a clear message, before any device work."""
    import block_sparse_long_causal_b200 as fp
    p = fp.fp_problem()
    host = np.array([0, 600_000], np.int32)
    assert fp._lib.fp_problem_init(C.byref(p), host.ctypes.data_as(C.c_void_p), 1, C.c_void_p(16),
                                   32, 8, 128, 128) == fp.FP_OK
    ok = C.c_void_p(4096)
    st = fp._lib.fp_sparse_prefill_noalloc(C.byref(p), ok, ok, ok, C.c_float(0.1), C.c_float(0.0), ok, None, None,
                                           None)
    assert st == fp.FP_ERR_INVALID_ARG
    assert "static array" in fp._lib.fp_last_error().decode()


def _workspace_lists(ws, p):
    """Counts and index lists inside a fp_sparse_prefill workspace (pooled Q, pooled K, counts,
    indices, work counter; each part 256-byte aligned)."""
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nb, hq, hkv, d = p.total_blocks, p.num_q_heads, p.num_kv_heads, p.head_dim
    off_c = a(a(nb * hq * d * 4) + nb * hkv * d * 4)
    off_i = a(off_c + hq * nb * 4)
    raw = ws.cpu().numpy()
    counts = raw[off_c:off_c + hq * nb * 4].view(np.int32).reshape(hq, nb)
    idx = raw[off_i:off_i + p.index_elems * 4].view(np.int32)
    return counts, idx


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    import torch
    import block_sparse_long_causal_b200 as fp
    from helpers import compare_attention, sample_rows
    assert torch.cuda.is_available()
    w = synth.WORKLOADS["llama3-8b-L32768"]
    # two different problems back to back: the second call finds the first call's leftovers in the
    # shared array and must not depend on them
    cases = [(w.with_lens([3000, 129, 1800]), 0.9), (w.with_lens([5000], seeds=[7]), 0.05)]
    for wl, tau in cases:
        x = synth.make_inputs(wl)
        p = fp.problem(x["cu_seqlens"], wl.hq, wl.hkv, 128, wl.block)
        assert fp.sparse_prefill_workspace(p) <= fp.FP_NOALLOC_MAX_BYTES
        q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
        T = p.total_tokens
        outs, lses = [], []
        for noalloc in (False, True):
            out = torch.empty((T, wl.hq, 128), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((wl.hq, T), dtype=torch.float32, device="cuda")
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            if noalloc:
                fp.sparse_prefill_noalloc(p, q, k, v, tau, 0.0, out, lse, st)
            else:
                ws = torch.empty(fp.sparse_prefill_workspace(p), dtype=torch.uint8, device="cuda")
                fp.sparse_prefill(p, q, k, v, tau, 0.0, ws, out, lse, st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            outs.append(bf16_to_np(out))
            lses.append(lse.cpu().numpy())
        # the same kernels on the same inputs with the same work-counter schedule: identical bits
        assert np.array_equal(outs[1], outs[0])
        assert np.array_equal(lses[1].view(np.uint32), lses[0].view(np.uint32))
        # and the output is the exact attention over the lists the call computed (oracle, sampled rows)
        counts, idx = _workspace_lists(ws, p)
        tok, head = sample_rows(x["cu_seqlens"], wl.hq, 256, seed=3)
        res = {"counts": counts, "indices": idx, "out": outs[1], "lse": lses[1]}
        compare_attention(x, res, wl.hq, wl.block, tok, head)
