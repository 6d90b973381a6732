"""FP8 attention (e4m3 Q and K, per-tensor scales, bf16 V): fp_block_sparse_attn_fp8 and
fp_dense_attn_fp8 against the oracle on the dequantised inputs.

e4m3 values are exactly representable in bf16, so the oracle runs its exact fp64 attention on the
bf16 bits of the e4m3 values with the softmax scale multiplied by q_scale * k_scale: the reference
is the exact attention of the quantised problem, and the GPU must match it to the same output
tolerance as the bf16 path (the only differences left are the bf16 rounding of P and O and the
fp32 accumulation)."""
import numpy as np
import pytest

import oracle
import synth
from helpers import ATOL_MAX, ATOL_MEAN, bf16_to_np, gpu_prefill, to_dev

pytestmark = pytest.mark.gpu


def quantise(bits_bf16, scale):
    x = synth.bf16_bits_to_f32(bits_bf16)
    codes = synth.to_e4m3_bits(x / scale)
    deq_bf16 = synth.to_bf16_bits(synth.e4m3_bits_to_f32(codes))  # exact: e4m3 values fit bf16
    return codes, deq_bf16


def run_fp8(x, hq, hkv, B, tau, dense=False, q_scale=None, k_scale=None):
    import torch
    import block_sparse_long_causal_b200 as fp
    q32, k32 = synth.bf16_bits_to_f32(x["q"]), synth.bf16_bits_to_f32(x["k"])
    q_scale = q_scale or float(np.abs(q32).max()) / 448.0
    k_scale = k_scale or float(np.abs(k32).max()) / 448.0
    qc, qd = quantise(x["q"], q_scale)
    kc, kd = quantise(x["k"], k_scale)
    cu = x["cu_seqlens"]
    lists = gpu_prefill(x, hq, hkv, B, tau, with_lse=False)  # lists from the bf16 search
    p = fp.problem(cu, hq, hkv, 128, B)
    T = p.total_tokens
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((hq, T), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    qg = torch.from_numpy(qc).cuda()
    kg = torch.from_numpy(kc).cuda()
    v = to_dev(x["v"])
    counts = torch.from_numpy(lists["counts"]).cuda().contiguous()
    indices = torch.from_numpy(lists["indices"]).cuda().contiguous()
    if dense:
        fp.dense_attn_fp8(p, qg, kg, v, q_scale, k_scale, 0.0, out, lse, st)
    else:
        fp.block_sparse_attn_fp8(p, qg, kg, v, q_scale, k_scale, counts, indices, 0.0, out, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    xq = {"q": qd, "k": kd, "v": x["v"], "cu_seqlens": cu}
    return xq, lists, bf16_to_np(out), lse.cpu().numpy(), q_scale * k_scale


def check(x, hq, hkv, B, tau, dense=False, **kw):
    xq, lists, out, lse, qk = run_fp8(x, hq, hkv, B, tau, dense, **kw)
    T = out.shape[0]
    rows_tok = np.repeat(np.arange(T, dtype=np.int64), hq)
    rows_head = np.tile(np.arange(hq, dtype=np.int32), T)
    scale = qk / np.sqrt(128.0)
    o_ref, lse_ref = oracle.attn_rows(xq["q"], xq["k"], xq["v"], xq["cu_seqlens"], B, rows_tok, rows_head,
                                      None if dense else lists["counts"], None if dense else lists["indices"],
                                      scale=scale)
    got = synth.bf16_bits_to_f32(out[rows_tok, rows_head]).astype(np.float64)
    err = np.abs(got - o_ref)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())
    assert np.abs(lse[rows_head, rows_tok] - lse_ref).max() <= 1e-2


@pytest.mark.parametrize("lens,hq,hkv,B,tau", [
    ((700, 300), 4, 2, 64, 0.5),
    ((1000, 129), 6, 2, 128, 0.3),    # G = 3
    ((640,), 4, 1, 128, 0.0),         # every causal block
])
def test_fp8_sparse_matches_the_oracle(lens, hq, hkv, B, tau):
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens), scale=1.5)
    check(x, hq, hkv, B, tau)


def test_fp8_dense_and_explicit_scales():
    x = synth.random_inputs((900, 257), 4, 2, 128, seed=77, scale=1.0)
    check(x, 4, 2, 128, 0.5, dense=True)
    check(x, 4, 2, 64, 0.5, q_scale=0.02, k_scale=0.015)  # codes saturate at 448 beyond |x| = 8.96 / 6.72


def quantise_blocks(bits_bf16, cu, B):
    """Per-(block, head) power-of-two scales: exponent e = ceil(log2(max|x| / 448)) of each B-token
    block of each head (blocks restart at every sequence), codes = e4m3(x / 2^e). Returns the codes,
    the int8 exponents [total_blocks, H] and the dequantised values 2^e * code as bf16 bits (exact)."""
    x = synth.bf16_bits_to_f32(bits_bf16).astype(np.float64)
    T, H, _ = x.shape
    exps, rows = [], []
    for s in range(len(cu) - 1):
        for t0 in range(int(cu[s]), int(cu[s + 1]), B):
            t1 = min(t0 + B, int(cu[s + 1]))
            amax = np.abs(x[t0:t1]).max(axis=(0, 2))
            e = np.where(amax > 0, np.ceil(np.log2(np.maximum(amax, 1e-30) / 448.0)), 0).astype(np.int8)
            exps.append(e)
            rows.append((t0, t1))
    exps = np.stack(exps) if exps else np.zeros((0, H), np.int8)
    codes = np.empty(x.shape, np.uint8)
    deq = np.empty(x.shape, np.float32)
    for b, (t0, t1) in enumerate(rows):
        sc = np.exp2(exps[b].astype(np.float64))[None, :, None]
        codes[t0:t1] = synth.to_e4m3_bits((x[t0:t1] / sc).astype(np.float32))
        deq[t0:t1] = (synth.e4m3_bits_to_f32(codes[t0:t1]).astype(np.float64) * sc).astype(np.float32)
    return codes, exps, synth.to_bf16_bits(deq)


@pytest.mark.parametrize("lens,hq,hkv,B,tau,dense", [
    ((700, 300), 4, 2, 64, 0.5, False),
    ((1000, 129), 6, 2, 128, 0.3, False),   # G = 3
    ((900, 257), 4, 2, 128, 0.5, True),
])
def test_fp8_per_block_scales_match_the_oracle(lens, hq, hkv, B, tau, dense):
    """Per-block scales follow each block's range (one query block and one key block are 64x smaller
    than the rest, where a per-tensor scale would leave them fewer significant code bits); the
    reference is the exact attention of the dequantised inputs (2^e * code, exact in bf16)."""
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + 5, scale=1.0)
    q32 = synth.bf16_bits_to_f32(x["q"]).copy()
    k32 = synth.bf16_bits_to_f32(x["k"]).copy()
    q32[B:2 * B] *= 0.015625
    k32[2 * B:3 * B] *= 0.015625
    x = dict(x, q=synth.to_bf16_bits(q32), k=synth.to_bf16_bits(k32))
    cu = x["cu_seqlens"]
    qc, qe, qd = quantise_blocks(x["q"], cu, B)
    kc, ke, kd = quantise_blocks(x["k"], cu, B)
    lists = gpu_prefill(x, hq, hkv, B, tau, with_lse=False)
    p = fp.problem(cu, hq, hkv, 128, B)
    assert qe.shape == (p.total_blocks, hq) and ke.shape == (p.total_blocks, hkv)
    T = p.total_tokens
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((hq, T), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (torch.from_numpy(qc).cuda(), torch.from_numpy(kc).cuda(), to_dev(x["v"]),
            torch.from_numpy(qe).cuda(), torch.from_numpy(ke).cuda())
    if dense:
        fp.dense_attn_fp8_blockscaled(p, *args, 0.0, out, lse, st)
    else:
        counts = torch.from_numpy(lists["counts"]).cuda().contiguous()
        indices = torch.from_numpy(lists["indices"]).cuda().contiguous()
        fp.block_sparse_attn_fp8_blockscaled(p, *args, counts, indices, 0.0, out, lse, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got_bits = bf16_to_np(out)
    rows_tok = np.repeat(np.arange(T, dtype=np.int64), hq)
    rows_head = np.tile(np.arange(hq, dtype=np.int32), T)
    o_ref, lse_ref = oracle.attn_rows(qd, kd, x["v"], cu, B, rows_tok, rows_head,
                                      None if dense else lists["counts"], None if dense else lists["indices"])
    got = synth.bf16_bits_to_f32(got_bits[rows_tok, rows_head]).astype(np.float64)
    err = np.abs(got - o_ref)
    assert err.max() <= ATOL_MAX and err.mean() <= ATOL_MEAN, (err.max(), err.mean())
    assert np.abs(lse.cpu().numpy()[rows_head, rows_tok] - lse_ref).max() <= 1e-2
