"""GPU search at the edge of its error bound.

The search kernel decides block j of row (h, i) from tensor-core pooled scores accurate to
eps = 2^-13 |qbar| max|kbar| (in dot-product units). Where 2 eps / sqrt(d) is below the tie band
(|p/max p - tau| <= 1e-4 tau, i.e. about 1e-4 in s - max s), that decision can only differ from the
exact one inside the band; rows with a wider bound take an exact fp32 pass. These cases put
hundreds of blocks just outside the band (1e-4 < |s - max s - ln tau| < 5e-4) with large pooled
norms, for both kinds of row, and require bit-exact lists there.

Inputs: every block's tokens take two values (a, b alternating), so its pooled mean (a + b) / 2 is
the same number in fp32 and fp64 but is generally not a bf16 value (its bf16 split has a non-zero
low part); keys share a large common vector plus small per-block perturbations, so their scores
are spread over a few hundredths while the norms stay large.
"""
import numpy as np
import pytest

import oracle
import synth
from helpers import compare_lists, keep_mask, to_dev

pytestmark = pytest.mark.gpu


def _two_valued(vals: np.ndarray, delta: float, B: int, rng) -> np.ndarray:
    """[nb, H, d] block means -> [nb * B, H, d] bf16 tokens alternating a = v + delta', b = v - delta'."""
    jit = delta * rng.standard_normal(vals.shape).astype(np.float32)
    a = synth.to_bf16_bits(vals + jit)
    b = synth.to_bf16_bits(vals - jit)
    tok = np.empty((vals.shape[0], B) + vals.shape[1:], np.uint16)
    tok[:, 0::2] = a[:, None]
    tok[:, 1::2] = b[:, None]
    return tok.reshape((-1,) + vals.shape[1:])


def _case(nb, hq, hkv, B, q_norm, c_norm, e_sigma, seed):
    rng = np.random.default_rng(seed)
    d = 128
    qv = rng.standard_normal((nb, hq, d)).astype(np.float32)
    qv *= q_norm / np.linalg.norm(qv, axis=2, keepdims=True)
    c = rng.standard_normal((1, hkv, d)).astype(np.float32)
    c *= c_norm / np.linalg.norm(c, axis=2, keepdims=True)
    kv = c + e_sigma * rng.standard_normal((nb, hkv, d)).astype(np.float32)
    q = _two_valued(qv, 0.01 * q_norm / np.sqrt(d), B, rng)
    k = _two_valued(kv, 0.01 * c_norm / np.sqrt(d), B, rng)
    v = synth.to_bf16_bits(rng.standard_normal((nb * B, hkv, d)).astype(np.float32))
    cu = np.array([0, nb * B], np.int32)
    return {"q": q, "k": k, "v": v, "cu_seqlens": cu}


def _tau_near_many_blocks(qb, kb, cu, B, hq):
    """A threshold with many blocks just outside its tie band; returns (tau, #blocks within
    1e-4 .. 5e-4 of ln tau)."""
    G = hq // kb.shape[1]
    ds = []
    for h in range(hq):
        s = qb[:, h, :] @ kb[:, h // G, :].T / np.sqrt(qb.shape[2])
        tri = np.tril(np.ones(s.shape, bool))
        s = np.where(tri, s, -np.inf)
        dd = s - s.max(axis=1, keepdims=True)
        ds.append(dd[tri & (dd < 0)])
    ds = np.concatenate(ds)
    lt = float(np.quantile(ds, 0.4))
    near = int(((np.abs(ds - lt) > 1e-4) & (np.abs(ds - lt) < 5e-4)).sum())
    return float(np.exp(lt)), near


@pytest.mark.parametrize("name,q_norm,c_norm,e_sigma", [
    # |qbar| |kbar| ~ 2.3: the tensor-core decision (2 eps / sqrt(d) ~ 4e-5 < 1e-4)
    ("tensor-core rows", 1.5, 1.5, 0.01),
    # |qbar| |kbar| ~ 30: bound wider than the band, every row takes the exact fp32 pass
    ("exact rows", 10.0, 3.0, 0.0015),
])
@pytest.mark.parametrize("B", [64, 128])
@pytest.mark.parametrize("key_split", [True, False], ids=["key_split", "tile_split"])
def test_lists_exact_just_outside_the_tie_band(name, q_norm, c_norm, e_sigma, B, key_split):
    import torch
    import block_sparse_long_causal_b200 as fp
    nb, hq, hkv = 200, 4, 2
    x = _case(nb, hq, hkv, B, q_norm, c_norm, e_sigma, seed=B + int(q_norm))
    cu = x["cu_seqlens"]
    qb, kb = oracle.pool(x["q"], cu, B), oracle.pool(x["k"], cu, B)
    tau, near = _tau_near_many_blocks(qb, kb, cu, B, hq)
    assert near >= 200, near  # the case has teeth: many blocks sit just outside the band
    oc, oi, band = oracle.search(qb, kb, cu, B, tau)
    p = fp.problem(cu, hq, hkv, 128, B, key_split=key_split)
    assert (p.key_split is not None) == key_split
    sp = fp.SparsePrefill(p)
    sp.search(to_dev(x["q"]), to_dev(x["k"]), tau)
    torch.cuda.synchronize()
    assert int(sp.dev_status.item()) == 0
    np.testing.assert_allclose(sp.k_pool[:nb].cpu().numpy(), kb, rtol=0, atol=1e-6)
    compare_lists(sp.counts.cpu().numpy(), sp.indices[: p.index_elems].cpu().numpy(), oc, oi, band, cu, B, hq)


@pytest.mark.parametrize("lens,hq,hkv,B,tau", [
    ((1000,), 4, 2, 128, 0.9),
    ((257, 1, 130, 640), 8, 2, 128, 0.7),
    ((700, 129), 4, 2, 64, 0.5),
    ((900, 385), 6, 2, 128, 0.6),      # G = 3
    ((2000,), 16, 2, 64, 0.95),        # G = 8
    ((3000,), 2, 2, 128, 0.05),        # every row certified all-kept
])
def test_key_split_and_tile_split_give_the_same_lists(lens, hq, hkv, B, tau):
    """The searches that split the pooled keys once per call (fp_problem.key_split) and per tile give
    the same lists bit for bit: same split, same error bound per key, same decisions."""
    import torch
    import block_sparse_long_causal_b200 as fp
    x = synth.random_inputs(lens, hq, hkv, 128, seed=sum(lens) + hq, scale=1.0)
    cu = x["cu_seqlens"]
    out = []
    for ks in (True, False):
        p = fp.problem(cu, hq, hkv, 128, B, key_split=ks)
        sp = fp.SparsePrefill(p)
        sp.search(to_dev(x["q"]), to_dev(x["k"]), tau)
        torch.cuda.synchronize()
        assert int(sp.dev_status.item()) == 0
        out.append((sp.counts.cpu().numpy().copy(), sp.indices[: p.index_elems].cpu().numpy().copy()))
    np.testing.assert_array_equal(out[0][0], out[1][0])
    # the lists (entries past a row's count are scratch of the exact pass, compared through the masks)
    np.testing.assert_array_equal(keep_mask(out[0][0], out[0][1], cu, B, hq), keep_mask(out[1][0], out[1][1], cu, B, hq))
