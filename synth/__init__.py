"""Seeded synthetic Q/K/V workloads for the block-sparse causal prefill path.

This module is the one piece shared by the CPU oracle side and the CUDA side: it
only draws random numbers and lays them out as bf16 bytes. It holds none of the
method's arithmetic (no pooling, no scores, no thresholds, no attention).

Recipe (the workloads of the FlashPrefill evaluation are described only in words,
so each step below is this repository's reading of that description):

* one shared direction per sequence: w ~ N(0, I_d), u = 3 * w / ||w||;
* V ~ N(0, 1) and K1 ~ N(0, 1) per kv-head; Q ~ N(0, 1) + 0.5 * u per q-head,
  except a seeded random subset of q-heads (``uniform_head_frac``) drawn with no
  u term ("near-uniform" heads);
* "vertical" keys: ``nvert`` distinct positions drawn uniformly from 1..L-1, plus
  position 0 (the sink); at those positions K1 += 4 * u on every kv-head;
* "slash" band: K[t] = K1[t] + 0.8 * sum_{o in offsets, t-o >= 0} K1[t-o]
  (non-recursive, from K1 after the vertical boost);
* every tensor is rounded once from float32 to bf16 (round to nearest even).

Random streams: every (sequence seed, tensor, chunk of CHUNK tokens) pair has its
own PCG64 stream keyed through numpy's SeedSequence, so the bytes do not depend
on how many threads fill the chunks.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Sequence

import numpy as np

CHUNK = 2048  # tokens per independent random stream

_T_V, _T_K, _T_Q, _T_DIR, _T_HEADS, _T_VERT = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic prefill problem: shapes, block size, tau and generator knobs."""

    name: str
    lens: tuple            # sequence lengths, packed back to back (cu_seqlens)
    hq: int                # query heads
    hkv: int               # key/value heads (GQA group size G = hq // hkv)
    d: int                 # head dim
    block: int             # pooling / attention block size B
    tau: float             # max-based threshold
    nvert: int             # number of vertical keys (besides the sink)
    offsets: tuple         # slash offsets
    uniform_head_frac: float = 0.0
    seeds: tuple = (0,)    # one seed per sequence

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lens))

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lens)]).astype(np.int32)

    def with_lens(self, lens: Sequence[int], seeds: Sequence[int] | None = None, **kw) -> "Workload":
        if seeds is None:
            seeds = tuple(range(len(lens)))
        return dataclasses.replace(self, lens=tuple(int(x) for x in lens), seeds=tuple(seeds), **kw)


# The five workloads of the evaluation, named by what they are.
WORKLOADS = {
    "mha4-L2048-B64": Workload("mha4-L2048-B64", (2048,), 4, 4, 128, 64, 0.1, 8, (256,)),
    "llama3-8b-L32768": Workload("llama3-8b-L32768", (32768,), 32, 8, 128, 128, 0.1, 64, (128, 1024)),
    "llama3-8b-L131072": Workload("llama3-8b-L131072", (131072,), 32, 8, 128, 128, 0.05, 256, (256,),
                                  uniform_head_frac=0.25),
    "llama3-8b-L262144": Workload("llama3-8b-L262144", (262144,), 32, 8, 128, 128, 0.05, 512,
                                  (128, 4096, 65536)),
    "llama3-8b-varlen8-T264192": Workload(
        "llama3-8b-varlen8-T264192", (4096, 8192, 16384, 32768, 65536, 4096, 131072, 2048),
        32, 8, 128, 128, 0.1, 64, (128, 1024), seeds=(0, 1, 2, 3, 4, 5, 6, 7)),
}
ORDER = list(WORKLOADS)  # evaluation order: small case first


def _rng(seed: int, tensor: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), tensor, chunk])))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---- FP8 e4m3 (OCP "E4M3": 1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinity,
# 0x7F / 0xFF are NaN; largest finite 448). Input-format conversion for the FP8 attention inputs.
def _e4m3_table() -> np.ndarray:
    """Values of the codes 0x00..0x7E (the non-negative finite e4m3 numbers), ascending."""
    vals = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        vals.append((m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, np.float64)


_E4M3 = _e4m3_table()


def to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """float -> e4m3 codes (uint8): round to nearest, ties to the even code, saturate to +-448."""
    x = np.asarray(x, np.float64)
    a = np.minimum(np.abs(x), _E4M3[-1])
    hi = np.clip(np.searchsorted(_E4M3, a, side="left"), 0, len(_E4M3) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo, dhi = a - _E4M3[lo], _E4M3[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def e4m3_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, np.uint8)
    v = _E4M3[np.minimum(b & 0x7F, 0x7E)].astype(np.float32)
    return np.where(b & 0x80, -v, v).astype(np.float32)


def _pool():
    return _cf.ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1)))


def _fill_normal(out: np.ndarray, seed: int, tensor: int, ex) -> None:
    """Fill out[L, H, d] (float32) chunk by chunk, one stream per chunk."""
    L = out.shape[0]
    futs = []
    for c in range(0, L, CHUNK):
        def job(c=c):
            _rng(seed, tensor, c // CHUNK).standard_normal(out=out[c:c + CHUNK], dtype=np.float32)
        futs.append(ex.submit(job))
    for f in futs:
        f.result()


def make_sequence(L: int, hq: int, hkv: int, d: int, seed: int, nvert: int, offsets: Sequence[int],
                  uniform_head_frac: float = 0.0, ex=None):
    """One sequence of the recipe above; returns bf16 bits q [L,hq,d], k [L,hkv,d], v [L,hkv,d]."""
    own = ex is None
    ex = ex or _pool()
    try:
        w = _rng(seed, _T_DIR, 0).standard_normal(d)
        u = (3.0 * w / np.linalg.norm(w)).astype(np.float32)

        n_uniform = int(round(uniform_head_frac * hq))
        uniform = set(_rng(seed, _T_HEADS, 0).choice(hq, size=n_uniform, replace=False).tolist()) if n_uniform else set()
        shift = np.zeros((hq, d), np.float32)
        for h in range(hq):
            if h not in uniform:
                shift[h] = 0.5 * u

        nv = min(nvert, max(L - 1, 0))
        vert = _rng(seed, _T_VERT, 0).choice(np.arange(1, L), size=nv, replace=False) if nv else np.zeros(0, np.int64)
        vert = np.concatenate([[0], np.sort(vert)]).astype(np.int64) if L > 0 else vert

        v32 = np.empty((L, hkv, d), np.float32)
        _fill_normal(v32, seed, _T_V, ex)
        v = _convert(v32, ex)
        del v32

        k1 = np.empty((L, hkv, d), np.float32)
        _fill_normal(k1, seed, _T_K, ex)
        if L > 0:
            k1[vert] += 4.0 * u
        k32 = k1.copy()
        for o in offsets:
            if o < L:
                k32[o:] += np.float32(0.8) * k1[:L - o]
        del k1
        k = _convert(k32, ex)
        del k32

        q = np.empty((L, hq, d), np.uint16)
        futs = []
        for c in range(0, L, CHUNK):
            def job(c=c):
                blk = _rng(seed, _T_Q, c // CHUNK).standard_normal((min(CHUNK, L - c), hq, d), dtype=np.float32)
                blk += shift
                q[c:c + CHUNK] = to_bf16_bits(blk)
            futs.append(ex.submit(job))
        for f in futs:
            f.result()
        return q, k, v
    finally:
        if own:
            ex.shutdown()


def _convert(x32: np.ndarray, ex) -> np.ndarray:
    out = np.empty(x32.shape, np.uint16)
    futs = [ex.submit(lambda c=c: out.__setitem__(slice(c, c + CHUNK), to_bf16_bits(x32[c:c + CHUNK])))
            for c in range(0, x32.shape[0], CHUNK)]
    for f in futs:
        f.result()
    return out


def make_inputs(w: Workload):
    """All sequences of a workload packed along tokens.

    Returns dict(q, k, v: uint16 bf16 bits [T, H, d]; cu_seqlens: int32 [S+1]).
    """
    T = w.total_tokens
    q = np.empty((T, w.hq, w.d), np.uint16)
    k = np.empty((T, w.hkv, w.d), np.uint16)
    v = np.empty((T, w.hkv, w.d), np.uint16)
    cu = w.cu_seqlens()
    with _pool() as ex:
        for s, (L, seed) in enumerate(zip(w.lens, w.seeds)):
            qs, ks, vs = make_sequence(L, w.hq, w.hkv, w.d, seed, w.nvert, w.offsets, w.uniform_head_frac, ex)
            a, b = cu[s], cu[s + 1]
            q[a:b], k[a:b], v[a:b] = qs, ks, vs
    return {"q": q, "k": k, "v": v, "cu_seqlens": cu}


def random_inputs(lens: Sequence[int], hq: int, hkv: int, d: int, seed: int, scale: float = 1.0):
    """Plain N(0, scale^2) bf16 inputs for small edge-case tests (no vertical/slash structure)."""
    T = int(sum(lens))
    g = _rng(seed, 99, 0)
    q = to_bf16_bits(scale * g.standard_normal((T, hq, d), dtype=np.float32))
    k = to_bf16_bits(scale * g.standard_normal((T, hkv, d), dtype=np.float32))
    v = to_bf16_bits(g.standard_normal((T, hkv, d), dtype=np.float32))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return {"q": q, "k": k, "v": v, "cu_seqlens": cu}
