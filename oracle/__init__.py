"""ctypes wrapper of the fp64 CPU oracle (fp_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline /
reference legs are the only callers. The CUDA product path never imports this package, and
the C source shares nothing with the CUDA sources.

The oracle restates the FlashPrefill block search (mean pooling, pooled block scores,
causal softmax with the max-based threshold, forced sink and diagonal blocks, ascending
index lists) and computes exact fp64 softmax attention over a given block mask.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libfp_oracle.so")
_lock = threading.Lock()
_lib = None

TIE_BAND_REL = 1e-4  # blocks with |p/max p - tau| <= 1e-4 * tau are exempt from exact list parity


def build(force: bool = False) -> str:
    """Compile fp_oracle.c with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            i32p, i64p = C.POINTER(C.c_int32), C.POINTER(C.c_int64)
            f64p, u16p, u8p = C.POINTER(C.c_double), C.POINTER(C.c_uint16), C.POINTER(C.c_uint8)
            L.orc_max_threads.restype = C.c_int
            L.orc_total_blocks.restype = C.c_int64
            L.orc_total_blocks.argtypes = [i32p, C.c_int, C.c_int]
            L.orc_index_elems.restype = C.c_int64
            L.orc_index_elems.argtypes = [i32p, C.c_int, C.c_int, C.c_int]
            L.orc_pool.restype = C.c_int
            L.orc_pool.argtypes = [u16p, i32p, C.c_int, C.c_int, C.c_int, C.c_int, f64p]
            L.orc_pooled_row.restype = C.c_int
            L.orc_pooled_row.argtypes = [f64p, f64p, i32p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                         C.c_int, C.c_int, C.c_int64, f64p, f64p, f64p]
            L.orc_search.restype = C.c_int
            L.orc_search.argtypes = [f64p, f64p, i32p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                     C.c_double, C.c_double, i32p, i32p, u8p]
            L.orc_search_topp.restype = C.c_int
            L.orc_search_topp.argtypes = [f64p, f64p, i32p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                          C.c_double, C.c_double, i32p, i32p, u8p]
            L.orc_attn_rows.restype = C.c_int
            L.orc_attn_rows.argtypes = [u16p, u16p, u16p, i32p, C.c_int, C.c_int, C.c_int, C.c_int,
                                        C.c_int, C.c_double, i32p, i32p, C.c_int64, i64p, i32p, f64p, f64p]
            _lib = L
    return _lib


def _p(a, t):
    return a.ctypes.data_as(C.POINTER(t)) if a is not None else None


def max_threads() -> int:
    return int(lib().orc_max_threads())


def total_blocks(cu: np.ndarray, B: int) -> int:
    cu = np.ascontiguousarray(cu, np.int32)
    return int(lib().orc_total_blocks(_p(cu, C.c_int32), len(cu) - 1, B))


def index_elems(cu: np.ndarray, B: int, hq: int) -> int:
    cu = np.ascontiguousarray(cu, np.int32)
    return int(lib().orc_index_elems(_p(cu, C.c_int32), len(cu) - 1, B, hq))


def pool(x: np.ndarray, cu: np.ndarray, B: int) -> np.ndarray:
    """Block means of bf16 bits x [T, H, d] -> float64 [NB, H, d]."""
    x = np.ascontiguousarray(x, np.uint16)
    cu = np.ascontiguousarray(cu, np.int32)
    T, H, d = x.shape
    out = np.empty((total_blocks(cu, B), H, d), np.float64)
    lib().orc_pool(_p(x, C.c_uint16), _p(cu, C.c_int32), len(cu) - 1, H, d, B, _p(out, C.c_double))
    return out


def pooled_row(qbar, kbar, cu, B, s, h, i):
    """(scores, p, p / max p) over j = 0..i for one (sequence, q-head, query block)."""
    qbar = np.ascontiguousarray(qbar, np.float64)
    kbar = np.ascontiguousarray(kbar, np.float64)
    cu = np.ascontiguousarray(cu, np.int32)
    hq, hkv, d = qbar.shape[1], kbar.shape[1], qbar.shape[2]
    sc, p, r = (np.empty(i + 1) for _ in range(3))
    rc = lib().orc_pooled_row(_p(qbar, C.c_double), _p(kbar, C.c_double), _p(cu, C.c_int32), len(cu) - 1,
                              B, hq, hkv, d, s, h, i, _p(sc, C.c_double), _p(p, C.c_double), _p(r, C.c_double))
    if rc:
        raise ValueError("bad pooled_row arguments")
    return sc, p, r


def search(qbar, kbar, cu, B: int, tau: float, want_band: bool = True):
    """Threshold + index emission.

    Returns (counts int32 [Hq, NB], indices int32 [index_elems], band uint8 [index_elems] or None).
    """
    qbar = np.ascontiguousarray(qbar, np.float64)
    kbar = np.ascontiguousarray(kbar, np.float64)
    cu = np.ascontiguousarray(cu, np.int32)
    hq, hkv, d = qbar.shape[1], kbar.shape[1], qbar.shape[2]
    nb = total_blocks(cu, B)
    n = index_elems(cu, B, hq)
    counts = np.zeros((hq, nb), np.int32)
    indices = np.full(n, -1, np.int32)
    band = np.zeros(n, np.uint8) if want_band else None
    rc = lib().orc_search(_p(qbar, C.c_double), _p(kbar, C.c_double), _p(cu, C.c_int32), len(cu) - 1, B,
                          hq, hkv, d, float(tau), TIE_BAND_REL, _p(counts, C.c_int32), _p(indices, C.c_int32),
                          _p(band, C.c_uint8))
    if rc:
        raise ValueError("bad search arguments")
    return counts, indices, band


def search_topp(qbar, kbar, cu, B: int, gamma: float, want_band: bool = True):
    """Cumulative top-p block selection on the pooled softmax (the comparison selector).

    Block j of row (h, i) is kept iff the probability mass of the strictly more probable blocks is
    below gamma (blocks tied at the cut kept together), plus the sink and the diagonal.
    Returns (counts, indices, band) in the layout of search().
    """
    qbar = np.ascontiguousarray(qbar, np.float64)
    kbar = np.ascontiguousarray(kbar, np.float64)
    cu = np.ascontiguousarray(cu, np.int32)
    hq, hkv, d = qbar.shape[1], kbar.shape[1], qbar.shape[2]
    nb = total_blocks(cu, B)
    n = index_elems(cu, B, hq)
    counts = np.zeros((hq, nb), np.int32)
    indices = np.full(n, -1, np.int32)
    band = np.zeros(n, np.uint8) if want_band else None
    rc = lib().orc_search_topp(_p(qbar, C.c_double), _p(kbar, C.c_double), _p(cu, C.c_int32), len(cu) - 1, B,
                               hq, hkv, d, float(gamma), TIE_BAND_REL, _p(counts, C.c_int32),
                               _p(indices, C.c_int32), _p(band, C.c_uint8))
    if rc:
        raise ValueError("bad search_topp arguments")
    return counts, indices, band


def attn_rows(q, k, v, cu, B: int, rows_tok, rows_head, counts=None, indices=None, scale: float = 0.0):
    """Exact fp64 attention for sampled (token, q-head) rows over a block mask.

    counts/indices None -> dense causal attention. Returns (out float64 [n, d], lse float64 [n]).
    """
    q = np.ascontiguousarray(q, np.uint16)
    k = np.ascontiguousarray(k, np.uint16)
    v = np.ascontiguousarray(v, np.uint16)
    cu = np.ascontiguousarray(cu, np.int32)
    rt = np.ascontiguousarray(rows_tok, np.int64)
    rh = np.ascontiguousarray(rows_head, np.int32)
    hq, hkv, d = q.shape[1], k.shape[1], q.shape[2]
    if counts is not None:
        counts = np.ascontiguousarray(counts, np.int32)
        indices = np.ascontiguousarray(indices, np.int32)
    out = np.empty((len(rt), d), np.float64)
    lse = np.empty(len(rt), np.float64)
    rc = lib().orc_attn_rows(_p(q, C.c_uint16), _p(k, C.c_uint16), _p(v, C.c_uint16), _p(cu, C.c_int32),
                             len(cu) - 1, B, hq, hkv, d, float(scale), _p(counts, C.c_int32),
                             _p(indices, C.c_int32), len(rt), _p(rt, C.c_int64), _p(rh, C.c_int32),
                             _p(out, C.c_double), _p(lse, C.c_double))
    if rc:
        raise ValueError("bad attn_rows arguments (row out of range or malformed index list)")
    return out, lse


def row_offset(cu, B: int, hq: int, s: int, h: int, i: int) -> int:
    """Start of row (s, h, i) in the triangular index buffer."""
    cu = np.asarray(cu, np.int64)
    base = 0
    for t in range(s):
        nbt = (int(cu[t + 1] - cu[t]) + B - 1) // B
        base += hq * nbt * (nbt + 1) // 2
    nbs = (int(cu[s + 1] - cu[s]) + B - 1) // B
    return base + h * nbs * (nbs + 1) // 2 + i * (i + 1) // 2


def block_base(cu, B: int, s: int) -> int:
    """Global id of block 0 of sequence s."""
    cu = np.asarray(cu, np.int64)
    return int(sum((int(cu[t + 1] - cu[t]) + B - 1) // B for t in range(s)))


def lists_as_sets(counts, indices, cu, B: int, hq: int):
    """Decode (counts, indices) into {(s, h, i): tuple(blocks)} for comparisons."""
    out = {}
    cu = np.asarray(cu, np.int64)
    for s in range(len(cu) - 1):
        nbs = (int(cu[s + 1] - cu[s]) + B - 1) // B
        gb0 = block_base(cu, B, s)
        for h in range(hq):
            for i in range(nbs):
                off = row_offset(cu, B, hq, s, h, i)
                n = int(counts[h, gb0 + i])
                out[(s, h, i)] = tuple(int(x) for x in indices[off:off + n])
    return out
