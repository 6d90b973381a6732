"""Thin Python binding of libfp (FlashPrefill-style block-sparse causal prefill on sm_100a).

Argument marshalling only: every step of the path (pooling, search, attention) runs in the
CUDA kernels of libfp.so; PyTorch supplies device memory and the current stream. There is no
CPU or PyTorch fallback: importing this module without the built library raises.

Entry points mirror the C ABI in include/fp.h:
    problem(...)            -> Problem (fp_problem_init)
    index_buffer_elems(...) -> fp_index_buffer_elems (index buffer length from sequence lengths)
    check_device_status(..) -> fp_check_device_status (dev_status word -> FpError)
    block_pool(...)         -> fp_block_pool
    block_search(...)       -> fp_block_search
    block_search_topp(...)  -> fp_block_search_topp (the cumulative top-p comparison selector)
    block_pool_search(...)  -> fp_block_pool_search (steps 1 + 2 fused)
    block_sparse_attn(...)  -> fp_block_sparse_attn
    block_sparse_attn_fp8 / dense_attn_fp8 -> e4m3 Q / K attention, per-tensor scales (fp_*_fp8)
    block_sparse_attn_fp8_blockscaled / dense_attn_fp8_blockscaled -> per-block power-of-two scales
    dense_attn(...)         -> fp_dense_attn
    sparse_prefill(...)     -> fp_sparse_prefill (all three steps, caller workspace)
    validate_lists(...)     -> fp_validate_lists
    paged_cache(...)        -> PagedCache (fp_paged_cache_init: chunked prefill onto a paged K/V cache)
    paged_block_pool / paged_block_search / paged_block_sparse_attn / paged_dense_attn /
    paged_validate_lists    -> the fp_paged_* calls
and SparsePrefill bundles the three steps with caller-side buffers.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp.so")

FP_OK, FP_ERR_INVALID_ARG, FP_ERR_UNSUPPORTED, FP_ERR_CUDA, FP_ERR_TIMEOUT = 0, 1, 2, 3, 4
FP_DEV_TIMEOUT, FP_DEV_BAD_LIST, FP_DEV_BAD_PROBLEM = 1, 2, 4
FP_MAX_SEQS = 1024
FP_SCHED_WORDS = 2  # int32 words of the attention work counter (fp_problem.sched)
FP_NOALLOC_MAX_BYTES = 64 << 20
EXPORTED = ("fp_problem_init", "fp_block_pool", "fp_block_search", "fp_block_pool_search", "fp_block_sparse_attn",
            "fp_dense_attn", "fp_sparse_prefill_workspace", "fp_sparse_prefill", "fp_sparse_prefill_noalloc",
            "fp_validate_lists", "fp_selftest_exp2", "fp_last_error", "fp_version", "fp_paged_cache_init",
            "fp_paged_block_pool", "fp_paged_block_search", "fp_paged_block_sparse_attn", "fp_paged_dense_attn",
            "fp_paged_validate_lists", "fp_block_search_topp", "fp_block_sparse_attn_fp8", "fp_dense_attn_fp8",
            "fp_index_buffer_elems", "fp_check_device_status", "fp_key_split_bytes", "fp_block_sparse_attn_fp8_blockscaled",
            "fp_dense_attn_fp8_blockscaled")


class FpError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"fp status {status}: {msg}")
        self.status = status


class fp_problem(C.Structure):
    _fields_ = [("cu_seqlens", C.c_void_p), ("num_seqs", C.c_int32), ("total_tokens", C.c_int32),
                ("total_blocks", C.c_int32), ("max_seq_blocks", C.c_int32), ("index_elems", C.c_int64),
                ("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("block_size", C.c_int32), ("sched", C.c_void_p), ("key_split", C.c_void_p),
                ("key_split_bytes", C.c_int64)]


class fp_paged_cache(C.Structure):
    _fields_ = [("prefix_lens", C.c_void_p), ("block_table", C.c_void_p), ("max_pages", C.c_int32),
                ("page_size", C.c_int32), ("num_pages", C.c_int32), ("total_kv_blocks", C.c_int32),
                ("index_elems", C.c_int64)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libfp.so is not built ({LIB_PATH}); run python block_sparse_long_causal_b200/build.py")
    lib = C.CDLL(LIB_PATH)
    vp, i32, f32 = C.c_void_p, C.c_int32, C.c_float
    P = C.POINTER(fp_problem)
    PC = C.POINTER(fp_paged_cache)
    sig = {
        "fp_paged_cache_init": [PC, P, vp, vp, vp, vp, i32, i32, i32],
        "fp_block_search_topp": [P, vp, vp, f32, vp, vp, vp, vp, vp],
        "fp_block_sparse_attn_fp8": [P, vp, vp, vp, f32, f32, vp, vp, f32, vp, vp, vp, vp],
        "fp_dense_attn_fp8": [P, vp, vp, vp, f32, f32, f32, vp, vp, vp, vp],
        "fp_block_sparse_attn_fp8_blockscaled": [P, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_dense_attn_fp8_blockscaled": [P, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_paged_block_pool": [P, PC, vp, vp, vp, vp, vp],
        "fp_paged_block_search": [P, PC, vp, vp, f32, vp, vp, vp, vp],
        "fp_paged_block_sparse_attn": [P, PC, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_paged_dense_attn": [P, PC, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_paged_validate_lists": [P, PC, vp, vp, vp, vp],
        "fp_problem_init": [P, vp, i32, vp, i32, i32, i32, i32],
        "fp_block_pool": [P, vp, vp, vp, vp, vp],
        "fp_block_search": [P, vp, vp, f32, vp, vp, vp, vp],
        "fp_block_pool_search": [P, vp, vp, f32, vp, vp, vp, vp, vp, vp],
        "fp_block_sparse_attn": [P, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_dense_attn": [P, vp, vp, vp, f32, vp, vp, vp, vp],
        "fp_validate_lists": [P, vp, vp, vp, vp],
        "fp_selftest_exp2": [vp, vp, vp, C.c_int64, vp],
        "fp_sparse_prefill_workspace": [P, C.POINTER(C.c_int64)],
        "fp_sparse_prefill": [P, vp, vp, vp, f32, f32, vp, C.c_int64, vp, vp, vp, vp],
        "fp_sparse_prefill_noalloc": [P, vp, vp, vp, f32, f32, vp, vp, vp, vp],
        "fp_index_buffer_elems": [vp, i32, i32, i32, C.POINTER(C.c_int64)],
        "fp_check_device_status": [i32],
        "fp_key_split_bytes": [P, vp, C.POINTER(C.c_int64)],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = C.c_int
    lib.fp_last_error.restype = C.c_char_p
    lib.fp_last_error.argtypes = []
    lib.fp_version.restype = C.c_int32
    lib.fp_version.argtypes = []
    return lib


_lib = _load()


def version() -> int:
    return int(_lib.fp_version())


def _check(st: int):
    if st != FP_OK:
        raise FpError(st, _lib.fp_last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return C.c_void_p(t.data_ptr())
    return C.c_void_p(int(t))


def _stream(stream):
    if stream is None:
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return C.c_void_p(stream.cuda_stream)
    return C.c_void_p(int(stream))


class Problem:
    """fp_problem plus the device tensors it points to (kept alive here): cu_seqlens and, with
    work_counter (the default on a CUDA device), the attention calls' work counter -- zeroed once,
    left at zero by every launch, so launches of this problem must be ordered (one stream, or
    events); give concurrent streams one Problem each. With key_split (the default on a CUDA device)
    the searches of the plain problem split the pooled keys once per call into a scratch buffer held
    here (fp_problem.key_split)."""

    def __init__(self, cu_seqlens_host, cu_seqlens_dev: torch.Tensor, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, work_counter: bool = True, key_split: bool = True):
        host = np.ascontiguousarray(cu_seqlens_host, np.int32)
        if cu_seqlens_dev.dtype != torch.int32:
            raise ValueError("cu_seqlens must be int32")
        self.cu_host = host
        self.cu_dev = cu_seqlens_dev
        self.c = fp_problem()
        _check(_lib.fp_problem_init(C.byref(self.c), host.ctypes.data_as(C.c_void_p), len(host) - 1,
                                    _ptr(cu_seqlens_dev), num_q_heads, num_kv_heads, head_dim, block_size))
        self.sched = None
        if work_counter and cu_seqlens_dev.is_cuda:
            self.sched = torch.zeros(FP_SCHED_WORDS, dtype=torch.int32, device=cu_seqlens_dev.device)
            self.c.sched = self.sched.data_ptr()
        self.key_split = None
        if key_split and cu_seqlens_dev.is_cuda:
            nbytes = key_split_bytes(self)
            self.key_split = torch.empty(nbytes, dtype=torch.uint8, device=cu_seqlens_dev.device)
            self.c.key_split = self.key_split.data_ptr()
            self.c.key_split_bytes = nbytes

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def ref(self):
        return C.byref(self.c)


def problem(cu_seqlens_host, num_q_heads: int, num_kv_heads: int, head_dim: int = 128, block_size: int = 128,
            device="cuda", work_counter: bool = True, key_split: bool = True) -> Problem:
    host = np.ascontiguousarray(cu_seqlens_host, np.int32)
    dev = torch.from_numpy(host.copy()).to(device)
    return Problem(host, dev, num_q_heads, num_kv_heads, head_dim, block_size, work_counter, key_split)


def _cache_ref(cache):
    return cache.ref if isinstance(cache, PagedCache) else C.byref(cache)


def key_split_bytes(p, cache=None) -> int:
    """fp_key_split_bytes: bytes of the search's key split scratch for this problem (and paged cache)."""
    n = C.c_int64(0)
    ref = p.ref if isinstance(p, Problem) else C.byref(p)
    _check(_lib.fp_key_split_bytes(ref, None if cache is None else _cache_ref(cache), C.byref(n)))
    return int(n.value)


def index_buffer_elems(seqlens, block_size: int, num_q_heads: int) -> int:
    """fp_index_buffer_elems: int32 entries of the index buffer for these sequence lengths."""
    lens = np.ascontiguousarray(seqlens, np.int32)
    n = C.c_int64(0)
    _check(_lib.fp_index_buffer_elems(lens.ctypes.data_as(C.c_void_p), len(lens), int(block_size), int(num_q_heads),
                                      C.byref(n)))
    return int(n.value)


def check_device_status(bits: int) -> None:
    """fp_check_device_status: raise FpError (status FP_ERR_TIMEOUT / FP_ERR_INVALID_ARG) for a
    non-zero dev_status word read back after the stream completed."""
    _check(_lib.fp_check_device_status(int(bits)))


def block_pool(p: Problem, q, k, q_pool, k_pool, stream=None):
    _check(_lib.fp_block_pool(p.ref, _ptr(q), _ptr(k), _ptr(q_pool), _ptr(k_pool), _stream(stream)))


def block_search(p: Problem, q_pool, k_pool, tau: float, counts, indices, dev_status=None, stream=None):
    _check(_lib.fp_block_search(p.ref, _ptr(q_pool), _ptr(k_pool), float(tau), _ptr(counts), _ptr(indices),
                                _ptr(dev_status), _stream(stream)))


def block_search_topp(p: Problem, q_pool, k_pool, gamma: float, scores, counts, indices, dev_status=None,
                      stream=None):
    """Cumulative top-p block selection (the comparison selector); scores: float32 [index_elems] scratch."""
    _check(_lib.fp_block_search_topp(p.ref, _ptr(q_pool), _ptr(k_pool), float(gamma), _ptr(scores), _ptr(counts),
                                     _ptr(indices), _ptr(dev_status), _stream(stream)))


def block_pool_search(p: Problem, q, k, tau: float, q_pool, k_pool, counts, indices, dev_status=None, stream=None):
    _check(_lib.fp_block_pool_search(p.ref, _ptr(q), _ptr(k), float(tau), _ptr(q_pool), _ptr(k_pool), _ptr(counts),
                                     _ptr(indices), _ptr(dev_status), _stream(stream)))


def block_sparse_attn(p: Problem, q, k, v, counts, indices, softmax_scale: float, out, lse=None, dev_status=None,
                      stream=None):
    _check(_lib.fp_block_sparse_attn(p.ref, _ptr(q), _ptr(k), _ptr(v), _ptr(counts), _ptr(indices),
                                     float(softmax_scale), _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def block_sparse_attn_fp8(p: Problem, q_e4m3, k_e4m3, v, q_scale: float, k_scale: float, counts, indices,
                          softmax_scale: float, out, lse=None, dev_status=None, stream=None):
    """FP8 attention: e4m3 Q / K codes (uint8 tensors) with per-tensor scales, bf16 V."""
    _check(_lib.fp_block_sparse_attn_fp8(p.ref, _ptr(q_e4m3), _ptr(k_e4m3), _ptr(v), float(q_scale), float(k_scale),
                                         _ptr(counts), _ptr(indices), float(softmax_scale), _ptr(out), _ptr(lse),
                                         _ptr(dev_status), _stream(stream)))


def dense_attn_fp8(p: Problem, q_e4m3, k_e4m3, v, q_scale: float, k_scale: float, softmax_scale: float, out, lse=None,
                   dev_status=None, stream=None):
    _check(_lib.fp_dense_attn_fp8(p.ref, _ptr(q_e4m3), _ptr(k_e4m3), _ptr(v), float(q_scale), float(k_scale),
                                  float(softmax_scale), _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def block_sparse_attn_fp8_blockscaled(p: Problem, q_e4m3, k_e4m3, v, q_exp, k_exp, counts, indices,
                                      softmax_scale: float, out, lse=None, dev_status=None, stream=None):
    """FP8 attention with per-block power-of-two scales: q_exp int8 [total_blocks, Hq], k_exp int8
    [total_blocks, Hkv] (dequantised value = 2^exp * e4m3 code)."""
    _check(_lib.fp_block_sparse_attn_fp8_blockscaled(p.ref, _ptr(q_e4m3), _ptr(k_e4m3), _ptr(v), _ptr(q_exp),
                                                     _ptr(k_exp), _ptr(counts), _ptr(indices), float(softmax_scale),
                                                     _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def dense_attn_fp8_blockscaled(p: Problem, q_e4m3, k_e4m3, v, q_exp, k_exp, softmax_scale: float, out, lse=None,
                               dev_status=None, stream=None):
    _check(_lib.fp_dense_attn_fp8_blockscaled(p.ref, _ptr(q_e4m3), _ptr(k_e4m3), _ptr(v), _ptr(q_exp), _ptr(k_exp),
                                              float(softmax_scale), _ptr(out), _ptr(lse), _ptr(dev_status),
                                              _stream(stream)))


def dense_attn(p: Problem, q, k, v, softmax_scale: float, out, lse=None, dev_status=None, stream=None):
    _check(_lib.fp_dense_attn(p.ref, _ptr(q), _ptr(k), _ptr(v), float(softmax_scale), _ptr(out), _ptr(lse),
                              _ptr(dev_status), _stream(stream)))


def validate_lists(p: Problem, counts, indices, dev_status, stream=None):
    _check(_lib.fp_validate_lists(p.ref, _ptr(counts), _ptr(indices), _ptr(dev_status), _stream(stream)))


def sparse_prefill_workspace(p: Problem) -> int:
    n = C.c_int64(0)
    _check(_lib.fp_sparse_prefill_workspace(p.ref, C.byref(n)))
    return int(n.value)


def sparse_prefill(p: Problem, q, k, v, tau: float, softmax_scale: float, workspace, out, lse=None, dev_status=None,
                   stream=None):
    _check(_lib.fp_sparse_prefill(p.ref, _ptr(q), _ptr(k), _ptr(v), float(tau), float(softmax_scale),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse),
                                  _ptr(dev_status), _stream(stream)))


def sparse_prefill_noalloc(p: Problem, q, k, v, tau: float, softmax_scale: float, out, lse=None, dev_status=None,
                           stream=None):
    """fp_sparse_prefill for callers that cannot allocate: intermediates in the library's static array."""
    _check(_lib.fp_sparse_prefill_noalloc(p.ref, _ptr(q), _ptr(k), _ptr(v), float(tau), float(softmax_scale),
                                          _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def selftest_exp2(x, y_poly, y_mufu, stream=None):
    _check(_lib.fp_selftest_exp2(_ptr(x), _ptr(y_poly), _ptr(y_mufu), x.numel(), _stream(stream)))


class PagedCache:
    """fp_paged_cache plus the device prefix-length and block-table tensors it points to."""

    def __init__(self, p: Problem, prefix_lens_host, prefix_lens_dev: torch.Tensor, block_table_dev: torch.Tensor,
                 page_size: int, num_pages: int):
        pre = np.ascontiguousarray(prefix_lens_host, np.int32)
        if prefix_lens_dev.dtype != torch.int32 or block_table_dev.dtype != torch.int32:
            raise ValueError("prefix_lens and block_table must be int32")
        if block_table_dev.dim() != 2 or block_table_dev.shape[0] != p.num_seqs:
            raise ValueError("block_table must be [num_seqs, max_pages]")
        self.p = p
        self.prefix_host = pre
        self.prefix_dev = prefix_lens_dev
        self.table_dev = block_table_dev.contiguous()
        self.c = fp_paged_cache()
        _check(_lib.fp_paged_cache_init(C.byref(self.c), p.ref, p.cu_host.ctypes.data_as(C.c_void_p),
                                        pre.ctypes.data_as(C.c_void_p), _ptr(prefix_lens_dev), _ptr(self.table_dev),
                                        int(self.table_dev.shape[1]), int(page_size), int(num_pages)))
        # the paged search's key split covers the cached prefixes' key blocks too
        self.key_split = None
        if p.key_split is not None:
            nbytes = key_split_bytes(p, self)
            self.key_split = torch.empty(nbytes, dtype=torch.uint8, device=prefix_lens_dev.device)
            self.search_problem = fp_problem.from_buffer_copy(p.c)
            self.search_problem.key_split = self.key_split.data_ptr()
            self.search_problem.key_split_bytes = nbytes

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def ref(self):
        return C.byref(self.c)


def paged_cache(p: Problem, prefix_lens_host, block_table, page_size: int, num_pages: int, device="cuda") -> PagedCache:
    pre = np.ascontiguousarray(prefix_lens_host, np.int32)
    table = block_table if isinstance(block_table, torch.Tensor) else torch.from_numpy(
        np.ascontiguousarray(block_table, np.int32))
    return PagedCache(p, pre, torch.from_numpy(pre.copy()).to(device), table.to(device=device, dtype=torch.int32),
                      page_size, num_pages)


def paged_block_pool(p: Problem, c: PagedCache, q, k_cache, q_pool, k_pool, stream=None):
    _check(_lib.fp_paged_block_pool(p.ref, c.ref, _ptr(q), _ptr(k_cache), _ptr(q_pool), _ptr(k_pool), _stream(stream)))


def paged_block_search(p: Problem, c: PagedCache, q_pool, k_pool, tau: float, counts, indices, dev_status=None,
                       stream=None):
    ref = C.byref(c.search_problem) if c.key_split is not None and p is c.p else p.ref
    _check(_lib.fp_paged_block_search(ref, c.ref, _ptr(q_pool), _ptr(k_pool), float(tau), _ptr(counts),
                                      _ptr(indices), _ptr(dev_status), _stream(stream)))


def paged_block_sparse_attn(p: Problem, c: PagedCache, q, k_cache, v_cache, counts, indices, softmax_scale: float, out,
                            lse=None, dev_status=None, stream=None):
    _check(_lib.fp_paged_block_sparse_attn(p.ref, c.ref, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(counts),
                                           _ptr(indices), float(softmax_scale), _ptr(out), _ptr(lse), _ptr(dev_status),
                                           _stream(stream)))


def paged_dense_attn(p: Problem, c: PagedCache, q, k_cache, v_cache, softmax_scale: float, out, lse=None,
                     dev_status=None, stream=None):
    _check(_lib.fp_paged_dense_attn(p.ref, c.ref, _ptr(q), _ptr(k_cache), _ptr(v_cache), float(softmax_scale),
                                    _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


def paged_validate_lists(p: Problem, c: PagedCache, counts, indices, dev_status, stream=None):
    _check(_lib.fp_paged_validate_lists(p.ref, c.ref, _ptr(counts), _ptr(indices), _ptr(dev_status),
                                        _stream(stream)))


class SparsePrefill:
    """Caller-side buffers for one problem shape, and the three-step sparse prefill.

    Buffers are allocated once (through PyTorch) and reused by every call; the library itself
    never allocates.
    """

    def __init__(self, p: Problem, device="cuda", with_lse: bool = False):
        self.p = p
        nb, hq, hkv, d = p.total_blocks, p.num_q_heads, p.num_kv_heads, p.head_dim
        self.q_pool = torch.empty((max(nb, 1), hq, d), dtype=torch.float32, device=device)
        self.k_pool = torch.empty((max(nb, 1), hkv, d), dtype=torch.float32, device=device)
        self.counts = torch.zeros((hq, max(nb, 1)), dtype=torch.int32, device=device)
        self.indices = torch.zeros(max(p.index_elems, 1), dtype=torch.int32, device=device)
        self.out = torch.empty((max(p.total_tokens, 1), hq, d), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((hq, max(p.total_tokens, 1)), dtype=torch.float32, device=device) if with_lse else None
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=device)

    def search(self, q, k, tau: float, stream=None, fused: bool = True):
        if fused:
            block_pool_search(self.p, q, k, tau, self.q_pool, self.k_pool, self.counts, self.indices,
                              self.dev_status, stream)
        else:
            block_pool(self.p, q, k, self.q_pool, self.k_pool, stream)
            block_search(self.p, self.q_pool, self.k_pool, tau, self.counts, self.indices, self.dev_status, stream)

    def attend(self, q, k, v, softmax_scale: float = 0.0, stream=None):
        block_sparse_attn(self.p, q, k, v, self.counts, self.indices, softmax_scale, self.out, self.lse,
                          self.dev_status, stream)
        return self.out

    def __call__(self, q, k, v, tau: float, softmax_scale: float = 0.0, stream=None):
        self.search(q, k, tau, stream)
        return self.attend(q, k, v, softmax_scale, stream)

    def dense(self, q, k, v, softmax_scale: float = 0.0, stream=None):
        dense_attn(self.p, q, k, v, softmax_scale, self.out, self.lse, self.dev_status, stream)
        return self.out
