"""The C-ABI library loads, exports every entry point declared in include/fp.h, and rejects bad
arguments on the host before any launch (no GPU needed for any of these)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import block_sparse_long_causal_b200 as fp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "fp.h")) as f:
        return sorted(set(re.findall(r"FP_API\s+[\w\s\*]+?\b(fp_\w+)\s*\(", f.read())))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("fp_block_pool", "fp_block_search", "fp_block_sparse_attn", "fp_dense_attn"):
        assert n in names
    assert set(names) == set(fp.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(fp.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert fp.version() >= 100


def _prob(cu=(0, 300), hq=4, hkv=2, d=128, B=128):
    p = fp.fp_problem()
    host = np.array(cu, np.int32)
    st = fp._lib.fp_problem_init(C.byref(p), host.ctypes.data_as(C.c_void_p), len(host) - 1, C.c_void_p(16),
                                 hq, hkv, d, B)
    return st, p


def _err():
    return fp._lib.fp_last_error().decode()


def test_problem_init_sizes():
    st, p = _prob((0, 300, 301, 700), hq=3, hkv=1, B=64)
    assert st == fp.FP_OK
    assert p.total_tokens == 700 and p.total_blocks == 5 + 1 + 7 and p.max_seq_blocks == 7
    assert p.index_elems == 3 * (15 + 1 + 28)


@pytest.mark.parametrize("kw,status", [
    (dict(d=64), fp.FP_ERR_UNSUPPORTED),
    (dict(B=32), fp.FP_ERR_UNSUPPORTED),
    (dict(hq=6, hkv=4), fp.FP_ERR_INVALID_ARG),
    (dict(hq=0, hkv=1), fp.FP_ERR_INVALID_ARG),
    (dict(cu=(1, 5)), fp.FP_ERR_INVALID_ARG),
    (dict(cu=(0, 9, 5)), fp.FP_ERR_INVALID_ARG),
    (dict(hq=128, hkv=1), fp.FP_ERR_UNSUPPORTED),
])
def test_problem_init_rejects(kw, status):
    st, _ = _prob(**kw)
    assert st == status, _err()
    assert _err()


def test_problem_init_rejects_too_many_sequences():
    st, _ = _prob(cu=tuple(range(fp.FP_MAX_SEQS + 2)))
    assert st == fp.FP_ERR_INVALID_ARG


def test_work_counter_is_null_after_init_and_checked_for_alignment():
    st, p = _prob()
    assert st == fp.FP_OK and not p.sched
    ok, null = C.c_void_p(4096), None
    p.sched = 4098  # not 4-byte aligned: rejected on the host, before any launch
    for dense in (False, True):
        if dense:
            r = fp._lib.fp_dense_attn(C.byref(p), ok, ok, ok, C.c_float(0), ok, null, null, null)
        else:
            r = fp._lib.fp_block_sparse_attn(C.byref(p), ok, ok, ok, ok, ok, C.c_float(0), ok, null, null, null)
        assert r == fp.FP_ERR_INVALID_ARG and "sched" in _err()


def test_empty_sequences_are_allowed():
    st, p = _prob(cu=(0, 0, 5, 5))
    assert st == fp.FP_OK and p.total_blocks == 1


def test_calls_reject_bad_arguments_before_launch():
    st, p = _prob()
    assert st == fp.FP_OK
    ok = C.c_void_p(4096)
    mis = C.c_void_p(4098)
    null = None
    pr = C.byref(p)
    s = None
    assert fp._lib.fp_block_pool(pr, null, ok, ok, ok, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_pool(pr, mis, ok, ok, ok, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_search(pr, ok, ok, C.c_float(float("nan")), ok, ok, null, s) == fp.FP_ERR_INVALID_ARG
    assert "tau" in _err()
    assert fp._lib.fp_block_search(pr, ok, ok, C.c_float(float("inf")), ok, ok, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_search(pr, ok, null, C.c_float(0.1), ok, ok, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_sparse_attn(pr, ok, ok, ok, null, ok, C.c_float(0), ok, null, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_sparse_attn(pr, ok, ok, mis, ok, ok, C.c_float(0), ok, null, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_dense_attn(pr, ok, ok, ok, C.c_float(float("nan")), ok, null, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_dense_attn(None, ok, ok, ok, C.c_float(0), ok, null, null, s) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_validate_lists(pr, ok, ok, null, s) == fp.FP_ERR_INVALID_ARG
    # a problem edited into an unsupported state is rejected by every call
    p.head_dim = 96
    assert fp._lib.fp_dense_attn(pr, ok, ok, ok, C.c_float(0), ok, null, null, s) == fp.FP_ERR_UNSUPPORTED


def test_binding_raises_fp_error():
    with pytest.raises(fp.FpError):
        fp.Problem(np.array([0, 10], np.int32), __import__("torch").zeros(2, dtype=__import__("torch").int32),
                   4, 2, 64, 128)


def test_sparse_prefill_workspace_and_argument_checks():
    st, p = _prob((0, 300, 301, 700), hq=4, hkv=2, B=128)
    assert st == fp.FP_OK
    n = C.c_int64(0)
    assert fp._lib.fp_sparse_prefill_workspace(C.byref(p), C.byref(n)) == fp.FP_OK
    nb = 3 + 1 + 4
    need = 0
    for nbytes in (nb * 4 * 128 * 4, nb * 2 * 128 * 4, 4 * nb * 4, p.index_elems * 4, fp.FP_SCHED_WORDS * 4,
                   nb * 2 * 512, nb * 2 * 4):  # ..., the work counter, the key split rows and their norms
        need += (nbytes + 255) // 256 * 256
    assert n.value == need
    ok, null = C.c_void_p(4096), None
    args = lambda ws, nbytes: (C.byref(p), ok, ok, ok, C.c_float(0.1), C.c_float(0), ws, nbytes, ok, null, null, null)
    assert fp._lib.fp_sparse_prefill(*args(null, n.value)) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_sparse_prefill(*args(C.c_void_p(4096 + 16), n.value)) == fp.FP_ERR_INVALID_ARG  # not 256-aligned
    assert fp._lib.fp_sparse_prefill(*args(ok, n.value - 1)) == fp.FP_ERR_INVALID_ARG
    assert "workspace" in _err()


def _paged(cu=(0, 300, 500), prefixes=(256, 0), hq=4, B=128, max_pages=8, page_size=256, num_pages=16):
    st, p = _prob(cu, hq=hq, hkv=2, B=B)
    assert st == fp.FP_OK
    c = fp.fp_paged_cache()
    host_cu = np.array(cu, np.int32)
    pre = np.array(prefixes, np.int32)
    st = fp._lib.fp_paged_cache_init(C.byref(c), C.byref(p), host_cu.ctypes.data_as(C.c_void_p),
                                     pre.ctypes.data_as(C.c_void_p), C.c_void_p(64), C.c_void_p(128), max_pages,
                                     page_size, num_pages)
    return st, p, c


def test_paged_cache_init_sizes():
    # sequence 0: 300 new tokens after 256 cached (pb 2, nb 3); sequence 1: 200 tokens, no prefix (nb 2)
    st, p, c = _paged()
    assert st == fp.FP_OK, _err()
    assert c.total_kv_blocks == (2 + 3) + (0 + 2)
    # trapezoidal rows: hq * (nb*pb + nb(nb+1)/2) per sequence
    assert c.index_elems == 4 * (3 * 2 + 6) + 4 * (0 + 3)
    assert c.page_size == 256 and c.max_pages == 8 and c.num_pages == 16


@pytest.mark.parametrize("kw,status", [
    (dict(prefixes=(200, 0)), fp.FP_ERR_INVALID_ARG),       # prefix not a multiple of B
    (dict(prefixes=(-128, 0)), fp.FP_ERR_INVALID_ARG),
    (dict(page_size=192), fp.FP_ERR_UNSUPPORTED),           # page not a multiple of B = 128
    (dict(page_size=0), fp.FP_ERR_UNSUPPORTED),
    (dict(max_pages=2), fp.FP_ERR_INVALID_ARG),             # sequence 0 needs ceil(556 / 256) = 3 pages
    (dict(num_pages=0), fp.FP_ERR_INVALID_ARG),
    (dict(num_pages=1 << 24, page_size=256), fp.FP_ERR_INVALID_ARG),  # rows past 2^31 - 1
])
def test_paged_cache_init_rejects(kw, status):
    st, _, _ = _paged(**kw)
    assert st == status, _err()


def test_paged_calls_reject_a_null_cache_before_launch():
    st, p = _prob()
    ok = C.c_void_p(4096)
    assert fp._lib.fp_paged_block_pool(C.byref(p), None, ok, ok, ok, ok, None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_paged_block_search(C.byref(p), None, ok, ok, C.c_float(0.1), ok, ok, None,
                                         None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_paged_block_sparse_attn(C.byref(p), None, ok, ok, ok, ok, ok, C.c_float(0.0), ok, None, None,
                                              None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_paged_dense_attn(C.byref(p), None, ok, ok, ok, C.c_float(0.0), ok, None, None,
                                       None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_paged_validate_lists(C.byref(p), None, ok, ok, ok, None) == fp.FP_ERR_INVALID_ARG
    assert "cache" in _err()


def test_paged_calls_check_the_cache_and_arguments():
    st, p, c = _paged()
    assert st == fp.FP_OK
    ok = C.c_void_p(4096)
    # NULL q: rejected on the host
    assert fp._lib.fp_paged_block_pool(C.byref(p), C.byref(c), None, ok, ok, ok, None) == fp.FP_ERR_INVALID_ARG
    # a hand-edited cache inconsistent with the problem
    c.page_size = 100
    assert fp._lib.fp_paged_block_pool(C.byref(p), C.byref(c), ok, ok, ok, ok, None) == fp.FP_ERR_INVALID_ARG


def test_fp8_blockscaled_calls_reject_missing_exponents_before_launch():
    st, p = _prob((0, 300), hq=4, hkv=2, B=128)
    ok = C.c_void_p(4096)
    assert fp._lib.fp_block_sparse_attn_fp8_blockscaled(C.byref(p), ok, ok, ok, None, ok, ok, ok, C.c_float(0.0), ok,
                                                        None, None, None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_dense_attn_fp8_blockscaled(C.byref(p), ok, ok, ok, ok, None, C.c_float(0.0), ok, None, None,
                                                 None) == fp.FP_ERR_INVALID_ARG


def test_fp8_calls_reject_bad_scales_before_launch():
    st, p = _prob()
    ok = C.c_void_p(4096)
    for qs, ks in ((0.0, 1.0), (1.0, -2.0), (float("nan"), 1.0), (1.0, float("inf")), (1e30, 1e30)):
        assert fp._lib.fp_block_sparse_attn_fp8(C.byref(p), ok, ok, ok, C.c_float(qs), C.c_float(ks), ok, ok,
                                                C.c_float(0.0), ok, None, None, None) == fp.FP_ERR_INVALID_ARG
        assert fp._lib.fp_dense_attn_fp8(C.byref(p), ok, ok, ok, C.c_float(qs), C.c_float(ks), C.c_float(0.0), ok,
                                         None, None, None) == fp.FP_ERR_INVALID_ARG
    assert "scale" in _err()


def test_topp_rejects_bad_arguments_before_launch():
    st, p = _prob()
    ok = C.c_void_p(4096)
    assert fp._lib.fp_block_search_topp(C.byref(p), ok, ok, C.c_float(float("nan")), ok, ok, ok, None,
                                        None) == fp.FP_ERR_INVALID_ARG
    assert fp._lib.fp_block_search_topp(C.byref(p), ok, ok, C.c_float(0.9), None, ok, ok, None,
                                        None) == fp.FP_ERR_INVALID_ARG


@pytest.mark.parametrize("lens,B,hq", [([300], 128, 4), ([300, 1, 400, 0], 64, 3), ([131072], 128, 32),
                                       ([4096, 8192, 16384, 32768, 65536, 4096, 131072, 2048], 128, 32)])
def test_index_buffer_elems_is_the_triangular_count(lens, B, hq):
    nb = [(L + B - 1) // B for L in lens]
    want = sum(hq * n * (n + 1) // 2 for n in nb)
    assert fp.index_buffer_elems(lens, B, hq) == want
    st, p = _prob(tuple(np.concatenate([[0], np.cumsum(lens)]).tolist()), hq=hq, hkv=1, B=B)
    assert st == fp.FP_OK and p.index_elems == want


@pytest.mark.parametrize("lens,B,hq,status", [([], 128, 4, fp.FP_ERR_INVALID_ARG),
                                              ([5, -1], 128, 4, fp.FP_ERR_INVALID_ARG),
                                              ([5], 128, 0, fp.FP_ERR_INVALID_ARG),
                                              ([5], 96, 4, fp.FP_ERR_UNSUPPORTED)])
def test_index_buffer_elems_rejects(lens, B, hq, status):
    arr = np.array(lens if lens else [0], np.int32)
    n = C.c_int64(-7)
    st = fp._lib.fp_index_buffer_elems(arr.ctypes.data_as(C.c_void_p), len(lens), B, hq, C.byref(n))
    assert st == status and _err()
    assert n.value == -7
    assert fp._lib.fp_index_buffer_elems(None, 1, 128, 4, C.byref(n)) == fp.FP_ERR_INVALID_ARG


@pytest.mark.parametrize("bits,status,words", [
    (0, fp.FP_OK, []),
    (fp.FP_DEV_TIMEOUT, fp.FP_ERR_TIMEOUT, ["bounded wait"]),
    (fp.FP_DEV_BAD_LIST, fp.FP_ERR_INVALID_ARG, ["out of range"]),
    (fp.FP_DEV_BAD_PROBLEM, fp.FP_ERR_INVALID_ARG, ["sequence tables"]),
    (fp.FP_DEV_TIMEOUT | fp.FP_DEV_BAD_LIST, fp.FP_ERR_TIMEOUT, ["bounded wait", "out of range"]),
])
def test_check_device_status_maps_the_device_bits(bits, status, words):
    assert fp._lib.fp_check_device_status(bits) == status
    if status != fp.FP_OK:
        msg = _err()
        assert all(w in msg for w in words), msg
        with pytest.raises(fp.FpError) as e:
            fp.check_device_status(bits)
        assert e.value.status == status
    else:
        fp.check_device_status(0)


def test_struct_layouts_match_the_header(tmp_path):
    """ctypes mirrors of fp_problem and fp_paged_cache have the C sizes and offsets (the header
    compiled by the host C compiler), and the ABI version is at least the one of this layout."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = {"fp_problem": [f[0] for f in fp.fp_problem._fields_],
              "fp_paged_cache": [f[0] for f in fp.fp_paged_cache._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "fp.h"', "int main(void) {"]
    for st, fl in fields.items():
        lines.append(f'  printf("{st} size %zu\\n", sizeof({st}));')
        for f in fl:
            lines.append(f'  printf("{st} {f} %zu\\n", offsetof({st}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = dict(line.rsplit(" ", 1) for line in subprocess.check_output([str(exe)], text=True).splitlines())
    for st, cls in (("fp_problem", fp.fp_problem), ("fp_paged_cache", fp.fp_paged_cache)):
        assert int(got[f"{st} size"]) == C.sizeof(cls)
        for f in fields[st]:
            assert int(got[f"{st} {f}"]) == getattr(cls, f).offset, (st, f)
    assert C.sizeof(fp.fp_problem) == 72 and C.sizeof(fp.fp_paged_cache) == 40
    assert fp.version() >= 500  # this layout of fp_problem (with sched, key_split) since 0.5.0


def test_key_split_sizes_and_checks():
    """fp_key_split_bytes: 512 bytes (bf16 hi + lo of 128 dims) and one float per (key block, kv-head),
    each part 256-byte aligned; the paged size counts the cached prefixes' key blocks. A search whose
    key_split is misaligned or too small is refused on the host, before any launch."""
    st, p = _prob((0, 300, 301, 700), hq=4, hkv=2, B=128)
    assert st == fp.FP_OK
    n = C.c_int64(0)
    assert fp._lib.fp_key_split_bytes(C.byref(p), None, C.byref(n)) == fp.FP_OK
    nb = 3 + 1 + 4
    rup = lambda x: (x + 255) // 256 * 256
    assert n.value == rup(nb * 2 * 512) + rup(nb * 2 * 4)
    assert fp._lib.fp_key_split_bytes(C.byref(p), None, None) == fp.FP_ERR_INVALID_ARG
    st, pp, c = _paged(cu=(0, 300, 500), prefixes=(256, 0))
    assert st == fp.FP_OK
    assert fp._lib.fp_key_split_bytes(C.byref(pp), C.byref(c), C.byref(n)) == fp.FP_OK
    nbk = (256 + 300 + 127) // 128 + (200 + 127) // 128
    assert n.value == rup(nbk * 2 * 512) + rup(nbk * 2 * 4)
    ok = C.c_void_p(4096)
    need = rup(nb * 2 * 512) + rup(nb * 2 * 4)
    search = lambda: fp._lib.fp_block_search(C.byref(p), ok, ok, C.c_float(0.5), ok, ok, None, None)
    p.key_split, p.key_split_bytes = 4096 + 16, need
    assert search() == fp.FP_ERR_INVALID_ARG and "key_split" in _err()
    p.key_split, p.key_split_bytes = 4096, need - 1
    assert search() == fp.FP_ERR_INVALID_ARG and "key_split" in _err()
