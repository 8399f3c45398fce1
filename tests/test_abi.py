"""The C-ABI library loads on a machine without a GPU, exports every entry
point of include/dsa.h, and rejects bad arguments on the host before any
CUDA call (pattern rule of the IndexCache explainer §1.1: the first layer
must be F).  CPU only."""
import ctypes
import os
import re

import pytest

from sparse_attention_13_b200 import dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z_]+)\s*\(", src)) - {"if", "sizeof"})


def test_library_exports_every_declared_symbol():
    lib = dsa.lib()
    names = _declared()
    assert "indexcache_forward" in names and "dsa_indexer_topk" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(dsa.EXPORTS) <= set(names)


def _fwd(pattern, n_layers=None, layers=None, dims=None, idx=1, ws=None, ws_bytes=0):
    lib = dsa.lib()
    n = len(pattern) if n_layers is None else n_layers
    arr = layers if layers is not None else (dsa.LayerIO * max(n, 1))()
    d = dims if dims is not None else dsa.Dims(B=1, Lq=8, Lk=8, start_pos=0, H_I=64, d_I=128, k=4,
                                              n_h=128, D_qk=576, D_v=512, scale=1.0,
                                              k_row_stride=576, v_row_stride=576)
    return lib.indexcache_forward(pattern.encode(), n, arr, ctypes.byref(d),
                                  ctypes.c_void_p(idx), ctypes.c_void_p(ws), ws_bytes, None)


@pytest.mark.parametrize("pattern", ["SFFF", "S", "FXSS", "fsss", "FF S"])
def test_bad_pattern_rejected(pattern):
    assert _fwd(pattern) == dsa.DSA_ERR_BAD_PATTERN
    assert dsa.lib().dsa_last_error()


def test_empty_pattern_rejected():
    assert _fwd("", n_layers=0) == dsa.DSA_ERR_BAD_PATTERN


def test_null_pointers_rejected_before_launch():
    # valid pattern, layer pointers all NULL
    d = dsa.Dims(B=1, Lq=8, Lk=8, start_pos=0, H_I=64, d_I=128, k=4, n_h=128, D_qk=576, D_v=512,
                 scale=1.0, k_row_stride=576, v_row_stride=576)
    need = dsa.lib().indexcache_forward_workspace(ctypes.byref(d))
    st = _fwd("FS", dims=d, ws=4096, ws_bytes=need)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_small_workspace_rejected():
    d = dsa.Dims(B=1, Lq=64, Lk=64, start_pos=0, H_I=64, d_I=128, k=16, n_h=128, D_qk=576, D_v=512,
                 scale=1.0, k_row_stride=576, v_row_stride=576)
    assert _fwd("FS", dims=d, ws=4096, ws_bytes=16) == dsa.DSA_ERR_WORKSPACE


def test_indexer_argument_checks():
    lib = dsa.lib()
    P = ctypes.c_void_p
    a = P(1 << 20)  # aligned, never dereferenced: the checks fail first
    # unsupported head count
    st = lib.dsa_indexer_topk(a, a, a, 1, 8, 8, 0, 12, 128, 4, a, a, 1 << 30, None)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    # k too large for the kernel
    st = lib.dsa_indexer_topk(a, a, a, 1, 8, 8, 0, 64, 128, 4096, a, a, 1 << 30, None)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    # query rows beyond the cache
    st = lib.dsa_indexer_topk(a, a, a, 1, 8, 8, 5, 64, 128, 4, a, a, 1 << 30, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    # misaligned pointer
    st = lib.dsa_indexer_topk(P((1 << 20) + 2), a, a, 1, 8, 8, 0, 64, 128, 4, a, a, 1 << 30, None)
    assert st == dsa.DSA_ERR_INVALID_ARG
    # null output
    st = lib.dsa_indexer_topk(a, a, a, 1, 8, 8, 0, 64, 128, 4, None, a, 1 << 30, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_attention_argument_checks():
    lib = dsa.lib()
    P = ctypes.c_void_p
    a = P(1 << 20)
    # unsupported head dims (not MLA, too wide for the small-dim kernel)
    st = lib.dsa_sparse_attn(a, a, 256, a, 256, a, 1, 8, 8, 0, 16, 256, 256, 4, 1.0, a, None, a,
                             1 << 20, None)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    # row stride shorter than the row
    st = lib.dsa_sparse_attn(a, a, 64, a, 576, a, 1, 8, 8, 0, 128, 576, 512, 4, 1.0, a, None, a,
                             1 << 20, None)
    assert st == dsa.DSA_ERR_INVALID_ARG


def test_workspace_sizes():
    lib = dsa.lib()
    small = lib.dsa_indexer_topk_workspace(1, 512, 512, 0, 4, 32, 64)
    big = lib.dsa_indexer_topk_workspace(1, 200000, 200000, 0, 64, 128, 2048)
    dec = lib.dsa_indexer_topk_workspace(8, 1, 200000, 200000, 64, 128, 2048)
    assert 0 < small < big
    assert dec > 0
    assert lib.dsa_indexer_topk_workspace(0, 1, 1, 0, 64, 128, 4) == 0


def test_launch_counter_starts_at_zero_without_launches():
    assert dsa.indexer_launch_count() >= 0


@pytest.mark.parametrize("limit", [0, -5, 3_000_000_000])
def test_selftest_limit_validated_on_host(limit):
    # the failure-detection self-test refuses out-of-range limits before any
    # CUDA call
    assert dsa.lib().dsa_selftest_wait_timeout(limit, None) == dsa.DSA_ERR_INVALID_ARG


def test_check_indices_validated_on_host():
    lib = dsa.lib()
    assert lib.dsa_check_indices(None, 1, 1, 0, 4, None, None) == dsa.DSA_ERR_INVALID_ARG
    fake = ctypes.c_void_p(16)  # never dereferenced: the sizes are refused first
    assert lib.dsa_check_indices(fake, 0, 1, 0, 4, fake, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_check_indices(fake, 1, 1, -1, 4, fake, None) == dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_check_indices(fake, 1, 1, 0, 0, fake, None) == dsa.DSA_ERR_INVALID_ARG


def test_selection_quality_tools_validated_on_host():
    lib = dsa.lib()
    fake = ctypes.c_void_p(16)  # never dereferenced: the arguments are refused first
    E = dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_dense_weights(None, fake, 576, 1, 1, 1, 0, 128, 576, 1.0, fake, None, None) == E
    assert lib.dsa_dense_weights(fake, fake, 576, 1, 3, 1, 0, 128, 576, 1.0, fake, None, None) == E
    assert lib.dsa_dense_weights(fake, fake, 576, 1, 1, 1, 0, 129, 576, 1.0, fake, None,
                                 None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_dense_weights(fake, fake, 576, 1, 1, 1, 0, 8, 100, 1.0, fake, None,
                                 None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_dense_weights(fake, fake, 60, 1, 1, 1, 0, 8, 64, 1.0, fake, None, None) == E
    assert lib.dsa_topk_rows(fake, 10, 1, 2, 10, 4, fake, None) == E     # t = 11 > row
    assert lib.dsa_topk_rows(fake, 10, 1, 2, 0, 0, fake, None) == E
    assert lib.dsa_index_overlap(fake, None, 4, 8, fake, None) == E
    assert lib.dsa_index_overlap(fake, fake, 0, 8, fake, None) == E
    assert lib.dsa_captured_mass(fake, fake, 0, fake, None) == E


def test_csa_entry_points_validated_on_host():
    lib = dsa.lib()
    fake = ctypes.c_void_p(16)  # never dereferenced: the arguments are refused first
    E = dsa.DSA_ERR_INVALID_ARG
    # (q, k_cmp, w, B, Lq, N_cmp, start_pos, m, H, d, k, idx, ws, ws_bytes, stream)
    assert lib.dsa_csa_indexer_topk(None, fake, fake, 1, 8, 2, 0, 4, 64, 128, 8, fake, fake, 1 << 20, None) == E
    assert lib.dsa_csa_indexer_topk(fake, fake, fake, 1, 8, 2, 0, 0, 64, 128, 8, fake, fake, 1 << 20, None) == E
    # floor((0 + 12 - 1) / 4) = 2 > N_cmp = 1
    assert lib.dsa_csa_indexer_topk(fake, fake, fake, 1, 12, 1, 0, 4, 64, 128, 8, fake, fake, 1 << 20, None) == E
    # several rows from a start that is not on a block boundary
    assert lib.dsa_csa_indexer_topk(fake, fake, fake, 1, 8, 10, 6, 4, 64, 128, 8, fake, fake, 1 << 20,
                                    None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_csa_indexer_topk_workspace(1, 8, 10, 0, 0, 64, 128, 8) == 0
    assert lib.dsa_csa_indexer_topk_workspace(2, 4096, 1024, 0, 4, 64, 128, 512) > \
        2 * 4096 * 64 * 128 * 2  # holds the phase-major copy of q_idx
    # (q, c, stride, idx, B, Lq, N, start, m, n_h, Dqk, Dv, k, scale, out, lse, ws, ws_bytes, stream)
    assert lib.dsa_csa_sparse_attn(None, fake, 576, fake, 1, 8, 2, 0, 4, 128, 576, 512, 8, 1.0,
                                   fake, None, fake, 0, None) == E
    assert lib.dsa_csa_sparse_attn(fake, fake, 576, fake, 1, 12, 1, 0, 4, 128, 576, 512, 8, 1.0,
                                   fake, None, fake, 0, None) == E
    assert lib.dsa_csa_sparse_attn(fake, fake, 500, fake, 1, 8, 2, 0, 4, 128, 576, 512, 8, 1.0,
                                   fake, None, fake, 0, None) == E


def _varlen(B=2, total_q=10, total_k=20, max_Lq=6, max_Lk=12, arrays=True):
    fake = 1 << 20  # never dereferenced on the host
    return dsa.Varlen(B=B, cu_q=fake if arrays else None, cu_k=fake if arrays else None,
                      start_pos=fake if arrays else None, total_q=total_q, total_k=total_k,
                      max_Lq=max_Lq, max_Lk=max_Lk)


def test_varlen_entry_points_validated_on_host():
    lib = dsa.lib()
    fake = ctypes.c_void_p(1 << 20)
    E = dsa.DSA_ERR_INVALID_ARG
    good = _varlen()
    for bad in (None, _varlen(arrays=False), _varlen(B=0), _varlen(max_Lq=11), _varlen(max_Lk=21),
                _varlen(total_q=0)):
        ref = ctypes.byref(bad) if bad is not None else None
        assert lib.dsa_indexer_topk_varlen(fake, fake, fake, ref, 64, 128, 8, fake, fake, 1 << 30, None) == E
        assert lib.dsa_sparse_attn_varlen(fake, fake, 576, fake, 576, fake, ref, 128, 576, 512, 8, 1.0, fake,
                                          None, fake, 1 << 30, None) == E
        assert lib.dsa_check_varlen(ref, fake, None) == E
        assert lib.dsa_indexer_topk_varlen_workspace(ref, 64, 128, 8) == 0
    # misaligned offset array
    mis = _varlen()
    mis.cu_q = (1 << 20) + 2
    assert lib.dsa_check_varlen(ctypes.byref(mis), fake, None) == E
    g = ctypes.byref(good)
    # the per-sequence limits of the uniform indexer apply
    assert lib.dsa_indexer_topk_varlen(fake, fake, fake, g, 12, 128, 8, fake, fake, 1 << 30,
                                       None) == dsa.DSA_ERR_UNSUPPORTED
    assert lib.dsa_indexer_topk_varlen(fake, fake, fake, g, 64, 128, 8, None, fake, 1 << 30, None) == E
    assert lib.dsa_indexer_topk_varlen(fake, fake, fake, g, 64, 128, 8, fake, fake, 16,
                                       None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_indexer_topk_varlen_workspace(g, 64, 128, 8) > 0
    # attention: row stride shorter than the row
    assert lib.dsa_sparse_attn_varlen(fake, fake, 64, fake, 576, fake, g, 128, 576, 512, 8, 1.0, fake, None, fake,
                                      1 << 30, None) == E
    # layer loop: the pattern rule holds for varlen batches too
    d = dsa.Dims(B=1, Lq=8, Lk=8, start_pos=0, H_I=64, d_I=128, k=4, n_h=128, D_qk=576, D_v=512,
                 scale=1.0, k_row_stride=576, v_row_stride=576)
    arr = (dsa.LayerIO * 2)()
    assert lib.indexcache_forward_varlen(b"SF", 2, arr, ctypes.byref(d), g, fake, fake, 1 << 30,
                                         None) == dsa.DSA_ERR_BAD_PATTERN
    assert lib.indexcache_forward_varlen(b"FS", 2, arr, ctypes.byref(d), g, fake, fake, 1 << 30, None) == E


def test_varlen_decode_batches_take_the_decode_workspace():
    # one query row per sequence (max_Lq = 1, total_q = B): the decode kernels
    # keep one row of score keys per sequence, sized by the longest cache
    lib = dsa.lib()
    dec = _varlen(B=8, total_q=8, total_k=8 * 200000, max_Lq=1, max_Lk=200000)
    ws = lib.dsa_indexer_topk_varlen_workspace(ctypes.byref(dec), 64, 128, 2048)
    assert ws == lib.dsa_indexer_topk_workspace(8, 1, 200000, 200000, 64, 128, 2048)


def test_lowprec_entry_points_validated_on_host():
    lib = dsa.lib()
    fake = ctypes.c_void_p(1 << 20)
    E, U = dsa.DSA_ERR_INVALID_ARG, dsa.DSA_ERR_UNSUPPORTED
    # (q, k, w, B, Lq, Lk, start, H, d, k, fmt, idx, ws, ws_bytes, stream)
    assert lib.dsa_indexer_topk_lowprec(None, fake, fake, 1, 8, 8, 0, 64, 128, 4, 0, fake, fake, 1 << 30, None) == E
    assert lib.dsa_indexer_topk_lowprec(fake, fake, fake, 1, 8, 8, 0, 64, 128, 4, 7, fake, fake, 1 << 30, None) == E
    assert lib.dsa_indexer_topk_lowprec(fake, fake, fake, 1, 8, 8, 0, 32, 128, 4, 0, fake, fake, 1 << 30, None) == U
    assert lib.dsa_indexer_topk_lowprec(fake, fake, fake, 1, 8, 8, 0, 64, 64, 4, 1, fake, fake, 1 << 30, None) == U
    assert lib.dsa_indexer_topk_lowprec(fake, fake, fake, 1, 8, 8, 5, 64, 128, 4, 0, fake, fake, 1 << 30, None) == E
    assert lib.dsa_indexer_topk_lowprec(fake, fake, fake, 1, 8, 8, 0, 64, 128, 4, 0, fake, fake, 16,
                                        None) == dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_indexer_topk_lowprec_workspace(1, 8, 8, 0, 64, 128, 4, 9) == 0
    assert lib.dsa_indexer_topk_lowprec_workspace(1, 8, 8, 0, 64, 128, 4, 1) > 8 * 64 * 128 + 8 * 128
    # (x, rows, cols, fmt, codes, scales, stream)
    assert lib.dsa_mx_quantize(fake, 0, 128, 0, fake, fake, None) == E
    assert lib.dsa_mx_quantize(fake, 4, 96, 0, fake, fake, None) == U
    assert lib.dsa_mx_quantize(fake, 4, 128, 3, fake, fake, None) == E
    assert lib.dsa_mx_quantize(None, 4, 128, 0, fake, fake, None) == E
