"""Python binding of the C ABI in include/dsa.h (argument marshalling only).

Every function takes torch CUDA tensors, checks dtypes/shapes/contiguity,
passes raw device pointers, sizes and the current stream to ``libdsa.so``
and raises ``DSAError`` on a non-OK status.  All compute runs in the
library's sm_100a kernels; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_BAD_PATTERN, DSA_ERR_UNSUPPORTED = 0, 1, 2, 3
DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT = 4, 5, 6
STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_BAD_PATTERN",
                3: "DSA_ERR_UNSUPPORTED", 4: "DSA_ERR_WORKSPACE", 5: "DSA_ERR_CUDA",
                6: "DSA_ERR_TIMEOUT"}

EXPORTS = ["dsa_last_error", "dsa_indexer_topk_workspace", "dsa_indexer_topk",
           "dsa_sparse_attn_workspace", "dsa_sparse_attn", "indexcache_forward_workspace",
           "indexcache_forward", "dsa_indexer_launch_count", "dsa_check_device_errors",
           "dsa_indexer_topk_noalloc", "dsa_selftest_wait_timeout", "dsa_check_indices",
           "dsa_dense_weights", "dsa_topk_rows", "dsa_index_overlap", "dsa_captured_mass",
           "dsa_csa_indexer_topk_workspace", "dsa_csa_indexer_topk", "dsa_csa_sparse_attn",
           "dsa_indexer_topk_varlen_workspace", "dsa_indexer_topk_varlen",
           "dsa_sparse_attn_varlen_workspace", "dsa_sparse_attn_varlen",
           "indexcache_forward_varlen_workspace", "indexcache_forward_varlen", "dsa_check_varlen",
           "dsa_indexer_topk_lowprec_workspace", "dsa_indexer_topk_lowprec", "dsa_mx_quantize"]

DSA_FMT_E4M3, DSA_FMT_E2M1 = 0, 1
FORMATS = {"e4m3": DSA_FMT_E4M3, "e2m1": DSA_FMT_E2M1}


class DSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("Lk", ctypes.c_int),
                ("start_pos", ctypes.c_int), ("H_I", ctypes.c_int), ("d_I", ctypes.c_int),
                ("k", ctypes.c_int), ("n_h", ctypes.c_int), ("D_qk", ctypes.c_int),
                ("D_v", ctypes.c_int), ("scale", ctypes.c_float),
                ("k_row_stride", ctypes.c_int64), ("v_row_stride", ctypes.c_int64)]


class LayerIO(ctypes.Structure):
    _fields_ = [("q_idx", ctypes.c_void_p), ("k_idx", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("kbuf", ctypes.c_void_p), ("vbuf", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


class Varlen(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("cu_q", ctypes.c_void_p), ("cu_k", ctypes.c_void_p),
                ("start_pos", ctypes.c_void_p), ("total_q", ctypes.c_int), ("total_k", ctypes.c_int),
                ("max_Lq", ctypes.c_int), ("max_Lk", ctypes.c_int)]


_lib = None


def lib():
    """Loads libdsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.dsa_last_error.restype = ctypes.c_char_p
        L.dsa_indexer_topk_workspace.argtypes = [I] * 7
        L.dsa_indexer_topk_workspace.restype = SZ
        L.dsa_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, P, P, SZ, P]
        L.dsa_indexer_topk.restype = I
        L.dsa_sparse_attn_workspace.argtypes = [I] * 5
        L.dsa_sparse_attn_workspace.restype = SZ
        L.dsa_sparse_attn.argtypes = [P, P, I64, P, I64, P, I, I, I, I, I, I, I, I,
                                      ctypes.c_float, P, P, P, SZ, P]
        L.dsa_sparse_attn.restype = I
        L.indexcache_forward_workspace.argtypes = [ctypes.POINTER(Dims)]
        L.indexcache_forward_workspace.restype = SZ
        L.indexcache_forward.argtypes = [ctypes.c_char_p, I, ctypes.POINTER(LayerIO),
                                         ctypes.POINTER(Dims), P, P, SZ, P]
        L.indexcache_forward.restype = I
        L.dsa_indexer_launch_count.restype = ctypes.c_longlong
        L.dsa_indexer_topk_noalloc.argtypes = [P, P, P, I, I, I, I, I, I, I, P, P]
        L.dsa_indexer_topk_noalloc.restype = I
        L.dsa_check_device_errors.argtypes = [P]
        L.dsa_check_device_errors.restype = I
        L.dsa_selftest_wait_timeout.argtypes = [ctypes.c_longlong, P]
        L.dsa_selftest_wait_timeout.restype = I
        L.dsa_check_indices.argtypes = [P, I, I, I, I, P, P]
        L.dsa_check_indices.restype = I
        F32 = ctypes.c_float
        L.dsa_dense_weights.argtypes = [P, P, I64, I, I, I, I, I, I, F32, P, P, P]
        L.dsa_dense_weights.restype = I
        L.dsa_topk_rows.argtypes = [P, I64, I, I, I, I, P, P]
        L.dsa_topk_rows.restype = I
        L.dsa_index_overlap.argtypes = [P, P, I64, I, P, P]
        L.dsa_index_overlap.restype = I
        L.dsa_captured_mass.argtypes = [P, P, I64, P, P]
        L.dsa_captured_mass.restype = I
        L.dsa_csa_indexer_topk_workspace.argtypes = [I, I, I, I, I, I, I, I]
        L.dsa_csa_indexer_topk_workspace.restype = SZ
        L.dsa_csa_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, SZ, P]
        L.dsa_csa_indexer_topk.restype = I
        L.dsa_csa_sparse_attn.argtypes = [P, P, I64, P, I, I, I, I, I, I, I, I, I, F32, P, P, P,
                                          SZ, P]
        L.dsa_csa_sparse_attn.restype = I
        VP = ctypes.POINTER(Varlen)
        L.dsa_indexer_topk_varlen_workspace.argtypes = [VP, I, I, I]
        L.dsa_indexer_topk_varlen_workspace.restype = SZ
        L.dsa_indexer_topk_varlen.argtypes = [P, P, P, VP, I, I, I, P, P, SZ, P]
        L.dsa_indexer_topk_varlen.restype = I
        L.dsa_sparse_attn_varlen_workspace.argtypes = [VP, I, I, I]
        L.dsa_sparse_attn_varlen_workspace.restype = SZ
        L.dsa_sparse_attn_varlen.argtypes = [P, P, I64, P, I64, P, VP, I, I, I, I, F32, P, P, P, SZ, P]
        L.dsa_sparse_attn_varlen.restype = I
        L.indexcache_forward_varlen_workspace.argtypes = [ctypes.POINTER(Dims), VP]
        L.indexcache_forward_varlen_workspace.restype = SZ
        L.indexcache_forward_varlen.argtypes = [ctypes.c_char_p, I, ctypes.POINTER(LayerIO),
                                                ctypes.POINTER(Dims), VP, P, P, SZ, P]
        L.indexcache_forward_varlen.restype = I
        L.dsa_check_varlen.argtypes = [VP, P, P]
        L.dsa_check_varlen.restype = I
        L.dsa_indexer_topk_lowprec_workspace.argtypes = [I] * 8
        L.dsa_indexer_topk_lowprec_workspace.restype = SZ
        L.dsa_indexer_topk_lowprec.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, SZ, P]
        L.dsa_indexer_topk_lowprec.restype = I
        L.dsa_mx_quantize.argtypes = [P, I64, I, I, P, P, P]
        L.dsa_mx_quantize.restype = I
        _lib = L
    return _lib


def _check(st: int) -> None:
    if st != DSA_OK:
        raise DSAError(st, lib().dsa_last_error().decode())


def _stream(t=None):
    import torch
    dev = t.device if t is not None else None
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, shape=None, name="tensor"):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def indexer_topk_workspace(B, Lq, Lk, start_pos, H_I, d_I, k) -> int:
    return int(lib().dsa_indexer_topk_workspace(B, Lq, Lk, start_pos, H_I, d_I, k))


def indexer_topk(q_idx, k_idx, w, k: int, *, start_pos: int = 0, out=None, ws=None):
    """Lightning indexer + top-k.  q_idx [B,Lq,H,d] bf16, k_idx [B,Lk,d] bf16,
    w [B,Lq,H] f32 -> idx [B,Lq,k] int32 (ascending positions, -1 padded)."""
    import torch
    B, Lq, H, d = q_idx.shape
    Lk = k_idx.shape[1]
    _need(q_idx, torch.bfloat16, name="q_idx")
    _need(k_idx, torch.bfloat16, (B, Lk, d), "k_idx")
    _need(w, torch.float32, (B, Lq, H), "w")
    if out is None:
        out = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device)
    _need(out, torch.int32, (B, Lq, k), "out")
    need = indexer_topk_workspace(B, Lq, Lk, start_pos, H, d, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_idx.device)
    _check(lib().dsa_indexer_topk(_ptr(q_idx), _ptr(k_idx), _ptr(w), B, Lq, Lk, start_pos, H, d, k,
                                  _ptr(out), _ptr(ws), ws.numel(), _stream(q_idx)))
    return out


NOALLOC_SCRATCH_BYTES = 72 * 1024 * 1024


def indexer_topk_noalloc(q_idx, k_idx, w, k: int, *, start_pos: int = 0, out=None):
    """Same as indexer_topk, for callers that cannot hand the library a
    workspace: the scratch comes from a fixed device array of
    NOALLOC_SCRATCH_BYTES inside the library (shared by every call; do not
    overlap calls on the GPU)."""
    import torch
    B, Lq, H, d = q_idx.shape
    Lk = k_idx.shape[1]
    _need(q_idx, torch.bfloat16, name="q_idx")
    _need(k_idx, torch.bfloat16, (B, Lk, d), "k_idx")
    _need(w, torch.float32, (B, Lq, H), "w")
    if out is None:
        out = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device)
    _need(out, torch.int32, (B, Lq, k), "out")
    _check(lib().dsa_indexer_topk_noalloc(_ptr(q_idx), _ptr(k_idx), _ptr(w), B, Lq, Lk, start_pos,
                                          H, d, k, _ptr(out), _stream(q_idx)))
    return out


def sparse_attn_workspace(B, Lq, n_h, D_v, k) -> int:
    return int(lib().dsa_sparse_attn_workspace(B, Lq, n_h, D_v, k))


def sparse_attn(q, kbuf, vbuf, idx, scale: float, *, D_v: int, start_pos: int = 0,
                out=None, lse=None, ws=None):
    """Sparse core attention.  q [B,Lq,n_h,D_qk] bf16; kbuf [B,Lk,Ck] and vbuf
    [B,Lk,Cv] bf16 rows (K = first D_qk columns, V = first D_v columns; pass
    the same latent tensor for MLA); idx [B,Lq,k] int32.
    Returns out [B,Lq,n_h,D_v] bf16 (and fills ``lse`` [B,Lq,n_h] f32 if given)."""
    import torch
    B, Lq, n_h, D_qk = q.shape
    Lk = kbuf.shape[1]
    k = idx.shape[2]
    _need(q, torch.bfloat16, name="q")
    _need(kbuf, torch.bfloat16, name="kbuf")
    _need(vbuf, torch.bfloat16, name="vbuf")
    _need(idx, torch.int32, (B, Lq, k), "idx")
    if out is None:
        out = torch.empty((B, Lq, n_h, D_v), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (B, Lq, n_h, D_v), "out")
    if lse is not None:
        _need(lse, torch.float32, (B, Lq, n_h), "lse")
    need = sparse_attn_workspace(B, Lq, n_h, D_v, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib().dsa_sparse_attn(_ptr(q), _ptr(kbuf), kbuf.shape[2], _ptr(vbuf), vbuf.shape[2],
                                 _ptr(idx), B, Lq, Lk, start_pos, n_h, D_qk, D_v, k, scale,
                                 _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(q)))
    return out


def make_dims(**kw) -> Dims:
    return Dims(**kw)


def indexcache_forward_workspace(dims: Dims) -> int:
    return int(lib().indexcache_forward_workspace(ctypes.byref(dims)))


def indexcache_forward(pattern: str, layers, dims: Dims, idx_cache, ws=None, stream=None):
    """Runs the F/S layer loop.  ``layers`` is a list of dicts with keys
    q_idx, k_idx, w (F layers), q, kbuf, vbuf, out and optionally lse."""
    import torch
    n = len(layers)
    arr = (LayerIO * max(n, 1))()
    for i, L in enumerate(layers):
        arr[i] = LayerIO(*[(L[f].data_ptr() if L.get(f) is not None else None) for f in
                           ("q_idx", "k_idx", "w", "q", "kbuf", "vbuf", "out", "lse")])
    need = indexcache_forward_workspace(dims)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=idx_cache.device)
    st = stream if stream is not None else _stream(idx_cache)
    _check(lib().indexcache_forward(pattern.encode(), n, arr, ctypes.byref(dims),
                                    _ptr(idx_cache), _ptr(ws), ws.numel(), st))
    return idx_cache


def indexer_launch_count() -> int:
    return int(lib().dsa_indexer_launch_count())


def check_device_errors(stream=None) -> None:
    _check(lib().dsa_check_device_errors(stream if stream is not None else _stream()))


def check_indices(idx, start_pos: int = 0) -> int:
    """Number of rows of idx [B, Lq, k] (int32, CUDA) that are not in the
    canonical form dsa_indexer_topk writes (ascending positions below t, then
    -1).  Synchronises the current stream."""
    import torch
    _need(idx, torch.int32, name="idx")
    B, Lq, k = idx.shape
    bad = torch.empty(1, dtype=torch.int32, device=idx.device)
    _check(lib().dsa_check_indices(_ptr(idx), B, Lq, start_pos, k, _ptr(bad), _stream(idx)))
    return int(bad.item())


def csa_indexer_topk_workspace(B, Lq, N_cmp, start_pos, m, H_I, d_I, k) -> int:
    return int(lib().dsa_csa_indexer_topk_workspace(B, Lq, N_cmp, start_pos, m, H_I, d_I, k))


def csa_indexer_topk(q_idx, k_cmp, w, k: int, *, m: int, start_pos: int = 0, out=None, ws=None):
    """CSA-style indexer + top-k over compressed blocks ([IDX] §5.2): row i at
    t = start_pos + i scores the blocks s < floor(t/m) of k_cmp [B, N_cmp,
    d_I].  q_idx [B, Lq, H_I, d_I] bf16, w [B, Lq, H_I] f32.  Returns idx
    [B, Lq, k] int32 (ascending block ids, then -1)."""
    import torch
    B, Lq, H, d = q_idx.shape
    N = k_cmp.shape[1]
    _need(q_idx, torch.bfloat16, name="q_idx")
    _need(k_cmp, torch.bfloat16, (B, N, d), "k_cmp")
    _need(w, torch.float32, (B, Lq, H), "w")
    if out is None:
        out = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device)
    _need(out, torch.int32, (B, Lq, k), "out")
    need = csa_indexer_topk_workspace(B, Lq, N, start_pos, m, H, d, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_idx.device)
    _check(lib().dsa_csa_indexer_topk(_ptr(q_idx), _ptr(k_cmp), _ptr(w), B, Lq, N, start_pos, m, H, d,
                                      k, _ptr(out), _ptr(ws), ws.numel(), _stream(q_idx)))
    return out


def csa_sparse_attn(q, c_cmp, idx, scale: float, *, m: int, D_v: int, start_pos: int = 0,
                    out=None, lse=None, ws=None):
    """Attention over the selected compressed entries ([IDX] §5.2): keys and
    values are the rows of c_cmp [B, N_cmp, C] (K = the first D_qk columns,
    V = the first D_v).  q [B, Lq, n_h, D_qk] bf16; idx from csa_indexer_topk."""
    import torch
    B, Lq, n_h, D_qk = q.shape
    N = c_cmp.shape[1]
    k = idx.shape[2]
    _need(q, torch.bfloat16, name="q")
    _need(c_cmp, torch.bfloat16, name="c_cmp")
    _need(idx, torch.int32, (B, Lq, k), "idx")
    if out is None:
        out = torch.empty((B, Lq, n_h, D_v), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (B, Lq, n_h, D_v), "out")
    if lse is not None:
        _need(lse, torch.float32, (B, Lq, n_h), "lse")
    need = sparse_attn_workspace(B, Lq, n_h, D_v, k)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib().dsa_csa_sparse_attn(_ptr(q), _ptr(c_cmp), c_cmp.shape[2], _ptr(idx), B, Lq, N,
                                     start_pos, m, n_h, D_qk, D_v, k, float(scale), _ptr(out),
                                     _ptr(lse), _ptr(ws), ws.numel(), _stream(q)))
    return out


def dense_weights(q, kv, *, Lk: int | None = None, start_pos: int = 0, scale: float,
                  D_qk: int | None = None, mean_weights: bool = True):
    """Dense causal attention statistics ([IDX] §8.1) of q [B, Lq, n_h, D_qk]
    against the rows of kv [B, Lk, row] (bf16, CUDA; the first D_qk columns
    are the keys).  Returns (lse_dense [B, Lq, n_h] f32, mean_w [B, Lq, Lk]
    f32 or None); mean_w holds the head-averaged dense weights for s < t and
    zeros elsewhere."""
    import torch
    _need(q, torch.bfloat16, name="q")
    _need(kv, torch.bfloat16, name="kv")
    B, Lq, n_h, Dq = q.shape
    D_qk = Dq if D_qk is None else D_qk
    assert D_qk == Dq, "q's last dimension is D_qk"
    Lk = kv.shape[1] if Lk is None else Lk
    lse = torch.empty((B, Lq, n_h), dtype=torch.float32, device=q.device)
    mw = torch.zeros((B, Lq, Lk), dtype=torch.float32, device=q.device) if mean_weights else None
    _check(lib().dsa_dense_weights(_ptr(q), _ptr(kv), kv.shape[2], B, Lq, Lk, start_pos, n_h, D_qk,
                                   float(scale), _ptr(lse), _ptr(mw), _stream(q)))
    return lse, mw


def topk_rows(scores, k: int, start_pos: int = 0):
    """TopK_k over dense score rows scores [B, Lq, W] (f32, CUDA); row i holds
    start_pos + i scores.  The oracle selection of [IDX] §8.2 when given the
    head-averaged dense weights.  Returns idx [B, Lq, k] int32."""
    import torch
    _need(scores, torch.float32, name="scores")
    B, Lq, W = scores.shape
    idx = torch.empty((B, Lq, k), dtype=torch.int32, device=scores.device)
    _check(lib().dsa_topk_rows(_ptr(scores), W, B, Lq, start_pos, k, _ptr(idx), _stream(scores)))
    return idx


def index_overlap(a, b):
    """|A & B| per row of two index tensors [..., k] (int32, CUDA, row form
    of indexer_topk).  Returns int32 counts of shape a.shape[:-1]."""
    import torch
    _need(a, torch.int32, name="a")
    _need(b, torch.int32, shape=a.shape, name="b")
    k = a.shape[-1]
    rows = a.numel() // k
    inter = torch.empty(a.shape[:-1], dtype=torch.int32, device=a.device)
    _check(lib().dsa_index_overlap(_ptr(a), _ptr(b), rows, k, _ptr(inter), _stream(a)))
    return inter


def captured_mass(lse_sel, lse_dense):
    """CapturedMass@k ([IDX] §8.1) = exp(lse_sel - lse_dense) elementwise (f32,
    CUDA, same shape); 1 where the row sees nothing."""
    import torch
    _need(lse_sel, torch.float32, name="lse_sel")
    _need(lse_dense, torch.float32, shape=lse_sel.shape, name="lse_dense")
    mass = torch.empty_like(lse_sel)
    _check(lib().dsa_captured_mass(_ptr(lse_sel), _ptr(lse_dense), lse_sel.numel(), _ptr(mass),
                                   _stream(lse_sel)))
    return mass


def selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Launches the library's bounded-wait self-test (a wait nothing completes,
    abandoned after `limit_cycles`); the next check_device_errors() raises
    DSA_ERR_TIMEOUT."""
    _check(lib().dsa_selftest_wait_timeout(int(limit_cycles), stream if stream is not None else _stream()))


# --------------------------------------------------------------------------
# Variable-length batches (packed rows; see dsa_varlen in include/dsa.h)
class VarlenBatch:
    """A variable-length batch: the device offset arrays and the host sizes
    of ``dsa_varlen``.  Keeps the device arrays alive with the descriptor."""

    def __init__(self, q_lens, k_lens, start_pos, device="cuda"):
        import torch
        q_lens, k_lens, start_pos = list(map(int, q_lens)), list(map(int, k_lens)), list(map(int, start_pos))
        if not (len(q_lens) == len(k_lens) == len(start_pos) >= 1):
            raise ValueError("q_lens, k_lens and start_pos need one entry per sequence")
        cu_q, cu_k = [0], [0]
        for a, b in zip(q_lens, k_lens):
            cu_q.append(cu_q[-1] + a)
            cu_k.append(cu_k[-1] + b)
        self.q_lens, self.k_lens, self.start_pos_list = q_lens, k_lens, start_pos
        self.cu_q_list, self.cu_k_list = cu_q, cu_k
        self.cu_q = torch.tensor(cu_q, dtype=torch.int32, device=device)
        self.cu_k = torch.tensor(cu_k, dtype=torch.int32, device=device)
        self.start_pos = torch.tensor(start_pos, dtype=torch.int32, device=device)
        self.desc = Varlen(B=len(q_lens), cu_q=self.cu_q.data_ptr(), cu_k=self.cu_k.data_ptr(),
                           start_pos=self.start_pos.data_ptr(), total_q=cu_q[-1], total_k=cu_k[-1],
                           max_Lq=max(max(q_lens), 1), max_Lk=max(max(k_lens), 1))

    @property
    def B(self):
        return self.desc.B

    @property
    def total_q(self):
        return self.desc.total_q

    @property
    def total_k(self):
        return self.desc.total_k


def indexer_topk_varlen(q_idx, k_idx, w, k: int, vb: VarlenBatch, *, out=None, ws=None):
    """Lightning indexer + top-k per sequence of a packed batch: q_idx
    [total_q, H, d] bf16, k_idx [total_k, d] bf16, w [total_q, H] f32 ->
    idx [total_q, k] int32."""
    import torch
    tq, H, d = q_idx.shape
    _need(q_idx, torch.bfloat16, (vb.total_q, H, d), "q_idx")
    _need(k_idx, torch.bfloat16, (vb.total_k, d), "k_idx")
    _need(w, torch.float32, (vb.total_q, H), "w")
    if out is None:
        out = torch.empty((vb.total_q, k), dtype=torch.int32, device=q_idx.device)
    _need(out, torch.int32, (vb.total_q, k), "out")
    need = int(lib().dsa_indexer_topk_varlen_workspace(ctypes.byref(vb.desc), H, d, k))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_idx.device)
    _check(lib().dsa_indexer_topk_varlen(_ptr(q_idx), _ptr(k_idx), _ptr(w), ctypes.byref(vb.desc), H, d, k,
                                         _ptr(out), _ptr(ws), ws.numel(), _stream(q_idx)))
    return out


def sparse_attn_varlen(q, kbuf, vbuf, idx, scale: float, vb: VarlenBatch, *, D_v: int, out=None, lse=None,
                       ws=None):
    """Sparse core attention per sequence of a packed batch: q [total_q, n_h,
    D_qk] bf16, kbuf/vbuf [total_k, C] bf16 rows, idx [total_q, k] int32 ->
    out [total_q, n_h, D_v] bf16 (and lse [total_q, n_h] f32 if given)."""
    import torch
    tq, n_h, D_qk = q.shape
    k = idx.shape[1]
    _need(q, torch.bfloat16, (vb.total_q, n_h, D_qk), "q")
    _need(kbuf, torch.bfloat16, name="kbuf")
    _need(vbuf, torch.bfloat16, name="vbuf")
    if kbuf.shape[0] != vb.total_k or vbuf.shape[0] != vb.total_k:
        raise ValueError("kbuf and vbuf need total_k rows")
    _need(idx, torch.int32, (vb.total_q, k), "idx")
    if out is None:
        out = torch.empty((vb.total_q, n_h, D_v), dtype=torch.bfloat16, device=q.device)
    _need(out, torch.bfloat16, (vb.total_q, n_h, D_v), "out")
    if lse is not None:
        _need(lse, torch.float32, (vb.total_q, n_h), "lse")
    need = int(lib().dsa_sparse_attn_varlen_workspace(ctypes.byref(vb.desc), n_h, D_v, k))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib().dsa_sparse_attn_varlen(_ptr(q), _ptr(kbuf), kbuf.shape[1], _ptr(vbuf), vbuf.shape[1], _ptr(idx),
                                        ctypes.byref(vb.desc), n_h, D_qk, D_v, k, float(scale), _ptr(out),
                                        _ptr(lse), _ptr(ws), ws.numel(), _stream(q)))
    return out


def indexcache_forward_varlen(pattern: str, layers, dims: Dims, vb: VarlenBatch, idx_cache, ws=None):
    """The F/S layer loop over a packed batch; ``layers`` as for
    indexcache_forward with packed per-layer tensors, idx_cache [total_q, k]."""
    import torch
    n = len(layers)
    arr = (LayerIO * max(n, 1))()
    for i, L in enumerate(layers):
        arr[i] = LayerIO(*[(L[f].data_ptr() if L.get(f) is not None else None) for f in
                           ("q_idx", "k_idx", "w", "q", "kbuf", "vbuf", "out", "lse")])
    need = int(lib().indexcache_forward_varlen_workspace(ctypes.byref(dims), ctypes.byref(vb.desc)))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=idx_cache.device)
    _check(lib().indexcache_forward_varlen(pattern.encode(), n, arr, ctypes.byref(dims), ctypes.byref(vb.desc),
                                           _ptr(idx_cache), _ptr(ws), ws.numel(), _stream(idx_cache)))
    return idx_cache


def check_varlen(vb: VarlenBatch) -> int:
    """Number of sequences of the batch that break the dsa_varlen contract
    (checked on the device).  Synchronises the current stream."""
    import torch
    bad = torch.empty(1, dtype=torch.int32, device=vb.cu_q.device)
    _check(lib().dsa_check_varlen(ctypes.byref(vb.desc), _ptr(bad), _stream(vb.cu_q)))
    return int(bad.item())


# --------------------------------------------------------------------------
# Low-precision selector ([IDX] §5.4; MX E4M3 / E2M1 operands, bf16 scores)
def indexer_topk_lowprec_workspace(B, Lq, Lk, start_pos, H_I, d_I, k, fmt: str) -> int:
    return int(lib().dsa_indexer_topk_lowprec_workspace(B, Lq, Lk, start_pos, H_I, d_I, k, FORMATS[fmt]))


def indexer_topk_lowprec(q_idx, k_idx, w, k: int, *, fmt: str, start_pos: int = 0, out=None, ws=None):
    """Low-precision selector: q_idx [B,Lq,64,128] bf16, k_idx [B,Lk,128]
    bf16, w [B,Lq,64] f32 quantised to MX ``fmt`` ("e4m3" or "e2m1") inside
    the call -> idx [B,Lq,k] int32 (bf16 scores, ascending, -1 padded)."""
    import torch
    B, Lq, H, d = q_idx.shape
    Lk = k_idx.shape[1]
    _need(q_idx, torch.bfloat16, name="q_idx")
    _need(k_idx, torch.bfloat16, (B, Lk, d), "k_idx")
    _need(w, torch.float32, (B, Lq, H), "w")
    if out is None:
        out = torch.empty((B, Lq, k), dtype=torch.int32, device=q_idx.device)
    _need(out, torch.int32, (B, Lq, k), "out")
    need = indexer_topk_lowprec_workspace(B, Lq, Lk, start_pos, H, d, k, fmt)
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=q_idx.device)
    _check(lib().dsa_indexer_topk_lowprec(_ptr(q_idx), _ptr(k_idx), _ptr(w), B, Lq, Lk, start_pos, H, d, k,
                                          FORMATS[fmt], _ptr(out), _ptr(ws), ws.numel(), _stream(q_idx)))
    return out


def mx_quantize(x, fmt: str):
    """MX quantisation of bf16 rows x [..., 128] -> (codes uint8 [rows, 128],
    scales uint8 [rows, 4]); see dsa_mx_quantize."""
    import torch
    _need(x, torch.bfloat16, name="x")
    rows = x.numel() // x.shape[-1]
    codes = torch.empty((rows, x.shape[-1]), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, x.shape[-1] // 32), dtype=torch.uint8, device=x.device)
    _check(lib().dsa_mx_quantize(_ptr(x), rows, x.shape[-1], FORMATS[fmt], _ptr(codes), _ptr(scales), _stream(x)))
    return codes, scales
