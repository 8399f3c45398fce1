"""CPU oracle for the DSA layer stack under IndexCache (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``dsa_oracle.c`` (plain C,
IEEE double, single-threaded) through ctypes and shares nothing with the CUDA
library.  bf16 tensors are passed as their uint16 bit patterns.

Sources: "读懂 IndexCache：从 DSA 的选词开销到跨层索引复用" (IndexCache
explainer, cited as [IC]) and "注意力机制中的 Index：从位置下标到预算检索"
(cited as [IDX]); each wrapper names the section it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-Wall", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_indexer_row.argtypes = [P, P, P, i32, i32, i32, P]
        lib.oracle_indexer_row.restype = ctypes.c_longlong
        lib.oracle_topk_row.argtypes = [P, i32, i32, P]
        lib.oracle_topk_row.restype = i32
        lib.oracle_sparse_attn_row.argtypes = [P, P, i64, P, i64, P, i32, i32, i32, i32, f64, P, P]
        lib.oracle_sparse_attn_row.restype = i32
        lib.oracle_dense_attn_row.argtypes = [P, P, i64, P, i64, i32, i32, i32, i32, f64, P, P]
        lib.oracle_dense_attn_row.restype = None
        lib.oracle_masked_attn_row.argtypes = [P, P, i64, P, i64, P, i32, i32, i32, i32, i32, i32, f64, P, P]
        lib.oracle_masked_attn_row.restype = None
        lib.oracle_dense_probs_row.argtypes = [P, P, i64, i32, i32, i32, f64, P]
        lib.oracle_dense_probs_row.restype = None
        lib.oracle_indexcache_forward.argtypes = [
            ctypes.c_char_p, i32, P, P, P, P, P, i64, P, i64, i32, i32, i32, i32,
            i32, i32, i32, i32, i32, i32, f64, P, P, P, P]
        lib.oracle_indexcache_forward.restype = i32
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 tensors are passed as uint16 bit patterns")
    return a


def indexer_row(q_row, k, w_row, T: int) -> np.ndarray:
    """[IDX] §4 index score: I[s] = sum_j w[j] * ReLU(q[j] . k[s]) for s < T.

    q_row [H, d] bf16 bits, k [>=T, d] bf16 bits, w_row [H] float32."""
    q_row, k = _bits(q_row), _bits(k)
    w_row = np.ascontiguousarray(w_row, dtype=np.float32)
    H, d = q_row.shape
    assert k.shape[1] == d and k.shape[0] >= T and w_row.shape == (H,)
    out = np.zeros(max(T, 1), dtype=np.float64)
    _load().oracle_indexer_row(_p(q_row), _p(k), _p(w_row), H, d, T, _p(out))
    return out[:T]


def topk_row(I, T: int, k: int) -> np.ndarray:
    """[IDX] §4 TopK over s < T; ties -> lower s; ascending s then -1 pad."""
    I = np.ascontiguousarray(I, dtype=np.float64)
    assert I.shape[0] >= T
    out = np.empty(k, dtype=np.int32)
    _load().oracle_topk_row(_p(I), T, k, _p(out))
    return out


def _attn_args(q_row, K, V):
    q_row, K, V = _bits(q_row), _bits(K), _bits(V)
    assert K.ndim == 2 and V.ndim == 2
    return q_row, K, V


def sparse_attn_row(q_row, K, V, idx, scale: float, Dv: int | None = None):
    """[IDX] §2 alpha-hat / o-hat over the selected set.  Returns (out, lse).

    q_row [n_h, Dqk]; K [Lk, >=Dqk] and V [Lk, >=Dv] (row-major; V may be a
    column view of the same latent rows); idx [k] int32 with -1 padding."""
    q_row, K, V = _attn_args(q_row, K, V)
    n_h, Dqk = q_row.shape
    Dv = V.shape[1] if Dv is None else Dv
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.zeros((n_h, Dv), dtype=np.float64)
    lse = np.zeros(n_h, dtype=np.float64)
    _load().oracle_sparse_attn_row(_p(q_row), _p(K), K.shape[1], _p(V), V.shape[1],
                                   _p(idx), idx.shape[0], n_h, Dqk, Dv, scale,
                                   _p(out), _p(lse))
    return out, lse


def dense_attn_row(q_row, K, V, T: int, scale: float, Dv: int | None = None):
    """[IDX] §1 dense causal attention over P_t = {s < T}.  Returns (out, lse)."""
    q_row, K, V = _attn_args(q_row, K, V)
    n_h, Dqk = q_row.shape
    Dv = V.shape[1] if Dv is None else Dv
    out = np.zeros((n_h, Dv), dtype=np.float64)
    lse = np.zeros(n_h, dtype=np.float64)
    _load().oracle_dense_attn_row(_p(q_row), _p(K), K.shape[1], _p(V), V.shape[1], T,
                                  n_h, Dqk, Dv, scale, _p(out), _p(lse))
    return out, lse


def masked_attn_row(q_row, K, V, idx, T: int, scale: float, Dv: int | None = None):
    """[IDX] §6.4 index-mask formulation (-inf scatter + causal mask)."""
    q_row, K, V = _attn_args(q_row, K, V)
    n_h, Dqk = q_row.shape
    Dv = V.shape[1] if Dv is None else Dv
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.zeros((n_h, Dv), dtype=np.float64)
    lse = np.zeros(n_h, dtype=np.float64)
    _load().oracle_masked_attn_row(_p(q_row), _p(K), K.shape[1], _p(V), V.shape[1],
                                   _p(idx), idx.shape[0], T, K.shape[0], n_h, Dqk, Dv,
                                   scale, _p(out), _p(lse))
    return out, lse


def dense_probs_row(q_row, K, T: int, scale: float) -> np.ndarray:
    """[IDX] §8.1: the dense attention weights alpha^dense_{t,s} of one query
    row over P_t = {0 <= s < T}, per head.  q_row [n_h, Dqk] and K [>=T, Dqk]
    (or a strided [rows, >=Dqk] view of the latent cache) as bf16 bits.
    Returns [n_h, T] float64."""
    q_row, K = _bits(q_row), _bits(K)
    n_h, Dqk = q_row.shape
    assert K.ndim == 2 and K.shape[1] >= Dqk and K.shape[0] >= T
    alpha = np.zeros((n_h, T), dtype=np.float64)
    _load().oracle_dense_probs_row(_p(q_row), _p(K), K.shape[1], T, n_h, Dqk,
                                   float(scale), _p(alpha))
    return alpha


def captured_mass_row(alpha, idx) -> np.ndarray:
    """[IDX] §8.1: CapturedMass@k = the dense weight that the selected set
    holds, sum over s in S_t of alpha^dense_{t,s}, for each head (alpha
    [n_h, T] from dense_probs_row; idx one index row, -1 entries skipped).
    MissedMass@k is 1 minus it.  A query that sees nothing (T = 0) has S_t =
    P_t = {} and is given mass 1: nothing of the dense weight is missed."""
    alpha = np.asarray(alpha, dtype=np.float64)
    sel = sorted({int(s) for s in np.asarray(idx) if s >= 0})
    if alpha.shape[1] == 0:
        assert not sel
        return np.ones(alpha.shape[0])
    assert all(s < alpha.shape[1] for s in sel)
    return alpha[:, sel].sum(axis=1) if sel else np.zeros(alpha.shape[0])


def overlap_row(a, b) -> int:
    """|A intersect B| for two index rows (-1 entries skipped): the numerator
    of [IDX] §8.4's adjacent-layer overlap |S^(l) & S^(l+1)| / k_idx and of
    [IDX] §8.2's Recall@k."""
    return len({int(s) for s in np.asarray(a) if s >= 0} & {int(s) for s in np.asarray(b) if s >= 0})


def recall_row(s_oracle, s_model) -> float:
    """[IDX] §8.2: Recall@k = |S^oracle & S^model| / |S^oracle|.  An empty
    oracle set (T = 0) is given recall 1: there is nothing to miss."""
    n = sum(1 for s in np.asarray(s_oracle) if s >= 0)
    return 1.0 if n == 0 else overlap_row(s_oracle, s_model) / n


def oracle_selection_row(alpha, T: int, k: int) -> np.ndarray:
    """[IDX] §8.2: S_t^oracle = TopK_k { alpha^dense_{t,s} : s < t }.  The
    page's alpha carries no head index; with n_h heads sharing one selection
    the weights are averaged over heads (sum over h, divided by n_h) before
    the top-k.  Same tie rule and row form as topk_row."""
    alpha = np.asarray(alpha, dtype=np.float64)
    mean = alpha.sum(axis=0) / alpha.shape[0] if T > 0 else np.zeros(0)
    return topk_row(mean, T, k)


def csa_visible(t: int, m: int) -> int:
    """[IDX] §5.2 (CSA indexer over compressed blocks): compressed block s is
    visible to query t iff s < floor(t / m), so query t sees floor(t / m)
    blocks."""
    assert t >= 0 and m >= 1
    return t // m


def csa_indexer_topk_row(q_row, k_cmp, w_row, t: int, m: int, k: int):
    """[IDX] §5.2: I[t,s] = sum_j w[t,j] ReLU(q[t,j] . K^IComp[s]) over the
    visible compressed blocks s < floor(t/m), then S_t^CSA = TopK_k.  Same
    score, tie rule and row form as the token-level indexer.  Returns (I, idx)."""
    T = csa_visible(t, m)
    I = indexer_row(q_row, k_cmp, w_row, T)
    return I, topk_row(I, T, k)


def csa_attn_row(q_row, c_cmp, idx, scale: float, Dv: int | None = None):
    """[IDX] §5.2: o_t = CoreAttn(q_t, {C_s^Comp : s in S_t^CSA}) with keys and
    values from the same compressed entries (shared-KV MQA; for the MLA shape
    V is the first Dv columns).  Returns (out, lse)."""
    return sparse_attn_row(q_row, c_cmp, c_cmp, idx, scale, Dv)


# Low-precision selector ([IDX] §5.4).  Element formats from the OCP 8-bit
# Floating Point (OFP8) and Microscaling (MX) v1.0 specifications:
# (mantissa bits, exponent of the smallest normal, largest exponent, largest
# finite value).
_LP_FORMATS = {"e4m3": (3, -6, 8, 448.0), "e2m1": (1, 0, 2, 6.0)}


def round_to_format(v, fmt: str) -> np.ndarray:
    """Rounds float64 values to the E4M3 or E2M1 element grid: nearest, ties to
    even, with subnormals below the smallest normal, saturating at the largest
    finite value (E4M3 keeps its top code for NaN, so 448 is the largest).
    Signs, including -0, are kept."""
    m, emin, _, vmax = _LP_FORMATS[fmt]
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), emin)
    ulp = np.exp2(e - m)
    q = np.minimum(np.round(a / ulp) * ulp, vmax)     # np.round: half to even
    return np.copysign(q, v)


def mx_quantize(x, fmt: str, block: int = 32) -> np.ndarray:
    """MX block quantization along the last axis: every run of `block`
    consecutive elements shares the power-of-two scale
    X = 2^(floor(log2 amax) - emax_elem) (emax_elem = 8 for E4M3, 2 for E2M1)
    and each element becomes round_to_format(x / X).  Returns the values the
    format represents, X * element, in float64.  (The 8-bit scale's range
    limits of +-127 are not reached by these inputs and are not modelled.)"""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % block == 0
    xb = x.reshape(x.shape[:-1] + (d // block, block))
    amax = np.abs(xb).max(axis=-1, keepdims=True)
    X = np.exp2(np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - _LP_FORMATS[fmt][2])
    return (round_to_format(xb / X, fmt) * X).reshape(x.shape)


def bf16_round(x) -> np.ndarray:
    """Rounds float64 values first to float32 and then to bfloat16 (each to
    nearest, ties to even): a score "quantised from FP32 to BF16".  Finite
    inputs; returns float64."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def _bf16_values(a) -> np.ndarray:
    u = _bits(a).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def lowprec_indexer_row(q_row, k, w_row, T: int, fmt: str) -> np.ndarray:
    """[IDX] §5.4: the §4 index score with the QK path in a low-precision
    format and the score quantised from FP32 to BF16.  q_row [H, d] and the
    keys are MX-quantised to `fmt` along d (blocks of 32), the head dots are
    formed exactly from the quantised values (a tensor-core product
    accumulates them in fp32), I = sum_j w_j ReLU(dot_j), and I is rounded to
    bf16.  q_row, k as bf16 bits; w_row float32.  Returns [T] float64."""
    qh = mx_quantize(_bf16_values(q_row), fmt)
    kh = mx_quantize(_bf16_values(k)[:T], fmt) if T > 0 else np.zeros((0, qh.shape[1]))
    w = np.asarray(w_row, dtype=np.float32).astype(np.float64)
    I = np.maximum(kh @ qh.T, 0.0) @ w
    return bf16_round(I)


def _ptr_array(arrs):
    arr = (ctypes.c_void_p * len(arrs))()
    for i, a in enumerate(arrs):
        arr[i] = None if a is None else a.ctypes.data
    return arr


def indexcache_forward(pattern: str, layers, *, B, Lq, Lk, start_pos, H, dI, k,
                       n_h, Dqk, Dv, scale, kv_cols_k=None, kv_cols_v=None):
    """[IC] §1.1-§1.2 (Figure 2 loop) over whole small inputs.

    ``layers`` is a list of dicts with keys q_idx, k_idx, w (F layers; may be
    None on S layers), q, and either kv (MLA latent rows: K = all columns, V
    = the first Dv columns) or k and v.  Returns (idx [L,B,Lq,k] int32,
    out [L,B,Lq,n_h,Dv] f64, lse [L,B,Lq,n_h] f64, counters dict) or raises
    ValueError for an invalid pattern."""
    n = len(layers)
    keep = []
    qi, ki, wi, qq, KK, VV = [], [], [], [], [], []
    ks = vs = None
    for L in layers:
        if L.get("q_idx") is not None:
            a, b_, c = _bits(L["q_idx"]), _bits(L["k_idx"]), np.ascontiguousarray(L["w"], np.float32)
            keep += [a, b_, c]
            qi.append(a); ki.append(b_); wi.append(c)
        else:
            qi.append(None); ki.append(None); wi.append(None)
        q = _bits(L["q"]); keep.append(q); qq.append(q)
        if "kv" in L:
            kv = _bits(L["kv"]); keep.append(kv)
            KK.append(kv); VV.append(kv)
            ks = vs = kv.shape[-1]
        else:
            K_, V_ = _bits(L["k"]), _bits(L["v"]); keep += [K_, V_]
            KK.append(K_); VV.append(V_)
            ks, vs = K_.shape[-1], V_.shape[-1]
    idx = np.zeros((n, B, Lq, k), dtype=np.int32)
    out = np.zeros((n, B, Lq, n_h, Dv), dtype=np.float64)
    lse = np.zeros((n, B, Lq, n_h), dtype=np.float64)
    counters = np.zeros(2, dtype=np.int64)
    rc = _load().oracle_indexcache_forward(
        pattern.encode(), n, _ptr_array(qi), _ptr_array(ki), _ptr_array(wi),
        _ptr_array(qq), _ptr_array(KK), ks, _ptr_array(VV), vs, B, Lq, Lk,
        start_pos, H, dI, k, n_h, Dqk, Dv, scale, _ptr_array(list(idx)),
        _ptr_array(list(out)), _ptr_array(list(lse)), _p(counters))
    if rc != 0:
        raise ValueError(f"invalid IndexCache pattern {pattern!r}")
    return idx, out, lse, {"indexer_calls": int(counters[0]), "scored_pairs": int(counters[1])}
