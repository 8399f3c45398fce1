"""Helpers shared by the GPU parity tests (inputs, oracle comparisons)."""
from __future__ import annotations

import numpy as np

from sparse_attention_13_b200 import synth


def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_f32(x: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def indexer_inputs_host(seed, B, Lq, Lk, H, d, layer=0, integer=True, corr=False):
    if integer:
        q = synth.tensor(seed, synth.Q_IDX, synth.INT9, layer, (B, Lq, H, d), corr=corr)
        k = synth.tensor(seed, synth.K_IDX, synth.INT9, layer, (B, Lk, d), corr=corr)
        w = synth.tensor(seed, synth.W, synth.POW2W, layer, (B, Lq, H), bf16=False)
    else:
        q = synth.tensor(seed, synth.Q_IDX, synth.NORMAL, layer, (B, Lq, H, d), sigma=1.0)
        k = synth.tensor(seed, synth.K_IDX, synth.NORMAL, layer, (B, Lk, d), sigma=1.0)
        w = synth.tensor(seed, synth.W, synth.NORMAL, layer, (B, Lq, H), sigma=1.0, bf16=False)
    return q, k, w


def score_error_bound(q_row, k, w_row, T):
    """Bound on |fp32 score - exact score| for the candidates s < T: each
    head dot sums d exact bf16 products in fp32 and the head sum adds H
    terms, so |err| <= (d + H + 2) * 2^-23 * sum_j |w_j| sum_c |q_jc k_sc|
    (first order), doubled for margin."""
    qf = synth.bf16_bits_to_f32(q_row).astype(np.float64)
    kf = synth.bf16_bits_to_f32(k[:T]).astype(np.float64)
    H, d = qf.shape
    mag = np.abs(kf) @ np.abs(qf).T                     # [T, H]
    return 2.0 * (d + H + 2) * 2.0 ** -23 * (mag @ np.abs(w_row.astype(np.float64)))


def check_topk_row(got, want, I, k, bound=None):
    """Exact equality, or (with ``bound``) agreement up to near-ties: every
    position in one set but not the other must score within the error bound
    of the oracle's k-th best score."""
    got = np.asarray(got)
    want = np.asarray(want)
    if bound is None:
        np.testing.assert_array_equal(got, want)
        return 0
    gv = got[got >= 0]
    wv = want[want >= 0]
    assert len(gv) == len(wv), "row length differs"
    assert np.all(np.diff(gv) > 0), "row not strictly ascending"
    if np.array_equal(gv, wv):
        return 0
    order = np.lexsort((np.arange(len(I)), -I))
    kth = I[order[min(k, len(I)) - 1]]
    diff = np.setxor1d(gv, wv)
    for s in diff:
        assert abs(I[s] - kth) <= 2 * bound[s] + 1e-30, (s, I[s], kth, bound[s])
    return len(diff)
