"""GPU parity of the selection-quality tools ([IDX] §8) against the oracle:
dense attention statistics (§8.1), the oracle selection TopK over the dense
weights (§8.2), the set intersections behind Recall@k (§8.2) and the
adjacent-layer overlap (§8.4), and CapturedMass@k (§8.1).

Where floating point decides an index (the top-k over dense weights), both
sides decide on the same fp32 values (the kernel's), so indices match bit for
bit; the weights themselves are compared against the fp64 oracle within the
fp32 dot-product bound derived in ``_weight_bound``."""
import math

import numpy as np
import pytest

from sparse_attention_13_b200 import synth

from gpu_util import indexer_inputs_host, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_13_b200 import dsa as _dsa
    _dsa.lib()
    return _dsa


def _weight_bound(q_row, K, T, scale):
    """|fp32 logit - exact logit| per (head, key): a D-term dot of exact bf16
    products accumulated by FMAs has error <= D * 2^-24 * sum_c |q_c k_c|
    (first order); scaled, doubled for margin.  Returns the max over the row."""
    if T == 0:
        return 0.0
    qf = synth.bf16_bits_to_f32(q_row).astype(np.float64)
    kf = synth.bf16_bits_to_f32(K[:T, :qf.shape[1]]).astype(np.float64)
    mag = np.abs(qf) @ np.abs(kf).T
    return float(2.0 * scale * (qf.shape[1] + 2) * 2.0 ** -24 * mag.max())


def _check_weights(oracle_mod, q, K, lse, mw, rows, scale, start_pos=0):
    for (b, i) in rows:
        T = start_pos + i
        _, l_ref = oracle_mod.dense_attn_row(q[b, i], K[b], K[b], T, scale, Dv=8)
        eb = _weight_bound(q[b, i], K[b], T, scale)
        if T == 0:
            assert np.all(np.isneginf(lse[b, i]))
            continue
        n_h = q.shape[2]
        u = 2.0 ** -24
        # the running sum of T positive exponentials: relative error <= (T + 4) u
        lse_tol = eb + (T + 4) * u + 2 * u * np.abs(l_ref).max()
        np.testing.assert_allclose(lse[b, i], l_ref, rtol=0, atol=lse_tol)
        want = oracle_mod.dense_probs_row(q[b, i], K[b], T, scale).mean(axis=0)
        # exp(logit - lse): errors of both, then a sum of n_h positive terms
        np.testing.assert_allclose(mw[b, i, :T], want, rtol=2 * (eb + lse_tol) + (n_h + 8) * u,
                                   atol=1e-30)
        assert np.all(mw[b, i, T:] == 0)


def _mla(seed, B, Lq, Lk, layer=0):
    q = synth.tensor(seed, synth.Q, synth.NORMAL, layer, (B, Lq, 128, 576), sigma=0.5, corr=True)
    kv = synth.tensor(seed, synth.KV, synth.NORMAL, layer, (B, Lk, 576), sigma=0.5, corr=True)
    return q, kv


def test_dense_weights_mla_rows(dsa, oracle_mod):
    # 300 rows span several 64-key tiles and a ragged tail.
    B, L = 1, 300
    q, kv = _mla(41, B, L, L)
    scale = 1 / math.sqrt(576)
    lse, mw = dsa.dense_weights(to_dev_bf16(q), to_dev_bf16(kv), scale=scale)
    dsa.check_device_errors()
    rows = [(0, i) for i in (0, 1, 2, 63, 64, 65, 128, 200, 299)]
    _check_weights(oracle_mod, q, kv, lse.cpu().numpy(), mw.cpu().numpy(), rows, scale)


def test_dense_weights_small_heads_and_decode(dsa, oracle_mod):
    rng = np.random.default_rng(5)
    # 4 heads x 64 (the tiny config's MQA), two sequences
    B, L, n_h, D = 2, 150, 4, 64
    q = synth.f32_to_bf16_bits(rng.normal(size=(B, L, n_h, D)).astype(np.float32))
    K = synth.f32_to_bf16_bits(rng.normal(size=(B, L, D)).astype(np.float32))
    lse, mw = dsa.dense_weights(to_dev_bf16(q), to_dev_bf16(K), scale=0.125)
    rows = [(b, i) for b in range(B) for i in (0, 1, 70, 149)]
    _check_weights(oracle_mod, q, K, lse.cpu().numpy(), mw.cpu().numpy(), rows, 0.125)
    # decode rows: one query per sequence at t = Lk
    Lk = 333
    q1, kv = _mla(43, 2, 1, Lk)
    lse, mw = dsa.dense_weights(to_dev_bf16(q1), to_dev_bf16(kv), start_pos=Lk, scale=1 / 24)
    _check_weights(oracle_mod, q1, kv, lse.cpu().numpy(), mw.cpu().numpy(),
                   [(0, 0), (1, 0)], 1 / 24, start_pos=Lk)


@pytest.mark.parametrize("T,k,levels", [(3000, 512, 0), (2500, 2048, 4), (700, 1, 2),
                                        (129, 128, 1), (64, 300, 0), (2049, 2048, 3)])
def test_topk_rows_exact(dsa, oracle_mod, T, k, levels):
    import torch
    rng = np.random.default_rng(T + k)
    B, Lq = 2, 3
    start = T - Lq + 1
    if levels:
        s = rng.integers(0, levels, size=(B, Lq, T)).astype(np.float32)
        s[rng.random(s.shape) < 0.2] = -0.0     # -0 ties with +0
    else:
        s = rng.normal(size=(B, Lq, T)).astype(np.float32)
    got = dsa.topk_rows(torch.from_numpy(s).cuda(), k, start_pos=start).cpu().numpy()
    for b in range(B):
        for i in range(Lq):
            t = start + i
            want = oracle_mod.topk_row(s[b, i].astype(np.float64), t, k)
            np.testing.assert_array_equal(got[b, i], want)


def test_oracle_selection_recall_and_overlap(dsa, oracle_mod):
    # Recall@k of the lightning indexer's selection against the dense
    # attention's own TopK (the oracle selection of [IDX] §8.2).
    import torch
    B, L, H, d, kk = 1, 400, 64, 128, 96
    scale = 1 / math.sqrt(576)
    q, kv = _mla(47, B, L, L)
    lse, mw = dsa.dense_weights(to_dev_bf16(q), to_dev_bf16(kv), scale=scale)
    s_or = dsa.topk_rows(mw, kk)
    qi, ki, w = indexer_inputs_host(47, B, L, L, H, d, integer=False)
    s_model = dsa.indexer_topk(to_dev_bf16(qi), to_dev_bf16(ki), to_dev_f32(w), kk)
    inter = dsa.index_overlap(s_or, s_model).cpu().numpy()
    mw_h, s_or_h, s_model_h = mw.cpu().numpy(), s_or.cpu().numpy(), s_model.cpu().numpy()
    assert dsa.check_indices(s_or) == 0
    for i in range(L):
        # the oracle selection, decided on the kernel's fp32 weights
        np.testing.assert_array_equal(
            s_or_h[0, i], oracle_mod.topk_row(mw_h[0, i, :i].astype(np.float64), i, kk))
        assert inter[0, i] == oracle_mod.overlap_row(s_or_h[0, i], s_model_h[0, i])
    n_or = np.minimum(np.arange(L), kk)
    recall = np.where(n_or > 0, inter[0] / np.maximum(n_or, 1), 1.0)
    for i in (0, 5, 95, 96, 97, 399):
        assert recall[i] == pytest.approx(oracle_mod.recall_row(s_or_h[0, i], s_model_h[0, i]))
    # rows with t <= k select all of P_t on both sides
    assert np.all(recall[:kk + 1] == 1.0)


def test_index_overlap_adjacent_layers(dsa, oracle_mod):
    # [IDX] §8.4 overlap |S^(l) & S^(l+1)| / k on correlated synthetic layers
    B, L, H, d, kk = 2, 1500, 64, 128, 256
    sel = []
    for layer in (0, 1):
        qi, ki, w = indexer_inputs_host(53, B, L, L, H, d, layer=layer, corr=True)
        sel.append(dsa.indexer_topk(to_dev_bf16(qi), to_dev_bf16(ki), to_dev_f32(w), kk))
    inter = dsa.index_overlap(sel[0], sel[1]).cpu().numpy()
    a, b = sel[0].cpu().numpy(), sel[1].cpu().numpy()
    for bb in range(B):
        for i in range(0, L, 37):
            assert inter[bb, i] == oracle_mod.overlap_row(a[bb, i], b[bb, i])
    assert np.all(inter[:, :kk + 1] == np.minimum(np.arange(kk + 1), kk))
    same = dsa.index_overlap(sel[0], sel[0]).cpu().numpy()
    np.testing.assert_array_equal(same, np.minimum(np.arange(L), kk)[None].repeat(B, 0))


def test_captured_mass(dsa, oracle_mod):
    import torch
    B, L, kk = 1, 260, 64
    scale = 1 / math.sqrt(576)
    q, kv = _mla(59, B, L, L)
    qd, kvd = to_dev_bf16(q), to_dev_bf16(kv)
    lse_d, mw = dsa.dense_weights(qd, kvd, scale=scale)
    qi, ki, w = indexer_inputs_host(59, B, L, L, 64, 128, integer=False)
    idx = dsa.indexer_topk(to_dev_bf16(qi), to_dev_bf16(ki), to_dev_f32(w), kk)
    lse_s = torch.empty_like(lse_d)
    dsa.sparse_attn(qd, kvd, kvd, idx, scale, D_v=512, lse=lse_s)
    mass = dsa.captured_mass(lse_s, lse_d).cpu().numpy()
    idx_h = idx.cpu().numpy()
    for i in (0, 1, 30, 64, 65, 150, 259):
        want = oracle_mod.captured_mass_row(oracle_mod.dense_probs_row(q[0, i], kv[0], i, scale),
                                            idx_h[0, i])
        # lse_s carries the attention kernel's bf16 probabilities (|dlse| <= 1e-3)
        np.testing.assert_allclose(mass[0, i], want, rtol=2.5e-3, atol=0)
    assert np.all(mass[0, :kk + 1] == pytest.approx(1.0, abs=2.5e-3))
    assert np.all((mass[0, kk + 1:] > 0) & (mass[0, kk + 1:] < 1.0 + 2.5e-3))
