"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a hand-worked example, a closed form, a special case that
reduces to a textbook/library routine, an invariant, or brute force on tiny
inputs.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from sparse_attention_13_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f32(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


# --------------------------------------------------------------------------
# indexer: I[t,s] = sum_j w_j ReLU(q_j . k_s)


def test_indexer_hand_example(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "indexer_hand_example.json")))
    q, k = bf16(g["q"]), bf16(g["k"])
    I = oracle_mod.indexer_row(q, k, np.array(g["w"], np.float32), g["T"])
    assert I.tolist() == g["scores"]
    for kk, want in g["topk"].items():
        assert oracle_mod.topk_row(I, g["T"], int(kk)).tolist() == want


def test_indexer_single_head_is_relu_dot(oracle_mod):
    # H = 1, w = 1 reduces to ReLU of a plain matrix-vector product.
    rng = np.random.default_rng(0)
    q = bf16(rng.normal(size=(1, 32)))
    k = bf16(rng.normal(size=(40, 32)))
    I = oracle_mod.indexer_row(q, k, np.ones(1, np.float32), 37)
    ref = np.maximum(f32(k)[:37] @ f32(q)[0], 0.0)
    np.testing.assert_allclose(I, ref, rtol=1e-13, atol=1e-13)


def test_indexer_linear_regime_folds_heads(oracle_mod):
    # All q, k >= 0: every dot is >= 0, ReLU is the identity and the head sum
    # folds into one combined query sum_j w_j q_j (catches transposed or
    # mis-indexed heads, a dropped weight, or a wrong key row).
    rng = np.random.default_rng(1)
    H, d, T = 6, 16, 25
    q = bf16(np.abs(rng.normal(size=(H, d))))
    k = bf16(np.abs(rng.normal(size=(T + 3, d))))
    w = rng.normal(size=H).astype(np.float32)
    I = oracle_mod.indexer_row(q, k, w, T)
    qc = (w.astype(np.float64)[:, None] * f32(q)).sum(0)
    np.testing.assert_allclose(I, f32(k)[:T] @ qc, rtol=1e-12, atol=1e-12)


def test_indexer_negative_dots_give_zero(oracle_mod):
    # q >= 0, k <= 0: every dot <= 0, so ReLU zeroes all heads (a sign error
    # in the ReLU would make the scores non-zero).
    rng = np.random.default_rng(2)
    q = bf16(np.abs(rng.normal(size=(4, 8))) + 0.1)
    k = bf16(-np.abs(rng.normal(size=(10, 8))) - 0.1)
    I = oracle_mod.indexer_row(q, k, rng.normal(size=4).astype(np.float32), 10)
    assert np.all(I == 0.0)


def test_indexer_integer_inputs_exact(oracle_mod):
    # Integer q/k in [-4,4] and w = +-2^-m: every score is a multiple of 1/8
    # and |I| <= 64 * 2048, so the double result must be exactly the integer
    # arithmetic result computed here with Python ints.
    rng = np.random.default_rng(3)
    H, d, T = 5, 12, 9
    qi = rng.integers(-4, 5, size=(H, d))
    ki = rng.integers(-4, 5, size=(T, d))
    m = rng.integers(0, 4, size=H)
    sgn = rng.choice([-1, 1], size=H)
    w = (sgn * 2.0 ** (-m)).astype(np.float32)
    I = oracle_mod.indexer_row(bf16(qi), bf16(ki), w, T)
    for s in range(T):
        acc8 = 0  # score * 8 as an exact integer
        for j in range(H):
            dot = int(sum(int(qi[j, c]) * int(ki[s, c]) for c in range(d)))
            acc8 += int(sgn[j]) * (8 >> int(m[j])) * max(dot, 0)
        assert I[s] * 8 == acc8


def test_indexer_positive_homogeneity_in_w(oracle_mod):
    rng = np.random.default_rng(4)
    q, k = bf16(rng.normal(size=(3, 8))), bf16(rng.normal(size=(12, 8)))
    w = rng.normal(size=3).astype(np.float32)
    I1 = oracle_mod.indexer_row(q, k, w, 12)
    I4 = oracle_mod.indexer_row(q, k, (4 * w).astype(np.float32), 12)
    np.testing.assert_array_equal(I4, 4 * I1)


# --------------------------------------------------------------------------
# top-k


def _rank_select(I, T, k):
    """Brute force: s is selected iff fewer than k candidates beat it, where
    u beats s when I[u] > I[s] or (I[u] == I[s] and u < s)."""
    sel = []
    for s in range(T):
        beats = sum(1 for u in range(T) if I[u] > I[s] or (I[u] == I[s] and u < s))
        if beats < k:
            sel.append(s)
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("T,k", [(0, 4), (1, 4), (3, 4), (4, 4), (9, 4), (40, 7), (64, 64), (65, 64)])
def test_topk_matches_rank_brute_force(oracle_mod, T, k):
    rng = np.random.default_rng(T * 131 + k)
    I = rng.integers(-3, 4, size=max(T, 1)).astype(np.float64)  # many ties
    got = oracle_mod.topk_row(I, T, k).tolist()
    assert got == _rank_select(I, T, k)


def test_topk_all_equal_takes_lowest_positions(oracle_mod):
    I = np.zeros(100)
    assert oracle_mod.topk_row(I, 100, 8).tolist() == list(range(8))


def test_topk_negative_zero_ties_positive_zero(oracle_mod):
    I = np.array([-0.0, 0.0, -0.0, 0.0, -1.0])
    assert oracle_mod.topk_row(I, 5, 2).tolist() == [0, 1]


def test_topk_negative_weights_pick_smallest_relu(oracle_mod):
    # With every head weight negative, I = -sum |w_j| ReLU(.), so the top-k
    # are the positions with the smallest non-negative ReLU mass.
    rng = np.random.default_rng(5)
    q = bf16(rng.normal(size=(1, 16)))
    k = bf16(rng.normal(size=(50, 16)))
    I = oracle_mod.indexer_row(q, k, np.array([-1.0], np.float32), 50)
    relu = np.maximum(f32(k) @ f32(q)[0], 0.0)
    order = sorted(range(50), key=lambda s: (relu[s], s))[:10]
    assert oracle_mod.topk_row(I, 50, 10).tolist() == sorted(order)


# --------------------------------------------------------------------------
# sparse / dense / masked attention


def _attn_inputs(seed, T, n_h=4, D=16, Dv=8):
    rng = np.random.default_rng(seed)
    q = bf16(rng.normal(size=(n_h, D)))
    K = bf16(rng.normal(size=(T, D)))
    V = bf16(rng.normal(size=(T, Dv)))
    return q, K, V


def test_attention_golden_closed_form(oracle_mod):
    # q = (1, 0), keys give logits 0, 1, 2; V = (1,0), (0,1), (1,1).
    q = bf16([[1, 0]])
    K = bf16([[0, 7], [1, -3], [2, 5]])
    V = bf16([[1, 0], [0, 1], [1, 1]])
    e = math.e
    out, lse = oracle_mod.dense_attn_row(q, K, V, 3, 1.0)
    z = 1 + e + e * e
    np.testing.assert_allclose(out[0], [(1 + e * e) / z, (e + e * e) / z], rtol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(z), rtol=1e-14)
    out, lse = oracle_mod.sparse_attn_row(q, K, V, np.array([0, 2, -1], np.int32), 1.0)
    np.testing.assert_allclose(out[0], [1.0, e * e / (1 + e * e)], rtol=1e-14)
    np.testing.assert_allclose(lse[0], math.log(1 + e * e), rtol=1e-14)


def test_dense_attention_matches_torch_sdpa(oracle_mod):
    T, n_h, D, Dv = 23, 3, 16, 8
    q, K, V = _attn_inputs(6, T + 1, n_h, D, Dv)
    scale = 0.3
    out, _ = oracle_mod.dense_attn_row(q, K, V, T, scale)
    qt = torch.tensor(f32(q))[None, :, None, :]            # [1, H, 1, D]
    kt = torch.tensor(f32(K)[:T])[None, None].expand(1, n_h, T, D)
    vt = torch.tensor(f32(V)[:T])[None, None].expand(1, n_h, T, Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    np.testing.assert_allclose(out, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,k", [(1, 4), (5, 8), (8, 8), (30, 64)])
def test_sparse_equals_dense_when_k_covers_history(oracle_mod, T, k):
    q, K, V = _attn_inputs(T, T + 2)
    I = np.random.default_rng(T).normal(size=T)
    idx = oracle_mod.topk_row(I, T, k)
    a, la = oracle_mod.sparse_attn_row(q, K, V, idx, 0.25)
    b, lb = oracle_mod.dense_attn_row(q, K, V, T, 0.25)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-13)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mask_formulation_equals_sparse(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    T, Lk, k = 40, 48, 12
    q, K, V = _attn_inputs(seed + 10, Lk)
    idx = np.sort(rng.choice(T, size=9, replace=False)).astype(np.int32)
    idx = np.concatenate([idx, -np.ones(k - 9, np.int32)])
    a, la = oracle_mod.sparse_attn_row(q, K, V, idx, 0.5)
    b, lb = oracle_mod.masked_attn_row(q, K, V, idx, T, 0.5)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-12)


def test_sparse_error_bound_holds_at_every_t(oracle_mod):
    # ||o_t - o_hat_t|| <= 2 V R_t(S_t), with V = max ||v_s|| and R_t the dense
    # attention mass outside S_t.
    T_max, n_h, D, Dv, k = 48, 2, 8, 8, 6
    q_all = [_attn_inputs(100 + t, 1, n_h, D, Dv)[0] for t in range(T_max)]
    _, K, V = _attn_inputs(7, T_max, n_h, D, Dv)
    Vf = f32(V)
    rng = np.random.default_rng(8)
    scale = 0.7
    for t in range(1, T_max):
        I = rng.normal(size=t)
        idx = oracle_mod.topk_row(I, t, k)
        o_hat, _ = oracle_mod.sparse_attn_row(q_all[t], K, V, idx, scale)
        o, _ = oracle_mod.dense_attn_row(q_all[t], K, V, t, scale)
        Vmax = np.linalg.norm(Vf[:t], axis=1).max()
        sel = set(int(s) for s in idx if s >= 0)
        for h in range(n_h):
            e = scale * (f32(K)[:t] @ f32(q_all[t])[h])
            a = np.exp(e - e.max()); a /= a.sum()
            R = sum(a[s] for s in range(t) if s not in sel)
            assert np.linalg.norm(o[h] - o_hat[h]) <= 2 * Vmax * R + 1e-12


def test_single_row_and_uniform_logits(oracle_mod):
    q, K, V = _attn_inputs(9, 20)
    out, lse = oracle_mod.sparse_attn_row(q, K, V, np.array([-1, 7, -1], np.int32), 1.0)
    np.testing.assert_array_equal(out, np.tile(f32(V)[7], (q.shape[0], 1)))
    np.testing.assert_allclose(lse, 1.0 * (f32(q) @ f32(K)[7]), rtol=1e-14)
    zero_q = bf16(np.zeros((2, 16)))
    sel = np.array([3, 11, 19, 2], np.int32)
    out, lse = oracle_mod.sparse_attn_row(zero_q, K, V, sel, 1.0)
    np.testing.assert_allclose(out[0], f32(V)[sel].mean(0), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse, math.log(4), rtol=1e-14)


def test_empty_selection_gives_zero(oracle_mod):
    q, K, V = _attn_inputs(10, 4)
    out, lse = oracle_mod.sparse_attn_row(q, K, V, -np.ones(5, np.int32), 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_selection_order_does_not_matter(oracle_mod):
    q, K, V = _attn_inputs(11, 30)
    idx = np.array([4, 9, 17, 22, -1, -1], np.int32)
    a, _ = oracle_mod.sparse_attn_row(q, K, V, idx, 0.5)
    b, _ = oracle_mod.sparse_attn_row(q, K, V, np.array([-1, 22, 4, -1, 17, 9], np.int32), 0.5)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# the IndexCache layer loop


def _stack(seed, pattern, B=2, L=24, H=3, dI=8, n_h=2, D=8, Dv=4, int_idx=True):
    layers = []
    for l in range(len(pattern)):
        # indexer inputs exist on every layer; the loop reads them on F layers only
        ent = {}
        ent["q_idx"] = synth.tensor(seed, synth.Q_IDX, synth.INT9, l, (B, L, H, dI))
        ent["k_idx"] = synth.tensor(seed, synth.K_IDX, synth.INT9, l, (B, L, dI))
        ent["w"] = synth.tensor(seed, synth.W, synth.POW2W, l, (B, L, H), bf16=False)
        ent["q"] = synth.tensor(seed, synth.Q, synth.NORMAL, l, (B, L, n_h, D), sigma=0.5)
        ent["k"] = synth.tensor(seed, synth.K_SEP, synth.NORMAL, l, (B, L, D), sigma=0.5)
        ent["v"] = synth.tensor(seed, synth.V_SEP, synth.NORMAL, l, (B, L, Dv), sigma=0.5)
        layers.append(ent)
    dims = dict(B=B, Lq=L, Lk=L, start_pos=0, H=H, dI=dI, k=5, n_h=n_h, Dqk=D, Dv=Dv,
                scale=1 / math.sqrt(D))
    return layers, dims


def test_pattern_validation_and_reuse_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "fsssfsss_reuse.json")))
    layers, dims = _stack(0, g["pattern"])
    idx, out, lse, cnt = oracle_mod.indexcache_forward(g["pattern"], layers, **dims)
    assert cnt["indexer_calls"] == g["indexer_runs"]
    for l, src in enumerate(g["source_layer_zero_based"]):
        np.testing.assert_array_equal(idx[l], idx[src])
    # layers 0 and 4 run their own indexers on different inputs
    assert not np.array_equal(idx[0], idx[4])
    for bad in g["invalid_patterns"]:
        n = max(len(bad), 1)
        with pytest.raises(ValueError):
            oracle_mod.indexcache_forward(bad, (layers * 2)[:n] if bad else layers[:1], **dims)


def test_all_f_equals_per_layer_dsa(oracle_mod):
    pattern = "FFF"
    layers, d = _stack(1, pattern)
    idx, out, lse, _ = oracle_mod.indexcache_forward(pattern, layers, **d)
    for l, L in enumerate(layers):
        for b in range(d["B"]):
            for i in range(d["Lq"]):
                I = oracle_mod.indexer_row(L["q_idx"][b, i], L["k_idx"][b], L["w"][b, i], i)
                sel = oracle_mod.topk_row(I, i, d["k"])
                np.testing.assert_array_equal(idx[l, b, i], sel)
                o, _ = oracle_mod.sparse_attn_row(L["q"][b, i], L["k"][b], L["v"][b], sel, d["scale"])
                np.testing.assert_array_equal(out[l, b, i], o)


def test_shared_layer_uses_own_kv_at_cached_positions(oracle_mod):
    # [IC] §1.2: an S layer reads the F layer's positions but its OWN K/V.
    layers, d = _stack(2, "FS")
    idx, out, _, _ = oracle_mod.indexcache_forward("FS", layers, **d)
    np.testing.assert_array_equal(idx[0], idx[1])
    assert not np.allclose(out[0], out[1])
    b, i = 1, 17
    o, _ = oracle_mod.sparse_attn_row(layers[1]["q"][b, i], layers[1]["k"][b], layers[1]["v"][b],
                                      idx[0, b, i], d["scale"])
    np.testing.assert_array_equal(out[1, b, i], o)


def test_first_row_attends_nothing(oracle_mod):
    layers, d = _stack(3, "F")
    idx, out, lse, _ = oracle_mod.indexcache_forward("F", layers, **d)
    assert np.all(idx[0, :, 0] == -1)
    assert np.all(out[0, :, 0] == 0) and np.all(np.isneginf(lse[0, :, 0]))
    # row i sees exactly min(i, k) positions, all < i
    for i in range(d["Lq"]):
        sel = idx[0, 0, i]
        valid = sel[sel >= 0]
        assert len(valid) == min(i, d["k"]) and np.all(valid < i)
        assert np.all(np.diff(valid) > 0)


@pytest.mark.parametrize("N", [4, 8, 16])
def test_indexer_work_scales_as_m_over_n(oracle_mod, N):
    # [IC] §1.2: keeping M of N indexers takes prefill indexer work from
    # O(N L^2) to O(M L^2); the oracle counts every scored (t, s) pair.
    L = 10
    pairs_per_layer = L * (L - 1) // 2
    for pat, M in [("F" * N, N), ("FS" * (N // 2), N // 2), ("FSSS" * (N // 4), N // 4)]:
        layers, d = _stack(4, pat, B=1, L=L, H=2, dI=4, n_h=1, D=4, Dv=4)
        _, _, _, cnt = oracle_mod.indexcache_forward(pat, layers, **d)
        assert cnt["indexer_calls"] == M
        assert cnt["scored_pairs"] == M * pairs_per_layer


def test_decode_rows_use_start_pos(oracle_mod):
    # Lq = 1 query at absolute position start_pos = Lk sees every cached key.
    B, Lk, H, dI = 1, 30, 2, 8
    qi = synth.tensor(5, synth.Q_IDX, synth.INT9, 0, (B, 1, H, dI))
    ki = synth.tensor(5, synth.K_IDX, synth.INT9, 0, (B, Lk, dI))
    w = synth.tensor(5, synth.W, synth.POW2W, 0, (B, 1, H), bf16=False)
    q = synth.tensor(5, synth.Q, synth.NORMAL, 0, (B, 1, 2, 8))
    kv = synth.tensor(5, synth.KV, synth.NORMAL, 0, (B, Lk, 8))
    layers = [dict(q_idx=qi, k_idx=ki, w=w, q=q, kv=kv)]
    idx, out, _, _ = oracle_mod.indexcache_forward(
        "F", layers, B=B, Lq=1, Lk=Lk, start_pos=Lk, H=H, dI=dI, k=64, n_h=2, Dqk=8, Dv=8,
        scale=0.3)
    assert idx[0, 0, 0].tolist() == list(range(Lk)) + [-1] * (64 - Lk)
    o, _ = oracle_mod.dense_attn_row(q[0, 0], kv[0], kv[0], Lk, 0.3)
    np.testing.assert_allclose(out[0, 0, 0], o, rtol=1e-13, atol=1e-15)


# --------------------------------------------------------------------------
# selection quality: dense weights, CapturedMass, Recall, cross-layer overlap


def test_dense_probs_two_keys_are_logistic(oracle_mod):
    # Two keys: alpha_1 = 1 / (1 + exp(-(e_1 - e_0))), a closed form.
    q = bf16([[1, 2], [-0.5, 1]])
    K = bf16([[3, -1], [0.25, 2]])
    scale = 0.7
    alpha = oracle_mod.dense_probs_row(q, K, 2, scale)
    qf, Kf = f32(q), f32(K)
    for h in range(2):
        d = scale * (qf[h] @ Kf[1] - qf[h] @ Kf[0])
        np.testing.assert_allclose(alpha[h, 1], 1.0 / (1.0 + math.exp(-d)), rtol=1e-14)
        np.testing.assert_allclose(alpha[h, 0], 1.0 / (1.0 + math.exp(d)), rtol=1e-14)


def test_dense_probs_match_torch_softmax(oracle_mod):
    T, n_h, D = 37, 3, 16
    q, K, _ = _attn_inputs(8, T + 5, n_h, D)
    alpha = oracle_mod.dense_probs_row(q, K, T, 0.4)
    ref = torch.softmax(0.4 * torch.tensor(f32(q)) @ torch.tensor(f32(K)[:T]).T, dim=-1)
    np.testing.assert_allclose(alpha, ref.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(alpha.sum(axis=1), 1.0, rtol=1e-14)
    # a zero query weighs every visible key alike
    flat = oracle_mod.dense_probs_row(np.zeros_like(q), K, T, 0.4)
    np.testing.assert_allclose(flat, 1.0 / T, rtol=1e-14)
    assert oracle_mod.dense_probs_row(q, K, 0, 0.4).shape == (n_h, 0)


@pytest.mark.parametrize("seed", [0, 1])
def test_captured_mass_equals_lse_ratio(oracle_mod, seed):
    # sum_{s in S} alpha_s = exp(lse_S - lse_{P_t}): the weights of one C
    # routine against the log-sum-exps of the attention routines.
    rng = np.random.default_rng(seed)
    T, k = 60, 16
    q, K, V = _attn_inputs(seed + 20, T + 3, 4, 16, 8)
    alpha = oracle_mod.dense_probs_row(q, K, T, 0.35)
    idx = oracle_mod.topk_row(rng.normal(size=T), T, k)
    mass = oracle_mod.captured_mass_row(alpha, idx)
    _, l_sel = oracle_mod.sparse_attn_row(q, K, V, idx, 0.35)
    _, l_all = oracle_mod.dense_attn_row(q, K, V, T, 0.35)
    np.testing.assert_allclose(mass, np.exp(l_sel - l_all), rtol=1e-12)
    assert np.all((mass > 0) & (mass < 1))


def test_captured_mass_full_empty_and_additive(oracle_mod):
    T, k = 25, 32
    q, K, _ = _attn_inputs(3, T, 2, 8)
    alpha = oracle_mod.dense_probs_row(q, K, T, 0.5)
    full = oracle_mod.topk_row(np.zeros(T), T, k)          # all of P_t
    np.testing.assert_allclose(oracle_mod.captured_mass_row(alpha, full), 1.0, rtol=1e-14)
    np.testing.assert_array_equal(oracle_mod.captured_mass_row(alpha, -np.ones(k, np.int32)), 0.0)
    a = np.array([0, 3, 7, -1], np.int32)
    b = np.array([1, 2, 20, 24], np.int32)
    ab = np.array([0, 1, 2, 3, 7, 20, 24, -1], np.int32)
    np.testing.assert_allclose(oracle_mod.captured_mass_row(alpha, a)
                               + oracle_mod.captured_mass_row(alpha, b),
                               oracle_mod.captured_mass_row(alpha, ab), rtol=1e-14)
    # T = 0: nothing visible, nothing missed
    np.testing.assert_array_equal(
        oracle_mod.captured_mass_row(np.zeros((2, 0)), -np.ones(4, np.int32)), 1.0)


def test_overlap_and_recall_hand_example(oracle_mod):
    a = np.array([1, 3, 5, -1], np.int32)
    b = np.array([3, 4, 5, 6], np.int32)
    assert oracle_mod.overlap_row(a, b) == 2
    assert oracle_mod.overlap_row(b, b) == 4
    assert oracle_mod.overlap_row(a, np.array([0, 2, 4, 6], np.int32)) == 0
    assert oracle_mod.recall_row(a, b) == pytest.approx(2 / 3)
    assert oracle_mod.recall_row(b, a) == pytest.approx(2 / 4)
    assert oracle_mod.recall_row(-np.ones(4, np.int32), b) == 1.0


def test_oracle_selection_is_topk_of_head_mean(oracle_mod):
    # brute force on a tiny row: sort by (mean weight desc, s asc), keep k
    T, k = 19, 6
    q, K, _ = _attn_inputs(12, T, 3, 8)
    alpha = oracle_mod.dense_probs_row(q, K, T, 0.6)
    mean = alpha.mean(axis=0)
    want = sorted(sorted(range(T), key=lambda s: (-mean[s], s))[:k])
    assert oracle_mod.oracle_selection_row(alpha, T, k).tolist() == want
    # one head: the head's own weights decide
    a1 = oracle_mod.dense_probs_row(q[:1], K, T, 0.6)
    want1 = sorted(sorted(range(T), key=lambda s: (-a1[0, s], s))[:k])
    assert oracle_mod.oracle_selection_row(a1, T, k).tolist() == want1
    # t < k: every visible position, then -1
    assert oracle_mod.oracle_selection_row(alpha[:, :4], 4, k).tolist() == [0, 1, 2, 3, -1, -1]


# --------------------------------------------------------------------------
# CSA indexer over compressed blocks: s < floor(t / m)


def test_csa_visibility_follows_floor_rule(oracle_mod):
    # one head, w = 1, block s scores s + 1: the top-2 of the visible blocks
    # are the last two below floor(t / 4)
    m, nb, d = 4, 8, 8
    q = bf16(np.eye(1, d))
    kc = bf16(np.arange(1, nb + 1)[:, None] * np.eye(1, d))
    w = np.ones(1, np.float32)
    for t in range(0, m * nb + 1):
        T = t // m
        assert oracle_mod.csa_visible(t, m) == T
        I, idx = oracle_mod.csa_indexer_topk_row(q, kc, w, t, m, 2)
        np.testing.assert_array_equal(I, np.arange(1, T + 1))
        want = [s for s in (T - 2, T - 1) if s >= 0]
        assert idx.tolist() == want + [-1] * (2 - len(want))
    # t = 7 sees block 0 only; t = 8 also block 1
    assert oracle_mod.csa_indexer_topk_row(q, kc, w, 7, m, 4)[1].tolist() == [0, -1, -1, -1]
    assert oracle_mod.csa_indexer_topk_row(q, kc, w, 8, m, 4)[1].tolist() == [0, 1, -1, -1]


def test_csa_with_m_1_is_the_token_indexer(oracle_mod):
    rng = np.random.default_rng(4)
    H, d, L, k = 4, 16, 40, 7
    q = bf16(rng.normal(size=(H, d)))
    kk = bf16(rng.normal(size=(L, d)))
    w = rng.normal(size=H).astype(np.float32)
    for t in (0, 1, 6, 7, 8, 39):
        I, idx = oracle_mod.csa_indexer_topk_row(q, kk, w, t, 1, k)
        I2 = oracle_mod.indexer_row(q, kk, w, t)
        np.testing.assert_array_equal(I, I2)
        np.testing.assert_array_equal(idx, oracle_mod.topk_row(I2, t, k))


def test_csa_attention_reads_selected_compressed_entries(oracle_mod):
    # keys and values both come from the selected compressed entries: with a
    # single selected entry the output is that entry's value columns
    q, C, _ = _attn_inputs(9, 6, 2, 16)
    out, lse = oracle_mod.csa_attn_row(q, C, np.array([3, -1, -1], np.int32), 0.5, Dv=8)
    np.testing.assert_allclose(out, np.broadcast_to(f32(C)[3, :8], out.shape), rtol=1e-15)
    np.testing.assert_allclose(lse, 0.5 * f32(q) @ f32(C)[3], rtol=1e-14)


# --------------------------------------------------------------------------
# low-precision selector: MX-quantised QK path, scores rounded to bf16


def test_e2m1_rounding_table(oracle_mod):
    # the E2M1 grid is {0, 0.5, 1, 1.5, 2, 3, 4, 6}; midpoints go to the even
    # code, anything beyond 6 saturates
    x = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 0.5, 3.0, -1.75, -0.0]
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 0.5, 3.0, -2.0, -0.0]
    got = oracle_mod.round_to_format(x, "e2m1")
    np.testing.assert_array_equal(got, want)
    assert math.copysign(1.0, got[-1]) == -1.0


def test_e4m3_rounding_table(oracle_mod):
    x = [448.0, 460.0, 1e6, 2.0 ** -9, 2.0 ** -10, 1.5 * 2.0 ** -10, 0.3, 17.0, 19.0, 2.0 ** -6, 240.0, 232.0]
    want = [448.0, 448.0, 448.0, 2.0 ** -9, 0.0, 2.0 ** -9, 0.3125, 16.0, 20.0, 2.0 ** -6, 240.0, 224.0]
    np.testing.assert_array_equal(oracle_mod.round_to_format(x, "e4m3"), want)
    # the positive finite E4M3 codes: 7 subnormals m 2^-9 and (1 + m/8) 2^(e-7)
    # for e = 1..15, without the top code of e = 15 (NaN): 126 values
    codes = sorted({m * 2.0 ** -9 for m in range(1, 8)} |
                   {(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)} - {480.0})
    assert len(codes) == 126 and codes[-1] == 448.0
    np.testing.assert_array_equal(oracle_mod.round_to_format(codes, "e4m3"), codes)
    image = np.unique(oracle_mod.round_to_format(np.geomspace(2.0 ** -12, 470.0, 200001), "e4m3"))
    np.testing.assert_array_equal(image, [0.0] + codes)
    # midpoints between neighbouring codes go to the one with the even mantissa
    mids = (np.array(codes[:-1]) + np.array(codes[1:])) / 2
    got = oracle_mod.round_to_format(mids, "e4m3")
    lo, hi = np.array(codes[:-1]), np.array(codes[1:])
    even_lo = np.array([round(c / 2.0 ** (max(math.floor(math.log2(c)), -6) - 3)) % 2 == 0 for c in lo])
    np.testing.assert_array_equal(got, np.where(even_lo, lo, hi))
    v = np.sort(np.random.default_rng(0).normal(scale=50, size=5000))
    assert np.all(np.diff(oracle_mod.round_to_format(v, "e4m3")) >= 0)


def test_mx_block_scale_rule(oracle_mod):
    # amax = 1 gives X = 2^-8 for E4M3 (1.0 is element 256) and 2^-2 for E2M1
    x = np.zeros(32)
    x[0], x[1], x[2] = 1.0, 1e-6, -0.7
    e4 = oracle_mod.mx_quantize(x, "e4m3")
    assert e4[0] == 1.0 and e4[1] == 0.0           # 1e-6 * 256 lies below 2^-10
    assert e4[2] == oracle_mod.round_to_format(-0.7 * 256, "e4m3") / 256
    e2 = oracle_mod.mx_quantize(x, "e2m1")
    assert e2[0] == 1.0 and e2[2] == -0.75          # -2.8 -> -3 on the E2M1 grid, times 2^-2
    # blocks are independent: a large value in block 1 leaves block 0 alone
    y = np.concatenate([x, 1000.0 * np.ones(32)])
    np.testing.assert_array_equal(oracle_mod.mx_quantize(y, "e4m3")[:32], e4)
    # integers in [-4, 4] are represented exactly in both formats
    ints = np.random.default_rng(1).integers(-4, 5, size=(3, 128)).astype(float)
    for fmt in ("e4m3", "e2m1"):
        np.testing.assert_array_equal(oracle_mod.mx_quantize(ints, fmt), ints)


def test_bf16_round(oracle_mod):
    got = oracle_mod.bf16_round([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -3.0, 257.0, 259.0, 2.0 ** 17 + 512])
    np.testing.assert_array_equal(got, [1.0, 1 + 2.0 ** -6, -3.0, 256.0, 260.0, 2.0 ** 17])


def test_lowprec_selector_on_integer_inputs(oracle_mod):
    # integer q, k lose nothing in either format, so the low-precision score is
    # the exact score rounded to bf16; many scores then tie and the lower
    # position wins
    rng = np.random.default_rng(2)
    H, d, T, k = 4, 64, 300, 40
    q = bf16(rng.integers(-4, 5, size=(H, d)))
    kk = bf16(rng.integers(-4, 5, size=(T, d)))
    w = (2.0 ** -rng.integers(0, 3, size=H) * rng.choice([-1, 1], size=H)).astype(np.float32)
    I = oracle_mod.indexer_row(q, kk, w, T)
    for fmt in ("e4m3", "e2m1"):
        Ilp = oracle_mod.lowprec_indexer_row(q, kk, w, T, fmt)
        np.testing.assert_array_equal(Ilp, oracle_mod.bf16_round(I))
    sel = oracle_mod.topk_row(Ilp, T, k)
    want = sorted(sorted(range(T), key=lambda s: (-Ilp[s], s))[:k])
    assert sel.tolist() == want
    assert 0.0 <= oracle_mod.recall_row(oracle_mod.topk_row(I, T, k), sel) <= 1.0


def test_lowprec_selector_recall_falls_with_precision(oracle_mod):
    # normal inputs: E4M3 keeps more of the exact selection than E2M1
    rng = np.random.default_rng(3)
    H, d, T, k = 8, 128, 2000, 128
    q = bf16(rng.normal(size=(H, d)))
    kk = bf16(rng.normal(size=(T, d)))
    w = rng.uniform(0.5, 1.5, size=H).astype(np.float32)
    exact = oracle_mod.topk_row(oracle_mod.indexer_row(q, kk, w, T), T, k)
    r = {fmt: oracle_mod.recall_row(exact, oracle_mod.topk_row(
        oracle_mod.lowprec_indexer_row(q, kk, w, T, fmt), T, k)) for fmt in ("e4m3", "e2m1")}
    assert 0.5 < r["e2m1"] < r["e4m3"] <= 1.0
