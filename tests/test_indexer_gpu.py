"""GPU parity of dsa_indexer_topk (fused indexer + top-k, through the C ABI)
against the CPU oracle.  Integer-valued inputs with power-of-two head
weights make every fp32 score exact, so indices must match bit for bit."""
import numpy as np
import pytest

from sparse_attention_13_b200 import synth

from gpu_util import (check_topk_row, indexer_inputs_host, score_error_bound, to_dev_bf16,
                      to_dev_f32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_13_b200 import dsa as _dsa
    _dsa.lib()
    return _dsa


def _run(dsa, q, k, w, kk, start_pos=0):
    out = dsa.indexer_topk(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), kk, start_pos=start_pos)
    dsa.check_device_errors()
    return out.cpu().numpy()


def _oracle_rows(oracle_mod, q, k, w, rows, kk, start_pos=0):
    res = {}
    for (b, i) in rows:
        T = start_pos + i
        I = oracle_mod.indexer_row(q[b, i], k[b], w[b, i], T)
        res[(b, i)] = (I, oracle_mod.topk_row(I, T, kk))
    return res


def test_synth_device_matches_host(dsa):
    import torch
    for (kind, dist, layer, corr, sig, bf) in [
            (synth.Q_IDX, synth.INT9, 2, True, 1.0, True), (synth.W, synth.POW2W, 1, False, 1.0, False),
            (synth.KV, synth.NORMAL, 3, True, 0.5, True), (synth.Q, synth.NORMAL, 0, False, 1.0, False)]:
        n = 100003
        host = synth.tensor(9, kind, dist, layer, (n,), sigma=sig, corr=corr, bf16=bf)
        t = torch.empty(n, dtype=torch.bfloat16 if bf else torch.float32, device="cuda")
        synth.fill_cuda(t, 9, kind, dist, layer, sigma=sig, corr=corr)
        dev = t.view(torch.int16).cpu().numpy().view(np.uint16) if bf else t.cpu().numpy()
        np.testing.assert_array_equal(dev, host)


def test_tiny_config_integer_exact(dsa, oracle_mod):
    # 4 indexer heads, d_I = 32, k = 64, L = 512 (the tiny stack's indexer).
    B, L, H, d, kk = 1, 512, 4, 32, 64
    q, k, w = indexer_inputs_host(11, B, L, L, H, d)
    got = _run(dsa, q, k, w, kk)
    for (b, i), (I, want) in _oracle_rows(oracle_mod, q, k, w, [(0, i) for i in range(L)], kk).items():
        check_topk_row(got[b, i], want, I, kk)


def test_tiny_config_float_near_ties(dsa, oracle_mod):
    # Tiny config with q/k/w ~ N(0,1) (q/k rounded to bf16): indices agree up to
    # candidates whose scores are within the fp32 rounding bound of the k-th.
    B, L, H, d, kk = 1, 512, 4, 32, 64
    q, k, w = indexer_inputs_host(12, B, L, L, H, d, integer=False)
    got = _run(dsa, q, k, w, kk)
    flips = 0
    for (b, i), (I, want) in _oracle_rows(oracle_mod, q, k, w, [(0, i) for i in range(L)], kk).items():
        bound = score_error_bound(q[b, i], k[b], w[b, i], i)
        flips += check_topk_row(got[b, i], want, I, kk, bound)
    assert flips <= 8


@pytest.mark.parametrize("B,L,H,d,kk", [
    (2, 1000, 64, 128, 256),    # ragged length, several 128-key tiles, compactions
    (1, 777, 16, 64, 100),      # odd k
    (1, 300, 64, 128, 2048),    # t <= k everywhere: rows written without scoring
    (3, 130, 32, 32, 7),        # tiny k, batch > 1, 64B swizzle
    (1, 2100, 8, 128, 64),      # many compactions per row (cap = 2k + 128)
])
def test_shapes_integer_exact(dsa, oracle_mod, B, L, H, d, kk):
    q, k, w = indexer_inputs_host(L + H, B, L, L, H, d)
    got = _run(dsa, q, k, w, kk)
    rows = [(b, i) for b in range(B) for i in range(L) if i % 5 == 0 or i > L - 10 or i < 10]
    for (b, i), (I, want) in _oracle_rows(oracle_mod, q, k, w, rows, kk).items():
        check_topk_row(got[b, i], want, I, kk)


def test_decode_split_path_exact(dsa, oracle_mod):
    # One query per sequence at t = Lk: the key range is split across CTAs and
    # the per-split top-k lists are merged.
    B, Lk, H, d, kk = 3, 20000, 64, 128, 2048
    q, k, w = indexer_inputs_host(21, B, 1, Lk, H, d)
    got = _run(dsa, q, k, w, kk, start_pos=Lk)
    for b in range(B):
        I = oracle_mod.indexer_row(q[b, 0], k[b], w[b, 0], Lk)
        check_topk_row(got[b, 0], oracle_mod.topk_row(I, Lk, kk), I, kk)


def test_full_size_single_f_layer_sampled(dsa, oracle_mod):
    # B = 1, L = 16384, H_I = 64, d_I = 128, k = 2048, integer inputs,
    # generated on the device; sampled rows checked against the oracle.
    import torch
    B, L, H, d, kk = 1, 16384, 64, 128, 2048
    seed = 2
    qd = torch.empty((B, L, H, d), dtype=torch.bfloat16, device="cuda")
    kd = torch.empty((B, L, d), dtype=torch.bfloat16, device="cuda")
    wd = torch.empty((B, L, H), dtype=torch.float32, device="cuda")
    synth.fill_cuda(qd, seed, synth.Q_IDX, synth.INT9, 0)
    synth.fill_cuda(kd, seed, synth.K_IDX, synth.INT9, 0)
    synth.fill_cuda(wd, seed, synth.W, synth.POW2W, 0)
    out = dsa.indexer_topk(qd, kd, wd, kk)
    dsa.check_device_errors()
    got = out.cpu().numpy()
    k_host = synth.tensor(seed, synth.K_IDX, synth.INT9, 0, (B, L, d))
    rows = [0, 1, 7, 8, 2047, 2048, 2049, 5000, 8191, 12345, 16383]
    for i in rows:
        qrow = synth.rows(seed, synth.Q_IDX, synth.INT9, 0, (B, L, H, d), np.arange(H) + i * H)
        wrow = synth.rows(seed, synth.W, synth.POW2W, 0, (B, L, H), [i], bf16=False)[0]
        I = oracle_mod.indexer_row(qrow, k_host[0], wrow, i)
        check_topk_row(got[0, i], oracle_mod.topk_row(I, i, kk), I, kk)


def test_deterministic_reruns(dsa):
    B, L, H, d, kk = 1, 3000, 64, 128, 512
    q, k, w = indexer_inputs_host(31, B, L, L, H, d, integer=False)
    a = _run(dsa, q, k, w, kk)
    b = _run(dsa, q, k, w, kk)
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("B,Lk,start_pos,H,d,kk", [
    (5, 20000, 20000, 64, 128, 2048),   # one query row per sequence at t = Lk
    (3, 9001, 7777, 32, 64, 300),       # t < Lk: the tail of the cache is not visible
    (2, 2100, 2100, 16, 128, 2048),     # T barely above k
    (2, 1500, 1500, 64, 64, 2048),      # T <= k: every visible position, no scoring
    (4, 130, 1, 16, 64, 5),             # T = 1: only position 0 (no scoring)
    (1, 50000, 49999, 64, 128, 1),      # k = 1
])
def test_decode_rows_integer_exact(dsa, oracle_mod, B, Lk, start_pos, H, d, kk):
    # Lq = 1 rows with T > k take the decode path (streamed score keys +
    # cluster radix select); integer inputs make every score exact.
    q, k, w = indexer_inputs_host(Lk + H + kk, B, 1, Lk, H, d)
    got = _run(dsa, q, k, w, kk, start_pos=start_pos)
    for b in range(B):
        I = oracle_mod.indexer_row(q[b, 0], k[b], w[b, 0], start_pos)
        check_topk_row(got[b, 0], oracle_mod.topk_row(I, start_pos, kk), I, kk)


@pytest.mark.parametrize("levels", [1, 2, 5])
def test_decode_rows_heavy_ties(dsa, oracle_mod, levels):
    # Scores take only `levels` distinct values, so the k-th score is shared by
    # thousands of positions spread over every CTA of the select cluster; the
    # lower positions must win.
    B, Lk, H, d, kk = 3, 40000, 16, 64, 2048
    rng = np.random.default_rng(100 + levels)
    q = np.zeros((B, 1, H, d), np.float32)
    q[:, :, :, 0] = 1.0
    k = np.zeros((B, Lk, d), np.float32)
    k[:, :, 0] = rng.integers(0, levels, size=(B, Lk))
    w = np.ones((B, 1, H), np.float32)
    qb, kb = synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k)
    got = _run(dsa, qb, kb, w, kk, start_pos=Lk)
    for b in range(B):
        I = oracle_mod.indexer_row(qb[b, 0], kb[b], w[b, 0], Lk)
        check_topk_row(got[b, 0], oracle_mod.topk_row(I, Lk, kk), I, kk)


def test_decode_full_size_rows(dsa, oracle_mod):
    # B = 8 sequences at 200000 cached positions, H_I = 64, d_I = 128,
    # k = 2048, integer inputs generated on the device; three rows checked
    # against the oracle, all eight for shape and order.
    import torch
    B, Lk, H, d, kk = 8, 200000, 64, 128, 2048
    seed, layer = 5, 3
    qd = torch.empty((B, 1, H, d), dtype=torch.bfloat16, device="cuda")
    kd = torch.empty((B, Lk, d), dtype=torch.bfloat16, device="cuda")
    wd = torch.empty((B, 1, H), dtype=torch.float32, device="cuda")
    synth.fill_cuda(qd, seed, synth.Q_IDX, synth.INT9, layer)
    synth.fill_cuda(kd, seed, synth.K_IDX, synth.INT9, layer)
    synth.fill_cuda(wd, seed, synth.W, synth.POW2W, layer)
    out = dsa.indexer_topk(qd, kd, wd, kk, start_pos=Lk)
    dsa.check_device_errors()
    got = out.cpu().numpy()
    assert np.all(np.diff(got[:, 0], axis=-1) > 0) and got.min() >= 0 and got.max() < Lk
    q_host = synth.tensor(seed, synth.Q_IDX, synth.INT9, layer, (B, 1, H, d))
    w_host = synth.tensor(seed, synth.W, synth.POW2W, layer, (B, 1, H), bf16=False)
    for b in [0, 3, 7]:
        k_host = synth.rows(seed, synth.K_IDX, synth.INT9, layer, (B, Lk, d), np.arange(Lk) + b * Lk)
        I = oracle_mod.indexer_row(q_host[b, 0], k_host, w_host[b, 0], Lk)
        check_topk_row(got[b, 0], oracle_mod.topk_row(I, Lk, kk), I, kk)


def test_prefill_200k_layer_sampled(dsa, oracle_mod):
    # One F layer at the benchmark's prefill length (L = 200,000, H_I = 64,
    # d_I = 128, k = 2048; the launch configuration bench.py times), integer
    # inputs generated on the device; sampled rows against the oracle.
    import torch
    B, L, H, d, kk = 1, 200000, 64, 128, 2048
    seed, layer = 4, 1
    qd = torch.empty((B, L, H, d), dtype=torch.bfloat16, device="cuda")
    kd = torch.empty((B, L, d), dtype=torch.bfloat16, device="cuda")
    wd = torch.empty((B, L, H), dtype=torch.float32, device="cuda")
    synth.fill_cuda(qd, seed, synth.Q_IDX, synth.INT9, layer)
    synth.fill_cuda(kd, seed, synth.K_IDX, synth.INT9, layer)
    synth.fill_cuda(wd, seed, synth.W, synth.POW2W, layer)
    out = dsa.indexer_topk(qd, kd, wd, kk)
    dsa.check_device_errors()
    k_host = synth.tensor(seed, synth.K_IDX, synth.INT9, layer, (B, L, d))
    for i in [1, 2048, 2049, 77777, 199999]:
        qrow = synth.rows(seed, synth.Q_IDX, synth.INT9, layer, (B, L, H, d), np.arange(H) + i * H)
        wrow = synth.rows(seed, synth.W, synth.POW2W, layer, (B, L, H), [i], bf16=False)[0]
        I = oracle_mod.indexer_row(qrow, k_host[0], wrow, i)
        check_topk_row(out[0, i].cpu().numpy(), oracle_mod.topk_row(I, i, kk), I, kk)


@pytest.mark.parametrize("T", [327680, 327681])
def test_decode_rows_at_the_slice_limit(dsa, oracle_mod, T):
    # The decode kernels hold 1/8 of a row's score keys per CTA (at most 40,960
    # keys each, i.e. T <= 327,680); one more key takes the split prefill path.
    # Both sides of the limit must give the oracle's rows.
    import torch
    B, H, d, kk = 1, 16, 64, 2048
    seed, layer = 8, 0
    qd = torch.empty((B, 1, H, d), dtype=torch.bfloat16, device="cuda")
    kd = torch.empty((B, T, d), dtype=torch.bfloat16, device="cuda")
    wd = torch.empty((B, 1, H), dtype=torch.float32, device="cuda")
    synth.fill_cuda(qd, seed, synth.Q_IDX, synth.INT9, layer)
    synth.fill_cuda(kd, seed, synth.K_IDX, synth.INT9, layer)
    synth.fill_cuda(wd, seed, synth.W, synth.POW2W, layer)
    out = dsa.indexer_topk(qd, kd, wd, kk, start_pos=T)
    dsa.check_device_errors()
    q_host = synth.tensor(seed, synth.Q_IDX, synth.INT9, layer, (B, 1, H, d))
    w_host = synth.tensor(seed, synth.W, synth.POW2W, layer, (B, 1, H), bf16=False)
    k_host = synth.tensor(seed, synth.K_IDX, synth.INT9, layer, (B, T, d))
    I = oracle_mod.indexer_row(q_host[0, 0], k_host[0], w_host[0, 0], T)
    check_topk_row(out[0, 0].cpu().numpy(), oracle_mod.topk_row(I, T, kk), I, kk)


def test_check_indices_accepts_output_and_counts_planted_rows(dsa):
    import torch
    B, L, H, d, kk = 2, 3000, 64, 128, 512
    q, k, w = indexer_inputs_host(37, B, L, L, H, d, integer=False)
    idx = dsa.indexer_topk(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), kk)
    assert dsa.check_indices(idx) == 0
    bad = idx.clone()
    bad[0, 5, 0] = 5            # position t itself is not visible
    bad[0, 2000, 10] = bad[0, 2000, 9]   # not strictly ascending
    bad[1, 100, 200] = 7        # padding must be -1 after min(t, k) entries
    bad[1, 2999, kk - 1] = -1   # a full row must hold k positions
    assert dsa.check_indices(bad) == 4
    dec = dsa.indexer_topk(to_dev_bf16(q[:, :1]), to_dev_bf16(k), to_dev_f32(w[:, :1]), kk,
                           start_pos=L)
    assert dsa.check_indices(dec, start_pos=L) == 0
    assert dsa.check_indices(torch.full_like(dec, -1), start_pos=L) == B
