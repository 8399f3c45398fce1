"""GPU parity of the CSA-style selection over compressed blocks ([IDX] §5.2)
against the oracle: the indexer over blocks s < floor(t/m) with TopK_k, and
the attention over the selected compressed entries.  Integer-valued indexer
inputs with power-of-two head weights make every fp32 score exact, so the
indices must match bit for bit."""
import math

import numpy as np
import pytest

from sparse_attention_13_b200 import synth

from gpu_util import to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_13_b200 import dsa as _dsa
    _dsa.lib()
    return _dsa


def _inputs(seed, B, Lq, N, H, d):
    q = synth.tensor(seed, synth.Q_IDX, synth.INT9, 0, (B, Lq, H, d))
    kc = synth.tensor(seed, synth.K_IDX, synth.INT9, 0, (B, N, d))
    w = synth.tensor(seed, synth.W, synth.POW2W, 0, (B, Lq, H), bf16=False)
    return q, kc, w


def _run(dsa, q, kc, w, kk, m, start_pos=0):
    out = dsa.csa_indexer_topk(to_dev_bf16(q), to_dev_bf16(kc), to_dev_f32(w), kk, m=m,
                               start_pos=start_pos)
    dsa.check_device_errors()
    return out.cpu().numpy()


@pytest.mark.parametrize("B,Lq,m,start_pos,H,d,kk", [
    (2, 600, 4, 0, 64, 128, 16),      # phases of 150 rows
    (1, 601, 4, 0, 64, 128, 64),      # a ragged last phase
    (2, 203, 3, 300, 32, 64, 40),     # chunked prefill from a block boundary
    (1, 130, 1, 0, 16, 128, 32),      # m = 1: the token indexer
])
def test_csa_indexer_integer_exact(dsa, oracle_mod, B, Lq, m, start_pos, H, d, kk):
    N = (start_pos + Lq - 1) // m + 1
    q, kc, w = _inputs(61 + m, B, Lq, N, H, d)
    got = _run(dsa, q, kc, w, kk, m, start_pos)
    for b in range(B):
        for i in range(Lq):
            t = start_pos + i
            _, want = oracle_mod.csa_indexer_topk_row(q[b, i], kc[b], w[b, i], t, m, kk)
            np.testing.assert_array_equal(got[b, i], want, err_msg=f"b={b} i={i} t={t}")


@pytest.mark.parametrize("t", [3, 4, 8191, 200003])
def test_csa_indexer_decode_rows(dsa, oracle_mod, t):
    # one query per sequence at t (t mod m need not be 0): blocks s < floor(t/4)
    B, H, d, kk, m = 2, 64, 128, 512, 4
    N = t // m
    q, kc, w = _inputs(67, B, 1, max(N, 1), H, d)
    got = _run(dsa, q, kc, w, kk, m, start_pos=t)
    for b in range(B):
        _, want = oracle_mod.csa_indexer_topk_row(q[b, 0], kc[b], w[b, 0], t, m, kk)
        np.testing.assert_array_equal(got[b, 0], want)


def test_csa_v4_shape_sampled(dsa, oracle_mod):
    # the V4 settings of [IDX] §5.3: m = 4, 64 heads x 128, k = 512 and 1024
    B, L, m, H, d = 1, 8192, 4, 64, 128
    N = L // m
    q, kc, w = _inputs(71, B, L, N, H, d)
    for kk in (512, 1024):
        got = _run(dsa, q, kc, w, kk, m)
        for i in (0, 3, 4, 7, 2051, 4099, 4100, 6000, L - 1):
            _, want = oracle_mod.csa_indexer_topk_row(q[0, i], kc[0], w[0, i], i, m, kk)
            np.testing.assert_array_equal(got[0, i], want, err_msg=f"k={kk} i={i}")


def test_csa_refuses_unaligned_chunk(dsa):
    B, Lq, N, H, d = 1, 8, 10, 64, 128
    q, kc, w = _inputs(73, B, Lq, N, H, d)
    with pytest.raises(dsa.DSAError) as e:
        dsa.csa_indexer_topk(to_dev_bf16(q), to_dev_bf16(kc), to_dev_f32(w), 8, m=4, start_pos=6)
    assert e.value.status == dsa.DSA_ERR_UNSUPPORTED


def test_csa_attention_mla(dsa, oracle_mod):
    # attention over the selected compressed latent entries (576 = K, first 512 = V)
    import torch
    B, L, m, kk = 1, 700, 4, 64
    N = L // m
    qi, kc, w = _inputs(79, B, L, N, 64, 128)
    idx = dsa.csa_indexer_topk(to_dev_bf16(qi), to_dev_bf16(kc), to_dev_f32(w), kk, m=m)
    q = synth.tensor(79, synth.Q, synth.NORMAL, 0, (B, L, 128, 576), sigma=0.5)
    c = synth.tensor(79, synth.KV, synth.NORMAL, 0, (B, N, 576), sigma=0.5)
    scale = 1 / math.sqrt(576)
    lse = torch.empty((B, L, 128), dtype=torch.float32, device="cuda")
    out = dsa.csa_sparse_attn(to_dev_bf16(q), to_dev_bf16(c), idx, scale, m=m, D_v=512, lse=lse)
    dsa.check_device_errors()
    got = out.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    idx_h = idx.cpu().numpy()
    for i in (0, 3, 4, 5, 255, 256, 257, 699):
        o, l = oracle_mod.csa_attn_row(q[0, i], c[0], idx_h[0, i], scale, Dv=512)
        assert np.all(np.abs(got[0, i] - o) <= 2e-2 + 1e-2 * np.abs(o)), i
        if i < m:
            assert np.all(np.isneginf(lse_h[0, i])) and np.all(got[0, i] == 0)
        else:
            np.testing.assert_allclose(lse_h[0, i], l, rtol=0, atol=1e-3)
