"""GPU parity of the variable-length batch entry points (packed rows with
device offsets, include/dsa.h dsa_varlen) against the oracle applied to each
sequence on its own: prefill sequences of different lengths, chunked
continuations, decode rows at different positions, an empty sequence, the
layer loop, agreement with the uniform entry points on equal lengths, and
the device-side contract check.  Source: "注意力机制中的 Index" §4.3 (prefill
and decode requests are served differently; a batch mixes them)."""
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


def _close(got, want):
    err = np.abs(np.asarray(got, np.float64) - want)
    assert (err <= 2e-2 + 1e-2 * np.abs(want)).all(), f"max abs err {err.max():.3e}"


def _indexer_batch(seed, q_lens, k_lens, H, d):
    """Per-sequence integer indexer inputs (sequence b drawn as layer b of
    the seeded tensors) and their packed concatenation."""
    qs, ks, ws = [], [], []
    for b, (lq, lk) in enumerate(zip(q_lens, k_lens)):
        qs.append(synth.tensor(seed, synth.Q_IDX, synth.INT9, b, (max(lq, 0), H, d)))
        ks.append(synth.tensor(seed, synth.K_IDX, synth.INT9, b, (lk, d)))
        ws.append(synth.tensor(seed, synth.W, synth.POW2W, b, (max(lq, 0), H), bf16=False))
    return qs, ks, ws, np.concatenate(qs), np.concatenate(ks), np.concatenate(ws)


def _oracle_rows(oracle_mod, q, k, w, start, rows, kk):
    return {i: oracle_mod.topk_row(oracle_mod.indexer_row(q[i], k, w[i], start + i), start + i, kk) for i in rows}


def _sample(n, extra=()):
    base = {0, 1, n // 2, n - 1, *extra}
    return sorted(i for i in base if 0 <= i < n)


def test_varlen_prefill_lengths_130_5000_20000(dsa, oracle_mod):
    # three prompts of very different lengths in one batch (k = 2048, the
    # 64 x 128 indexer): indices bit-exact per sequence
    q_lens = k_lens = [130, 5000, 20000]
    H, d, kk = 64, 128, 2048
    qs, ks, ws, qp, kp, wp = _indexer_batch(71, q_lens, k_lens, H, d)
    vb = dsa.VarlenBatch(q_lens, k_lens, [0, 0, 0])
    assert dsa.check_varlen(vb) == 0
    got = dsa.indexer_topk_varlen(to_dev_bf16(qp), to_dev_bf16(kp), to_dev_f32(wp), kk, vb).cpu().numpy()
    dsa.check_device_errors()
    for b, lq in enumerate(q_lens):
        rows = range(lq) if lq <= 130 else _sample(lq, (2047, 2048, 2049, 4999))
        want = _oracle_rows(oracle_mod, qs[b], ks[b], ws[b], 0, rows, kk)
        for i in rows:
            np.testing.assert_array_equal(got[vb.cu_q_list[b] + i], want[i], err_msg=f"seq {b} row {i}")


def test_varlen_mixed_chunks_decode_and_empty(dsa, oracle_mod):
    # a chunked continuation (rows 2700..2999 of a 3000-token cache), a single
    # decode-style row inside a prefill batch, a short prompt, and a sequence
    # with no query rows at all
    q_lens = [300, 1, 64, 0, 257]
    k_lens = [3000, 10000, 64, 500, 4097]
    starts = [2700, 10000, 0, 500, 3840]
    H, d, kk = 32, 64, 512
    qs, ks, ws, qp, kp, wp = _indexer_batch(72, q_lens, k_lens, H, d)
    vb = dsa.VarlenBatch(q_lens, k_lens, starts)
    assert dsa.check_varlen(vb) == 0
    got = dsa.indexer_topk_varlen(to_dev_bf16(qp), to_dev_bf16(kp), to_dev_f32(wp), kk, vb).cpu().numpy()
    dsa.check_device_errors()
    for b, lq in enumerate(q_lens):
        rows = _sample(lq, (7, 8, 255, 256))
        want = _oracle_rows(oracle_mod, qs[b], ks[b], ws[b], starts[b], rows, kk)
        for i in rows:
            np.testing.assert_array_equal(got[vb.cu_q_list[b] + i], want[i], err_msg=f"seq {b} row {i}")


def test_varlen_decode_rows_at_different_positions(dsa, oracle_mod):
    # one row per sequence (the streaming decode kernels), positions on both
    # sides of k and up to a 30,000-token cache; every row bit-exact
    T = [1, 100, 2047, 2048, 2049, 30000]
    H, d, kk = 64, 128, 2048
    qs, ks, ws, qp, kp, wp = _indexer_batch(73, [1] * len(T), T, H, d)
    vb = dsa.VarlenBatch([1] * len(T), T, T)
    got = dsa.indexer_topk_varlen(to_dev_bf16(qp), to_dev_bf16(kp), to_dev_f32(wp), kk, vb).cpu().numpy()
    dsa.check_device_errors()
    for b, t in enumerate(T):
        want = oracle_mod.topk_row(oracle_mod.indexer_row(qs[b][0], ks[b], ws[b][0], t), t, kk)
        np.testing.assert_array_equal(got[b], want, err_msg=f"decode row {b} at t = {t}")


def test_varlen_equal_lengths_reproduce_the_uniform_entry_points(dsa):
    # three sequences of the same length as a packed batch give the uniform
    # batch's indices and attention outputs bit for bit
    import torch
    B, L, H, d, kk = 3, 1000, 64, 128, 256
    qi = torch.empty((B, L, H, d), dtype=torch.bfloat16, device="cuda")
    ki = torch.empty((B, L, d), dtype=torch.bfloat16, device="cuda")
    w = torch.empty((B, L, H), dtype=torch.float32, device="cuda")
    synth.fill_cuda(qi, 74, synth.Q_IDX, synth.INT9, 0)
    synth.fill_cuda(ki, 74, synth.K_IDX, synth.INT9, 0)
    synth.fill_cuda(w, 74, synth.W, synth.POW2W, 0)
    q = torch.empty((B, L, 128, 576), dtype=torch.bfloat16, device="cuda")
    kv = torch.empty((B, L, 576), dtype=torch.bfloat16, device="cuda")
    synth.fill_cuda(q, 74, synth.Q, synth.NORMAL, 0, sigma=0.5)
    synth.fill_cuda(kv, 74, synth.KV, synth.NORMAL, 0, sigma=0.5)
    uni = dsa.indexer_topk(qi, ki, w, kk)
    out_u = dsa.sparse_attn(q, kv, kv, uni, 1 / 24, D_v=512)
    vb = dsa.VarlenBatch([L] * B, [L] * B, [0] * B)
    var = dsa.indexer_topk_varlen(qi.view(B * L, H, d), ki.view(B * L, d), w.view(B * L, H), kk, vb)
    out_v = dsa.sparse_attn_varlen(q.view(B * L, 128, 576), kv.view(B * L, 576), kv.view(B * L, 576), var,
                                   1 / 24, vb, D_v=512)
    dsa.check_device_errors()
    assert torch.equal(uni.view(B * L, kk), var)
    assert torch.equal(out_u.view(B * L, 128, 512), out_v)


@pytest.mark.parametrize("mla", [True, False])
def test_varlen_attention_against_the_oracle(dsa, oracle_mod, mla):
    # attention of a mixed batch (a continuation chunk, a decode row, a short
    # prompt, an empty sequence) through oracle-selected index rows
    import torch
    q_lens = [200, 1, 70, 0, 130]
    k_lens = [2500, 6000, 70, 40, 130]
    starts = [2300, 6000, 0, 40, 0]
    kk = 256
    n_h, Dq, Dv = (128, 576, 512) if mla else (4, 64, 64)
    rng = np.random.default_rng(75)
    idx_rows, qs, kvs, vs = [], [], [], []
    for b, (lq, lk, st) in enumerate(zip(q_lens, k_lens, starts)):
        qs.append(synth.tensor(75, synth.Q, synth.NORMAL, b, (lq, n_h, Dq), sigma=0.5))
        kvs.append(synth.tensor(75, synth.KV if mla else synth.K_SEP, synth.NORMAL, b, (lk, Dq), sigma=0.5))
        vs.append(kvs[-1] if mla else synth.tensor(75, synth.V_SEP, synth.NORMAL, b, (lk, Dv), sigma=0.5))
        for i in range(lq):
            t = st + i
            n = min(t, kk)
            row = -np.ones(kk, np.int32)
            row[:n] = np.sort(rng.choice(t, size=n, replace=False))
            idx_rows.append(row)
    idx = np.stack(idx_rows)
    vb = dsa.VarlenBatch(q_lens, k_lens, starts)
    scale = 1 / math.sqrt(Dq)
    lse = torch.empty((vb.total_q, n_h), dtype=torch.float32, device="cuda")
    kd = to_dev_bf16(np.concatenate(kvs))
    vd = kd if mla else to_dev_bf16(np.concatenate(vs))
    out = dsa.sparse_attn_varlen(to_dev_bf16(np.concatenate(qs)), kd, vd, torch.from_numpy(idx).cuda(), scale,
                                 vb, D_v=Dv, lse=lse)
    dsa.check_device_errors()
    got, lse_h = out.float().cpu().numpy(), lse.cpu().numpy()
    for b, lq in enumerate(q_lens):
        for i in _sample(lq, (63, 64, 129)):
            r = vb.cu_q_list[b] + i
            o, l = oracle_mod.sparse_attn_row(qs[b][i], kvs[b], vs[b], idx[r], scale, Dv=Dv)
            _close(got[r], o)
            np.testing.assert_allclose(lse_h[r], l, rtol=1e-4, atol=1e-5 + kk * 2.0 ** -24 + 3.6e-4)


def test_indexcache_forward_varlen_tiny_stack(dsa, oracle_mod):
    # the FSFS layer loop over a batch of three sequences (tiny shapes: 4
    # indexer heads of 32, k = 64, 4 query heads of 64 sharing one K and one
    # V head) against the oracle's loop run on each sequence
    import torch
    q_lens, k_lens, starts = [160, 90, 1], [160, 400, 700], [0, 310, 700]
    H, dI, kk, n_h, D = 4, 32, 64, 4, 64
    pattern = "FSFS"
    seqs = []
    for b, (lq, lk) in enumerate(zip(q_lens, k_lens)):
        layers = []
        for l in range(4):
            s = 1000 + 10 * b + l
            layers.append(dict(q_idx=synth.tensor(s, synth.Q_IDX, synth.INT9, 0, (1, lq, H, dI)),
                               k_idx=synth.tensor(s, synth.K_IDX, synth.INT9, 0, (1, lk, dI)),
                               w=synth.tensor(s, synth.W, synth.POW2W, 0, (1, lq, H), bf16=False),
                               q=synth.tensor(s, synth.Q, synth.NORMAL, 0, (1, lq, n_h, D), sigma=0.5),
                               k=synth.tensor(s, synth.K_SEP, synth.NORMAL, 0, (1, lk, D), sigma=0.5),
                               v=synth.tensor(s, synth.V_SEP, synth.NORMAL, 0, (1, lk, D), sigma=0.5)))
        seqs.append(layers)
    vb = dsa.VarlenBatch(q_lens, k_lens, starts)
    scale = 1 / math.sqrt(D)
    dl = []
    for l in range(4):
        cat = {f: np.concatenate([seqs[b][l][f][0] for b in range(3)]) for f in seqs[0][l]}
        dl.append(dict(q_idx=to_dev_bf16(cat["q_idx"]), k_idx=to_dev_bf16(cat["k_idx"]), w=to_dev_f32(cat["w"]),
                       q=to_dev_bf16(cat["q"]), kbuf=to_dev_bf16(cat["k"]), vbuf=to_dev_bf16(cat["v"]),
                       out=torch.empty((vb.total_q, n_h, D), dtype=torch.bfloat16, device="cuda")))
    dims = dsa.make_dims(B=0, Lq=0, Lk=0, start_pos=0, H_I=H, d_I=dI, k=kk, n_h=n_h, D_qk=D, D_v=D, scale=scale,
                         k_row_stride=D, v_row_stride=D)
    idx = torch.empty((vb.total_q, kk), dtype=torch.int32, device="cuda")
    before = dsa.indexer_launch_count()
    dsa.indexcache_forward_varlen(pattern, dl, dims, vb, idx)
    dsa.check_device_errors()
    assert dsa.indexer_launch_count() - before == 2
    idx_h = idx.cpu().numpy()
    for b in range(3):
        o_idx, o_out, _, _ = oracle_mod.indexcache_forward(
            pattern, seqs[b], B=1, Lq=q_lens[b], Lk=k_lens[b], start_pos=starts[b], H=H, dI=dI, k=kk, n_h=n_h,
            Dqk=D, Dv=D, scale=scale)
        r0, r1 = vb.cu_q_list[b], vb.cu_q_list[b + 1]
        np.testing.assert_array_equal(idx_h[r0:r1], o_idx[3][0])
        for l in range(4):
            _close(dl[l]["out"][r0:r1].float().cpu().numpy(), o_out[l][0])


def test_check_varlen_counts_broken_sequences(dsa):
    # cu_q = [0, 4, 7, 12], cu_k = [0, 10, 13, 22], starts [6, 0, 4], bounds
    # max_Lq = 5, max_Lk = 10: every sequence keeps t <= its cache length
    vb = dsa.VarlenBatch([4, 3, 5], [10, 3, 9], [6, 0, 4])
    assert dsa.check_varlen(vb) == 0
    # sequence 1 starting at 2: its last row would sit at t = 4 > 3 cached rows
    vb.start_pos[1] = 2
    assert dsa.check_varlen(vb) == 1
    vb.start_pos[1] = 0
    # cu_q[2] = 3 < cu_q[1]: sequence 1 gets a negative length and sequence 2
    # nine rows, beyond max_Lq = 5
    vb.cu_q[2] = 3
    assert dsa.check_varlen(vb) == 2
    vb.cu_q[2] = 7
    # the last offset must equal total_q
    vb.cu_q[3] = 11
    assert dsa.check_varlen(vb) == 1
