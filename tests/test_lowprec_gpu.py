"""GPU parity of the low-precision selector ("注意力机制中的 Index" §5.4:
FP4/FP8 QK path, scores quantised from FP32 to BF16) against the oracle's
lowprec_indexer_row + topk_row: the MX quantiser value for value on normal
inputs (both formats, with zero blocks, saturating and tied values), the
selector's indices bit for bit on integer inputs (where MX quantisation is
lossless and the score is the exact one rounded to bf16, so ties abound),
and, on normal inputs, the selection's recall of the exact selector."""
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


def _decode_e4m3(c):
    c = c.astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    return s * np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))


def _decode_e2m1(byte):
    # 16 codes per 16-byte slot, packed in its first 8 bytes, low nibble first
    rows, cols = byte.shape
    slot = byte.astype(np.int64).reshape(rows, cols // 16, 16)
    assert np.all(slot[:, :, 8:] == 0)
    c = np.stack([slot[:, :, :8] & 15, slot[:, :, :8] >> 4], axis=-1).reshape(rows, cols)
    s = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    return s * np.where(e == 0, m * 0.5, (1 + m / 2.0) * np.exp2(e - 1.0))


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_mx_quantize_matches_the_oracle(dsa, oracle_mod, fmt):
    rows = 3000
    x = synth.tensor(81, synth.Q_IDX, synth.NORMAL, 0, (rows, 128), sigma=3.0)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    # special blocks: all zero, one huge value (others underflow), ties at
    # half the element grid, negative zero
    xf[0, :32] = 0.0
    xf[1, 32:64] = 0.0
    xf[1, 40] = 1000.0
    xf[2, :32] = np.array([0.75, 1.25, -2.5, 3.5, 5.0, -0.25, 448.0, 7.0] * 4)
    xf[3, 64:96] = -0.0
    x = synth.f32_to_bf16_bits(xf.astype(np.float32))
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    codes, scales = dsa.mx_quantize(to_dev_bf16(x), fmt)
    dsa.check_device_errors()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    dec = _decode_e4m3(codes) if fmt == "e4m3" else _decode_e2m1(codes)
    X = np.exp2(scales.astype(np.float64) - 127.0)
    got = dec * np.repeat(X, 32, axis=1)
    want = oracle_mod.mx_quantize(xf, fmt)
    np.testing.assert_array_equal(got, want)


def _int_inputs(seed, B, Lq, Lk):
    q = synth.tensor(seed, synth.Q_IDX, synth.INT9, 0, (B, Lq, 64, 128))
    k = synth.tensor(seed, synth.K_IDX, synth.INT9, 0, (B, Lk, 128))
    w = synth.tensor(seed, synth.W, synth.POW2W, 0, (B, Lq, 64), bf16=False)
    return q, k, w


@pytest.mark.parametrize("fmt,L,kk", [("e4m3", 2100, 512), ("e2m1", 2100, 512), ("e4m3", 4500, 2048),
                                       ("e2m1", 1000, 2048)])
def test_lowprec_selector_integer_inputs_bit_exact(dsa, oracle_mod, fmt, L, kk):
    B = 1
    q, k, w = _int_inputs(82, B, L, L)
    got = dsa.indexer_topk_lowprec(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), kk, fmt=fmt).cpu().numpy()
    dsa.check_device_errors()
    for t in sorted({0, 1, 2, 127, 128, 129, kk - 1, kk, kk + 1, L // 2, L - 2, L - 1}):
        if t >= L:
            continue
        I = oracle_mod.lowprec_indexer_row(q[0, t], k[0], w[0, t], t, fmt)
        np.testing.assert_array_equal(got[0, t], oracle_mod.topk_row(I, t, kk), err_msg=f"{fmt} row {t}")


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_lowprec_selector_chunk_and_decode_rows(dsa, oracle_mod, fmt):
    # a continuation chunk (rows 3000..3299 of 5000 keys, two sequences) and
    # single rows at t = 20,000 (the key range split over several CTAs)
    q, k, w = _int_inputs(83, 2, 300, 5000)
    got = dsa.indexer_topk_lowprec(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), 1024, fmt=fmt,
                                   start_pos=3000).cpu().numpy()
    for b in range(2):
        for i in (0, 1, 150, 299):
            I = oracle_mod.lowprec_indexer_row(q[b, i], k[b], w[b, i], 3000 + i, fmt)
            np.testing.assert_array_equal(got[b, i], oracle_mod.topk_row(I, 3000 + i, 1024))
    q, k, w = _int_inputs(84, 3, 1, 20000)
    got = dsa.indexer_topk_lowprec(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), 2048, fmt=fmt,
                                   start_pos=20000).cpu().numpy()
    dsa.check_device_errors()
    for b in range(3):
        I = oracle_mod.lowprec_indexer_row(q[b, 0], k[b], w[b, 0], 20000, fmt)
        np.testing.assert_array_equal(got[b, 0], oracle_mod.topk_row(I, 20000, 2048))


def test_lowprec_recall_of_the_exact_selection(dsa, oracle_mod):
    # normal inputs: the low-precision selection keeps most of the exact
    # selection, E4M3 more than E2M1; on sampled rows each GPU selection
    # agrees with the oracle's own low-precision selection up to scores
    # within the rounding of the k-th value
    import torch
    B, L, kk = 1, 4096, 512
    q = synth.tensor(85, synth.Q_IDX, synth.NORMAL, 0, (B, L, 64, 128), sigma=1.0)
    k = synth.tensor(85, synth.K_IDX, synth.NORMAL, 0, (B, L, 128), sigma=1.0)
    w = np.abs(synth.tensor(85, synth.W, synth.NORMAL, 0, (B, L, 64), sigma=1.0, bf16=False)) / 64.0
    qd, kd, wd = to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w)
    exact = dsa.indexer_topk(qd, kd, wd, kk)
    rec = {}
    for fmt in ("e4m3", "e2m1"):
        sel = dsa.indexer_topk_lowprec(qd, kd, wd, kk, fmt=fmt)
        inter = dsa.index_overlap(exact[:, kk:], sel[:, kk:])
        rec[fmt] = float(inter.float().mean()) / kk
        got = sel.cpu().numpy()
        for t in (kk + 1, 2000, L - 1):
            I = oracle_mod.lowprec_indexer_row(q[0, t], k[0], w[0, t], t, fmt)
            want = oracle_mod.topk_row(I, t, kk)
            diff = np.setxor1d(got[0, t][got[0, t] >= 0], want[want >= 0])
            kth = np.sort(I)[::-1][kk - 1]
            # fp32 accumulation of the head dots before the bf16 rounding may
            # land one bf16 step (2^-7 relative at most) from the oracle's
            # exact value; doubled for the k-th value's own step
            assert np.all(np.abs(I[diff] - kth) <= 2.0 ** -6 * abs(kth) + 1e-12), (fmt, t)
    dsa.check_device_errors()
    assert rec["e4m3"] > 0.9 and rec["e2m1"] > 0.6 and rec["e4m3"] > rec["e2m1"], rec
