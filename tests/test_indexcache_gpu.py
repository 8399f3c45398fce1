"""GPU parity of indexcache_forward (the F/S layer loop, through the C ABI)
against the oracle's loop: the tiny FSFS stack in full, FSSSFSSS MLA stacks
with correlated layers on sampled rows (L = 4,096, and the eight-layer stack
at L = 32,768), four-layer FFFF and FSFS stacks at L = 200,000, the reuse
identity of the IndexCache explainer (§1.1: S layers attend through the last
F layer's indices with their own K/V) and the indexer launch count (two for
FSSSFSSS)."""
import math

import numpy as np
import pytest

from sparse_attention_13_b200 import synth

from gpu_util import check_topk_row, indexer_inputs_host, to_dev_bf16, to_dev_f32

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


def test_tiny_stack_fsfs_full(dsa, oracle_mod):
    # 4 layers FSFS, L = 512, H_I = 4, d_I = 32, k = 64, 4 query heads of 64
    # sharing one K and one V head; integer indexer inputs (exact top-k).
    import torch
    B, L, H, dI, k, n_h, D = 1, 512, 4, 32, 64, 4, 64
    pattern, seed = "FSFS", 21
    hl, dl = [], []
    for l in range(4):
        h = dict(q_idx=synth.tensor(seed, synth.Q_IDX, synth.INT9, l, (B, L, H, dI)),
                 k_idx=synth.tensor(seed, synth.K_IDX, synth.INT9, l, (B, L, dI)),
                 w=synth.tensor(seed, synth.W, synth.POW2W, l, (B, L, H), bf16=False),
                 q=synth.tensor(seed, synth.Q, synth.NORMAL, l, (B, L, n_h, D)),
                 k=synth.tensor(seed, synth.K_SEP, synth.NORMAL, l, (B, L, D)),
                 v=synth.tensor(seed, synth.V_SEP, synth.NORMAL, l, (B, L, D)))
        hl.append(h)
        dl.append(dict(q_idx=to_dev_bf16(h["q_idx"]), k_idx=to_dev_bf16(h["k_idx"]),
                       w=to_dev_f32(h["w"]), q=to_dev_bf16(h["q"]), kbuf=to_dev_bf16(h["k"]),
                       vbuf=to_dev_bf16(h["v"]),
                       out=torch.empty((B, L, n_h, D), dtype=torch.bfloat16, device="cuda"),
                       lse=torch.empty((B, L, n_h), dtype=torch.float32, device="cuda")))
    scale = 1 / math.sqrt(D)
    dims = dsa.make_dims(B=B, Lq=L, Lk=L, start_pos=0, H_I=H, d_I=dI, k=k, n_h=n_h, D_qk=D, D_v=D,
                         scale=scale, k_row_stride=D, v_row_stride=D)
    idx = torch.empty((B, L, k), dtype=torch.int32, device="cuda")
    before = dsa.indexer_launch_count()
    dsa.indexcache_forward(pattern, dl, dims, idx)
    dsa.check_device_errors()
    assert dsa.indexer_launch_count() - before == 2
    o_idx, o_out, o_lse, cnt = oracle_mod.indexcache_forward(
        pattern, hl, B=B, Lq=L, Lk=L, start_pos=0, H=H, dI=dI, k=k, n_h=n_h, Dqk=D, Dv=D, scale=scale)
    assert cnt["indexer_calls"] == 2
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx[3])
    for l in range(4):
        _close(dl[l]["out"].float().cpu().numpy(), o_out[l])
        lse = dl[l]["lse"].cpu().numpy()
        fin = np.isfinite(o_lse[l])
        assert np.array_equal(np.isfinite(lse), fin)
        np.testing.assert_allclose(lse[fin], o_lse[l][fin], rtol=1e-4, atol=1e-4)


def test_fsssfsss_mla_stack_sampled(dsa, oracle_mod):
    # 8 layers FSSSFSSS, MLA shape, correlated layers (k_l = 0.9 k_{l-1} +
    # 0.44 noise), L = 4096, k = 2048: per-layer outputs on sampled rows and
    # the index cache after each F segment.
    import torch
    B, L, H, dI, k = 1, 4096, 64, 128, 2048
    pattern, seed = "FSSSFSSS", 22
    scale = 1 / math.sqrt(576)
    dl = []
    for l in range(8):
        ent = dict(q=torch.empty((B, L, 128, 576), dtype=torch.bfloat16, device="cuda"),
                   kbuf=torch.empty((B, L, 576), dtype=torch.bfloat16, device="cuda"),
                   out=torch.empty((B, L, 128, 512), dtype=torch.bfloat16, device="cuda"))
        synth.fill_cuda(ent["q"], seed, synth.Q, synth.NORMAL, l, sigma=0.5, corr=True)
        synth.fill_cuda(ent["kbuf"], seed, synth.KV, synth.NORMAL, l, sigma=0.5, corr=True)
        ent["vbuf"] = ent["kbuf"]
        if pattern[l] == "F":
            ent["q_idx"] = torch.empty((B, L, H, dI), dtype=torch.bfloat16, device="cuda")
            ent["k_idx"] = torch.empty((B, L, dI), dtype=torch.bfloat16, device="cuda")
            ent["w"] = torch.empty((B, L, H), dtype=torch.float32, device="cuda")
            synth.fill_cuda(ent["q_idx"], seed, synth.Q_IDX, synth.INT9, l, corr=True)
            synth.fill_cuda(ent["k_idx"], seed, synth.K_IDX, synth.INT9, l, corr=True)
            synth.fill_cuda(ent["w"], seed, synth.W, synth.POW2W, l)
        dl.append(ent)
    dims = dsa.make_dims(B=B, Lq=L, Lk=L, start_pos=0, H_I=H, d_I=dI, k=k, n_h=128, D_qk=576,
                         D_v=512, scale=scale, k_row_stride=576, v_row_stride=576)
    idx = torch.empty((B, L, k), dtype=torch.int32, device="cuda")
    # first segment alone: the cache after layer 3 is layer 0's top-k
    before = dsa.indexer_launch_count()
    dsa.indexcache_forward(pattern[:4], dl[:4], dims, idx)
    seg0 = idx.cpu().numpy()
    dsa.indexcache_forward(pattern, dl, dims, idx)
    dsa.check_device_errors()
    assert dsa.indexer_launch_count() - before == 1 + 2
    seg1 = idx.cpu().numpy()
    rows = [1, 2, 100, 2047, 2048, 3000, 4095]
    for F, seg in ((0, seg0), (4, seg1)):
        kh = synth.tensor(seed, synth.K_IDX, synth.INT9, F, (B, L, dI), corr=True)
        for i in rows:
            qr = synth.rows(seed, synth.Q_IDX, synth.INT9, F, (B, L, H, dI), np.arange(H) + H * i, corr=True)
            wr = synth.rows(seed, synth.W, synth.POW2W, F, (B, L, H), [i], bf16=False)[0]
            I = oracle_mod.indexer_row(qr, kh[0], wr, i)
            np.testing.assert_array_equal(seg[0, i], oracle_mod.topk_row(I, i, k))
    for l in (0, 1, 3, 4, 7):
        cache = seg0 if l < 4 else seg1
        kvh = synth.tensor(seed, synth.KV, synth.NORMAL, l, (B, L, 576), sigma=0.5, corr=True)
        got = dl[l]["out"]
        for i in rows[:4]:
            qr = synth.rows(seed, synth.Q, synth.NORMAL, l, (B, L, 128, 576), np.arange(128) + 128 * i,
                            sigma=0.5, corr=True)
            o, _ = oracle_mod.sparse_attn_row(qr, kvh[0], kvh[0], cache[0, i], scale, Dv=512)
            _close(got[0, i].float().cpu().numpy(), o)


def test_bad_pattern_launches_nothing(dsa):
    import torch
    dims = dsa.make_dims(B=1, Lq=8, Lk=8, start_pos=0, H_I=64, d_I=128, k=4, n_h=128, D_qk=576,
                         D_v=512, scale=1.0, k_row_stride=576, v_row_stride=576)
    idx = torch.empty((1, 8, 4), dtype=torch.int32, device="cuda")
    before = dsa.indexer_launch_count()
    with pytest.raises(dsa.DSAError) as e:
        dsa.indexcache_forward("SF", [{}, {}], dims, idx)
    assert e.value.status == dsa.DSA_ERR_BAD_PATTERN
    assert dsa.indexer_launch_count() == before


def test_bounded_wait_expiry_reports_timeout_and_context_survives(dsa, oracle_mod):
    # A wait that nothing completes gives up after ~1e6 cycles (about half a
    # millisecond) and records the expiry; the host sees DSA_ERR_TIMEOUT once,
    # the error word is cleared, and the next library call still works.
    dsa.selftest_wait_timeout(1_000_000)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_errors()
    assert e.value.status == dsa.DSA_ERR_TIMEOUT
    dsa.check_device_errors()  # cleared
    B, L, H, d, kk = 1, 300, 16, 64, 32
    q, k, w = indexer_inputs_host(77, B, L, L, H, d)
    got = dsa.indexer_topk(to_dev_bf16(q), to_dev_bf16(k), to_dev_f32(w), kk).cpu().numpy()
    dsa.check_device_errors()
    for i in (0, 31, 32, 299):
        I = oracle_mod.indexer_row(q[0, i], k[0], w[0, i], i)
        check_topk_row(got[0, i], oracle_mod.topk_row(I, i, kk), I, kk)


def _sampled_stack(dsa, oracle_mod, pattern, L, seed, rows, att_rows, corr, shared_q):
    """Runs `pattern` through indexcache_forward at B = 1, length L, with the
    MLA shape and k = 2048, and checks sampled rows against the oracle:
      - the index cache after each F layer's segment, bit for bit (the segment
        is run as a prefix of the pattern: the cache then holds that F layer's
        selection);
      - every layer's LSE, through the oracle's selection of the F layer that
        governs it (the reuse rule of [IC] §1.1-§1.2);
      - the last layer's output.
    With shared_q every layer reads one query tensor and writes one output
    buffer (the L = 200,000 stacks would not fit otherwise); the per-layer
    LSE then checks each layer's attention."""
    import torch
    B, H, dI, k = 1, 64, 128, 2048
    assert set(att_rows) <= set(rows)
    scale = 1 / math.sqrt(576)
    kw = dict(sigma=0.5, corr=corr)
    dl = []
    q_shared = out_shared = None
    if shared_q:
        q_shared = torch.empty((B, L, 128, 576), dtype=torch.bfloat16, device="cuda")
        synth.fill_cuda(q_shared, seed, synth.Q, synth.NORMAL, 0, sigma=0.5)
        out_shared = torch.empty((B, L, 128, 512), dtype=torch.bfloat16, device="cuda")
    for l, role in enumerate(pattern):
        ent = dict(kbuf=torch.empty((B, L, 576), dtype=torch.bfloat16, device="cuda"),
                   lse=torch.empty((B, L, 128), dtype=torch.float32, device="cuda"))
        synth.fill_cuda(ent["kbuf"], seed, synth.KV, synth.NORMAL, l, **kw)
        ent["vbuf"] = ent["kbuf"]
        if shared_q:
            ent["q"], ent["out"] = q_shared, out_shared
        else:
            ent["q"] = torch.empty((B, L, 128, 576), dtype=torch.bfloat16, device="cuda")
            synth.fill_cuda(ent["q"], seed, synth.Q, synth.NORMAL, l, **kw)
            ent["out"] = torch.empty((B, L, 128, 512), dtype=torch.bfloat16, device="cuda")
        if role == "F":
            ent["q_idx"] = torch.empty((B, L, H, dI), dtype=torch.bfloat16, device="cuda")
            ent["k_idx"] = torch.empty((B, L, dI), dtype=torch.bfloat16, device="cuda")
            ent["w"] = torch.empty((B, L, H), dtype=torch.float32, device="cuda")
            synth.fill_cuda(ent["q_idx"], seed, synth.Q_IDX, synth.INT9, l, corr=corr)
            synth.fill_cuda(ent["k_idx"], seed, synth.K_IDX, synth.INT9, l, corr=corr)
            synth.fill_cuda(ent["w"], seed, synth.W, synth.POW2W, l)
        dl.append(ent)
    dims = dsa.make_dims(B=B, Lq=L, Lk=L, start_pos=0, H_I=H, d_I=dI, k=k, n_h=128, D_qk=576,
                         D_v=512, scale=scale, k_row_stride=576, v_row_stride=576)
    idx = torch.empty((B, L, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(dsa.indexcache_forward_workspace(dims), dtype=torch.uint8, device="cuda")
    f_layers = [l for l, r in enumerate(pattern) if r == "F"]
    caches = {}
    for F in f_layers:
        # prefix up to F's segment end: the cache then holds F's selection
        end = next((g for g in f_layers if g > F), len(pattern))
        before = dsa.indexer_launch_count()
        dsa.indexcache_forward(pattern[:end], dl[:end], dims, idx, ws=ws)
        dsa.check_device_errors()
        assert dsa.indexer_launch_count() - before == pattern[:end].count("F")
        caches[F] = idx[0, rows].cpu().numpy()
    lse_all = [dl[l]["lse"][0, att_rows].cpu().numpy() for l in range(len(pattern))]
    out_last = dl[-1]["out"][0, att_rows].float().cpu().numpy()
    sel = {}
    for F in f_layers:
        kh = synth.tensor(seed, synth.K_IDX, synth.INT9, F, (B, L, dI), corr=corr)
        for n, i in enumerate(rows):
            qr = synth.rows(seed, synth.Q_IDX, synth.INT9, F, (B, L, H, dI), np.arange(H) + H * i, corr=corr)
            wr = synth.rows(seed, synth.W, synth.POW2W, F, (B, L, H), [i], bf16=False)[0]
            I = oracle_mod.indexer_row(qr, kh[0], wr, i)
            sel[F, i] = oracle_mod.topk_row(I, i, k)
            np.testing.assert_array_equal(caches[F][n], sel[F, i])
        del kh
    gov = {}
    for l, role in enumerate(pattern):
        gov[l] = l if role == "F" else gov[l - 1]
    for l in range(len(pattern)):
        ql = 0 if shared_q else l
        qkw = dict(sigma=0.5) if shared_q else kw
        for n, i in enumerate(att_rows):
            s_row = sel[gov[l], i]
            valid = s_row[s_row >= 0]
            qr = synth.rows(seed, synth.Q, synth.NORMAL, ql, (B, L, 128, 576), np.arange(128) + 128 * i, **qkw)
            kr = synth.rows(seed, synth.KV, synth.NORMAL, l, (B, L, 576), valid.astype(np.uint64), **kw)
            o, lse_o = oracle_mod.sparse_attn_row(qr, kr, kr, np.arange(len(valid), dtype=np.int32), scale, Dv=512)
            fin = np.isfinite(lse_o)
            assert np.array_equal(np.isfinite(lse_all[l][n]), fin)
            np.testing.assert_allclose(lse_all[l][n][fin], lse_o[fin], rtol=0, atol=1e-5 + 2048 * 2.0 ** -24 + 3.6e-4)
            if l == len(pattern) - 1:
                _close(out_last[n], o)


def test_config3_stack_fsssfsss_l32768(dsa, oracle_mod):
    # The eight-layer FSSSFSSS stack at its stated size (B = 1, L = 32,768,
    # k = 2048, correlated layers): the index cache after both F segments and
    # every layer's attention on rows stratified over t.
    _sampled_stack(dsa, oracle_mod, "FSSSFSSS", 32768, 61,
                   rows=[1, 2047, 2048, 2049, 16384, 32767], att_rows=[1, 2048, 16384, 32767],
                   corr=True, shared_q=False)


@pytest.mark.parametrize("pattern", ["FFFF", "FSFS"])
def test_long_stacks_l200k(dsa, oracle_mod, pattern):
    # Four-layer stacks of the 1/1 and 1/2 patterns at L = 200,000 (the long
    # prefill of the sweep), uncorrelated layers as in the benchmark.
    _sampled_stack(dsa, oracle_mod, pattern, 200000, 62,
                   rows=[1, 2048, 99999, 199999], att_rows=[1, 2048, 199999],
                   corr=False, shared_q=True)
