"""Zig-zag query sharding of one sequence on the product path: each rank's
two chunks run as chunked prefills (start_pos = the chunk's first row, the
full per-layer caches) through indexcache_forward, and together they
reproduce the whole-sequence run bit for bit (indices and every layer's
output), with sampled rows checked against the oracle.  Two and four ranks
are emulated one after another on one GPU (no rank waits on another: the
chunks are independent)."""
import math

import numpy as np
import pytest

from sparse_attention_13_b200 import shard, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_13_b200 import dsa as _dsa
    _dsa.lib()
    return _dsa


def test_zigzag_chunks_reproduce_the_whole_sequence(dsa, oracle_mod):
    import torch
    B, L, H, dI, kk = 1, 4096, 64, 128, 2048
    pattern, seed = "FSSSFSSS", 91
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
    dims = dsa.make_dims(B=B, Lq=L, Lk=L, start_pos=0, H_I=H, d_I=dI, k=kk, n_h=128, D_qk=576, D_v=512,
                         scale=scale, k_row_stride=576, v_row_stride=576)
    idx = torch.empty((B, L, kk), dtype=torch.int32, device="cuda")
    dsa.indexcache_forward(pattern, dl, dims, idx)
    dsa.check_device_errors()
    whole_idx = idx.clone()
    whole_out = [d["out"].clone() for d in dl]
    for G in (2, 4):
        seen = torch.zeros(L, dtype=torch.int32, device="cuda")
        for r in range(G):
            for (s, n) in shard.zigzag_chunks(L, G, r):
                layers = []
                for l, d in enumerate(dl):
                    ent = dict(q=d["q"][:, s:s + n], kbuf=d["kbuf"], vbuf=d["vbuf"],
                               out=torch.empty((B, n, 128, 512), dtype=torch.bfloat16, device="cuda"))
                    if pattern[l] == "F":
                        ent.update(q_idx=d["q_idx"][:, s:s + n], k_idx=d["k_idx"], w=d["w"][:, s:s + n])
                    layers.append(ent)
                cdims = dsa.make_dims(B=B, Lq=n, Lk=L, start_pos=s, H_I=H, d_I=dI, k=kk, n_h=128, D_qk=576,
                                      D_v=512, scale=scale, k_row_stride=576, v_row_stride=576)
                cidx = torch.empty((B, n, kk), dtype=torch.int32, device="cuda")
                dsa.indexcache_forward(pattern, layers, cdims, cidx)
                dsa.check_device_errors()
                assert torch.equal(cidx, whole_idx[:, s:s + n]), (G, r, s)
                for l in range(8):
                    assert torch.equal(layers[l]["out"], whole_out[l][:, s:s + n]), (G, r, s, l)
                seen[s:s + n] += 1
        assert bool(torch.all(seen == 1))
    # the whole-sequence run against the oracle on rows of the first and last chunks
    kh = synth.tensor(seed, synth.K_IDX, synth.INT9, 4, (B, L, dI), corr=True)
    kvh = synth.tensor(seed, synth.KV, synth.NORMAL, 7, (B, L, 576), sigma=0.5, corr=True)
    got_idx = whole_idx.cpu().numpy()
    for i in (5, 1030, 3071, 4095):
        qr = synth.rows(seed, synth.Q_IDX, synth.INT9, 4, (B, L, H, dI), np.arange(H) + H * i, corr=True)
        wr = synth.rows(seed, synth.W, synth.POW2W, 4, (B, L, H), [i], bf16=False)[0]
        sel = oracle_mod.topk_row(oracle_mod.indexer_row(qr, kh[0], wr, i), i, kk)
        np.testing.assert_array_equal(got_idx[0, i], sel)
        q7 = synth.rows(seed, synth.Q, synth.NORMAL, 7, (B, L, 128, 576), np.arange(128) + 128 * i, sigma=0.5,
                        corr=True)
        o, _ = oracle_mod.sparse_attn_row(q7, kvh[0], kvh[0], sel, scale, Dv=512)
        got = whole_out[7][0, i].float().cpu().numpy()
        assert np.all(np.abs(got - o) <= 2e-2 + 1e-2 * np.abs(o))
