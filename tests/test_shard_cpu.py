"""Query sharding of one sequence (zig-zag chunks), on CPU: every row is owned
by exactly one rank, the indexer work is balanced, and two gloo ranks that each
run only their chunks as chunked prefills (start_pos = chunk start) reproduce
the whole-sequence layer loop of the oracle."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sparse_attention_13_b200 import shard, synth  # noqa: E402


@pytest.mark.parametrize("L", [1, 7, 96, 512, 200000])
@pytest.mark.parametrize("G", [1, 2, 3, 4, 8])
def test_zigzag_covers_every_row_once(L, G):
    rows = np.zeros(L, dtype=np.int64)
    for r in range(G):
        for (s, n) in shard.zigzag_chunks(L, G, r):
            assert n > 0
            rows[s:s + n] += 1
    assert np.all(rows == 1)


def test_work_counts_match_brute_force():
    for (s, n, k) in [(0, 10, 4), (3, 5, 100), (90, 20, 95), (0, 1, 1)]:
        t = np.arange(s, s + n)
        assert shard.indexer_pairs(s, n) == t.sum()
        assert shard.attention_rows(s, n, k) == np.minimum(t, k).sum()


@pytest.mark.parametrize("G", [2, 4, 8])
def test_zigzag_balances_work_at_200k(G):
    L, k = 200000, 2048
    pairs = [sum(shard.indexer_pairs(s, n) for s, n in shard.zigzag_chunks(L, G, r)) for r in range(G)]
    rows = [sum(shard.attention_rows(s, n, k) for s, n in shard.zigzag_chunks(L, G, r)) for r in range(G)]
    assert sum(pairs) == L * (L - 1) // 2
    assert max(pairs) / min(pairs) < 1.001
    # only rank 0's first chunk holds rows with t < k: it misses about k^2/2
    # of the L k / G entries a rank holds
    x = G * k / (2 * L)
    assert rows.index(min(rows)) == 0
    assert max(rows) / min(rows) < 1 / (1 - x) + 1e-3
    # contiguous slices would be far worse
    slices = [shard.indexer_pairs(r * L // G, (r + 1) * L // G - r * L // G) for r in range(G)]
    assert max(slices) / min(slices) > 2.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# tiny two-layer stack: F then S
DIMS = dict(L=96, H=4, dI=32, k=16, n_h=2, D=16, pattern="FS", scale=0.25)


def _stack(seed=5):
    d = DIMS
    layers = []
    for l, role in enumerate(d["pattern"]):
        lay = dict(q=synth.tensor(seed, synth.Q, synth.NORMAL, l, (1, d["L"], d["n_h"], d["D"])),
                   kv=synth.tensor(seed, synth.KV, synth.NORMAL, l, (1, d["L"], d["D"])))
        if role == "F":
            lay.update(q_idx=synth.tensor(seed, synth.Q_IDX, synth.INT9, l, (1, d["L"], d["H"], d["dI"])),
                       k_idx=synth.tensor(seed, synth.K_IDX, synth.INT9, l, (1, d["L"], d["dI"])),
                       w=synth.tensor(seed, synth.W, synth.POW2W, l, (1, d["L"], d["H"]), bf16=False))
        else:
            lay.update(q_idx=None, k_idx=None, w=None)
        layers.append(lay)
    return layers


def _run_rows(oracle_mod, layers, start, n):
    """The layer loop over rows start .. start + n - 1 only (a chunked
    prefill against the whole caches)."""
    d = DIMS
    sub = []
    for lay in layers:
        s = dict(q=lay["q"][:, start:start + n], kv=lay["kv"])
        if lay["q_idx"] is not None:
            s.update(q_idx=lay["q_idx"][:, start:start + n], k_idx=lay["k_idx"], w=lay["w"][:, start:start + n])
        else:
            s.update(q_idx=None, k_idx=None, w=None)
        sub.append(s)
    idx, out, _, _ = oracle_mod.indexcache_forward(
        d["pattern"], sub, B=1, Lq=n, Lk=d["L"], start_pos=start, H=d["H"], dI=d["dI"], k=d["k"],
        n_h=d["n_h"], Dqk=d["D"], Dv=d["D"], scale=d["scale"])
    return idx, out


def _worker(rank, world, port, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle as oracle_mod
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", init_method="env://", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    layers = _stack()
    mine = [(s, n, *_run_rows(oracle_mod, layers, s, n)) for (s, n) in shard.zigzag_chunks(DIMS["L"], world, rank)]
    gathered = [None] * world
    dist.all_gather_object(gathered, mine)
    dist.destroy_process_group()
    if rank == 0:
        out_q.put(gathered)


def test_two_ranks_reproduce_the_whole_sequence(oracle_mod):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d = DIMS
    idx_full, out_full = _run_rows(oracle_mod, _stack(), 0, d["L"])
    seen = np.zeros(d["L"], dtype=int)
    for chunks in gathered:
        for (s, n, idx, out) in chunks:
            np.testing.assert_array_equal(idx, idx_full[:, :, s:s + n])
            np.testing.assert_array_equal(out, out_full[:, :, s:s + n])
            seen[s:s + n] += 1
    assert np.all(seen == 1)
