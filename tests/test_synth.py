"""Host side of the seeded input generator: published SplitMix64 outputs,
value ranges of each law, and the layer-correlation recursion.  CPU only."""
import numpy as np

from sparse_attention_13_b200 import synth


def test_splitmix64_reference_outputs():
    # SplitMix64 started from state 0 (key 0): first outputs of the
    # published generator.
    z = synth._mix64(np.arange(1, 4, dtype=np.uint64) * synth.GAMMA)
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_int9_range_and_balance():
    v = synth.bf16_bits_to_f32(synth.tensor(1, synth.K_IDX, synth.INT9, 0, (200000,)))
    assert set(np.unique(v).tolist()) == set(range(-4, 5))
    counts = np.bincount((v + 4).astype(int))
    assert counts.min() > 0.95 * len(v) / 9


def test_pow2_weights():
    w = synth.tensor(1, synth.W, synth.POW2W, 0, (100000,), bf16=False)
    assert set(np.unique(np.abs(w)).tolist()) == {1.0, 0.5, 0.25, 0.125}
    assert abs((w > 0).mean() - 0.5) < 0.01


def test_normal_moments():
    x = synth.bf16_bits_to_f32(synth.tensor(2, synth.Q, synth.NORMAL, 0, (400000,), sigma=0.5))
    assert abs(x.mean()) < 0.005 and abs(x.std() - 0.5) < 0.005


def test_layer_correlation():
    a = synth.bf16_bits_to_f32(synth.tensor(3, synth.KV, synth.NORMAL, 2, (100000,), sigma=0.5, corr=True))
    b = synth.bf16_bits_to_f32(synth.tensor(3, synth.KV, synth.NORMAL, 3, (100000,), sigma=0.5, corr=True))
    c = np.corrcoef(a, b)[0, 1]
    assert 0.85 < c < 0.95
    ia = synth.bf16_bits_to_f32(synth.tensor(3, synth.K_IDX, synth.INT9, 1, (100000,), corr=True))
    assert set(np.unique(ia).tolist()) <= set(range(-4, 5))


def test_rows_match_full_tensor():
    full = synth.tensor(4, synth.Q_IDX, synth.INT9, 1, (7, 5, 3), corr=True)
    r = synth.rows(4, synth.Q_IDX, synth.INT9, 1, (7, 5, 3), [0, 9, 34], corr=True)
    np.testing.assert_array_equal(r, full.reshape(35, 3)[[0, 9, 34]])
