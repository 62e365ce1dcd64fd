"""The seeded generators produce the shapes, distributions and structure of the five workloads."""
import numpy as np

from hstu_sequential_transducer_jagged_b200 import workloads as W


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5e-3], np.float32)
    r = W.round_to_bf16(x)
    assert r[0] == 1.0
    assert r[1] == 1.0                    # tie -> even mantissa
    assert r[2] == 1.0 + 4 * 2 ** -8      # tie -> even (up)
    assert r[3] == 1.0
    assert np.all(W.round_to_bf16(r) == r)
    assert np.all((r.view(np.uint32) & 0xFFFF) == 0)


def test_small_layer_workload_shapes():
    w = W.make("layer_fp32_b4")
    assert w.num_seqs == 4 and w.dtype == "fp32"
    assert np.all((w.lengths >= 16) & (w.lengths <= 128))
    assert w.x.shape == (w.total_tokens, 64)
    assert w.layers[0].w1.shape == (64, 2 * 2 * (32 + 32))
    assert w.layers[0].rab_pos.shape == (257,) and w.layers[0].rab_time.shape == (128,)
    for b in range(4):
        s, e = w.seq_offsets[b], w.seq_offsets[b + 1]
        ts = w.timestamps[s:e]
        assert ts[0] == 0 and np.all(np.diff(ts) >= 0)


def test_truncated_geometric_mean():
    rng = np.random.default_rng(0)
    x = W.truncated_geometric(rng, 200000)
    assert x.min() >= 1 and x.max() <= 1024
    assert abs(x.mean() - 300) < 3


def test_interleaved_timestamps_shared_per_pair():
    w = W.make("stack4_bf16_b8_inter", B=2, lo=64, hi=96, num_layers=1)
    for b in range(2):
        s, e = w.seq_offsets[b], w.seq_offsets[b + 1]
        ts = w.timestamps[s:e]
        L = e - s
        assert np.all(ts[0:L - 1:2] == ts[1:L:2])


def test_mfalcon_candidates_share_last_history_timestamp():
    w = W.make("mfalcon_bf16_b16", B=2, n_hist=64, m=16, num_layers=1)
    for b in range(2):
        s = w.seq_offsets[b]
        ts = w.timestamps[s:s + 80]
        assert np.all(ts[64:] == ts[63])
    assert w.mask == W.MASK_MFALCON and w.num_candidates == 16


def test_seeded_streams_are_deterministic_and_independent():
    a = W.random_attention_case(5, [10, 20], H=2, d=8)
    b = W.random_attention_case(5, [10, 20], H=2, d=8)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.timestamps, b.timestamps)
    c = W.random_attention_case(6, [10, 20], H=2, d=8)
    assert not np.array_equal(a.q, c.q)
