"""GPU-vs-oracle parity through the C ABI (needs a B200 and the built library).

Tolerance (floating point): per element |gpu - ref| <= 2e-2 * max|ref row| + 1e-3 and relative
Frobenius error <= 5e-3 (bf16 inputs, fp32 accumulation); time buckets and jagged copies are
compared bit-exactly.  Sizes span several 128-row tiles with ragged tails; full-size workloads are
checked on sampled rows (or whole sampled sequences) that the oracle computes directly.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W

pytestmark = pytest.mark.gpu

ROW_TOL = 2e-2
ABS_TOL = 1e-3
FRO_TOL = 5e-3


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from hstu_sequential_transducer_jagged_b200 import binding
    binding.lib()  # fails loudly if the library is missing
    return binding


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def act(case):
    return torch.bfloat16 if case.dtype == "bf16" else torch.float32


def assert_close(gpu, ref, what=""):
    g = gpu.detach().float().cpu().numpy().astype(np.float64) if torch.is_tensor(gpu) else gpu
    ref = np.asarray(ref, dtype=np.float64)
    g = g.reshape(ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    if ref.ndim == 1:
        bound = ROW_TOL * np.abs(ref).max(initial=0.0) + ABS_TOL
    else:
        bound = ROW_TOL * np.abs(ref).max(axis=-1, keepdims=True) + ABS_TOL
    bad = err > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} elements out of tolerance, max err "
                           f"{err.max():.3e}")
    nref = np.linalg.norm(ref)
    if nref > 0:
        fro = np.linalg.norm(g - ref) / nref
        assert fro <= FRO_TOL, f"{what}: relative Frobenius error {fro:.3e}"


def attn_kw(case):
    return dict(num_heads=case.num_heads, d_qk=case.d_qk, d_v=case.d_v,
                max_pos_dist=case.max_pos_dist, num_time_buckets=case.num_time_buckets,
                alpha=case.alpha, mask=case.mask, num_candidates=case.num_candidates)


def gpu_attention(B, case, use_time=True, use_pos=True, microbatch=None):
    dt = act(case)
    q, k, v = dev(case.q, dt), dev(case.k, dt), dev(case.v, dt)
    off = dev(case.seq_offsets)
    ts = dev(case.timestamps) if use_time else None
    rp = dev(case.rab_pos) if use_pos else None
    rt = dev(case.rab_time) if use_time else None
    out = B.attention_forward(q, k, v, off, case.max_seq_len, ts, rp, rt,
                              num_heads=case.num_heads, max_pos_dist=case.max_pos_dist,
                              num_time_buckets=case.num_time_buckets, alpha=case.alpha,
                              mask=case.mask, num_candidates=case.num_candidates,
                              microbatch=microbatch or max(case.microbatch, 1))
    torch.cuda.synchronize()
    return out


def oracle_attention(case, use_time=True, use_pos=True, rows=None):
    return O.attention_forward(case.q, case.k, case.v, case.seq_offsets,
                               case.timestamps if use_time else None,
                               case.rab_pos if use_pos else None,
                               case.rab_time if use_time else None, rows=rows, **attn_kw(case))


# ------------------------------------------------------------------------ bias indices
def test_time_buckets_bit_exact(B):
    vals = [0, 1, -1, -(2 ** 62), 2 ** 63 - 1]
    for k in range(1, 63):
        vals += [2 ** k - 1, 2 ** k, 2 ** k + 1]
    rng = np.random.default_rng(0)
    vals += list(rng.integers(-2 ** 40, 2 ** 62, size=5000))
    dt = np.array(vals, dtype=np.int64)
    for nb in (1, 16, 64, 128):
        got = B.debug_time_buckets(dev(dt), nb).cpu().numpy()
        assert np.array_equal(got, O.time_bucket(dt, nb)), nb


def _edges(kmax, lo=-3):
    """Differences around every power of two up to 2^kmax, plus zero and negatives."""
    v = {0, 1, -1, -2, lo}
    for k in range(1, kmax + 1):
        v |= {2 ** k - 1, 2 ** k, 2 ** k + 1, -(2 ** k)}
    return v


@pytest.mark.parametrize("nb", [1, 16, 64, 128])
def test_bias_time_rules_bit_exact(B, nb):
    """Each time-bucket form the attention kernels evaluate (64-bit, per-row fp32-exponent,
    per-element table entry, classifier, two-bucket threshold) equals the integer rule of
    [FunRec 7.1] §7.1.4 innovation 2 with log2 buckets, on every power-of-two edge of its range
    (the 2^23 and 2^30 switch points included) and on random differences."""
    rng = np.random.default_rng(nb)
    small = sorted(x for x in _edges(22) | {2 ** 23 - 1, -(2 ** 23 - 1)} if abs(x) < 2 ** 23)
    small = np.array(small + list(rng.integers(-2 ** 23 + 1, 2 ** 23, size=4000)), np.int64)
    cls = sorted(x for x in _edges(30) | {2 ** 31 - 1, -(2 ** 31 - 1), 2 ** 23 - 1, 2 ** 23,
                                           2 ** 23 + 1} if abs(x) < 2 ** 31)
    cls = np.array(cls + list(rng.integers(-2 ** 31 + 1, 2 ** 31, size=4000)), np.int64)
    wide = sorted(_edges(62) | {2 ** 63 - 1, -(2 ** 63) + 1})
    wide = np.array(wide + list(rng.integers(-2 ** 62, 2 ** 62, size=4000)), np.int64)
    for rule, vals in (("bucket64", wide), ("bucket_row", small), ("time_elem", small),
                       ("bucket_cls", cls)):
        got = B.debug_bias_index(rule, dev(vals), nb).cpu().numpy()
        assert np.array_equal(got, O.time_bucket(vals, nb)), (rule, nb)
    # threshold rows: [dt_lo, dt_hi] spans, one dt inside; bounds near powers of two
    lo = rng.integers(-2 ** 23 + 1, 2 ** 23, size=6000)
    span = np.where(rng.random(6000) < 0.5, rng.integers(0, 4, size=6000),
                    rng.integers(0, 2 ** 22, size=6000))
    edge = np.array(sorted(x for x in _edges(22) if abs(x) < 2 ** 23))
    lo[:len(edge)] = edge
    hi = np.minimum(lo + span, 2 ** 23 - 1)
    dt = lo + (rng.random(6000) * (hi - lo + 1)).astype(np.int64)
    dt = np.minimum(dt, hi)
    trip = np.stack([lo, hi, dt], axis=1).astype(np.int64)
    got = B.debug_bias_index("threshold", dev(trip), nb).cpu().numpy()
    b_lo, b_hi = O.time_bucket(lo, nb), O.time_bucket(hi, nb)
    want = np.where(b_hi <= b_lo + 1, O.time_bucket(dt, nb), -1)
    assert np.array_equal(got, want), nb
    assert (got >= 0).sum() > 1000  # the threshold path itself was exercised


@pytest.mark.parametrize("P", [0, 1, 5, 96, 1024, 3000])
def test_bias_position_rules_bit_exact(B, P):
    """Each position-index form (the 4-wide shifted table of the paired forward with its lane
    offset, the M-FALCON candidate form, the constant-segment decision, the direct clamp)
    equals clamp(p_i - p_j, -P, P) + P on distances -P-1 .. P+1 and at every tile offset."""
    rng = np.random.default_rng(P)
    p_i = rng.integers(0, 12000, size=8000)
    dist = np.concatenate([np.array([-P - 2, -P - 1, -P, -P + 1, -1, 0, 1, P - 1, P, P + 1,
                                     P + 2, P + 3, P + 4]),
                           rng.integers(-P - 300, P + 300, size=8000 - 13)])
    p_i[:13] = 5000
    j = np.clip(p_i - dist, 0, None)
    # every residue of j modulo the 96-key tile and the 4-wide lanes, near the clamp
    j[13:13 + 192] = 6000 + np.arange(192)
    p_i[13:13 + 192] = 6000 + 96 + P - 1
    n = rng.integers(0, 12000, size=8000)
    trip = np.stack([p_i, j, n], axis=1).astype(np.int64)
    got = B.debug_bias_index("pos_table", dev(trip), P).cpu().numpy()
    assert np.array_equal(got, O.position_index(p_i - j, P)), "pos_table"
    got = B.debug_bias_index("pos_general", dev(trip), P).cpu().numpy()
    assert np.array_equal(got, O.position_index(p_i - np.minimum(j, n), P)), "pos_general"
    got = B.debug_bias_index("pos_direct", dev(trip), P).cpu().numpy()
    assert np.array_equal(got, O.position_index(p_i - j, P)), "pos_direct"
    # The constant-segment decision is the documented rule p_min - j_last >= P, and it is sound:
    # where it fires, every query at p >= p_min and key at j <= j_last has the index 2P.  (At
    # P = 0 a negative distance also clamps to 2P; the kernel then keeps the exact per-element
    # path, which is why this is compared with the rule rather than with the index alone.)
    got = B.debug_bias_index("pos_segment", dev(trip), P).cpu().numpy()
    assert np.array_equal(got, np.where(p_i - j >= P, 2 * P, -1)), "pos_segment"
    assert np.all(O.position_index((p_i - j)[got >= 0], P) == 2 * P), "pos_segment sound"


# --------------------------------------------------------------------- attention forward
CAUSAL_LENGTHS = [1, 127, 128, 129, 0, 300, 513, 64]


@pytest.mark.parametrize("d", [64, 128, 32])
def test_attention_forward_causal_small(B, d):
    case = W.random_attention_case(100 + d, CAUSAL_LENGTHS, H=2, d=d, P=40, NB=16,
                                   gap_mean=20.0, table_std=0.5)
    assert_close(gpu_attention(B, case), oracle_attention(case), f"causal d={d}")


@pytest.mark.parametrize("use_time,use_pos", [(False, True), (True, False), (False, False)])
def test_attention_forward_bias_switches(B, use_time, use_pos):
    case = W.random_attention_case(7, [200, 77, 256], H=3, d=64, P=8, NB=12, gap_mean=5.0)
    assert_close(gpu_attention(B, case, use_time, use_pos),
                 oracle_attention(case, use_time, use_pos), f"time={use_time} pos={use_pos}")


def test_attention_forward_alpha_and_wide_scores(B):
    case = W.random_attention_case(8, [333, 129], H=2, d=64, P=100, NB=32, qkv_std=1.0)
    case.alpha = 0.125
    assert_close(gpu_attention(B, case), oracle_attention(case), "alpha")


def test_attention_forward_interleaved_timestamps(B):
    case = W.random_attention_case(9, [700, 451], H=2, d=64, P=64, NB=32, interleaved=True)
    assert_close(gpu_attention(B, case), oracle_attention(case), "interleaved")


def test_attention_forward_large_position_clamp(B):
    # P beyond the shared-memory table limit takes the global-memory table path
    case = W.random_attention_case(10, [600, 260], H=2, d=64, P=3000, NB=64)
    assert_close(gpu_attention(B, case), oracle_attention(case), "P=3000")


@pytest.mark.parametrize("m,lengths", [(40, [240, 190, 128, 300]), (64, [64 + 64, 5 + 64, 30]),
                                       (200, [456, 200, 1])])
def test_attention_forward_mfalcon(B, m, lengths):
    case = W.random_attention_case(11 + m, lengths, H=2, d=64, P=50, NB=16, mask=W.MASK_MFALCON,
                                   num_candidates=m, gap_mean=30.0)
    assert_close(gpu_attention(B, case), oracle_attention(case), f"mfalcon m={m}")


def test_attention_forward_mfalcon_microbatch_invariance(B):
    case = W.random_attention_case(12, [300, 420], H=2, d=64, P=32, NB=16, mask=W.MASK_MFALCON,
                                   num_candidates=150)
    outs = [gpu_attention(B, case, microbatch=mb) for mb in (1, 64, 128, 150)]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    ref = O.attention_forward_mfalcon_microbatched(
        case.q, case.k, case.v, case.seq_offsets, case.timestamps, case.rab_pos, case.rab_time,
        num_heads=2, d_qk=64, d_v=64, max_pos_dist=32, num_time_buckets=16,
        num_candidates=150, microbatch=64)
    assert_close(outs[0], ref, "mfalcon microbatched oracle")


def _wide_timestamps(case, seed, gap_mean, base=1_700_000_000_000):
    """Epoch-millisecond-scale timestamps with exponential gaps (30 % of them zero, so equal
    timestamps still occur)."""
    rng = np.random.default_rng(seed)
    ts = np.empty(int(case.seq_offsets[-1]), np.int64)
    for b in range(case.num_seqs):
        s, e = int(case.seq_offsets[b]), int(case.seq_offsets[b + 1])
        g = rng.exponential(gap_mean, size=e - s)
        g[rng.random(e - s) < 0.3] = 0.0
        ts[s:e] = base + np.floor(np.cumsum(g)).astype(np.int64)
    case.timestamps = ts


@pytest.mark.parametrize("gap_mean,d", [(3.0e4, 64), (2.0e8, 64), (2.0e8, 128)])
def test_attention_forward_wide_timestamps(B, gap_mean, d):
    # time differences past 2^23 (the limit of the 32-bit per-element forms) and past 2^30 (the
    # classifier's 32-bit reductions) on epoch-scale absolute values; NB = 128 reaches the
    # high buckets
    case = W.random_attention_case(14, [700, 129, 300], H=2, d=d, P=64, NB=128)
    _wide_timestamps(case, 14, gap_mean)
    assert_close(gpu_attention(B, case), oracle_attention(case), f"wide timestamps {gap_mean:g}")


def test_attention_forward_long_sequence_sampled_rows(B):
    # one 20000-token sequence beside short ones: over 200 KV tiles per late query tile, and the
    # longest work items first
    case = W.random_attention_case(15, [20000, 3, 700], H=2, d=64, P=1024, NB=128)
    out = gpu_attention(B, case).float().cpu().numpy()
    rng = np.random.default_rng(15)
    rows = [0, 1, 127, 128, 129, 9999, 10000, 19871, 19998, 19999, 20000, 20002, 20003, 20702]
    rows = np.unique(np.array(rows + list(rng.integers(0, 20000, size=24))))
    ref = oracle_attention(case, rows=rows)
    assert_close(out[rows], ref[rows], "long sequence sampled rows")


def test_attention_forward_empty_batch(B):
    # sequences that are all empty: nothing to compute, and zero-row views (whatever strides
    # they report) are accepted
    case = W.random_attention_case(16, [0, 0, 0], H=2, d=64, P=8, NB=8)
    out = gpu_attention(B, case)
    assert out.shape[0] == 0
    dq, dk, dv, dp, dt = gpu_backward(B, case)
    assert dq.shape[0] == 0 and float(dp.abs().sum()) == 0.0 and float(dt.abs().sum()) == 0.0


def test_layer_forward_empty_batch(B):
    case = W.random_layer_case(17, [0, 0], d_model=128, H=2, d=64, P=8, NB=8)
    y = gpu_layer(B, case)
    assert y.shape[0] == 0


def test_attention_forward_fp32(B):
    case = W.random_attention_case(13, [100, 17, 130], H=2, d=32, P=20, NB=16, bf16=False)
    assert_close(gpu_attention(B, case), oracle_attention(case), "fp32")


def test_attention_forward_full_size_sampled_rows(B):
    """The 4-layer stack's attention shape (B=8, L~U{2048..8192}, H=8, d=64) at full size, with
    the attention workload's own score distribution (unit-variance Q, K, V)."""
    case = W.make_attn_fwdbwd_bf16_b64(seed=3, B=8, lo=2048, hi=8192)
    out = gpu_attention(B, case).float().cpu().numpy()
    off = case.seq_offsets
    rng = np.random.default_rng(5)
    rows = []
    for b in range(case.num_seqs):
        s, e = int(off[b]), int(off[b + 1])
        rows += [s, s + 127, s + 128, e - 1] + list(rng.integers(s, e, size=4))
    rows = np.unique(np.array(rows))
    ref = oracle_attention(case, rows=rows)
    assert_close(out[rows], ref[rows], "full-size sampled rows")


# -------------------------------------------------------------------------- layer forward
def gpu_layer(B, case, layer_idx=0, x=None, out=None):
    dt = act(case)
    lp = case.layers[layer_idx]
    xx = dev(case.x, dt) if x is None else x
    y = B.layer_forward(xx, dev(lp.w1, dt), dev(lp.w2, dt), dev(case.seq_offsets),
                        case.max_seq_len, dev(case.timestamps), dev(lp.rab_pos),
                        dev(lp.rab_time), num_heads=case.num_heads, d_qk=case.d_qk,
                        d_v=case.d_v, max_pos_dist=case.max_pos_dist,
                        num_time_buckets=case.num_time_buckets, alpha=case.alpha,
                        mask=case.mask, num_candidates=case.num_candidates,
                        microbatch=max(case.microbatch, 1), out=out)
    return y


def oracle_layer(case, layer_idx=0, x=None):
    lp = case.layers[layer_idx]
    return O.layer_forward(case.x if x is None else x, lp.w1, lp.w2, case.seq_offsets,
                           case.timestamps, lp.rab_pos, lp.rab_time, **attn_kw(case))


@pytest.mark.parametrize("bf16", [True, False])
def test_layer_forward_small(B, bf16):
    case = W.random_layer_case(20, [150, 1, 129, 64, 0, 260], d_model=128, H=2, d=64, P=30,
                               NB=16, bf16=bf16, w_std=0.05)
    y = gpu_layer(B, case)
    torch.cuda.synchronize()
    assert_close(y, oracle_layer(case), f"layer bf16={bf16}")


@pytest.mark.parametrize("d_model,H,d", [(264, 3, 32), (200, 2, 64), (128, 8, 128)])
def test_layer_forward_f2_shapes(B, d_model, H, d):
    # the fused output projection at its edges: a partial second 256-column unit (264), a
    # single partial unit (200), F = H d_v not a multiple of 64 (96) and the largest F (1024);
    # 507 tokens leave a partial 128-row block
    case = W.random_layer_case(22, [300, 1, 129, 0, 77], d_model=d_model, H=H, d=d, P=30,
                               NB=16, w_std=0.05)
    y = gpu_layer(B, case)
    torch.cuda.synchronize()
    assert_close(y, oracle_layer(case), f"layer f2 d_model={d_model} H={H} d={d}")


def test_layer_forward_mfalcon_small(B):
    case = W.random_layer_case(21, [300, 250], d_model=128, H=2, d=64, P=30, NB=16,
                               mask=W.MASK_MFALCON, num_candidates=100)
    y = gpu_layer(B, case)
    torch.cuda.synchronize()
    assert_close(y, oracle_layer(case), "layer mfalcon")


def test_layer_fp32_b4_workload(B):
    case = W.make("layer_fp32_b4")
    y = gpu_layer(B, case)
    torch.cuda.synchronize()
    assert_close(y, oracle_layer(case), "layer_fp32_b4")


def test_layer_bf16_b32_geo_workload(B):
    case = W.make("layer_bf16_b32_geo")
    y = gpu_layer(B, case)
    torch.cuda.synchronize()
    assert_close(y, oracle_layer(case), "layer_bf16_b32_geo")


def _sequence_subcase(case, b):
    """The single sequence b of a workload as its own jagged batch (sequences are independent)."""
    s, e = int(case.seq_offsets[b]), int(case.seq_offsets[b + 1])
    return s, e, np.array([0, e - s], dtype=np.int64)


def test_stack4_workload_sampled_sequence(B):
    """Full 4-layer stack on the GPU; the shortest and longest sequences checked in fp64."""
    case = W.make("stack4_bf16_b8_inter")
    dt = act(case)
    x = dev(case.x, dt)
    for l in range(len(case.layers)):
        x = gpu_layer(B, case, l, x=x)
    torch.cuda.synchronize()
    y = x.float().cpu().numpy()
    for b in (int(np.argmin(case.lengths)), int(np.argmax(case.lengths))):
        s, e, off = _sequence_subcase(case, b)
        ref = O.stack_forward(case.x[s:e], case.layers, off, case.timestamps[s:e],
                              round_between=W.round_to_bf16, **attn_kw(case))
        assert_close(y[s:e], ref, f"stack4 sequence {b}")


def test_mfalcon_workload_sampled_sequence(B):
    case = W.make("mfalcon_bf16_b16")
    dt = act(case)
    x = dev(case.x, dt)
    for l in range(len(case.layers)):
        x = gpu_layer(B, case, l, x=x)
    torch.cuda.synchronize()
    y = x.float().cpu().numpy()
    for b in (0, 5, case.num_seqs - 1):
        s, e, off = _sequence_subcase(case, b)
        ref = O.stack_forward(case.x[s:e], case.layers, off, case.timestamps[s:e],
                              round_between=W.round_to_bf16, **attn_kw(case))
        assert_close(y[s:e], ref, f"mfalcon sequence {b}")


# ----------------------------------------------------------------------- attention backward
def gpu_backward(B, case, use_time=True, use_pos=True):
    dt = act(case)
    q, k, v, d_o = (dev(case.q, dt), dev(case.k, dt), dev(case.v, dt), dev(case.d_o, dt))
    res = B.attention_backward(q, k, v, d_o, dev(case.seq_offsets), case.max_seq_len,
                               dev(case.timestamps), dev(case.rab_pos) if use_pos else None,
                               dev(case.rab_time) if use_time else None,
                               num_heads=case.num_heads, max_pos_dist=case.max_pos_dist,
                               num_time_buckets=case.num_time_buckets, alpha=case.alpha,
                               mask=case.mask, num_candidates=case.num_candidates,
                               microbatch=max(case.microbatch, 1))
    torch.cuda.synchronize()
    return res


def oracle_backward(case, use_time=True, use_pos=True):
    return O.attention_backward(case.q, case.k, case.v, case.d_o, case.seq_offsets,
                                case.timestamps, case.rab_pos if use_pos else None,
                                case.rab_time if use_time else None, **attn_kw(case))


@pytest.mark.parametrize("mask,m", [(W.MASK_CAUSAL, 0), (W.MASK_MFALCON, 50)])
def test_attention_backward_small(B, mask, m):
    case = W.random_attention_case(30 + m, [200, 1, 129, 77], H=2, d=64, P=20, NB=16,
                                   mask=mask, num_candidates=m, gap_mean=20.0, qkv_std=0.5)
    got = gpu_backward(B, case)
    ref = oracle_backward(case)
    for name, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time"), got, ref):
        assert_close(g, r, f"backward {name}")


def test_attention_backward_wide_timestamps(B):
    # the backward's time buckets from 64-bit differences past 2^30, epoch-scale values
    case = W.random_attention_case(31, [300, 129, 1], H=2, d=64, P=20, NB=64, qkv_std=0.5)
    _wide_timestamps(case, 31, 2.0e8)
    got = gpu_backward(B, case)
    ref = oracle_backward(case)
    for name, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time"), got, ref):
        assert_close(g, r, f"backward wide timestamps {name}")


@pytest.mark.parametrize("use_time,use_pos,mask,m,wide", [
    (True, True, W.MASK_CAUSAL, 0, False),
    (False, True, W.MASK_CAUSAL, 0, False),
    (True, False, W.MASK_CAUSAL, 0, False),
    (True, True, W.MASK_MFALCON, 40, False),
    (True, True, W.MASK_CAUSAL, 0, True),
    (True, False, W.MASK_CAUSAL, 0, True),
])
def test_attention_backward_band_blocks(B, use_time, use_pos, mask, m, wide):
    # P = 160 over sequences of up to 740 tokens: 32 x 32 blocks whose distances all lie in the
    # position band sum the position bins by diagonal, with one time bucket or per-element
    # buckets from 32-bit differences; blocks past the band, with candidates, on the diagonal or
    # (wide) with differences past 2^23 take the other paths
    case = W.random_attention_case(33 + m, [700 + m, 300 + m, 65 + m, 1], H=2, d=64, P=160,
                                   NB=32, mask=mask, num_candidates=m, gap_mean=20.0,
                                   qkv_std=0.5)
    if wide:
        _wide_timestamps(case, 33, 2.0e4)
    got = gpu_backward(B, case, use_time, use_pos)
    ref = oracle_backward(case, use_time, use_pos)
    names = ("dq", "dk", "dv", "d_rab_pos", "d_rab_time")
    for name, g, r in zip(names, got, ref):
        if g is None:
            assert (name == "d_rab_pos" and not use_pos) or (name == "d_rab_time" and not use_time)
            continue
        assert_close(g, r, f"backward band blocks {name}")


def test_attention_backward_mid_size(B):
    case = W.make_attn_fwdbwd_bf16_b64(seed=1, B=4, lo=512, hi=2048)
    got = gpu_backward(B, case)
    ref = oracle_backward(case)
    for name, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time"), got, ref):
        assert_close(g, r, f"backward mid {name}")


def test_attention_backward_full_size_sampled(B):
    """Full attention-only backward workload; per-sequence gradients of sampled sequences, and
    the invariant that both bias-table gradients total Σ dS over every visible pair."""
    case = W.make("attn_fwdbwd_bf16_b64")
    dq, dk, dv, dp, dtm = gpu_backward(B, case)
    for b in (0, int(np.argmax(case.lengths))):
        s, e, off = _sequence_subcase(case, b)
        ref = O.attention_backward(case.q[s:e], case.k[s:e], case.v[s:e], case.d_o[s:e], off,
                                   case.timestamps[s:e], case.rab_pos, case.rab_time,
                                   **attn_kw(case))
        for name, g, r in zip(("dq", "dk", "dv"), (dq[s:e], dk[s:e], dv[s:e]), ref[:3]):
            assert_close(g, r, f"full backward seq {b} {name}")
    tp, tt = float(dp.double().sum()), float(dtm.double().sum())
    assert abs(tp - tt) <= 1e-3 * max(abs(tp), abs(tt), 1.0)
    # table entries compared element by element, each summed over every sequence: offsets
    # 0..31 of the position table and the time buckets of differences below 512 s
    P = case.max_pos_dist
    ref_p, ref_t = O.bias_grad_entries(case.q, case.k, case.v, case.d_o, case.seq_offsets,
                                       case.timestamps, case.rab_pos, case.rab_time,
                                       max_delta=31, max_bucket=8, **_attn_kw_causal(case))
    assert_close(dp[P:P + 32], ref_p, "full backward d_rab_pos entries P..P+31")
    assert_close(dtm[:9], ref_t, "full backward d_rab_time buckets 0..8")


def _attn_kw_causal(case):
    assert case.mask == W.MASK_CAUSAL
    kw = attn_kw(case)
    del kw["mask"], kw["num_candidates"]
    return kw


# ---------------------------------------------------------------------------- misc kernels
def test_jagged_padded_roundtrip(B):
    lengths = np.array([5, 0, 130, 1, 64])
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    vals = torch.randn(T, 24, device="cuda").to(torch.bfloat16)  # 48-byte rows
    padded = B.jagged_to_padded(vals, dev(off), 130)
    ref = torch.zeros(5, 130, 24, dtype=torch.bfloat16, device="cuda")
    for b in range(5):
        ref[b, :lengths[b]] = vals[off[b]:off[b + 1]]
    assert torch.equal(padded, ref)
    back = B.padded_to_jagged(padded, dev(off), T)
    assert torch.equal(back, vals)
    trunc = B.jagged_to_padded(vals, dev(off), 64)
    assert torch.equal(trunc, ref[:, :64])


def test_malformed_offsets_set_device_check(B):
    case = W.random_attention_case(40, [100, 50], H=1, d=64)
    dt = act(case)
    q = dev(case.q, dt)
    bad = dev(np.array([0, 120, 150], dtype=np.int32))  # first length 120 > max_seq_len 100
    ws = B.Workspace(1 << 20, q.device)
    out = torch.full_like(q, 7.0)
    B.attention_forward(q, q, q, bad, 100, None, None, None, num_heads=1, out=out, ws=ws)
    assert ws.sync_status() == 6
    assert torch.all(out == 7.0)
    assert ws.sync_status() == 0  # reading the status clears it
