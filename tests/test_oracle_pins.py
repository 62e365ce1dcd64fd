"""Pins of the fp64 oracle against facts fixed by the HSTU pages and by mathematics.

None of these tests retypes the oracle's formula: each checks a closed form, an invariant, a
brute force on tiny inputs or a hand-derived value, chosen so that a dropped term, a wrong sign or
index, a transposed operand or a swapped split block fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _attn(case, **kw):
    args = dict(num_heads=case.num_heads, d_qk=case.d_qk, d_v=case.d_v,
                max_pos_dist=case.max_pos_dist, num_time_buckets=case.num_time_buckets,
                mask=case.mask, num_candidates=case.num_candidates, alpha=case.alpha)
    args.update(kw)
    return args


# ---------------------------------------------------------------------------------- SiLU
def test_silu_special_values_and_limits():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert O.silu_grad(np.array([0.0]))[0] == 0.5
    # x·σ(x) -> x for large x, -> 0 for very negative x; σ(1) = e/(1+e)
    np.testing.assert_allclose(O.silu(np.array([40.0])), [40.0], rtol=1e-15)
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15
    np.testing.assert_allclose(O.silu(np.array([1.0])), [math.e / (1 + math.e)], rtol=1e-15)
    np.testing.assert_allclose(O.silu(np.array([-1.0])), [-1.0 / (1 + math.e)], rtol=1e-15)


def test_silu_grad_is_derivative():
    x = np.linspace(-12, 12, 97)
    h = 1e-6
    fd = (O.silu(x + h) - O.silu(x - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_grad(x), fd, rtol=1e-7, atol=1e-9)


# ---------------------------------------------------------------------------- bias indices
def _golden_buckets():
    rows = []
    with open(os.path.join(GOLDEN, "time_buckets.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            dt, b = line.split()[:2]
            rows.append((int(dt), int(b)))
    return rows


def test_time_bucket_hand_values():
    for dt, b in _golden_buckets():
        assert int(O.time_bucket(np.array([dt]), 128)[0]) == b, dt


def test_time_bucket_bruteforce_powers_of_two():
    vals = [0, 1, -1, -(2 ** 40)]
    for k in range(1, 63):
        vals += [2 ** k - 1, 2 ** k, 2 ** k + 1]
    vals = [v for v in vals if v < 2 ** 63]
    got = O.time_bucket(np.array(vals, dtype=np.int64), 128)
    for v, g in zip(vals, got):
        # smallest k with 2^(k+1) > max(1, v), by Python's exact integer bit length
        ref = max(1, v).bit_length() - 1
        assert int(g) == ref, v
    # clamp at NB-1
    assert int(O.time_bucket(np.array([2 ** 40]), 16)[0]) == 15
    assert int(O.time_bucket(np.array([2 ** 14]), 16)[0]) == 14


def test_position_index_bruteforce():
    P = 5
    L = 2 * P + 3
    for mask, m in ((O.MASK_CAUSAL, 0), (O.MASK_MFALCON, 4)):
        p = O.positions(L, mask, m)
        n = L - m
        for i in range(L):
            for j in range(L):
                pi = i if i < n else n
                pj = j if j < n else n
                ref = min(max(pi - pj, -P), P) + P
                assert int(O.position_index(p[i] - p[j], P)) == ref


def test_allowed_pairs_bruteforce():
    L, m = 9, 3
    ok = O.allowed_pairs(L, O.MASK_MFALCON, m)
    n = L - m
    for i in range(L):
        for j in range(L):
            if i < n:
                exp = j <= i
            else:
                exp = (j < n) or (j == i)
            assert bool(ok[i, j]) == exp
    assert np.array_equal(O.allowed_pairs(L, O.MASK_CAUSAL, 0), np.tril(np.ones((L, L), bool)))


# ------------------------------------------------------------------------------ attention
def test_attention_closed_form_zero_keys_constant_bias():
    """K = 0 and constant tables: out_i = SiLU(c1 + c2) · Σ_{j<=i} V_j."""
    case = W.random_attention_case(1, [7, 1, 12, 0, 5], H=2, d=4, P=4, NB=8, bf16=False)
    c1, c2 = 0.7, -0.25
    out = O.attention_forward(case.q, np.zeros_like(case.k), case.v, case.seq_offsets,
                              case.timestamps, np.full(9, c1), np.full(8, c2), **_attn(case))
    ref = np.zeros_like(out)
    off = case.seq_offsets
    for b in range(len(off) - 1):
        s, e = off[b], off[b + 1]
        ref[s:e] = np.cumsum(case.v[s:e].astype(np.float64), axis=0)
    ref *= (c1 + c2) / (1 + math.exp(-(c1 + c2)))
    np.testing.assert_allclose(out, ref, rtol=1e-13, atol=1e-13)


def test_attention_single_token():
    case = W.random_attention_case(2, [1], H=3, d=5, P=4, NB=8, bf16=False)
    out = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, **_attn(case, alpha=0.5))
    for h in range(3):
        qh = case.q[0, h * 5:(h + 1) * 5].astype(np.float64)
        kh = case.k[0, h * 5:(h + 1) * 5].astype(np.float64)
        s = 0.5 * float(qh @ kh) + float(case.rab_pos[4]) + float(case.rab_time[0])
        a = s / (1 + math.exp(-s))
        np.testing.assert_allclose(out[0, h * 5:(h + 1) * 5],
                                   a * case.v[0, h * 5:(h + 1) * 5].astype(np.float64),
                                   rtol=1e-13)


def _padded_dense(case, alpha=1.0):
    """Brute force: every pair (i, j) of a padded batch, with explicit loops and math.exp."""
    H, d = case.num_heads, case.d_qk
    off = case.seq_offsets
    T = int(off[-1])
    out = np.zeros((T, H * d))
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        L = e - s
        n = L - case.num_candidates if case.mask == O.MASK_MFALCON else L
        for h in range(H):
            for i in range(L):
                acc = np.zeros(d)
                for j in range(L):
                    visible = j <= i and (j < n or j == i)
                    if not visible:
                        continue
                    pi, pj = min(i, n), min(j, n)
                    dp = min(max(pi - pj, -case.max_pos_dist), case.max_pos_dist)
                    dt = int(case.timestamps[s + i]) - int(case.timestamps[s + j])
                    bk = min(max(1, dt).bit_length() - 1, case.num_time_buckets - 1)
                    qv = case.q[s + i, h * d:(h + 1) * d].astype(np.float64)
                    kv = case.k[s + j, h * d:(h + 1) * d].astype(np.float64)
                    sc = alpha * float(qv @ kv) + float(case.rab_pos[dp + case.max_pos_dist]) + \
                        float(case.rab_time[bk])
                    a = sc / (1.0 + math.exp(-sc))
                    acc += a * case.v[s + j, h * d:(h + 1) * d].astype(np.float64)
                out[s + i, h * d:(h + 1) * d] = acc
    return out


@pytest.mark.parametrize("mask,m", [(O.MASK_CAUSAL, 0), (O.MASK_MFALCON, 3)])
def test_attention_matches_pairwise_bruteforce(mask, m):
    case = W.random_attention_case(3, [6, 9, 5], H=2, d=3, P=3, NB=6, mask=mask,
                                   num_candidates=m, bf16=False, gap_mean=3.0)
    out = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, **_attn(case, alpha=0.8))
    np.testing.assert_allclose(out, _padded_dense(case, alpha=0.8), rtol=1e-12, atol=1e-12)


def test_attention_causality_bit_exact():
    case = W.random_attention_case(4, [10, 13], H=2, d=4, P=4, NB=8, bf16=False)
    base = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    s = int(case.seq_offsets[1])
    i = 6  # perturb every later token of sequence 1
    q2, k2, v2 = case.q.copy(), case.k.copy(), case.v.copy()
    q2[s + i + 1:] += 3.0
    k2[s + i + 1:] -= 2.0
    v2[s + i + 1:] *= -5.0
    pert = O.attention_forward(q2, k2, v2, case.seq_offsets, case.timestamps, case.rab_pos,
                               case.rab_time, **_attn(case))
    assert np.array_equal(pert[:s + i + 1], base[:s + i + 1])
    assert not np.allclose(pert[s + i + 1:], base[s + i + 1:])


def test_attention_masked_pairs_contribute_zero():
    """Changing a candidate's K/V leaves every other candidate (and the history) bit-identical."""
    case = W.random_attention_case(5, [12], H=1, d=4, P=4, NB=8, mask=O.MASK_MFALCON,
                                   num_candidates=4, bf16=False)
    base = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    k2, v2 = case.k.copy(), case.v.copy()
    k2[9] += 10.0
    v2[9] += 10.0
    pert = O.attention_forward(case.q, k2, v2, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    others = [r for r in range(12) if r != 9]
    assert np.array_equal(pert[others], base[others])


def test_attention_timestamp_shift_invariance_and_linearity_in_v():
    case = W.random_attention_case(6, [11, 4], H=2, d=4, P=4, NB=12, bf16=False, gap_mean=5.0)
    kw = _attn(case)
    base = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **kw)
    shifted = O.attention_forward(case.q, case.k, case.v, case.seq_offsets,
                                  case.timestamps + 123456789, case.rab_pos, case.rab_time, **kw)
    assert np.array_equal(base, shifted)
    v2 = np.random.default_rng(0).standard_normal(case.v.shape)
    a = O.attention_forward(case.q, case.k, 2.0 * case.v + v2, case.seq_offsets,
                            case.timestamps, case.rab_pos, case.rab_time, **kw)
    b = O.attention_forward(case.q, case.k, v2, case.seq_offsets, case.timestamps,
                            case.rab_pos, case.rab_time, **kw)
    np.testing.assert_allclose(a, 2.0 * base + b, rtol=1e-12, atol=1e-12)


def test_attention_keeps_interaction_intensity():
    """The worked example of "HSTU：Scaling Law 的首次探索" §7.1.4, innovation 1: user A clicks
    technology 10 times and entertainment once, user B 100 and 10 times.  A softmax gives both
    the same 90 % / 10 % mixture; pointwise aggregation keeps B's tenfold intensity.  With the
    same key and value per interest, no bias terms and a final query token whose own key is zero
    (its own term is SiLU(0) = 0), B's output there is exactly ten times A's, while the weights
    normalised to sum 1 (what a softmax would use) are the same for both users."""
    rng = np.random.default_rng(3)
    d = 8
    k_tech, k_ent, v_tech, v_ent, q = (rng.normal(size=d) for _ in range(5))

    def user(n_tech, n_ent):
        L = n_tech + n_ent + 1
        K = np.vstack([np.tile(k_tech, (n_tech, 1)), np.tile(k_ent, (n_ent, 1)), np.zeros(d)])
        V = np.vstack([np.tile(v_tech, (n_tech, 1)), np.tile(v_ent, (n_ent, 1)),
                       rng.normal(size=d)])
        Q = np.zeros((L, d))
        Q[-1] = q
        out = O.attention_forward(Q, K, V, np.array([0, L]), None, None, None, num_heads=1,
                                  d_qk=d, d_v=d, max_pos_dist=0, num_time_buckets=1,
                                  rows=np.array([L - 1]))
        w = O.silu(np.array([q @ k_tech, q @ k_ent]))
        mix = np.array([n_tech, n_ent]) * w
        return out[L - 1], mix / mix.sum()

    out_a, mix_a = user(10, 1)
    out_b, mix_b = user(100, 10)
    assert np.allclose(out_b, 10.0 * out_a, rtol=1e-12, atol=0)
    assert np.allclose(mix_a, mix_b, rtol=1e-12, atol=0)
    assert not np.allclose(out_b, out_a)


def test_attention_rows_subset_equals_full():
    case = W.random_attention_case(7, [20, 3, 17], H=2, d=4, P=6, NB=10, bf16=False)
    full = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    rows = np.array([0, 5, 19, 21, 30, 39])
    sub = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, rows=rows, **_attn(case))
    np.testing.assert_allclose(sub[rows], full[rows], rtol=1e-14)


# ------------------------------------------------------------------------------- M-FALCON
def test_mfalcon_candidate_equals_single_candidate_causal_forward():
    n, m = 9, 5
    case = W.random_attention_case(8, [n + m], H=2, d=3, P=4, NB=8, mask=O.MASK_MFALCON,
                                   num_candidates=m, bf16=False, gap_mean=4.0)
    full = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    kw = _attn(case, mask=O.MASK_CAUSAL, num_candidates=0)
    for c in range(m):
        idx = np.concatenate([np.arange(n), [n + c]])
        one = O.attention_forward(case.q[idx], case.k[idx], case.v[idx],
                                  np.array([0, n + 1]), case.timestamps[idx], case.rab_pos,
                                  case.rab_time, **kw)
        np.testing.assert_allclose(full[n + c], one[n], rtol=1e-13, atol=1e-14)
        if c == 0:
            np.testing.assert_allclose(full[:n], one[:n], rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("bm", [1, 2, 3, 128])
def test_mfalcon_microbatch_independence(bm):
    n, m = 7, 6
    case = W.random_attention_case(9, [n + m, n + m], H=2, d=3, P=4, NB=8,
                                   mask=O.MASK_MFALCON, num_candidates=m, bf16=False)
    full = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, **_attn(case))
    mb = O.attention_forward_mfalcon_microbatched(
        case.q, case.k, case.v, case.seq_offsets, case.timestamps, case.rab_pos, case.rab_time,
        num_heads=2, d_qk=3, d_v=3, max_pos_dist=4, num_time_buckets=8, num_candidates=m,
        microbatch=bm)
    np.testing.assert_allclose(mb, full, rtol=1e-13, atol=1e-14)


# ------------------------------------------------------------------------------- backward
def test_attention_backward_finite_differences():
    case = W.random_attention_case(10, [5, 4], H=2, d=3, P=3, NB=6, bf16=False, gap_mean=3.0,
                                   table_std=0.7)
    kw = _attn(case, alpha=0.9)
    rng = np.random.default_rng(1)
    d_o = rng.standard_normal((case.total_tokens, 6))

    def loss(q, k, v, rp, rt):
        out = O.attention_forward(q, k, v, case.seq_offsets, case.timestamps, rp, rt, **kw)
        return float((out * d_o).sum())

    q, k, v = (case.q.astype(np.float64), case.k.astype(np.float64), case.v.astype(np.float64))
    rp, rt = case.rab_pos.astype(np.float64), case.rab_time.astype(np.float64)
    dq, dk, dv, dp, dt = O.attention_backward(q, k, v, d_o, case.seq_offsets, case.timestamps,
                                              rp, rt, **kw)
    h = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("rp", rp, dp),
                            ("rt", rt, dt)):
        flat = arr.reshape(-1)
        for idx in range(flat.size):
            old = flat[idx]
            flat[idx] = old + h
            lp = loss(q, k, v, rp, rt)
            flat[idx] = old - h
            lm = loss(q, k, v, rp, rt)
            flat[idx] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad.reshape(-1)[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_attention_backward_bias_grad_totals():
    """Both bias tables see every allowed pair once: their gradients sum to the same total."""
    case = W.random_attention_case(11, [9, 6], H=2, d=3, P=2, NB=4, mask=O.MASK_MFALCON,
                                   num_candidates=2, bf16=False)
    dq, dk, dv, dp, dt = O.attention_backward(case.q, case.k, case.v, case.d_o,
                                              case.seq_offsets, case.timestamps, case.rab_pos,
                                              case.rab_time, **_attn(case))
    np.testing.assert_allclose(dp.sum(), dt.sum(), rtol=1e-12)
    assert dp[:2].sum() == 0.0  # causal and candidate pairs never have p_i < p_j


# -------------------------------------------------------------------------------- layer
def test_matmul_matches_explicit_loops():
    rng = np.random.default_rng(2)
    x, w, b = rng.standard_normal((3, 4)), rng.standard_normal((4, 5)), rng.standard_normal(5)
    ref = np.zeros((3, 5))
    for i in range(3):
        for j in range(5):
            ref[i, j] = b[j] + sum(x[i, t] * w[t, j] for t in range(4))
    np.testing.assert_allclose(O.linear(x, w, b), ref, rtol=1e-14)


def test_layer_norm_moments():
    a = np.random.default_rng(3).standard_normal((7, 48)) * 5 + 2
    n = O.layer_norm(a, eps=0.0)
    np.testing.assert_allclose(n.mean(-1), 0, atol=1e-13)
    np.testing.assert_allclose((n ** 2).mean(-1), 1, atol=1e-12)
    g, bt = np.arange(48.0), -np.ones(48)
    np.testing.assert_allclose(O.layer_norm(a, 0.0, g, bt), n * g + bt, rtol=1e-14)


def _layer_case(seed=12):
    return W.random_layer_case(seed, [8, 5], d_model=6, H=2, d=3, P=3, NB=6, bf16=False,
                               w_std=0.4)


def _layer_kw(c):
    return dict(num_heads=c.num_heads, d_qk=c.d_qk, d_v=c.d_v, max_pos_dist=c.max_pos_dist,
                num_time_buckets=c.num_time_buckets)


def test_layer_zero_w2_is_identity():
    c = _layer_case()
    lp = c.layers[0]
    y = O.layer_forward(c.x, lp.w1, np.zeros_like(lp.w2), c.seq_offsets, c.timestamps,
                        lp.rab_pos, lp.rab_time, **_layer_kw(c))
    assert np.array_equal(y, c.x.astype(np.float64))


def test_layer_split_order_u_block_gates():
    """Zeroing the U block (first) or the V block (second) of W1 gives U = 0 or AV = 0, hence
    G = Norm(AV) ⊙ U = 0 and Y = X exactly; zeroing Q or K (third, fourth) does not."""
    c = _layer_case()
    lp = c.layers[0]
    hd = c.num_heads * c.d_v
    for blk in range(4):
        w1 = lp.w1.astype(np.float64).copy()
        w1[:, blk * hd:(blk + 1) * hd] = 0.0
        y = O.layer_forward(c.x, w1, lp.w2, c.seq_offsets, c.timestamps, lp.rab_pos,
                            lp.rab_time, **_layer_kw(c))
        if blk < 2:
            assert np.array_equal(y, c.x.astype(np.float64))
        else:
            assert not np.allclose(y, c.x, rtol=1e-3, atol=1e-3)


def test_layer_split_order_q_before_k():
    """The attention inside the layer uses block 3 of SiLU(X W1) as Q and block 4 as K (a swap
    transposes the score matrix, which the causal mask does not forgive)."""
    c = _layer_case()
    lp = c.layers[0]
    H, d = c.num_heads, c.d_v
    y, mid = O.layer_forward(c.x, lp.w1, lp.w2, c.seq_offsets, c.timestamps, lp.rab_pos,
                             lp.rab_time, return_intermediates=True, **_layer_kw(c))
    blocks = [O.silu(c.x.astype(np.float64) @ lp.w1[:, i * H * d:(i + 1) * H * d].astype(
        np.float64)) for i in range(4)]
    kw = dict(_layer_kw(c))
    ref = O.attention_forward(blocks[2], blocks[3], blocks[1], c.seq_offsets, c.timestamps,
                              lp.rab_pos, lp.rab_time, **kw)
    swapped = O.attention_forward(blocks[3], blocks[2], blocks[1], c.seq_offsets, c.timestamps,
                                  lp.rab_pos, lp.rab_time, **kw)
    np.testing.assert_allclose(mid["av"], ref, rtol=1e-13, atol=1e-13)
    assert not np.allclose(mid["av"], swapped, rtol=1e-6, atol=1e-6)


def test_layer_zero_qk_blocks_closed_form():
    """Q = K = 0 (blocks 3 and 4 of W1 zeroed): AV_i = SiLU(bias_ii... ) reduces to the bias-only
    attention; with constant tables it is SiLU(c)·Σ_{j<=i} V_j, V = SiLU(X W1[:, V block])."""
    c = _layer_case()
    lp = c.layers[0]
    H, d = c.num_heads, c.d_v
    w1 = lp.w1.astype(np.float64).copy()
    w1[:, 2 * H * d:] = 0.0
    cst = 0.3
    y, mid = O.layer_forward(c.x, w1, lp.w2, c.seq_offsets, c.timestamps,
                             np.full(2 * c.max_pos_dist + 1, cst), np.zeros(c.num_time_buckets),
                             return_intermediates=True, **_layer_kw(c))
    xv = c.x.astype(np.float64) @ w1[:, H * d:2 * H * d]
    vv = xv / (1 + np.exp(-xv))
    ref_av = np.zeros_like(vv)
    off = c.seq_offsets
    for b in range(len(off) - 1):
        ref_av[off[b]:off[b + 1]] = np.cumsum(vv[off[b]:off[b + 1]], axis=0)
    ref_av *= cst / (1 + math.exp(-cst))
    np.testing.assert_allclose(mid["av"], ref_av, rtol=1e-12, atol=1e-14)
    xu = c.x.astype(np.float64) @ w1[:, :H * d]
    uu = xu / (1 + np.exp(-xu))
    mu = ref_av.mean(-1, keepdims=True)
    sd = np.sqrt(((ref_av - mu) ** 2).mean(-1, keepdims=True) + 1e-5)
    ref_y = c.x + (((ref_av - mu) / sd) * uu) @ lp.w2
    np.testing.assert_allclose(y, ref_y, rtol=1e-12, atol=1e-12)


def test_layer_rows_equals_full_and_stack_composes():
    c = W.random_layer_case(13, [9, 14, 4], d_model=8, H=2, d=4, P=5, NB=8, bf16=False,
                            num_layers=2, w_std=0.3)
    lp = c.layers[0]
    full = O.layer_forward(c.x, lp.w1, lp.w2, c.seq_offsets, c.timestamps, lp.rab_pos,
                           lp.rab_time, **_layer_kw(c))
    rows = np.array([0, 8, 9, 20, 26])
    sub = O.layer_forward_rows(c.x, lp.w1, lp.w2, c.seq_offsets, c.timestamps, lp.rab_pos,
                               lp.rab_time, rows, **_layer_kw(c))
    np.testing.assert_allclose(sub, full[rows], rtol=1e-13, atol=1e-13)
    st = O.stack_forward(c.x, c.layers, c.seq_offsets, c.timestamps, **_layer_kw(c))
    l2 = c.layers[1]
    ref = O.layer_forward(full, l2.w1, l2.w2, c.seq_offsets, c.timestamps, l2.rab_pos,
                          l2.rab_time, **_layer_kw(c))
    np.testing.assert_allclose(st, ref, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------------- layer backward
def _tiny_layer(seed=7, mask=O.MASK_CAUSAL, m=0):
    rng = np.random.default_rng(seed)
    H, d, dm = 2, 3, 5
    offsets = np.array([0, 4, 5, 9])
    T = int(offsets[-1])
    ts = np.concatenate([np.cumsum(rng.integers(0, 9, size=int(b - a)))
                         for a, b in zip(offsets[:-1], offsets[1:])]).astype(np.int64)
    p = dict(x=rng.normal(size=(T, dm)), w1=0.5 * rng.normal(size=(dm, 4 * H * d)),
             w2=0.5 * rng.normal(size=(H * d, dm)), b1=0.1 * rng.normal(size=4 * H * d),
             b2=0.1 * rng.normal(size=dm), rab_pos=0.3 * rng.normal(size=2 * 2 + 1),
             rab_time=0.3 * rng.normal(size=4), ln_gamma=1 + 0.2 * rng.normal(size=H * d),
             ln_beta=0.1 * rng.normal(size=H * d))
    kw = dict(num_heads=H, d_qk=d, d_v=d, max_pos_dist=2, num_time_buckets=4, alpha=0.7,
              mask=mask, num_candidates=m, ln_eps=1e-5)
    return p, offsets, ts, kw, rng.normal(size=(T, dm))


def _layer_loss(p, offsets, ts, kw, dy):
    y = O.layer_forward(p["x"], p["w1"], p["w2"], offsets, ts, p["rab_pos"], p["rab_time"],
                        b1=p["b1"], b2=p["b2"], ln_gamma=p["ln_gamma"], ln_beta=p["ln_beta"],
                        **kw)
    return float((dy * y).sum())


@pytest.mark.parametrize("mask,m", [(O.MASK_CAUSAL, 0), (O.MASK_MFALCON, 2)])
def test_layer_backward_finite_differences(mask, m):
    """Every gradient of the layer (input, both projections and biases, both bias tables, the
    LayerNorm affine) against central finite differences of Σ dY ⊙ Y in fp64."""
    p, offsets, ts, kw, dy = _tiny_layer(mask=mask, m=m)
    g = O.layer_backward(p["x"], p["w1"], p["w2"], offsets, ts, p["rab_pos"], p["rab_time"], dy,
                         b1=p["b1"], b2=p["b2"], ln_gamma=p["ln_gamma"], ln_beta=p["ln_beta"],
                         **kw)
    names = dict(x="dx", w1="dw1", w2="dw2", b1="db1", b2="db2", rab_pos="d_rab_pos",
                 rab_time="d_rab_time", ln_gamma="d_ln_gamma", ln_beta="d_ln_beta")
    h = 1e-6
    for key, gname in names.items():
        arr = p[key]
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = _layer_loss(p, offsets, ts, kw, dy)
            arr[idx] = old - h
            lm = _layer_loss(p, offsets, ts, kw, dy)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        scale = max(np.abs(num).max(), 1e-3)
        assert np.abs(g[gname] - num).max() <= 1e-6 * scale + 1e-8, key


def test_layer_backward_zero_w2_passes_dy_through():
    """With W2 = 0 the branch contributes nothing: dX = dY exactly (the residual edge), and
    every gradient upstream of f2 vanishes while dW2 = Gᵀ dY does not."""
    p, offsets, ts, kw, dy = _tiny_layer(seed=8)
    p["w2"][:] = 0.0
    g = O.layer_backward(p["x"], p["w1"], p["w2"], offsets, ts, p["rab_pos"], p["rab_time"], dy,
                         b1=p["b1"], b2=p["b2"], ln_gamma=p["ln_gamma"], ln_beta=p["ln_beta"],
                         **kw)
    assert np.array_equal(g["dx"], dy)
    for name in ("dw1", "db1", "d_rab_pos", "d_rab_time", "d_ln_gamma", "d_ln_beta"):
        assert not np.any(g[name]), name
    assert np.abs(g["dw2"]).max() > 0


# ----------------------------------------------------------------- Stochastic Length (§7.1.5)
def test_stochastic_length_alpha_two_keeps_everything():
    """α = 2: N^{α/2} = N, so no sequence of at most N tokens is truncated."""
    rng = np.random.default_rng(0)
    lengths = rng.integers(0, 512, size=20)
    off = W.offsets_from_lengths(lengths)
    sub_len, n_alpha = O.stochastic_length_params(512, 2.0)
    assert sub_len == 512 and n_alpha == 512.0 ** 2
    new_off, kept = O.stochastic_length(off, rng.random(20).astype(np.float32),
                                        rng.integers(0, 2 ** 32, int(off[-1]), dtype=np.uint64)
                                        .astype(np.uint32), sub_len, n_alpha)
    assert np.array_equal(new_off, off) and np.array_equal(kept, np.arange(off[-1]))


def test_stochastic_length_selection_brute_force():
    """A truncated sequence keeps exactly the sub_len tokens of smallest (key, index), counted
    pair by pair, in index order; ties in the keys go to the lower index."""
    rng = np.random.default_rng(1)
    for trial in range(30):
        n = int(rng.integers(2, 60))
        sub_len = int(rng.integers(1, n))
        keys = rng.integers(0, 8 if trial % 2 else 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
        off = np.array([0, n])
        _, kept = O.stochastic_length(off, np.array([0.0], np.float32), keys, sub_len, 0.0)
        rank = np.array([sum((int(keys[s]), s) < (int(keys[t]), t) for s in range(n))
                         for t in range(n)])
        assert np.array_equal(kept, np.nonzero(rank < sub_len)[0])


def test_stochastic_length_probability():
    """A sequence longer than N^{α/2} is truncated with probability 1 - N^α / n² (binomial
    check over 20 000 sequences, 5 standard deviations)."""
    N, alpha, n = 4096, 1.7, 3000
    sub_len, n_alpha = O.stochastic_length_params(N, alpha)
    rng = np.random.default_rng(2)
    B = 20000
    off = np.arange(B + 1, dtype=np.int64) * n
    keys = np.zeros(B * n, dtype=np.uint32)
    new_off, _ = O.stochastic_length(off, rng.random(B).astype(np.float32), keys, sub_len, n_alpha)
    frac = np.mean(np.diff(new_off) == sub_len)
    p = 1.0 - n_alpha / n ** 2
    assert abs(frac - p) <= 5 * np.sqrt(p * (1 - p) / B)


def test_stochastic_length_sparsity_claim():
    """The page reports 80%+ sequence sparsity at α about 1.6-1.7: for sequences of the longest
    length N = 8192 the expected fraction of causal attention pairs kept is below 20 %."""
    N = 8192
    for alpha in (1.6, 1.7):
        k, n_alpha = O.stochastic_length_params(N, alpha)
        p = 1.0 - n_alpha / N ** 2
        kept_pairs = p * k * (k + 1) / 2 + (1 - p) * N * (N + 1) / 2
        assert kept_pairs / (N * (N + 1) / 2) < 0.2, alpha


# ------------------------------------------------------- token-type bias ([FunRec 7.1] §7.1.4)
def _typed_case(seed, lengths, NT, mask=O.MASK_CAUSAL, m=0):
    case = W.random_attention_case(seed, lengths, H=2, d=8, P=6, NB=8, mask=mask,
                                   num_candidates=m, gap_mean=30.0)
    rng = np.random.default_rng(seed + 1)
    types = rng.integers(0, NT, size=case.total_tokens)
    rab_type = rng.normal(0.0, 0.5, size=NT * NT)
    return case, types, rab_type


def _akw(case):
    return dict(num_heads=case.num_heads, d_qk=case.d_qk, d_v=case.d_v,
                max_pos_dist=case.max_pos_dist, num_time_buckets=case.num_time_buckets,
                alpha=case.alpha, mask=case.mask, num_candidates=case.num_candidates)


def test_type_bias_explicit_pairwise_loop():
    """The type term inside the SiLU, against a pair-by-pair loop of the whole bias
    rab_pos + rab_time + rab_type[type_i NT + type_j]."""
    for mask, m in ((O.MASK_CAUSAL, 0), (O.MASK_MFALCON, 3)):
        case, types, rt = _typed_case(31, [9, 1, 12], 3, mask, m)
        got = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                  case.rab_pos, case.rab_time, token_types=types, rab_type=rt,
                                  num_types=3, **_akw(case))
        H, d, P, NB = 2, 8, 6, 8
        want = np.zeros_like(got)
        off = case.seq_offsets
        for b in range(len(off) - 1):
            s, e = int(off[b]), int(off[b + 1])
            L = e - s
            n = L - m if mask == O.MASK_MFALCON else L
            for i in range(L):
                for j in range(L):
                    vis = j <= i and (mask == O.MASK_CAUSAL or j < n or j == i)
                    if not vis:
                        continue
                    pi, pj = min(i, n), min(j, n)
                    dt = int(case.timestamps[s + i]) - int(case.timestamps[s + j])
                    bkt = min(max(max(dt, 1).bit_length() - 1, 0), NB - 1)
                    bias = (float(case.rab_pos[min(max(pi - pj, -P), P) + P])
                            + float(case.rab_time[bkt]) + float(rt[types[s + i] * 3 + types[s + j]]))
                    for h in range(H):
                        sc = float(np.dot(case.q[s + i, h * d:(h + 1) * d].astype(np.float64),
                                          case.k[s + j, h * d:(h + 1) * d].astype(np.float64)))
                        x = sc + bias
                        want[s + i, h * d:(h + 1) * d] += x / (1 + math.exp(-x)) * \
                            case.v[s + j, h * d:(h + 1) * d].astype(np.float64)
        assert np.allclose(got, want, rtol=1e-10, atol=1e-12)


def test_type_bias_single_type_is_a_constant_shift():
    """One token type: the type term is the constant rab_type[0] on every pair, the same as
    adding it to every position-table entry."""
    case, types, rt = _typed_case(32, [10, 7], 1)
    got = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, token_types=np.zeros_like(types),
                              rab_type=rt, num_types=1, **_akw(case))
    want = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                               case.rab_pos + rt[0], case.rab_time, **_akw(case))
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_type_bias_gradient_finite_differences():
    """d rab_type against central differences of Σ dO ⊙ out, and its total equal to the other
    two tables' totals (every visible pair has one index in each table)."""
    case, types, rt = _typed_case(33, [8, 5], 2)
    d_o = np.random.default_rng(4).standard_normal(case.q.shape)
    res = O.attention_backward(case.q, case.k, case.v, d_o, case.seq_offsets, case.timestamps,
                               case.rab_pos, case.rab_time, token_types=types, rab_type=rt,
                               num_types=2, **_akw(case))
    d_type = res[5]

    def loss(tab):
        o = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                case.rab_pos, case.rab_time, token_types=types, rab_type=tab,
                                num_types=2, **_akw(case))
        return float(np.sum(o * d_o))

    for c in range(4):
        e = np.zeros(4)
        e[c] = 1e-6
        fd = (loss(rt + e) - loss(rt - e)) / 2e-6
        assert abs(fd - d_type[c]) <= 1e-6 * max(1.0, abs(fd))
    assert abs(d_type.sum() - res[3].sum()) <= 1e-9 * max(1.0, abs(res[3].sum()))
    assert abs(d_type.sum() - res[4].sum()) <= 1e-9 * max(1.0, abs(res[4].sum()))


def test_bias_grad_entries_match_full_backward():
    # the pair-enumerating restatement of the bias-table gradient entries agrees with the full
    # backward (itself pinned by finite differences) on a small causal case whose timestamps
    # repeat and step by a few seconds, so that every selected bucket and offset is populated
    rng = np.random.default_rng(17)
    lengths = [37, 1, 90, 64]
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T, H, d, P, NB = int(off[-1]), 2, 8, 12, 10
    q, k, v, d_o = (rng.normal(0, 0.7, (T, H * d)) for _ in range(4))
    ts = np.concatenate([np.cumsum(rng.integers(0, 9, size=n)) for n in lengths]).astype(np.int64)
    rab_pos = rng.normal(0, 0.5, 2 * P + 1)
    rab_time = rng.normal(0, 0.5, NB)
    kw = dict(num_heads=H, d_qk=d, d_v=d, max_pos_dist=P, num_time_buckets=NB, alpha=0.6)
    full = O.attention_backward(q, k, v, d_o, off, ts, rab_pos, rab_time, **kw)
    dp, dt = O.bias_grad_entries(q, k, v, d_o, off, ts, rab_pos, rab_time, max_delta=7,
                                 max_bucket=4, **kw)
    assert np.abs(dt).min() > 0  # every selected bucket has pairs
    np.testing.assert_allclose(dp, full[3][P:P + 8], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dt, full[4][:5], rtol=1e-10, atol=1e-12)
