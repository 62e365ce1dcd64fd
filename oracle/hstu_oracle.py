"""fp64 CPU oracle for the HSTU jagged layer, attention forward and attention backward.

TEST INFRASTRUCTURE ONLY.  This module is the slow, literal statement of what the CUDA library
computes.  Only the tests, the graft entry's smoke check and the benchmark's CPU-baseline leg may
import it; the library never calls it and shares no code with it.

Sources (web pages on HSTU; cited by page title and section):

* [FunRec 7.1] "HSTU：Scaling Law 的首次探索" (fun-rec mdbook, part 7):
  §7.1.4 innovation 1 (pointwise aggregation with SiLU instead of softmax, gated output
  LayerNorm(A(X)V(X)) ⊙ U(X)), innovation 2 (relative bias from position and time differences),
  §7.1.5 M-FALCON (candidates attend to the history but not to one another; microbatches of
  b_m candidates; history K/V reused across microbatches).
* [Review §2.1] "万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" (paper review),
  §2.1: U,V,Q,K = Split(φ1(f1(X))); A(X)V(X) = φ2(Q Kᵀ + rab) V; Y = f2(Norm(AV) ⊙ U);
  f1, f2 single linear layers, φ1, φ2 SiLU; the block diagram's residual edge from input to output.
* [Explainer] "从自注意力到 HSTU：解构下一代推荐系统引擎", part 2, steps 1-3 (same three formulas).
* [GenRank §6.2.2-6.2.3] "6.2 HSTU的工程突破": the candidate mask (history causal, candidates
  see all history, not each other) and the relative-bias score of Eq. (6.2.3), whose backward pass
  needs the gradient of the N×N bias.

Readings where the pages are silent or garbled (each is restated in the design notes):

* score scale alpha = 1 by default (the HSTU formulas carry no 1/sqrt(d)); causal mask includes
  the diagonal (j <= i);
* rab_{p,t}(i, j) = rab_pos[clamp(p_i - p_j, -P, P) + P] + rab_time[bucket(t_i - t_j)], shared by
  all heads, with bucket(dt) = clamp(floor(log2(max(1, dt))), 0, NB - 1) computed on integers;
* M-FALCON candidates all sit at the position index n (the history length), so a candidate's
  pairs with history use p_i - p_j = n - j and its self pair uses 0; its timestamp is an input;
* LayerNorm over the H*d_v features of a token, biased variance, eps = 1e-5, optional affine;
* the split order is [U | V | Q | K], head-major inside each block; f1/f2 biases optional.

Every function computes in float64 from the given (already bf16-rounded) input values.
"""
from __future__ import annotations

import numpy as np

MASK_CAUSAL = 0
MASK_MFALCON = 1


# --------------------------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------------------------

def sigmoid(x):
    """σ(x) = 1 / (1 + e^{-x}), evaluated without overflow for either sign of x."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def silu(x):
    """φ(x) = x·σ(x): the SiLU used for both φ1 and φ2 ([Review §2.1])."""
    x = np.asarray(x, dtype=np.float64)
    return x * sigmoid(x)


def silu_grad(x):
    """dφ/dx = σ(x)·(1 + x·(1 - σ(x)))."""
    x = np.asarray(x, dtype=np.float64)
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


# --------------------------------------------------------------------------------------------
# relative attention bias indices ([FunRec 7.1] §7.1.4 innovation 2; [GenRank §6.2.3])
# --------------------------------------------------------------------------------------------

def time_bucket(dt, num_buckets: int):
    """bucket(dt) = clamp(floor(log2(max(1, dt))), 0, NB-1), exactly, on integers.

    floor(log2(d)) for an integer d >= 1 is the number of k >= 1 with 2^k <= d; it is counted
    with integer comparisons only, so no floating-point rounding can move a bucket edge.
    """
    d = np.maximum(np.asarray(dt, dtype=np.int64), 1)
    b = np.zeros(d.shape, dtype=np.int64)
    for k in range(1, 63):
        b += (d >= (np.int64(1) << np.int64(k))).astype(np.int64)
    return np.minimum(b, num_buckets - 1)


def positions(L: int, mask: int, num_candidates: int):
    """Position index of every token: k for history tokens; n (history length) for candidates."""
    n = L - num_candidates if mask == MASK_MFALCON else L
    p = np.arange(L, dtype=np.int64)
    return np.minimum(p, n)


def position_index(dp, max_pos_dist: int):
    """Table index clamp(dp, -P, P) + P of the position bias."""
    return np.clip(np.asarray(dp, dtype=np.int64), -max_pos_dist, max_pos_dist) + max_pos_dist


def allowed_pairs(L: int, mask: int, num_candidates: int):
    """Boolean [L, L]: token i attends to token j.

    Causal: j <= i.  M-FALCON ([FunRec 7.1] §7.1.5 batched inference; [GenRank §6.2.2]):
    history tokens are causal among themselves; a candidate sees every history token and itself.
    """
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    causal = j <= i
    if mask == MASK_CAUSAL:
        return causal
    n = L - num_candidates
    return causal & ((j < n) | (j == i))


def type_bias_matrix(rows, types, rab_type, num_types):
    """The token-type term of bias_{i,j} = f(p_i - p_j, t_i - t_j, type_i, type_j) ([FunRec 7.1]
    §7.1.4 innovation 2: content and action tokens relate differently).  Reading: a learned
    table over (type_i, type_j) pairs, rab_type[type_i * NT + type_j], added to the position and
    time terms.  types: int [L] of one sequence, values in [0, NT)."""
    types = np.asarray(types, dtype=np.int64)
    idx = types[np.asarray(rows, dtype=np.int64)][:, None] * num_types + types[None, :]
    return np.asarray(rab_type, dtype=np.float64)[idx]


def bias_matrix(rows, L, ts, rab_pos, rab_time, max_pos_dist, num_buckets, mask, num_candidates):
    """rab_{p,t}(i, j) for the given query rows i and all keys j of one sequence (fp64)."""
    p = positions(L, mask, num_candidates)
    dp = p[rows][:, None] - p[None, :]
    out = np.zeros((len(rows), L), dtype=np.float64)
    if rab_pos is not None:
        out += np.asarray(rab_pos, dtype=np.float64)[position_index(dp, max_pos_dist)]
    if rab_time is not None and ts is not None:
        ts = np.asarray(ts, dtype=np.int64)
        dt = ts[rows][:, None] - ts[None, :]
        out += np.asarray(rab_time, dtype=np.float64)[time_bucket(dt, num_buckets)]
    return out


# --------------------------------------------------------------------------------------------
# attention: A(X)V(X) = φ2(α Q Kᵀ + rab) V per head, masked pairs contribute exactly zero
# ([Review §2.1] second formula; [FunRec 7.1] §7.1.4 innovation 1; [Explainer] step 2)
# --------------------------------------------------------------------------------------------

def _heads(a, H, d):
    return np.asarray(a, dtype=np.float64).reshape(a.shape[0], H, d)


def attention_forward(q, k, v, seq_offsets, timestamps, rab_pos, rab_time, *, num_heads,
                      d_qk, d_v, max_pos_dist, num_time_buckets, alpha=1.0,
                      mask=MASK_CAUSAL, num_candidates=0, rows=None, token_types=None,
                      rab_type=None, num_types=0):
    """Jagged pointwise attention.  q,k: [T, H*d_qk], v: [T, H*d_v] -> out [T, H*d_v] (fp64).

    If ``rows`` is given (global token indices), only those output rows are computed (others 0).
    With token_types [T] and rab_type [NT*NT] the bias also carries the type term
    (type_bias_matrix).
    """
    H = num_heads
    T = int(seq_offsets[-1])
    Q, K, V = _heads(q, H, d_qk), _heads(k, H, d_qk), _heads(v, H, d_v)
    out = np.zeros((T, H, d_v), dtype=np.float64)
    want = None if rows is None else np.zeros(T, dtype=bool)
    if want is not None:
        want[np.asarray(rows, dtype=np.int64)] = True
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = e - s
        if L == 0:
            continue
        local = np.arange(L) if want is None else np.nonzero(want[s:e])[0]
        if local.size == 0:
            continue
        ts = None if timestamps is None else np.asarray(timestamps[s:e], dtype=np.int64)
        ok = allowed_pairs(L, mask, num_candidates)[local]
        for blk in range(0, local.size, 512):
            r = local[blk:blk + 512]
            okb = ok[blk:blk + 512]
            bias = bias_matrix(r, L, ts, rab_pos, rab_time, max_pos_dist, num_time_buckets,
                               mask, num_candidates)
            if rab_type is not None:
                bias = bias + type_bias_matrix(r, token_types[s:e], rab_type, num_types)
            for h in range(H):
                scores = alpha * (Q[s + r, h, :] @ K[s:e, h, :].T) + bias
                a = np.where(okb, silu(scores), 0.0)
                out[s + r, h, :] = a @ V[s:e, h, :]
    return out.reshape(T, H * d_v)


def attention_forward_mfalcon_microbatched(q, k, v, seq_offsets, timestamps, rab_pos, rab_time,
                                           *, num_heads, d_qk, d_v, max_pos_dist,
                                           num_time_buckets, num_candidates, microbatch,
                                           alpha=1.0):
    """M-FALCON as the pages lay it out ([FunRec 7.1] §7.1.5): the m candidates of a request
    are scored ⌈m/b_m⌉ microbatches at a time; each microbatch is one forward over
    [history, that microbatch's candidates] with the candidate mask, and reuses the history
    keys/values (they do not depend on the candidates).  History outputs come from the first
    microbatch.  The result must not depend on b_m.
    """
    H = num_heads
    T = int(seq_offsets[-1])
    out = np.zeros((T, H * d_v), dtype=np.float64)
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = e - s
        m = num_candidates
        n = L - m
        first = True
        for c0 in range(0, max(m, 1), microbatch):
            c1 = min(c0 + microbatch, m)
            idx = np.concatenate([np.arange(s, s + n), np.arange(s + n + c0, s + n + c1)])
            sub_off = np.array([0, idx.size], dtype=np.int64)
            ts = None if timestamps is None else np.asarray(timestamps)[idx]
            o = attention_forward(np.asarray(q)[idx], np.asarray(k)[idx], np.asarray(v)[idx],
                                  sub_off, ts, rab_pos, rab_time, num_heads=H, d_qk=d_qk,
                                  d_v=d_v, max_pos_dist=max_pos_dist,
                                  num_time_buckets=num_time_buckets, alpha=alpha,
                                  mask=MASK_MFALCON, num_candidates=c1 - c0)
            if first:
                out[s:s + n] = o[:n]
                first = False
            out[s + n + c0:s + n + c1] = o[n:]
            if m == 0:
                break
    return out


def attention_backward(q, k, v, d_o, seq_offsets, timestamps, rab_pos, rab_time, *, num_heads,
                       d_qk, d_v, max_pos_dist, num_time_buckets, alpha=1.0, mask=MASK_CAUSAL,
                       num_candidates=0, token_types=None, rab_type=None, num_types=0):
    """Gradients of L = Σ dO ⊙ out through the pointwise attention (chain rule, fp64).

    With S = α QKᵀ + rab, A = φ2(S) on allowed pairs (0 elsewhere), out = A V:
      dV = Aᵀ dO;  dA = dO Vᵀ;  dS = dA ⊙ φ2'(S) on allowed pairs;
      dQ = α dS K;  dK = α dSᵀ Q;
      d rab_pos[k]  = Σ over allowed pairs with position index k of dS (all heads, all sequences);
      d rab_time[b] = Σ over allowed pairs with time bucket b of dS.
    The bias backward is the N×N rab gradient that [GenRank §6.2.3] names as RAB's cost.
    With the type term (rab_type given) a sixth result d rab_type[a NT + b] = Σ over allowed
    pairs with type_i = a, type_j = b of dS is returned.
    """
    H = num_heads
    T = int(seq_offsets[-1])
    Q, K, V = _heads(q, H, d_qk), _heads(k, H, d_qk), _heads(v, H, d_v)
    dO = _heads(d_o, H, d_v)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    d_pos = np.zeros(2 * max_pos_dist + 1, dtype=np.float64)
    d_time = np.zeros(num_time_buckets, dtype=np.float64)
    d_type = None if rab_type is None else np.zeros(num_types * num_types, dtype=np.float64)
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = e - s
        if L == 0:
            continue
        ts = None if timestamps is None else np.asarray(timestamps[s:e], dtype=np.int64)
        rows = np.arange(L)
        ok = allowed_pairs(L, mask, num_candidates)
        bias = bias_matrix(rows, L, ts, rab_pos, rab_time, max_pos_dist, num_time_buckets,
                           mask, num_candidates)
        yidx = None
        if rab_type is not None:
            bias = bias + type_bias_matrix(rows, token_types[s:e], rab_type, num_types)
            ty = np.asarray(token_types[s:e], dtype=np.int64)
            yidx = ty[:, None] * num_types + ty[None, :]
        p = positions(L, mask, num_candidates)
        pidx = position_index(p[:, None] - p[None, :], max_pos_dist)
        tidx = None
        if ts is not None:
            tidx = time_bucket(ts[:, None] - ts[None, :], num_time_buckets)
        for h in range(H):
            S = alpha * (Q[s:e, h] @ K[s:e, h].T) + bias
            A = np.where(ok, silu(S), 0.0)
            dV[s:e, h] = A.T @ dO[s:e, h]
            dA = dO[s:e, h] @ V[s:e, h].T
            dS = np.where(ok, dA * silu_grad(S), 0.0)
            dQ[s:e, h] = alpha * (dS @ K[s:e, h])
            dK[s:e, h] = alpha * (dS.T @ Q[s:e, h])
            if rab_pos is not None:
                d_pos += np.bincount(pidx[ok], weights=dS[ok], minlength=d_pos.size)
            if tidx is not None and rab_time is not None:
                d_time += np.bincount(tidx[ok], weights=dS[ok], minlength=d_time.size)
            if yidx is not None:
                d_type += np.bincount(yidx[ok], weights=dS[ok], minlength=d_type.size)
    out = (dQ.reshape(T, H * d_qk), dK.reshape(T, H * d_qk), dV.reshape(T, H * d_v), d_pos,
           d_time)
    return out if d_type is None else out + (d_type,)


def bias_grad_entries(q, k, v, d_o, seq_offsets, timestamps, rab_pos, rab_time, *, num_heads,
                      d_qk, d_v, max_pos_dist, num_time_buckets, alpha=1.0, max_delta=31,
                      max_bucket=5):
    """Selected entries of the causal attention's bias-table gradients, exactly as
    attention_backward defines them, by enumerating only the pairs that reach those entries.

    Returns (d_rab_pos[P .. P + max_delta], d_rab_time[0 .. max_bucket]) (fp64).
      * position entry P + Δ (Δ < P, so not clamped) collects the pairs (i, i - Δ);
      * time bucket b <= max_bucket collects the pairs with ts_i - ts_j < 2^(max_bucket + 1)
        (bucket(dt) <= max_bucket exactly there), found per row by a search over the
        sequence's non-decreasing timestamps.
    Each pair contributes dS = (dO_i · V_j) φ2'(α q_i·k_j + rab) summed over heads, as in
    attention_backward (causal mask, no type term).
    """
    H, P = num_heads, max_pos_dist
    assert 0 <= max_delta < P and 0 <= max_bucket < num_time_buckets - 1
    Q, K, V = _heads(q, H, d_qk), _heads(k, H, d_qk), _heads(v, H, d_v)
    dO = _heads(d_o, H, d_v)
    d_pos = np.zeros(max_delta + 1, dtype=np.float64)
    d_time = np.zeros(max_bucket + 1, dtype=np.float64)
    rp = np.asarray(rab_pos, dtype=np.float64)
    rt = np.asarray(rab_time, dtype=np.float64)

    def d_s(s, I, J):
        """dS of the pairs (s + I, s + J) summed over heads."""
        dt = np.asarray(timestamps[s + I], dtype=np.int64) - np.asarray(timestamps[s + J],
                                                                         dtype=np.int64)
        bias = rp[position_index(I - J, P)] + rt[time_bucket(dt, num_time_buckets)]
        sc = alpha * np.einsum("phd,phd->ph", Q[s + I], K[s + J]) + bias[:, None]
        da = np.einsum("phd,phd->ph", dO[s + I], V[s + J])
        return (da * silu_grad(sc)).sum(axis=1), dt

    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = e - s
        if L == 0:
            continue
        ts = np.asarray(timestamps[s:e], dtype=np.int64)
        assert np.all(np.diff(ts) >= 0), "timestamps must not decrease within a sequence"
        for delta in range(min(max_delta, L - 1) + 1):
            I = np.arange(delta, L)
            ds, _ = d_s(s, I, I - delta)
            d_pos[delta] += ds.sum()
        # rows i and the first key j with ts_i - ts_j < 2^(max_bucket + 1)
        lim = np.int64(1) << np.int64(max_bucket + 1)
        first = np.searchsorted(ts, ts - lim, side="right")
        counts = np.arange(L) - first + 1
        I = np.repeat(np.arange(L), counts)
        J = np.concatenate([np.arange(f, i + 1) for i, f in enumerate(first)]) if L else I
        ds, dt = d_s(s, I, J)
        bk = time_bucket(dt, num_time_buckets)
        d_time += np.bincount(bk, weights=ds, minlength=max_bucket + 1)[:max_bucket + 1]
    return d_pos, d_time


# --------------------------------------------------------------------------------------------
# the layer: U,V,Q,K = Split(φ1(f1(X)));  Y = X + f2(Norm(A(X)V(X)) ⊙ U(X))
# ([Review §2.1] first and third formula + the block diagram's residual edge;
#  [FunRec 7.1] §7.1.4 innovation 1 output formula; [Explainer] steps 1 and 3)
# --------------------------------------------------------------------------------------------

def linear(x, w, b=None):
    """f(x) = x W (+ b): a single linear layer."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64)
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)
    return y


def split_uvqk(z, num_heads, d_qk, d_v):
    """Split the f1 output columns as [U | V | Q | K]."""
    hv, hq = num_heads * d_v, num_heads * d_qk
    return z[:, :hv], z[:, hv:2 * hv], z[:, 2 * hv:2 * hv + hq], z[:, 2 * hv + hq:2 * hv + 2 * hq]


def layer_norm(a, eps=1e-5, gamma=None, beta=None):
    """Norm(a) over the last axis: (a - mean) / sqrt(var + eps), biased variance, then affine."""
    a = np.asarray(a, dtype=np.float64)
    mu = a.mean(axis=-1, keepdims=True)
    var = ((a - mu) ** 2).mean(axis=-1, keepdims=True)
    out = (a - mu) / np.sqrt(var + eps)
    if gamma is not None:
        out = out * np.asarray(gamma, dtype=np.float64)
    if beta is not None:
        out = out + np.asarray(beta, dtype=np.float64)
    return out


def layer_forward(x, w1, w2, seq_offsets, timestamps, rab_pos, rab_time, *, num_heads, d_qk,
                  d_v, max_pos_dist, num_time_buckets, alpha=1.0, mask=MASK_CAUSAL,
                  num_candidates=0, b1=None, b2=None, ln_eps=1e-5, ln_gamma=None,
                  ln_beta=None, return_intermediates=False, token_types=None, rab_type=None,
                  num_types=0):
    z = silu(linear(x, w1, b1))                                        # φ1(f1(X))
    u, v, q, k = split_uvqk(z, num_heads, d_qk, d_v)                   # Split
    av = attention_forward(q, k, v, seq_offsets, timestamps, rab_pos, rab_time,
                           num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_pos_dist=max_pos_dist,
                           num_time_buckets=num_time_buckets, alpha=alpha, mask=mask,
                           num_candidates=num_candidates, token_types=token_types,
                           rab_type=rab_type, num_types=num_types)     # A(X)V(X)
    g = layer_norm(av, ln_eps, ln_gamma, ln_beta) * u                  # Norm(AV) ⊙ U
    y = np.asarray(x, dtype=np.float64) + linear(g, w2, b2)            # X + f2(·)
    if return_intermediates:
        return y, dict(z=z, u=u, v=v, q=q, k=k, av=av, g=g)
    return y


def layer_forward_rows(x, w1, w2, seq_offsets, timestamps, rab_pos, rab_time, rows, *,
                       num_heads, d_qk, d_v, max_pos_dist, num_time_buckets, alpha=1.0,
                       mask=MASK_CAUSAL, num_candidates=0, b1=None, b2=None, ln_eps=1e-5,
                       ln_gamma=None, ln_beta=None):
    """One layer evaluated only at the given output rows (same arithmetic as layer_forward).

    An output row needs U, Q of that row and K, V of every token its sequence can attend to, so
    K and V are formed for the sequences that contain the requested rows.
    """
    rows = np.asarray(rows, dtype=np.int64)
    x = np.asarray(x)
    T = int(seq_offsets[-1])
    need = np.zeros(T, dtype=bool)
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        if np.any((rows >= s) & (rows < e)):
            need[s:e] = True
    z = np.zeros((T, w1.shape[1]), dtype=np.float64)
    z[need] = silu(linear(x[need], w1, b1))
    u, v, q, k = split_uvqk(z, num_heads, d_qk, d_v)
    av = attention_forward(q, k, v, seq_offsets, timestamps, rab_pos, rab_time,
                           num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_pos_dist=max_pos_dist,
                           num_time_buckets=num_time_buckets, alpha=alpha, mask=mask,
                           num_candidates=num_candidates, rows=rows)
    g = layer_norm(av[rows], ln_eps, ln_gamma, ln_beta) * u[rows]
    return np.asarray(x[rows], dtype=np.float64) + linear(g, w2, b2)


def stack_forward(x, layers, seq_offsets, timestamps, *, num_heads, d_qk, d_v, max_pos_dist,
                  num_time_buckets, alpha=1.0, mask=MASK_CAUSAL, num_candidates=0,
                  ln_eps=1e-5, round_between=None):
    """L identical-shape layers applied in sequence ([FunRec 7.1] §7.1.6: depth up to 24).

    ``layers`` holds objects with w1, w2, rab_pos, rab_time (b1, b2 optional).  If
    ``round_between`` is given, it is applied to each layer's output before the next layer
    (e.g. rounding to the storage precision of the activations).
    """
    h = np.asarray(x, dtype=np.float64)
    for lp in layers:
        h = layer_forward(h, lp.w1, lp.w2, seq_offsets, timestamps, lp.rab_pos, lp.rab_time,
                          num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_pos_dist=max_pos_dist,
                          num_time_buckets=num_time_buckets, alpha=alpha, mask=mask,
                          num_candidates=num_candidates, b1=getattr(lp, "b1", None),
                          b2=getattr(lp, "b2", None), ln_eps=ln_eps)
        if round_between is not None:
            h = np.asarray(round_between(h), dtype=np.float64)
    return h


# --------------------------------------------------------------------------------------------
# the layer's backward, for training the stack end to end ([FunRec 7.1] §7.1.3: the whole
# user sequence is trained in one causal pass; [Review §2.1] the three layer formulas): the
# chain rule through Y = X + f2(Norm(A(X)V(X)) ⊙ U(X)), written out step by step in fp64
# --------------------------------------------------------------------------------------------

def layer_norm_backward(a, d_out, eps=1e-5, gamma=None):
    """Gradient of Σ d_out ⊙ Norm(a) with respect to a, gamma and beta (last axis normalised).

    With n = (a - mean) / sqrt(var + eps) and out = n ⊙ gamma + beta: dn = d_out ⊙ gamma;
    da = (dn - mean(dn) - n ⊙ mean(dn ⊙ n)) / sqrt(var + eps); dgamma = Σ_rows d_out ⊙ n;
    dbeta = Σ_rows d_out.
    """
    a = np.asarray(a, dtype=np.float64)
    d_out = np.asarray(d_out, dtype=np.float64)
    mu = a.mean(axis=-1, keepdims=True)
    xc = a - mu
    rstd = 1.0 / np.sqrt((xc ** 2).mean(axis=-1, keepdims=True) + eps)
    n = xc * rstd
    dn = d_out if gamma is None else d_out * np.asarray(gamma, dtype=np.float64)
    da = rstd * (dn - dn.mean(axis=-1, keepdims=True) - n * (dn * n).mean(axis=-1, keepdims=True))
    return da, (d_out * n).sum(axis=0), d_out.sum(axis=0)


def layer_backward(x, w1, w2, seq_offsets, timestamps, rab_pos, rab_time, d_y, *, num_heads,
                   d_qk, d_v, max_pos_dist, num_time_buckets, alpha=1.0, mask=MASK_CAUSAL,
                   num_candidates=0, b1=None, b2=None, ln_eps=1e-5, ln_gamma=None,
                   ln_beta=None):
    """Gradients of L = Σ d_y ⊙ Y for one layer, Y = layer_forward(...).

    Forward: pre = X W1 + b1, Z = SiLU(pre) = [U | V | Q | K], AV = A(X)V(X),
    G = Norm(AV) ⊙ U, Y = X + G W2 + b2.  Backward, in reverse order:
      dW2 = Gᵀ dY, db2 = Σ dY, dG = dY W2ᵀ;
      dU = dG ⊙ Norm(AV), dNorm = dG ⊙ U, (dAV, dgamma, dbeta) = Norm backward;
      (dQ, dK, dV, d rab_pos, d rab_time) = attention backward of dAV;
      dZ = [dU | dV | dQ | dK], dpre = dZ ⊙ SiLU'(pre);
      dW1 = Xᵀ dpre, db1 = Σ dpre, dX = dY (residual edge) + dpre W1ᵀ.
    Returns a dict with dx, dw1, db1, dw2, db2, d_rab_pos, d_rab_time, d_ln_gamma, d_ln_beta.
    """
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    dy = np.asarray(d_y, dtype=np.float64)
    pre = linear(x, w1, b1)
    z = silu(pre)
    u, v, q, k = split_uvqk(z, num_heads, d_qk, d_v)
    av = attention_forward(q, k, v, seq_offsets, timestamps, rab_pos, rab_time,
                           num_heads=num_heads, d_qk=d_qk, d_v=d_v, max_pos_dist=max_pos_dist,
                           num_time_buckets=num_time_buckets, alpha=alpha, mask=mask,
                           num_candidates=num_candidates)
    nrm = layer_norm(av, ln_eps, ln_gamma, ln_beta)
    g = nrm * u
    dw2 = g.T @ dy
    db2 = dy.sum(axis=0)
    dg = dy @ w2.T
    du = dg * nrm
    d_av, d_gamma, d_beta = layer_norm_backward(av, dg * u, ln_eps, ln_gamma)
    dq, dk, dv, d_pos, d_time = attention_backward(
        q, k, v, d_av, seq_offsets, timestamps, rab_pos, rab_time, num_heads=num_heads,
        d_qk=d_qk, d_v=d_v, max_pos_dist=max_pos_dist, num_time_buckets=num_time_buckets,
        alpha=alpha, mask=mask, num_candidates=num_candidates)
    dz = np.concatenate([du, dv, dq, dk], axis=1)
    dpre = dz * silu_grad(pre)
    return dict(dx=dy + dpre @ w1.T, dw1=x.T @ dpre, db1=dpre.sum(axis=0), dw2=dw2, db2=db2,
                d_rab_pos=d_pos, d_rab_time=d_time, d_ln_gamma=d_gamma, d_ln_beta=d_beta)


# --------------------------------------------------------------------------------------------
# the parameter-free relative bias of [GenRank §6.2.3], Eq. (6.2.6), in place of the learned
# tables: bias_{i,j} = -m_p (p_i - p_j) - m_t bucket(t_i - t_j)  (ALiBi extended to time)
# --------------------------------------------------------------------------------------------

def alibi_bias_matrix(rows, L, ts, m_p, m_t, num_buckets, mask, num_candidates):
    """Eq. (6.2.6) for the given query rows and all keys of one sequence (fp64), with the same
    positions (candidates at n) and the same time-bucket rule as the learned-table bias."""
    p = positions(L, mask, num_candidates)
    out = -float(m_p) * (p[rows][:, None] - p[None, :]).astype(np.float64)
    if ts is not None:
        ts = np.asarray(ts, dtype=np.int64)
        out -= float(m_t) * time_bucket(ts[rows][:, None] - ts[None, :], num_buckets)
    return out


def attention_forward_alibi(q, k, v, seq_offsets, timestamps, m_p, m_t, *, num_heads, d_qk,
                            d_v, num_time_buckets, alpha=1.0, mask=MASK_CAUSAL,
                            num_candidates=0):
    """The pointwise attention with Eq. (6.2.6)'s bias inside the SiLU:
    out_i = Σ_{j allowed} SiLU(alpha <q_i, k_j> + bias_{i,j}) v_j, per head (fp64)."""
    H = num_heads
    T = int(seq_offsets[-1])
    Q, K, V = _heads(q, H, d_qk), _heads(k, H, d_qk), _heads(v, H, d_v)
    out = np.zeros((T, H, d_v), dtype=np.float64)
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = e - s
        if L == 0:
            continue
        rows = np.arange(L)
        ts = None if timestamps is None else np.asarray(timestamps[s:e], dtype=np.int64)
        ok = allowed_pairs(L, mask, num_candidates)
        bias = alibi_bias_matrix(rows, L, ts, m_p, m_t, num_time_buckets, mask, num_candidates)
        for h in range(H):
            scores = alpha * (Q[s:e, h, :] @ K[s:e, h, :].T) + bias
            out[s:e, h, :] = np.where(ok, silu(scores), 0.0) @ V[s:e, h, :]
    return out.reshape(T, H * d_v)


# --------------------------------------------------------------------------------------------
# Stochastic Length ([FunRec 7.1] §7.1.5): long sequences are, at random, replaced by a shorter
# subsequence during training.  The page's formula is garbled; the reading used here:
#   a sequence of length n is left whole when n <= N^{α/2}; otherwise, with probability
#   p = 1 - N^α / n², it is replaced by a subsequence of N^{α/2} of its tokens (keeping their
#   order), and with probability 1 - p it is left whole.  N is the longest sequence length the
#   data allows, α in (1, 2] (α = 2: never truncated).  The page selects the subsequence "by
#   feature weighting" without saying how; the plainest reading, a uniformly random subset, is
#   taken: the N^{α/2} tokens with the smallest random keys (ties broken by the lower index).
# The random draws are inputs: u[b] (uniform on [0, 1)) decides per sequence, key[t] (uint32)
# orders the tokens.  sub_len = floor(N^{α/2}) and n_alpha = N^α are passed as numbers, so that
# the decision u < 1 - n_alpha / n² is taken in fp64 from the same operands on every side.
# --------------------------------------------------------------------------------------------

def stochastic_length_params(max_len_N: int, alpha: float):
    """(sub_len, n_alpha) = (floor(N^{α/2}), N^α) for the longest length N and exponent α."""
    return int(np.floor(float(max_len_N) ** (alpha / 2.0))), float(max_len_N) ** alpha


def stochastic_length(seq_offsets, u, keys, sub_len: int, n_alpha: float):
    """Per sequence: whole, or the sub_len tokens with the smallest (key, index), in index order.

    Returns (new_offsets int64 [B+1], kept int64 [T']): kept lists the global index of every
    token that stays, sequence by sequence, in increasing order; new_offsets delimits them.
    """
    seq_offsets = np.asarray(seq_offsets, dtype=np.int64)
    keys = np.asarray(keys, dtype=np.uint32)
    u = np.asarray(u, dtype=np.float32)
    new_off = [0]
    kept = []
    for b in range(len(seq_offsets) - 1):
        s, e = int(seq_offsets[b]), int(seq_offsets[b + 1])
        n = e - s
        idx = np.arange(s, e, dtype=np.int64)
        p = 1.0 - float(n_alpha) / (float(n) * float(n)) if n > 0 else 0.0
        if n > sub_len and float(u[b]) < p:
            # sort by (key, index) and keep the first sub_len, then restore the index order
            order = np.lexsort((idx, keys[s:e].astype(np.int64)))
            idx = np.sort(idx[order[:sub_len]])
        kept.append(idx)
        new_off.append(new_off[-1] + len(idx))
    kept = np.concatenate(kept) if kept else np.zeros(0, np.int64)
    return np.array(new_off, dtype=np.int64), kept
