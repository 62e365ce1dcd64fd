"""The tensor-core backward's data movement, modelled on the CPU (tests/bwd_tc_model.py),
against the oracle's chain rule for the attention backward ("6.2 HSTU的工程突破" §6.2.3 names the
rab gradient it includes).

The model uses the kernel's own address arithmetic for every shared- and tensor-memory access
and the canonical operand layouts for what the MMAs read.  So it checks that each operand lands
where its reader expects it, for both epilogue forms (per element, and classified 32 x 32
blocks), before the kernel runs on hardware.  Each planted layout mistake must make it fail.
"""
import numpy as np
import pytest

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
import bwd_tc_model as M  # noqa: E402  (tests/ is on sys.path under pytest)

ROW_TOL, ABS_TOL, FRO_TOL = 2e-2, 1e-3, 5e-3


def within(got, ref, bf16_out):
    g = M.bits_to_f32(M.bf16_bits(got)) if bf16_out else got
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    bound = ROW_TOL * (np.abs(r).max(axis=-1, keepdims=True) if r.ndim > 1
                       else np.abs(r).max()) + ABS_TOL
    fro = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    return bool((np.abs(g - r) <= bound).all() and fro <= FRO_TOL)


def oracle(case):
    return O.attention_backward(case.q, case.k, case.v, case.d_o, case.seq_offsets,
                                case.timestamps, case.rab_pos, case.rab_time,
                                num_heads=case.num_heads, d_qk=case.d_qk, d_v=case.d_v,
                                max_pos_dist=case.max_pos_dist,
                                num_time_buckets=case.num_time_buckets, alpha=case.alpha,
                                mask=case.mask, num_candidates=case.num_candidates)


CASES = {
    "causal": lambda: W.random_attention_case(30, [200, 1, 129, 77], H=2, d=64, P=20, NB=16,
                                              gap_mean=20.0, qkv_std=0.5),
    "mfalcon": lambda: W.random_attention_case(80, [200, 1, 129, 77], H=2, d=64, P=20, NB=16,
                                               mask=W.MASK_MFALCON, num_candidates=50,
                                               gap_mean=20.0, qkv_std=0.5),
    "far pairs": lambda: W.random_attention_case(31, [700, 300], H=1, d=64, P=64, NB=32,
                                                 gap_mean=600.0, qkv_std=0.5),
}


@pytest.mark.parametrize("fast", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_model_matches_oracle(name, fast):
    case = CASES[name]()
    got = M.run(case, fast)
    ref = oracle(case)
    for nm, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time"), got, ref):
        assert within(g, r, nm in ("dq", "dk", "dv")), f"{name} fast={fast}: {nm}"


@pytest.mark.parametrize("knob", [dict(ds_swizzle=False), dict(dq_lbo=8192),
                                  dict(split_pc=False), dict(p_col_step=16)])
def test_planted_layout_mistakes_fail(knob):
    case = CASES["causal"]()
    with np.errstate(all="ignore"):  # misplaced operands read garbage
        got = M.run(case, True, knob)
    ref = oracle(case)
    with np.errstate(all="ignore"):
        assert not all(within(g, r, nm in ("dq", "dk", "dv"))
                       for nm, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time"), got,
                                           ref))


def test_block_classes_exact():
    """Brute force over random blocks: every pair of a constant block is visible and has the
    claimed position bin and time bucket; every pair of a zero block is hidden (causal and
    M-FALCON masks, sorted and shuffled timestamps, gaps from 1 s to 10^7 s)."""
    rng = np.random.default_rng(1)
    seen = set()
    for _ in range(400):
        L = int(rng.integers(1, 700))
        mfal = bool(rng.random() < 0.4)
        m = int(rng.integers(0, min(L, 200) + 1)) if mfal else 0
        mask = O.MASK_MFALCON if mfal else O.MASK_CAUSAL
        n = max(L - m, 0) if mfal else L
        P, NB = int(rng.choice([4, 20, 64, 300])), int(rng.choice([8, 16, 64]))
        ts = np.floor(np.cumsum(rng.exponential(float(rng.choice([1.0, 600.0, 1e7])), L)))
        ts = ts.astype(np.int64)
        if mfal and n > 0:
            ts[n:] = ts[n - 1]
        if rng.random() < 0.2:
            rng.shuffle(ts)
        ok = O.allowed_pairs(L, mask, m)
        pidx = O.position_index(O.positions(L, mask, m)[:, None] - O.positions(L, mask, m)[None, :], P)
        tidx = O.time_bucket(ts[:, None] - ts[None, :], NB)
        tpad = np.concatenate([ts, np.zeros(256, np.int64)])
        tabp, tabt = np.zeros(2 * P + 1, np.float32), np.zeros(NB, np.float32)
        nt = (L + 127) // 128
        for _ in range(4):
            kt = int(rng.integers(0, nt))
            qt = int(rng.integers(kt, nt))
            i0 = qt * 128 + int(rng.choice([0, 32, 64, 96]))
            j0 = kt * 128 + 32 * int(rng.integers(0, 4))
            jrow = j0 + np.arange(32)
            cls, _, cp, ct = M.chunk_class(i0, j0, L, n, P, NB, tpad[i0:i0 + 32],
                                           tpad[np.minimum(jrow, len(tpad) - 1)], jrow < L,
                                           tabp, tabt)
            seen.add(cls)
            ii, jj = np.meshgrid(np.arange(i0, i0 + 32), jrow, indexing="ij")
            inside = (ii < L) & (jj < L)
            vis = np.zeros_like(inside)
            vis[inside] = ok[ii[inside], jj[inside]]
            if cls == "zero":
                assert not vis.any()
            elif cls in ("const", "timeconst"):
                assert vis.all()
                assert (tidx[ii, jj] == ct).all()
                if cls == "const":
                    assert (pidx[ii, jj] == cp).all()
    assert seen == {"zero", "general", "const", "timeconst"}


# ------------------------------------------------------------ diagonal position-bin sums
def diag_bins_by_shuffle(v, src_offset=-1):
    """The band blocks' position-bin sums as the kernel forms them (DiagBins in attn_bwd_tc.cu):
    lane m keeps diagonals m (lo) and m + 32 (hi); at block column e it takes the value of lane
    (e + src_offset - m) mod 32 from the warp shuffle and adds it to lo when m >= e, else to hi.
    v[l, e] is the dS of key row l (lane) and block column e.  Returns the 63 diagonal sums,
    diagonal k = e - l + 31."""
    lo = np.zeros(32)
    hi = np.zeros(32)
    lanes = np.arange(32)
    for e in range(v.shape[1]):
        src = (e + src_offset - lanes) & 31
        w = v[src, e]
        lo += np.where(lanes >= e, w, 0.0)
        hi += np.where(lanes >= e, 0.0, w)
    return np.concatenate([lo, hi[:31]])


@pytest.mark.parametrize("width", [16, 32])
def test_diag_bins_shuffle_mapping(width):
    """Brute force: every pair (l, e) lands on diagonal e - l + 31; the kernel's mapping gives
    the same 63 sums for a full block and for the first 16 columns (one half)."""
    rng = np.random.default_rng(7 + width)
    v = rng.standard_normal((32, width))
    ref = np.zeros(63)
    for l in range(32):
        for e in range(width):
            ref[e - l + 31] += v[l, e]
    np.testing.assert_allclose(diag_bins_by_shuffle(v), ref, rtol=0, atol=1e-12)
    # the planted mistake: a source lane off by one must not reproduce the sums
    assert not np.allclose(diag_bins_by_shuffle(v, src_offset=0), ref)
