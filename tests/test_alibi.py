"""The parameter-free relative bias of "6.2 HSTU的工程突破" §6.2.3, Eq. (6.2.6), on the CPU:
the oracle's direct formula, the reading that it is the two-table bias with linear tables, and
the library's host table builder (hstu_alibi_tables)."""
import ctypes

import numpy as np
import pytest

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import binding as B
from hstu_sequential_transducer_jagged_b200 import build as BUILD
from hstu_sequential_transducer_jagged_b200 import workloads as W


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load_library()


def test_library_tables_are_the_linear_tables(lib):
    B._LIB = lib
    for m_p, m_t, P, NB in [(0.05, 0.02, 7, 16), (1.5e-3, -0.25, 1024, 128), (0.0, 0.0, 0, 1)]:
        pos, tim = B.alibi_tables(m_p, m_t, P, NB)
        k = np.arange(2 * P + 1)
        assert np.array_equal(pos, np.float32(-m_p) * (k - P).astype(np.float32))
        assert np.array_equal(tim, np.float32(-m_t) * np.arange(NB).astype(np.float32))


def test_library_tables_reject_bad_arguments(lib):
    buf = (ctypes.c_float * 64)()
    assert lib.hstu_alibi_tables(float("nan"), 0.0, 3, 4, buf, buf) == 1
    assert lib.hstu_alibi_tables(0.1, float("inf"), 3, 4, buf, buf) == 1
    assert lib.hstu_alibi_tables(0.1, 0.1, -1, 4, buf, buf) == 1
    assert lib.hstu_alibi_tables(0.1, 0.1, 3, 0, buf, buf) == 1
    # 2P would overflow int32 past 2^30: P is bounded by 2^24 (nothing is written)
    assert lib.hstu_alibi_tables(0.1, 0.1, 2 ** 31 - 1, 4, None, None) == 1
    assert lib.hstu_alibi_tables(0.1, 0.1, (1 << 24) + 1, 4, None, None) == 1
    assert lib.hstu_alibi_tables(0.1, 0.1, 3, 4, None, None) == 0


@pytest.mark.parametrize("mask,m", [(O.MASK_CAUSAL, 0), (O.MASK_MFALCON, 3)])
def test_alibi_is_the_table_bias_with_linear_tables(mask, m):
    """Eq. (6.2.6) is linear in the integer distance and in the bucket index, so it equals the
    learned-table bias with rab_pos[k] = -m_p (k - P) and rab_time[b] = -m_t b when no distance
    exceeds P: the direct formula and the table path agree (fp64)."""
    case = W.random_attention_case(21, [40, 1, 17], H=2, d=8, P=4, NB=16, mask=mask,
                                   num_candidates=m, gap_mean=50.0)
    m_p, m_t, P = 0.07, 0.11, 39
    direct = O.attention_forward_alibi(case.q, case.k, case.v, case.seq_offsets,
                                       case.timestamps, m_p, m_t, num_heads=2, d_qk=8, d_v=8,
                                       num_time_buckets=16, mask=mask, num_candidates=m)
    tabp = -m_p * (np.arange(2 * P + 1) - P)
    tabt = -m_t * np.arange(16)
    table = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                tabp, tabt, num_heads=2, d_qk=8, d_v=8, max_pos_dist=P,
                                num_time_buckets=16, mask=mask, num_candidates=m)
    assert np.allclose(direct, table, rtol=1e-12, atol=1e-12)
    # with a clamp shorter than the longest distance the table path differs
    short = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                -m_p * (np.arange(9) - 4), tabt, num_heads=2, d_qk=8, d_v=8,
                                max_pos_dist=4, num_time_buckets=16, mask=mask,
                                num_candidates=m)
    assert not np.allclose(direct, short)


def test_alibi_page_example_ordering():
    """The page's example: predicting the 8th interaction from 7, the 7th (distance 1, 5 minutes
    earlier) weighs most, the 5th (distance 3, one hour) less, the 1st (distance 7, one day)
    least.  Every key scores 2 against the query, so each weight is SiLU(2 + bias); one-hot
    values read the weights out."""
    L = 8
    t8 = 10 ** 6
    ts = np.full(L, t8 - 3 * 3600, dtype=np.int64)
    ts[0], ts[4], ts[6], ts[7] = t8 - 86400, t8 - 3600, t8 - 300, t8
    q = np.ones((L, 1))
    k = 2.0 * np.ones((L, 1))
    v = np.eye(L)
    out = O.attention_forward_alibi(q, k, v, np.array([0, L]), ts, 0.05, 0.02, num_heads=1,
                                    d_qk=1, d_v=L, num_time_buckets=32)
    w = out[L - 1]
    assert w[6] > w[4] > w[0] > 0

    def expect(dp, dt):  # buckets by hand: 2^8 <= 300 < 2^9, 2^11 <= 3600, 2^16 <= 86400
        b = {300: 8, 3600: 11, 86400: 16}[dt]
        return O.silu(np.array([2.0 - 0.05 * dp - 0.02 * b]))[0]

    assert np.isclose(w[6], expect(1, 300), rtol=1e-14)
    assert np.isclose(w[4], expect(3, 3600), rtol=1e-14)
    assert np.isclose(w[0], expect(7, 86400), rtol=1e-14)


def test_alibi_zero_slopes_is_no_bias():
    case = W.random_attention_case(22, [30, 9], H=1, d=8, P=4, NB=8)
    direct = O.attention_forward_alibi(case.q, case.k, case.v, case.seq_offsets,
                                       case.timestamps, 0.0, 0.0, num_heads=1, d_qk=8, d_v=8,
                                       num_time_buckets=8)
    plain = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, None, None, None,
                                num_heads=1, d_qk=8, d_v=8, max_pos_dist=0, num_time_buckets=1)
    assert np.allclose(direct, plain, rtol=1e-13, atol=1e-13)
