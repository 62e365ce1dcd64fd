"""GPU parity of the attention with the parameter-free bias of "6.2 HSTU的工程突破" §6.2.3,
Eq. (6.2.6), through the C ABI: the library's linear tables (hstu_alibi_tables, span P at least
the longest sequence) fed to the attention forward, against the oracle's direct formula.  Kept
in a file that runs after the main parity suite."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
from test_gpu_parity import B, assert_close, dev  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,mask,m", [(64, W.MASK_CAUSAL, 0), (128, W.MASK_CAUSAL, 0),
                                       (64, W.MASK_MFALCON, 30)])
def test_attention_forward_alibi_bias(B, d, mask, m):
    case = W.random_attention_case(23 + d + m, [300, 129, 41, 1], H=2, d=d, P=8, NB=32,
                                   mask=mask, num_candidates=m, gap_mean=600.0, qkv_std=0.5)
    m_p, m_t, NB = 0.01, 0.05, 32
    P = int(case.max_seq_len)
    pos, tim = B.alibi_tables(m_p, m_t, P, NB)
    bf = torch.bfloat16
    out = B.attention_forward(dev(case.q, bf), dev(case.k, bf), dev(case.v, bf),
                              dev(case.seq_offsets), case.max_seq_len, dev(case.timestamps),
                              dev(pos), dev(tim), num_heads=2, max_pos_dist=P,
                              num_time_buckets=NB, alpha=case.alpha, mask=mask,
                              num_candidates=m, microbatch=max(case.microbatch, 1))
    torch.cuda.synchronize()
    ref = O.attention_forward_alibi(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                    m_p, m_t, num_heads=2, d_qk=d, d_v=d, num_time_buckets=NB,
                                    alpha=case.alpha, mask=mask, num_candidates=m)
    assert_close(out, ref, f"alibi d={d} m={m}")


def test_attention_forward_alibi_bias_long_sequences(B):
    # tables spanning P = 2599 >= the longest sequence: too wide for the paired kernel's shared
    # copy, so the single-tile tensor-core forward reads the table from global memory
    case = W.random_attention_case(29, [2600, 700, 1], H=2, d=64, P=8, NB=32, gap_mean=600.0,
                                   qkv_std=0.5)
    m_p, m_t, NB = 0.002, 0.05, 32
    P = int(case.max_seq_len) - 1
    pos, tim = B.alibi_tables(m_p, m_t, P, NB)
    bf = torch.bfloat16
    out = B.attention_forward(dev(case.q, bf), dev(case.k, bf), dev(case.v, bf),
                              dev(case.seq_offsets), case.max_seq_len, dev(case.timestamps),
                              dev(pos), dev(tim), num_heads=2, max_pos_dist=P,
                              num_time_buckets=NB, alpha=case.alpha)
    torch.cuda.synchronize()
    ref = O.attention_forward_alibi(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                                    m_p, m_t, num_heads=2, d_qk=64, d_v=64, num_time_buckets=NB,
                                    alpha=case.alpha)
    assert_close(out, ref, "alibi long sequences")
