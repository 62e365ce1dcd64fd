"""GPU-vs-oracle parity of the attention forward for timestamps in epoch milliseconds (through
the C ABI; needs a B200).  Sequences spanning more than 2^30 take the 64-bit time-difference
path; ordinary gaps on large absolute values take the relative 32-bit path.  Same tolerance as
tests/test_gpu_parity.py.  Kept in a file that runs after the main parity suite.
"""
import numpy as np
import pytest

from hstu_sequential_transducer_jagged_b200 import workloads as W
from test_gpu_parity import B, assert_close, gpu_attention, oracle_attention  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d,mask,m", [(64, W.MASK_CAUSAL, 0), (128, W.MASK_CAUSAL, 0),
                                       (64, W.MASK_MFALCON, 40)])
def test_attention_forward_wide_time_span(B, d, mask, m):
    """Timestamps in epoch milliseconds with sequences spanning more than 2^30: the time
    buckets then come from 64-bit differences (relative 32-bit values no longer fit)."""
    case = W.random_attention_case(11 + d + m, [300, 129, 41], H=2, d=d, P=64, NB=64,
                                   mask=mask, num_candidates=m, gap_mean=3.0e7)
    case.timestamps = case.timestamps + np.int64(1_700_000_000_000)
    spans = [int(case.timestamps[e - 1] - case.timestamps[s])
             for s, e in zip(case.seq_offsets[:-1], case.seq_offsets[1:]) if e > s]
    assert max(spans) > 2 ** 30
    assert_close(gpu_attention(B, case), oracle_attention(case), f"wide span d={d} m={m}")


def test_attention_forward_epoch_timestamps(B):
    """Large absolute timestamps with ordinary gaps: relative 32-bit time differences."""
    case = W.random_attention_case(12, [300, 129, 41], H=2, d=64, P=64, NB=64, gap_mean=600.0)
    case.timestamps = case.timestamps + np.int64(1_700_000_000_000)
    assert_close(gpu_attention(B, case), oracle_attention(case), "epoch timestamps")
