"""Failure path of the boundary on a B200: a bounded device wait that runs out.

The probe kernel waits, with the same bounded wait every kernel of the library uses, on a
barrier phase that nothing completes.  The wait must give up after its limit, the status word
must then report HSTU_ERR_TIMEOUT through hstu_sync_status (and be cleared by it), and the
context must stay usable: a small attention forward afterwards still matches the oracle.
No fault, trap or endless loop is involved.
"""
import time

import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W

pytestmark = pytest.mark.gpu

HSTU_ERR_TIMEOUT = 5


def test_bounded_wait_times_out_and_context_survives():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from hstu_sequential_transducer_jagged_b200 import binding as B
    ws = B.Workspace(256, torch.device("cuda", 0))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    B.debug_wait_timeout(ws)
    assert ws.sync_status() == HSTU_ERR_TIMEOUT
    elapsed = time.perf_counter() - t0
    assert 1.5 < elapsed < 30.0, elapsed  # the wait limit is 2 s
    assert ws.sync_status() == 0  # read and cleared

    case = W.random_attention_case(5, [130, 7], H=2, d=64, P=16, NB=16)
    def dev(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.to(dt) if dt is not None else t).cuda()

    bf = torch.bfloat16
    out = B.attention_forward(dev(case.q, bf), dev(case.k, bf), dev(case.v, bf),
                              dev(case.seq_offsets), case.max_seq_len, dev(case.timestamps),
                              dev(case.rab_pos), dev(case.rab_time), num_heads=case.num_heads,
                              max_pos_dist=case.max_pos_dist,
                              num_time_buckets=case.num_time_buckets, alpha=case.alpha)
    torch.cuda.synchronize()
    ref = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, num_heads=case.num_heads,
                              d_qk=case.d_qk, d_v=case.d_v, max_pos_dist=case.max_pos_dist,
                              num_time_buckets=case.num_time_buckets, alpha=case.alpha)
    got = out.float().cpu().numpy().astype(np.float64)
    bound = 2e-2 * np.abs(ref).max(axis=-1, keepdims=True) + 1e-3
    assert (np.abs(got - ref) <= bound).all()
