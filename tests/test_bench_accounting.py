"""bench.py's work accounting (the numerator of every reported TFLOP/s and roofline fraction)
against brute force: visible pairs counted one by one from the oracle's mask, the attention's
4 d FLOPs per visible pair and head, and the two projections' 2 m n k each."""
import sys
import types
from pathlib import Path

import numpy as np
import pytest

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from oracle import hstu_oracle as O  # noqa: E402
from hstu_sequential_transducer_jagged_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("mask,m", [(W.MASK_CAUSAL, 0), (W.MASK_MFALCON, 5),
                                    (W.MASK_MFALCON, 40)])
def test_attention_pairs_match_mask_count(mask, m):
    lengths = np.array([1, 7, 33, 128, 129, 300, 0, 12])
    wl = types.SimpleNamespace(lengths=lengths, mask=mask, num_candidates=m, d_qk=64,
                               num_heads=8)
    brute = sum(int(O.allowed_pairs(int(L), mask, m).sum()) for L in lengths if L > 0)
    assert bench.attention_pairs(wl) == brute
    assert bench.attention_flops(wl) == 4.0 * 64 * 8 * brute


def test_projection_flops_count_every_multiply_add():
    wl = types.SimpleNamespace(num_heads=3, d_qk=5, d_v=7, d_model=11, total_tokens=13)
    n1 = 2 * 3 * (5 + 7)            # U, V, Q, K columns of f1
    f1 = 2 * 13 * 11 * n1           # [T, d_model] x [d_model, n1]
    f2 = 2 * 13 * (3 * 7) * 11      # [T, H d_v] x [H d_v, d_model]
    assert bench.gemm_flops(wl) == f1 + f2


def test_four_layer_workload_flops():
    wl = W.make("stack4_bf16_b8_inter")
    L = wl.lengths.astype(np.int64)
    assert bench.attention_flops(wl) == 4.0 * 64 * 8 * float((L * (L + 1) // 2).sum())
