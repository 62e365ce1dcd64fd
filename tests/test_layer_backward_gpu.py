"""GPU parity of the layer backward (hstu_layer_backward) against the oracle's fp64 chain rule.

Gradients of L = Σ dY ⊙ Y through Y = X + f2(Norm(A(X)V(X)) ⊙ U(X)) ("万亿参数推荐大模型：HSTU 架构
如何超越传统 Self-Attention" §2.1; the training pass of "HSTU：Scaling Law 的首次探索" §7.1.3).
Same tolerance as the other parity tests: per element |err| <= 2e-2 max|ref row| + 1e-3 and
relative Frobenius error <= 5e-3 (bias and weight gradients are compared as whole arrays), except
the relative Frobenius bound of the two bias-table gradients, 1e-2: in a layer the attention
backward's tensor-core operands dO = dAV and Q, K, V are bf16 roundings of intermediate results
(relative error up to 2^-9 each, which the fp64 oracle does not have), and a table entry sums
dS over up to ~10^5 pairs of both signs, so it keeps the ~3 x 2^-9 relative error of its terms
instead of averaging it away.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
import test_gpu_parity as P
from test_gpu_parity import B, assert_close, dev  # noqa: F401

pytestmark = pytest.mark.gpu

TABLE_FRO_TOL = 1e-2  # bias-table gradients of the layer backward (module docstring)

NAMES = ("dx", "dw1", "db1", "dw2", "db2", "d_rab_pos", "d_rab_time", "d_ln_gamma", "d_ln_beta")


def _run(B, case, d_y, lp, b1=None, b2=None, gamma=None, beta=None, x=None, off=None, ts=None):
    bf = torch.bfloat16
    return B.layer_backward(
        dev(case.x if x is None else x, bf), dev(lp.w1, bf), dev(lp.w2, bf), dev(d_y, bf),
        dev(case.seq_offsets if off is None else off), case.max_seq_len,
        dev(case.timestamps if ts is None else ts), dev(lp.rab_pos), dev(lp.rab_time),
        num_heads=case.num_heads, d_qk=case.d_qk, d_v=case.d_v, max_pos_dist=case.max_pos_dist,
        num_time_buckets=case.num_time_buckets, alpha=case.alpha, mask=case.mask,
        num_candidates=case.num_candidates, b1=None if b1 is None else dev(b1),
        b2=None if b2 is None else dev(b2), ln_gamma=None if gamma is None else dev(gamma),
        ln_beta=None if beta is None else dev(beta))


def _oracle(case, d_y, lp, b1=None, b2=None, gamma=None, beta=None):
    return O.layer_backward(case.x, lp.w1, lp.w2, case.seq_offsets, case.timestamps, lp.rab_pos,
                            lp.rab_time, d_y, num_heads=case.num_heads, d_qk=case.d_qk,
                            d_v=case.d_v, max_pos_dist=case.max_pos_dist,
                            num_time_buckets=case.num_time_buckets, alpha=case.alpha,
                            mask=case.mask, num_candidates=case.num_candidates, b1=b1, b2=b2,
                            ln_gamma=gamma, ln_beta=beta)


def _compare(got, ref, what):
    torch.cuda.synchronize()
    for name in NAMES:
        if ref.get(name) is None or got.get(name) is None:
            continue
        if name in ("d_rab_pos", "d_rab_time"):
            saved = P.FRO_TOL
            P.FRO_TOL = TABLE_FRO_TOL
            try:
                assert_close(got[name], ref[name], f"{what} {name}")
            finally:
                P.FRO_TOL = saved
        else:
            assert_close(got[name], ref[name], f"{what} {name}")


@pytest.mark.parametrize("mask,m", [(W.MASK_CAUSAL, 0), (W.MASK_MFALCON, 60)])
def test_layer_backward_small(B, mask, m):
    case = W.random_layer_case(50 + m, [150, 1, 129, 64, 0, 260], d_model=128, H=2, d=64,
                               P=30, NB=16, w_std=0.05, mask=mask, num_candidates=m)
    lp = case.layers[0]
    d_y = W.round_to_bf16(np.random.default_rng(7).standard_normal(case.x.shape))
    _compare(_run(B, case, d_y, lp), _oracle(case, d_y, lp), f"layer backward mask={mask}")


def test_layer_backward_biases_and_affine(B):
    case = W.random_layer_case(61, [200, 77, 256], d_model=128, H=2, d=64, P=20, NB=16,
                               w_std=0.05)
    lp = case.layers[0]
    rng = np.random.default_rng(8)
    d_y = W.round_to_bf16(rng.standard_normal(case.x.shape))
    n1, hv = lp.w1.shape[1], lp.w2.shape[0]
    b1 = (0.1 * rng.standard_normal(n1)).astype(np.float32)
    b2 = (0.1 * rng.standard_normal(128)).astype(np.float32)
    gamma = (1.0 + 0.2 * rng.standard_normal(hv)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(hv)).astype(np.float32)
    got = _run(B, case, d_y, lp, b1, b2, gamma, beta)
    ref = _oracle(case, d_y, lp, b1, b2, gamma, beta)
    _compare(got, ref, "layer backward with biases and affine")


def test_layer_backward_mid_size(B):
    """The geometric-length layer's shapes (d_model 256, H 4, d 64, P 1024, NB 128) on a
    mid-size batch spanning many tiles."""
    case = W.random_layer_case(62, [700, 1024, 33, 300, 512], d_model=256, H=4, d=64, P=1024,
                               NB=128, w_std=0.02, table_std=0.02)
    lp = case.layers[0]
    d_y = W.round_to_bf16(np.random.default_rng(9).standard_normal(case.x.shape))
    _compare(_run(B, case, d_y, lp), _oracle(case, d_y, lp), "layer backward mid")


def test_layer_backward_full_size_sampled_sequence(B):
    """Layer 0 of the 4-layer workload at full size (41808 tokens, d_model 512, H 8): the input
    gradient of the shortest sequence checked against the oracle run on that sequence alone
    (sequences are independent, so its dX rows depend on it and the weights only), and every
    gradient finite."""
    case = W.make("stack4_bf16_b8_inter")
    lp = case.layers[0]
    d_y = W.round_to_bf16(np.random.default_rng(10).standard_normal(case.x.shape)
                          .astype(np.float32))
    got = _run(B, case, d_y, lp)
    torch.cuda.synchronize()
    for name in NAMES:
        if got.get(name) is not None:
            assert torch.isfinite(got[name].float()).all(), name
    b = int(np.argmin(case.lengths))
    s, e = int(case.seq_offsets[b]), int(case.seq_offsets[b + 1])
    ref = O.layer_backward(case.x[s:e], lp.w1, lp.w2, np.array([0, e - s]), case.timestamps[s:e],
                           lp.rab_pos, lp.rab_time, d_y[s:e], num_heads=8, d_qk=64, d_v=64,
                           max_pos_dist=case.max_pos_dist,
                           num_time_buckets=case.num_time_buckets)
    assert_close(got["dx"][s:e], ref["dx"], "full-size layer backward dx")
