"""GPU parity of the token-type bias term ("HSTU：Scaling Law 的首次探索" §7.1.4 innovation 2:
bias_{i,j} = f(p_i - p_j, t_i - t_j, type_i, type_j), read as rab_pos + rab_time +
rab_type[type_i NT + type_j]) against the oracle: attention forward on the tensor-core (head
widths 64, 128) and CUDA-core (32) paths, the typed backward, and a layer forward."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
from test_gpu_parity import B, assert_close, attn_kw, dev  # noqa: F401

pytestmark = pytest.mark.gpu


def _types(case, NT, interleaved):
    if interleaved:  # item / action tokens alternate within each sequence
        off = case.seq_offsets
        t = np.concatenate([np.arange(int(off[b + 1]) - int(off[b])) % 2
                            for b in range(len(off) - 1)]) if case.total_tokens else np.zeros(0)
    else:
        t = np.random.default_rng(case.total_tokens).integers(0, NT, size=case.total_tokens)
    rab = np.random.default_rng(NT).normal(0.0, 0.5, size=NT * NT).astype(np.float32)
    return t.astype(np.int32), rab


@pytest.mark.parametrize("d,mask,m,NT,inter", [(64, W.MASK_CAUSAL, 0, 2, True),
                                                (64, W.MASK_MFALCON, 40, 3, False),
                                                (128, W.MASK_CAUSAL, 0, 4, False),
                                                (32, W.MASK_CAUSAL, 0, 2, True)])
def test_attention_forward_type_bias(B, d, mask, m, NT, inter):
    case = W.random_attention_case(90 + d + m, [300, 129, 41, 1, 0], H=2, d=d, P=40, NB=16,
                                   mask=mask, num_candidates=m, gap_mean=30.0, qkv_std=0.5)
    types, rab = _types(case, NT, inter)
    bf = torch.bfloat16
    out = B.attention_forward(dev(case.q, bf), dev(case.k, bf), dev(case.v, bf),
                              dev(case.seq_offsets), case.max_seq_len, dev(case.timestamps),
                              dev(case.rab_pos), dev(case.rab_time), num_heads=2,
                              max_pos_dist=40, num_time_buckets=16, mask=mask,
                              num_candidates=m, token_types=dev(types), rab_type=dev(rab),
                              num_types=NT)
    torch.cuda.synchronize()
    ref = O.attention_forward(case.q, case.k, case.v, case.seq_offsets, case.timestamps,
                              case.rab_pos, case.rab_time, token_types=types, rab_type=rab,
                              num_types=NT, **attn_kw(case))
    assert_close(out, ref, f"type bias d={d}")


@pytest.mark.parametrize("mask,m", [(W.MASK_CAUSAL, 0), (W.MASK_MFALCON, 30)])
def test_attention_backward_type_bias(B, mask, m):
    case = W.random_attention_case(95 + m, [200, 1, 129, 77], H=2, d=64, P=20, NB=16,
                                   mask=mask, num_candidates=m, gap_mean=20.0, qkv_std=0.5)
    types, rab = _types(case, 3, False)
    bf = torch.bfloat16
    got = B.attention_backward(dev(case.q, bf), dev(case.k, bf), dev(case.v, bf),
                               dev(case.d_o, bf), dev(case.seq_offsets), case.max_seq_len,
                               dev(case.timestamps), dev(case.rab_pos), dev(case.rab_time),
                               num_heads=2, max_pos_dist=20, num_time_buckets=16, mask=mask,
                               num_candidates=m, token_types=dev(types), rab_type=dev(rab),
                               num_types=3)
    torch.cuda.synchronize()
    ref = O.attention_backward(case.q, case.k, case.v, case.d_o, case.seq_offsets,
                               case.timestamps, case.rab_pos, case.rab_time, token_types=types,
                               rab_type=rab, num_types=3, **attn_kw(case))
    for name, g, r in zip(("dq", "dk", "dv", "d_rab_pos", "d_rab_time", "d_rab_type"), got, ref):
        assert_close(g, r, f"typed backward {name}")


def test_layer_forward_type_bias(B):
    case = W.random_layer_case(97, [150, 1, 129, 64, 260], d_model=128, H=2, d=64, P=30, NB=16,
                               w_std=0.05)
    types, rab = _types(case, 2, True)
    lp = case.layers[0]
    bf = torch.bfloat16
    y = B.layer_forward(dev(case.x, bf), dev(lp.w1, bf), dev(lp.w2, bf), dev(case.seq_offsets),
                        case.max_seq_len, dev(case.timestamps), dev(lp.rab_pos),
                        dev(lp.rab_time), num_heads=2, d_qk=64, d_v=64, max_pos_dist=30,
                        num_time_buckets=16, token_types=dev(types), rab_type=dev(rab),
                        num_types=2)
    torch.cuda.synchronize()
    ref = O.layer_forward(case.x, lp.w1, lp.w2, case.seq_offsets, case.timestamps, lp.rab_pos,
                          lp.rab_time, token_types=types, rab_type=rab, num_types=2,
                          **attn_kw(case))
    assert_close(y, ref, "layer with type bias")
