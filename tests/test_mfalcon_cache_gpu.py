"""M-FALCON cross-request cache ("HSTU：Scaling Law 的首次探索" §7.1.5: the history's K/V are
computed once; later microbatches and requests compute only their candidates): a prefill with one
set of candidates, then a candidates-only pass with another set, through a 2-layer stack, against
a full forward over the new request and against the oracle."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
from test_gpu_parity import B, assert_close, attn_kw, dev  # noqa: F401

pytestmark = pytest.mark.gpu


def _cand_rows(off, m):
    return np.concatenate([np.arange(int(off[b + 1]) - m, int(off[b + 1]))
                           for b in range(len(off) - 1)])


@pytest.mark.parametrize("lengths,m", [([300, 250, 64 + 64], 64), ([4096 + 512, 700], 512)])
def test_candidates_only_pass_matches_full_forward(B, lengths, m):
    case = W.random_layer_case(70 + m, lengths, d_model=128, H=2, d=64, P=64, NB=32,
                               mask=W.MASK_MFALCON, num_candidates=m, num_layers=2, w_std=0.05)
    bf = torch.bfloat16
    off, ts = dev(case.seq_offsets), dev(case.timestamps)
    kw = dict(num_heads=2, d_qk=64, d_v=64, max_pos_dist=case.max_pos_dist,
              num_time_buckets=case.num_time_buckets, num_candidates=m)
    rows = _cand_rows(case.seq_offsets, m)
    # request 1 fills the caches; request 2 has new candidates on the same history
    x1 = case.x.copy()
    x2 = case.x.copy()
    x2[rows] = W.round_to_bf16(np.random.default_rng(3).standard_normal((len(rows), 128))
                               .astype(np.float32))
    layers = [dict(w1=dev(lp.w1, bf), w2=dev(lp.w2, bf), rp=dev(lp.rab_pos), rt=dev(lp.rab_time))
              for lp in case.layers]
    T = case.total_tokens
    caches = [torch.empty((T, 2 * 2 * 128), dtype=bf, device="cuda") for _ in layers]
    cur = dev(x1, bf)
    for l, ly in enumerate(layers):
        cur = B.layer_forward_cached(cur, ly["w1"], ly["w2"], caches[l], off, case.max_seq_len,
                                     ts, ly["rp"], ly["rt"], **kw)
    xc = dev(x2[rows], bf)
    for l, ly in enumerate(layers):
        xc = B.layer_forward_candidates(xc, ly["w1"], ly["w2"], caches[l], off, T,
                                        case.max_seq_len, ts, ly["rp"], ly["rt"], **kw)
    # full forward over request 2
    full = dev(x2, bf)
    for ly in layers:
        full = B.layer_forward(full, ly["w1"], ly["w2"], off, case.max_seq_len, ts, ly["rp"],
                               ly["rt"], mask=W.MASK_MFALCON, **kw)
    torch.cuda.synchronize()
    got = xc.float().cpu().numpy()
    ref_gpu = full.float().cpu().numpy()[rows]
    # the same kernels on the same tiles: identical up to the f1 GEMM's row blocking
    assert np.abs(got - ref_gpu).max() <= 1e-2 * np.abs(ref_gpu).max() + 1e-3
    ref = O.stack_forward(x2, case.layers, case.seq_offsets, case.timestamps,
                          round_between=W.round_to_bf16, **attn_kw(case))[rows]
    assert_close(got, ref, "candidates-only pass vs oracle")
