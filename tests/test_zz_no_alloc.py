"""hstu_attention_forward_static_ws (the attention forward on the library's built-in scratch
array, for callers that may not allocate device memory while running) gives the same output
as hstu_attention_forward with a caller workspace, on two different problems in a row: the
shared array keeps the first call's contents, so the second call must not depend on them."""
import pytest
import torch

from hstu_sequential_transducer_jagged_b200 import binding as B
from hstu_sequential_transducer_jagged_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _to(dev, a, dtype=None):
    t = torch.from_numpy(a).to(dev)
    return t.to(dtype) if dtype is not None else t


def _case_args(wl, dev):
    bf = torch.bfloat16
    tensors = dict(q=_to(dev, wl.q, bf), k=_to(dev, wl.k, bf), v=_to(dev, wl.v, bf),
                   seq_offsets=_to(dev, wl.seq_offsets), timestamps=_to(dev, wl.timestamps),
                   rab_pos=_to(dev, wl.rab_pos), rab_time=_to(dev, wl.rab_time))
    kw = dict(num_heads=wl.num_heads, max_pos_dist=wl.max_pos_dist,
              num_time_buckets=wl.num_time_buckets, mask=wl.mask,
              num_candidates=wl.num_candidates, microbatch=max(1, wl.microbatch))
    return tensors, kw


def _run_both(wl, dev):
    t, kw = _case_args(wl, dev)
    T = t["q"].shape[0]
    max_len = int(wl.lengths.max())
    # everything the scratch call touches is allocated before it
    out_ref = torch.full((T, t["v"].shape[1]), float("nan"), dtype=torch.bfloat16, device=dev)
    out_new = torch.full_like(out_ref, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    B.attention_forward(t["q"], t["k"], t["v"], t["seq_offsets"], max_len, t["timestamps"],
                        t["rab_pos"], t["rab_time"], out=out_ref, **kw)
    B.attention_forward_static_ws(t["q"], t["k"], t["v"], t["seq_offsets"], max_len,
                                  t["timestamps"], t["rab_pos"], t["rab_time"], out=out_new,
                                  status_out=status, **kw)
    torch.cuda.synchronize()
    return out_ref.float().cpu(), out_new.float().cpu(), int(status.item())


def _assert_close(ref, got):
    # the tolerance the attention parity tests use: per element 2e-2 x max |row| + 1e-3
    assert torch.isfinite(got).all()
    row_scale = ref.abs().amax(dim=1, keepdim=True)
    assert ((got - ref).abs() <= 2e-2 * row_scale + 1e-3).all()


def test_static_scratch_matches_workspace_call_twice():
    dev = torch.device("cuda", 0)
    # first: causal, ragged lengths, time + position bias, interleaved timestamps
    wl1 = W.random_attention_case(seed=901, lengths=[300, 1, 517, 64, 200], H=2, d=64, P=40,
                                  NB=24, interleaved=True)
    # second: a different problem (M-FALCON, other sizes) on the same shared array
    wl2 = W.random_attention_case(seed=902, lengths=[260, 45, 130], H=3, d=64, P=16, NB=16,
                                  mask=W.MASK_MFALCON, num_candidates=40)
    for wl in (wl1, wl2):
        ref, got, status = _run_both(wl, dev)
        assert status == 0
        _assert_close(ref, got)
    # and the first problem again, after the second left its contents in the array
    ref, got, status = _run_both(wl1, dev)
    assert status == 0
    _assert_close(ref, got)
