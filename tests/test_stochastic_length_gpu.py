"""Stochastic Length ("HSTU：Scaling Law 的首次探索" §7.1.5) on the GPU against the oracle:
new offsets and kept-token indices bit-exact (integer work), and the gathered rows identical."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W
from test_gpu_parity import B, dev  # noqa: F401

pytestmark = pytest.mark.gpu


def _draws(seed, B_, T, tie_every=0):
    rng = np.random.default_rng(seed)
    u = rng.random(B_).astype(np.float32)
    keys = rng.integers(0, 2 ** 32, size=T, dtype=np.uint64).astype(np.uint32)
    if tie_every:
        keys[::tie_every] = keys[0]  # many equal keys: the lower index must win
    return u, keys


def _check(B, lengths, N, alpha, seed, tie_every=0, u=None):
    off = W.offsets_from_lengths(np.asarray(lengths, np.int64))
    T = int(off[-1])
    uu, keys = _draws(seed, len(lengths), T, tie_every)
    if u is not None:
        uu = u
    sub_len, n_alpha = O.stochastic_length_params(N, alpha)
    ref_off, ref_kept = O.stochastic_length(off, uu, keys, sub_len, n_alpha)
    new_off, kept = B.stochastic_length(dev(off), max(lengths), dev(uu), dev(keys),
                                        sub_len=sub_len, n_alpha=n_alpha)
    torch.cuda.synchronize()
    new_off = new_off.cpu().numpy()
    assert np.array_equal(new_off, ref_off)
    assert np.array_equal(kept.cpu().numpy()[:new_off[-1]], ref_kept)
    return off, new_off, kept, sub_len


def test_stochastic_length_edges_bit_exact(B):
    N, alpha = 4096, 1.7
    sub_len, n_alpha = O.stochastic_length_params(N, alpha)
    lengths = [0, 1, sub_len - 1, sub_len, sub_len + 1, 2 * sub_len, 4096, 3000, 5, 4095]
    # u just below / above the threshold 1 - N^α / n² of each long sequence
    u = []
    for n in lengths:
        p = 1.0 - n_alpha / (n * n) if n > 0 else 0.0
        u.append(np.nextafter(np.float32(p), np.float32(0)) if len(u) % 2 else np.float32(p))
    _check(B, lengths, N, alpha, 1, u=np.array(u, np.float32))
    _check(B, lengths, N, alpha, 2)
    _check(B, lengths, N, alpha, 3, tie_every=3)
    _check(B, [4096] * 3, N, 2.0, 4)  # alpha = 2: nothing is truncated


def test_stochastic_length_workload_and_gather(B):
    """The 4-layer workload's batch (8 users, L~U{2048..8192}) with N = 8192, α = 1.6: offsets and
    indices bit-exact, and the gathered embeddings / timestamps equal a host gather."""
    wl = W.make("stack4_bf16_b8_inter")
    off, new_off, kept, sub_len = _check(B, wl.lengths.tolist(), 8192, 1.6, 5)
    n_new = int(new_off[-1])
    count = torch.tensor([n_new], dtype=torch.int32, device="cuda")
    x = dev(wl.x, torch.bfloat16)
    ts = dev(wl.timestamps)
    xg = B.gather_rows(x, kept, count=count, max_rows=wl.total_tokens)
    tg = B.gather_rows(ts, kept, count=count, max_rows=wl.total_tokens)
    torch.cuda.synchronize()
    k = kept.cpu().numpy()[:n_new].astype(np.int64)
    assert torch.equal(xg[:n_new].cpu(), x.cpu()[k])
    assert np.array_equal(tg[:n_new].cpu().numpy(), wl.timestamps[k])
    assert torch.count_nonzero(xg[n_new:].float()) == 0  # rows past *count untouched (zeros)
