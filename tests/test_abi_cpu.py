"""The C-ABI library loads, exports every symbol include/hstu.h declares, and rejects bad
arguments on the host before touching the GPU (these tests need no GPU)."""
import ctypes
import os
import re

import pytest

from hstu_sequential_transducer_jagged_b200 import binding as B
from hstu_sequential_transducer_jagged_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(hstu_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_header_and_binding_agree():
    assert set(_declared_functions()) == set(B.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert lib.hstu_version().decode().startswith("hstu_b200")


def test_status_strings(lib):
    for code in range(7):
        assert lib.hstu_status_string(code)
    assert lib.hstu_status_string(99) == b"unknown status"


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: argument checks fail before any launch


def _desc(**kw):
    base = dict(num_seqs=2, total_tokens=100, max_seq_len=64, seq_offsets=1 << 20,
                timestamps=None, num_heads=2, d_qk=64, d_v=64, ld_q=128, ld_k=128, ld_v=128,
                ld_o=128, mask=0, num_candidates=0, mfalcon_microbatch=1, rab_pos=None,
                max_pos_dist=0, rab_time=None, num_time_buckets=1, alpha=1.0, dtype=0)
    base.update(kw)
    return B.AttnDesc(**base)


@pytest.mark.parametrize("bad", [
    dict(num_seqs=-1), dict(total_tokens=-5), dict(num_heads=0), dict(d_qk=0),
    dict(mask=7), dict(mask=1, num_candidates=-1), dict(mask=1, mfalcon_microbatch=0),
    dict(alpha=float("nan")), dict(dtype=5), dict(ld_q=64), dict(seq_offsets=None),
    dict(max_seq_len=10),  # 2 sequences of <= 10 tokens cannot hold 100 tokens
])
def test_attention_forward_rejects_bad_arguments(lib, bad):
    d = _desc(**bad)
    st = lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == 1


@pytest.mark.parametrize("bad", [dict(d_qk=48, d_v=48), dict(d_qk=64, d_v=32)])
def test_attention_forward_unsupported_widths(lib, bad):
    d = _desc(**bad)
    st = lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == 2


def test_attention_workspace_checks(lib):
    d = _desc()
    need = lib.hstu_attention_workspace_size(ctypes.byref(d))
    assert need >= 256 and need % 256 == 0
    # too small, misaligned, missing
    assert lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, need - 1,
                                      None) == 3
    assert lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE,
                                      ctypes.c_void_p((1 << 20) + 16), need, None) == 3
    assert lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, None, need,
                                      None) == 3
    assert lib.hstu_attention_forward(None, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == 1


def test_empty_batch_accepts_any_row_strides(lib):
    # zero tokens: nothing to compute, and zero-row views report arbitrary strides (0 for an
    # empty torch tensor); the call succeeds without touching any buffer
    d = _desc(total_tokens=0, max_seq_len=0, ld_q=0, ld_k=0, ld_v=0, ld_o=0)
    need = lib.hstu_attention_workspace_size(ctypes.byref(d))
    assert lib.hstu_attention_forward(ctypes.byref(d), None, None, None, None, FAKE, need,
                                      None) == 0
    # with tokens the same strides are rejected
    d = _desc(ld_q=0)
    assert lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                      None) == 1


def test_workspace_size_grows_with_batch(lib):
    small = lib.hstu_attention_workspace_size(ctypes.byref(_desc()))
    big = lib.hstu_attention_workspace_size(ctypes.byref(_desc(num_seqs=64, total_tokens=81920,
                                                               max_seq_len=2048)))
    assert big > small


def _ldesc(**kw):
    base = dict(num_seqs=2, total_tokens=100, max_seq_len=64, seq_offsets=1 << 20,
                timestamps=None, d_model=64, num_heads=2, d_qk=32, d_v=32, mask=0,
                num_candidates=0, mfalcon_microbatch=1, rab_pos=None, max_pos_dist=0,
                rab_time=None, num_time_buckets=1, alpha=1.0, ln_eps=1e-5, ln_gamma=None,
                ln_beta=None, dtype=1)
    base.update(kw)
    return B.LayerDesc(**base)


def test_layer_rejects_bad_arguments(lib):
    d = _ldesc()
    need = lib.hstu_layer_workspace_size(ctypes.byref(d))
    # layer workspace holds f1 output + AV + G in fp32
    assert need >= 100 * (2 * 2 * 64 + 2 * 64) * 4
    ok_ws = ctypes.c_void_p(1 << 20)
    assert lib.hstu_layer_forward(ctypes.byref(_ldesc(d_model=0)), FAKE, FAKE, None, FAKE, None,
                                  ctypes.c_void_p(2 << 20), ok_ws, need, None) == 1
    assert lib.hstu_layer_forward(ctypes.byref(_ldesc(ln_eps=-1.0)), FAKE, FAKE, None, FAKE,
                                  None, ctypes.c_void_p(2 << 20), ok_ws, need, None) == 1
    # y aliasing x
    assert lib.hstu_layer_forward(ctypes.byref(d), FAKE, FAKE, None, FAKE, None, FAKE, ok_ws,
                                  need, None) == 1
    # H * d_v beyond the LayerNorm row limit
    big = _ldesc(num_heads=16, d_qk=128, d_v=128)
    assert lib.hstu_layer_forward(ctypes.byref(big), FAKE, FAKE, None, FAKE, None,
                                  ctypes.c_void_p(2 << 20), ok_ws, 1 << 40, None) == 2


def test_position_clamp_is_bounded(lib):
    # 2P + 1 table entries must stay inside int32 arithmetic
    d = _desc(rab_pos=1 << 20, max_pos_dist=(1 << 24) + 1)
    st = lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == 1


def test_backward_requires_grad_buffers(lib):
    d = _desc(rab_pos=1 << 20, max_pos_dist=4)
    st = lib.hstu_attention_backward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                     None, None, FAKE, 1 << 30, None)
    assert st == 1


def test_misc_entry_points_validate(lib):
    assert lib.hstu_debug_time_buckets(FAKE, -1, FAKE, 8, None) == 1
    assert lib.hstu_debug_time_buckets(FAKE, 4, FAKE, 0, None) == 1
    assert lib.hstu_debug_time_buckets(None, 0, None, 8, None) == 0
    # bias-index export: unknown rule, n < 0, NB < 1 (time rules), P out of range (position rules)
    assert lib.hstu_debug_bias_index(9, FAKE, 4, 8, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(-1, FAKE, 4, 8, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(0, FAKE, -1, 8, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(2, FAKE, 4, 0, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(5, FAKE, 4, -1, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(5, FAKE, 4, (1 << 24) + 1, FAKE, None) == 1
    assert lib.hstu_debug_bias_index(5, None, 4, 8, None, None) == 1
    assert lib.hstu_debug_bias_index(5, None, 0, 8, None, None) == 0
    # row_bytes not a multiple of 16
    assert lib.hstu_jagged_padded_copy(FAKE, 2, 8, FAKE, 32, FAKE, 32, 24, 1, None) == 1
    assert lib.hstu_jagged_padded_copy(FAKE, 0, 8, FAKE, 32, FAKE, 32, 32, 1, None) == 0
    assert lib.hstu_sync_status(ctypes.c_void_p((1 << 20) + 8), None) == 3
    assert lib.hstu_workspace_init(None, 256, None) == 3


def test_static_scratch_call_rejects_on_the_host(lib):
    # the built-in scratch call checks its arguments and its size limit before touching CUDA
    assert lib.hstu_attention_forward_static_ws(None, FAKE, FAKE, FAKE, FAKE, None, None) == 1
    assert lib.hstu_attention_forward_static_ws(ctypes.byref(_desc(mask=7)), FAKE, FAKE, FAKE,
                                                FAKE, None, None) == 1
    assert lib.hstu_attention_forward_static_ws(ctypes.byref(_desc()), FAKE, FAKE, FAKE, FAKE,
                                                ctypes.c_void_p((1 << 20) + 2), None) == 1
    limit = 1 << 20  # HSTU_STATIC_SCRATCH_BYTES
    assert f"HSTU_STATIC_SCRATCH_BYTES ((size_t)1 << 20)" in open(HEADER).read()
    big = _desc(num_seqs=100000, total_tokens=100000, max_seq_len=1)
    need = lib.hstu_attention_workspace_size(ctypes.byref(big))
    assert need > limit
    assert lib.hstu_attention_forward_static_ws(ctypes.byref(big), FAKE, FAKE, FAKE, FAKE, None,
                                                None) == 3
    msg = lib.hstu_last_error_string().decode()
    assert str(need) in msg and str(limit) in msg


def test_wait_timeout_probe_rejects_bad_workspace(lib):
    assert lib.hstu_debug_wait_timeout(None, 256, None) == 3
    assert lib.hstu_debug_wait_timeout(ctypes.c_void_p((1 << 20) + 8), 256, None) == 3
    assert lib.hstu_debug_wait_timeout(FAKE, 100, None) == 3


def test_static_scratch_rejects_bad_strides_before_touching_the_array(lib):
    # a stride below the row width is rejected on the host (the shared array is not touched)
    assert lib.hstu_attention_forward_static_ws(ctypes.byref(_desc(ld_q=64)), FAKE, FAKE, FAKE,
                                                FAKE, None, None) == 1
    assert lib.hstu_attention_forward_static_ws(ctypes.byref(_desc()), None, FAKE, FAKE, FAKE,
                                                None, None) == 1


def test_layer_backward_validates_on_the_host(lib):
    bf = dict(dtype=0, d_model=128, num_heads=2, d_qk=64, d_v=64)
    d = _ldesc(**bf)
    need = lib.hstu_layer_backward_workspace_size(ctypes.byref(d))
    assert need > lib.hstu_layer_workspace_size(ctypes.byref(d))
    ws = ctypes.c_void_p(1 << 20)
    args = [FAKE, FAKE, None, FAKE, None, FAKE, ctypes.c_void_p(3 << 20), FAKE, None, FAKE,
            None, None, None, None, None]
    # fp32 layers and rows of H*d_v outside {128, 256, 512, 1024} are not supported
    assert lib.hstu_layer_backward(ctypes.byref(_ldesc()), *args, ws, 1 << 40, None) == 2
    assert lib.hstu_layer_backward(ctypes.byref(_ldesc(**dict(bf, d_v=48, d_qk=48))), *args, ws,
                                   1 << 40, None) == 2
    # too small a workspace
    assert lib.hstu_layer_backward(ctypes.byref(d), *args, ws, need - 1, None) == 3
    # d_x aliasing x
    bad = list(args)
    bad[6] = FAKE
    assert lib.hstu_layer_backward(ctypes.byref(d), *bad, ws, need, None) == 1
    # a LayerNorm affine without its gradient buffer
    d2 = _ldesc(ln_gamma=1 << 20, **bf)
    assert lib.hstu_layer_backward(ctypes.byref(d2), *args, ws, 1 << 40, None) == 1


def test_stochastic_length_and_gather_validate(lib):
    ws = ctypes.c_void_p(1 << 20)
    need = lib.hstu_stochastic_length_workspace_size(4, 100)
    assert need >= 256 + 400 + 16
    ok = [FAKE, 4, 100, 64, 10, 1000.0, FAKE, FAKE, FAKE, FAKE, ws, need, None]
    for i, bad in ((4, 0), (5, float("nan")), (5, -1.0), (3, -1), (2, -1)):
        a = list(ok)
        a[i] = bad
        assert lib.hstu_stochastic_length(*a) == 1, (i, bad)
    a = list(ok)
    a[3] = 10  # 4 sequences of <= 10 tokens cannot hold 100
    assert lib.hstu_stochastic_length(*a) == 1
    a = list(ok)
    a[11] = need - 1
    assert lib.hstu_stochastic_length(*a) == 3
    # gather: misaligned rows, negative sizes, nothing to do
    assert lib.hstu_gather_rows(FAKE, 16, FAKE, None, 4, FAKE, 16, 6, None) == 1
    assert lib.hstu_gather_rows(FAKE, 16, FAKE, None, -1, FAKE, 16, 16, None) == 1
    assert lib.hstu_gather_rows(FAKE, 16, FAKE, None, 0, FAKE, 16, 16, None) == 0
    assert lib.hstu_gather_rows(None, 16, FAKE, None, 4, FAKE, 16, 16, None) == 1


def test_mfalcon_cache_calls_validate(lib):
    d = _ldesc(dtype=0, d_model=128, num_heads=2, d_qk=64, d_v=64, mask=1, num_candidates=16)
    assert lib.hstu_layer_cache_bytes(ctypes.byref(d)) == 100 * 2 * 2 * 128 * 2
    need = lib.hstu_layer_candidates_workspace_size(ctypes.byref(d))
    ws = ctypes.c_void_p(1 << 20)
    # the candidates pass needs the M-FALCON mask and at least one candidate
    causal = _ldesc(dtype=0, d_model=128, num_heads=2, d_qk=64, d_v=64)
    assert lib.hstu_layer_forward_candidates(ctypes.byref(causal), FAKE, FAKE, None, FAKE, None,
                                             ctypes.c_void_p(2 << 20), FAKE, ws, 1 << 40,
                                             None) == 1
    # B * m above T
    many = _ldesc(dtype=0, d_model=128, num_heads=2, d_qk=64, d_v=64, mask=1, num_candidates=60)
    assert lib.hstu_layer_forward_candidates(ctypes.byref(many), FAKE, FAKE, None, FAKE, None,
                                             ctypes.c_void_p(2 << 20), FAKE, ws, 1 << 40,
                                             None) == 1
    assert lib.hstu_layer_forward_candidates(ctypes.byref(d), FAKE, FAKE, None, FAKE, None,
                                             ctypes.c_void_p(2 << 20), FAKE, ws, need - 1,
                                             None) == 3
    # the cached forward needs a cache
    assert lib.hstu_layer_forward_cached(ctypes.byref(d), FAKE, FAKE, None, FAKE, None,
                                         ctypes.c_void_p(2 << 20), None, ws, 1 << 40, None) == 1


def test_type_bias_arguments(lib):
    # rab_type without token types, or NT outside [1, 64]
    for kw in (dict(rab_type=1 << 20, num_types=2, token_types=None),
               dict(rab_type=1 << 20, num_types=0, token_types=1 << 20),
               dict(rab_type=1 << 20, num_types=65, token_types=1 << 20)):
        d = _desc(**kw)
        assert lib.hstu_attention_forward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                          None) == 1
    d = _desc(rab_type=1 << 20, num_types=2, token_types=1 << 20)
    # the plain backward has no place for the type gradient; the typed one needs its buffer
    assert lib.hstu_attention_backward(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                       None, None, FAKE, 1 << 30, None) == 1
    assert lib.hstu_attention_backward_typed(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                             FAKE, None, None, None, FAKE, 1 << 30, None) == 1
