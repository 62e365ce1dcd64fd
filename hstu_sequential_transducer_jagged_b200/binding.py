"""Thin ctypes binding of libhstu_b200.so (the C ABI in include/hstu.h).

Argument marshalling only: every step of the HSTU path runs in the library's CUDA kernels.
PyTorch is used for device memory and streams.  If the shared library is missing the import of
this module fails; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhstu_b200.so")

HSTU_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
                3: "workspace", 4: "CUDA error", 5: "device wait timed out",
                6: "device-side check failed"}
MASK_CAUSAL, MASK_MFALCON = 0, 1
DTYPE_BF16, DTYPE_FP32 = 0, 1

EXPORTED = [
    "hstu_attention_workspace_size", "hstu_attention_forward",
    "hstu_attention_backward_workspace_size", "hstu_attention_backward",
    "hstu_layer_workspace_size", "hstu_layer_forward", "hstu_layer_forward_stage",
    "hstu_jagged_padded_copy",
    "hstu_debug_time_buckets", "hstu_workspace_init", "hstu_sync_status",
    "hstu_status_string", "hstu_version", "hstu_last_error_string",
    "hstu_attention_forward_static_ws", "hstu_debug_wait_timeout", "hstu_alibi_tables",
    "hstu_debug_bias_index", "hstu_layer_backward_workspace_size", "hstu_layer_backward",
    "hstu_stochastic_length_workspace_size", "hstu_stochastic_length", "hstu_gather_rows",
    "hstu_layer_cache_bytes", "hstu_layer_forward_cached", "hstu_layer_candidates_workspace_size",
    "hstu_layer_forward_candidates", "hstu_attention_backward_typed",
]

# Rules of hstu_debug_bias_index (hstu_bias_rule_t)
BIAS_RULES = {"bucket64": 0, "bucket_row": 1, "time_elem": 2, "bucket_cls": 3, "threshold": 4,
              "pos_table": 5, "pos_general": 6, "pos_segment": 7, "pos_direct": 8}


class HstuError(RuntimeError):
    def __init__(self, status: int, where: str):
        detail = ""
        if status == 4 and _LIB is not None:
            detail = ": " + _LIB.hstu_last_error_string().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, 'unknown')} (status {status})"
                         f"{detail}")
        self.status = status


class AttnDesc(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32), ("seq_offsets", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p), ("num_heads", ctypes.c_int32),
        ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("ld_q", ctypes.c_int64), ("ld_k", ctypes.c_int64), ("ld_v", ctypes.c_int64),
        ("ld_o", ctypes.c_int64), ("mask", ctypes.c_int32), ("num_candidates", ctypes.c_int32),
        ("mfalcon_microbatch", ctypes.c_int32), ("rab_pos", ctypes.c_void_p),
        ("max_pos_dist", ctypes.c_int32), ("rab_time", ctypes.c_void_p),
        ("num_time_buckets", ctypes.c_int32), ("alpha", ctypes.c_float),
        ("dtype", ctypes.c_int32), ("token_types", ctypes.c_void_p),
        ("rab_type", ctypes.c_void_p), ("num_types", ctypes.c_int32),
    ]


class LayerDesc(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32), ("seq_offsets", ctypes.c_void_p),
        ("timestamps", ctypes.c_void_p), ("d_model", ctypes.c_int32),
        ("num_heads", ctypes.c_int32), ("d_qk", ctypes.c_int32), ("d_v", ctypes.c_int32),
        ("mask", ctypes.c_int32), ("num_candidates", ctypes.c_int32),
        ("mfalcon_microbatch", ctypes.c_int32), ("rab_pos", ctypes.c_void_p),
        ("max_pos_dist", ctypes.c_int32), ("rab_time", ctypes.c_void_p),
        ("num_time_buckets", ctypes.c_int32), ("alpha", ctypes.c_float),
        ("ln_eps", ctypes.c_float), ("ln_gamma", ctypes.c_void_p), ("ln_beta", ctypes.c_void_p),
        ("dtype", ctypes.c_int32), ("token_types", ctypes.c_void_p),
        ("rab_type", ctypes.c_void_p), ("num_types", ctypes.c_int32),
    ]


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m hstu_sequential_transducer_jagged_b200.build`")
    lib = ctypes.CDLL(path)
    vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int64
    adp, ldp = ctypes.POINTER(AttnDesc), ctypes.POINTER(LayerDesc)
    sigs = {
        "hstu_attention_workspace_size": (sz, [adp]),
        "hstu_attention_forward": (i32, [adp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_attention_backward_workspace_size": (sz, [adp]),
        "hstu_attention_backward": (i32, [adp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_attention_backward_typed": (i32, [adp] + [vp] * 11 + [sz, vp]),
        "hstu_layer_workspace_size": (sz, [ldp]),
        "hstu_layer_forward": (i32, [ldp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_layer_forward_stage": (i32, [ldp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_layer_backward_workspace_size": (sz, [ldp]),
        "hstu_layer_cache_bytes": (sz, [ldp]),
        "hstu_layer_forward_cached": (i32, [ldp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_layer_candidates_workspace_size": (sz, [ldp]),
        "hstu_layer_forward_candidates": (i32, [ldp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "hstu_stochastic_length_workspace_size": (sz, [i32, i32]),
        "hstu_stochastic_length": (i32, [vp, i32, i32, i32, i32, ctypes.c_double, vp, vp, vp, vp,
                                         vp, sz, vp]),
        "hstu_gather_rows": (i32, [vp, i64, vp, vp, i32, vp, i64, i64, vp]),
        "hstu_layer_backward": (i32, [ldp] + [vp] * 15 + [vp, sz, vp]),
        "hstu_jagged_padded_copy": (i32, [vp, i32, i32, vp, i64, vp, i64, i64, i32, vp]),
        "hstu_debug_time_buckets": (i32, [vp, i32, vp, i32, vp]),
        "hstu_debug_bias_index": (i32, [i32, vp, i32, i32, vp, vp]),
        "hstu_workspace_init": (i32, [vp, sz, vp]),
        "hstu_sync_status": (i32, [vp, vp]),
        "hstu_status_string": (ctypes.c_char_p, [i32]),
        "hstu_version": (ctypes.c_char_p, []),
        "hstu_last_error_string": (ctypes.c_char_p, []),
        "hstu_attention_forward_static_ws": (i32, [adp, vp, vp, vp, vp, vp, vp]),
        "hstu_debug_wait_timeout": (i32, [vp, sz, vp]),
        "hstu_alibi_tables": (i32, [ctypes.c_float, ctypes.c_float, i32, i32, vp, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load_library()
    return _LIB


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != HSTU_OK:
        raise HstuError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DTYPE_BF16
    if t.dtype == torch.float32:
        return DTYPE_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


class Workspace:
    """A device workspace (a torch uint8 buffer) with its status word zeroed once."""

    def __init__(self, nbytes: int, device):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.view = self.buf[off:off + self.nbytes]
        _check(lib().hstu_workspace_init(ctypes.c_void_p(self.view.data_ptr()),
                                         self.nbytes, _stream_ptr(None)), "workspace_init")

    def ensure(self, nbytes: int) -> "Workspace":
        return self if nbytes <= self.nbytes else Workspace(nbytes, self.buf.device)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.view.data_ptr())

    def sync_status(self, stream=None) -> int:
        return int(lib().hstu_sync_status(self.ptr, _stream_ptr(stream)))


_WS_CACHE = {}


def workspace(nbytes: int, device) -> Workspace:
    key = (str(device), threading_id())
    ws = _WS_CACHE.get(key)
    if ws is None or ws.nbytes < nbytes:
        ws = Workspace(nbytes, device)
        _WS_CACHE[key] = ws
    return ws


def threading_id() -> int:
    import threading
    return threading.get_ident()


def attn_desc(*, seq_offsets, total_tokens, max_seq_len, timestamps, num_heads, d_qk, d_v,
              ld_q, ld_k, ld_v, ld_o, mask=MASK_CAUSAL, num_candidates=0, microbatch=1,
              rab_pos=None, max_pos_dist=0, rab_time=None, num_time_buckets=1, alpha=1.0,
              dtype=DTYPE_BF16, token_types=None, rab_type=None, num_types=0) -> AttnDesc:
    return AttnDesc(
        num_seqs=seq_offsets.numel() - 1, total_tokens=int(total_tokens),
        max_seq_len=int(max_seq_len), seq_offsets=seq_offsets.data_ptr(),
        timestamps=None if timestamps is None else timestamps.data_ptr(), num_heads=num_heads,
        d_qk=d_qk, d_v=d_v, ld_q=ld_q, ld_k=ld_k, ld_v=ld_v, ld_o=ld_o, mask=mask,
        num_candidates=num_candidates, mfalcon_microbatch=max(1, int(microbatch)),
        rab_pos=None if rab_pos is None else rab_pos.data_ptr(), max_pos_dist=max_pos_dist,
        rab_time=None if rab_time is None else rab_time.data_ptr(),
        num_time_buckets=num_time_buckets, alpha=alpha, dtype=dtype,
        token_types=None if token_types is None else token_types.data_ptr(),
        rab_type=None if rab_type is None else rab_type.data_ptr(),
        num_types=int(num_types) if rab_type is not None else 0)


def attention_forward(q, k, v, seq_offsets, max_seq_len, timestamps=None, rab_pos=None,
                      rab_time=None, *, num_heads, max_pos_dist=0, num_time_buckets=1,
                      alpha=1.0, mask=MASK_CAUSAL, num_candidates=0, microbatch=128, out=None,
                      ws: Optional[Workspace] = None, stream=None, token_types=None,
                      rab_type=None, num_types=0):
    """O = hstu_attention_forward(...) for [T, H*d] views q, k, v (row strides taken from them)."""
    T = q.shape[0]
    d = q.shape[1] // num_heads if q.dim() == 2 else q.shape[-1]
    if out is None:
        out = torch.empty((T, num_heads * v.shape[1] // num_heads), dtype=q.dtype,
                          device=q.device)
    desc = attn_desc(seq_offsets=seq_offsets, total_tokens=T, max_seq_len=max_seq_len,
                     timestamps=timestamps, num_heads=num_heads, d_qk=d, d_v=v.shape[1] // num_heads,
                     ld_q=q.stride(0), ld_k=k.stride(0), ld_v=v.stride(0), ld_o=out.stride(0),
                     mask=mask, num_candidates=num_candidates, microbatch=microbatch,
                     rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                     num_time_buckets=num_time_buckets, alpha=alpha, dtype=_dtype_code(q),
                     token_types=token_types, rab_type=rab_type, num_types=num_types)
    need = lib().hstu_attention_workspace_size(ctypes.byref(desc))
    ws = workspace(need, q.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_attention_forward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                        ws.ptr, ws.nbytes, _stream_ptr(stream)),
           "hstu_attention_forward")
    return out


def attention_forward_static_ws(q, k, v, seq_offsets, max_seq_len, timestamps=None,
                                rab_pos=None, rab_time=None, *, num_heads, max_pos_dist=0,
                                num_time_buckets=1, alpha=1.0, mask=MASK_CAUSAL,
                                num_candidates=0, microbatch=128, out=None, status_out=None,
                                stream=None):
    """O = hstu_attention_forward_static_ws(...): the attention forward on the library's
    built-in scratch array instead of a workspace.  For callers that may not allocate device
    memory while running; `out` (and `status_out`, a device int32 tensor) must then be passed in
    preallocated.  Calls that overlap in time on one device race on the shared array."""
    T = q.shape[0]
    d = q.shape[1] // num_heads
    if out is None:
        out = torch.empty((T, v.shape[1]), dtype=q.dtype, device=q.device)
    desc = attn_desc(seq_offsets=seq_offsets, total_tokens=T, max_seq_len=max_seq_len,
                     timestamps=timestamps, num_heads=num_heads, d_qk=d, d_v=v.shape[1] // num_heads,
                     ld_q=q.stride(0), ld_k=k.stride(0), ld_v=v.stride(0), ld_o=out.stride(0),
                     mask=mask, num_candidates=num_candidates, microbatch=microbatch,
                     rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                     num_time_buckets=num_time_buckets, alpha=alpha, dtype=_dtype_code(q))
    st = lib().hstu_attention_forward_static_ws(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v),
                                                _ptr(out), _ptr(status_out), _stream_ptr(stream))
    if st != HSTU_OK:
        detail = lib().hstu_last_error_string().decode(errors="replace")
        raise HstuError(st, f"hstu_attention_forward_static_ws ({detail})")
    return out


def attention_backward(q, k, v, d_o, seq_offsets, max_seq_len, timestamps=None, rab_pos=None,
                       rab_time=None, *, num_heads, max_pos_dist=0, num_time_buckets=1,
                       alpha=1.0, mask=MASK_CAUSAL, num_candidates=0, microbatch=128,
                       ws: Optional[Workspace] = None, stream=None, token_types=None,
                       rab_type=None, num_types=0):
    """(dq, dk, dv, d_rab_pos, d_rab_time) of hstu_attention_backward; with the token-type term
    (rab_type given) hstu_attention_backward_typed, and d_rab_type appended."""
    T = q.shape[0]
    d = q.shape[1] // num_heads
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    d_pos = None if rab_pos is None else torch.empty_like(rab_pos)
    d_time = None if rab_time is None else torch.empty_like(rab_time)
    if T > 0 and (dq.stride(0) != q.stride(0) or dk.stride(0) != k.stride(0)
                  or dv.stride(0) != v.stride(0)):
        raise ValueError("q, k, v must be contiguous for the backward binding")
    desc = attn_desc(seq_offsets=seq_offsets, total_tokens=T, max_seq_len=max_seq_len,
                     timestamps=timestamps, num_heads=num_heads, d_qk=d, d_v=v.shape[1] // num_heads,
                     ld_q=q.stride(0), ld_k=k.stride(0), ld_v=v.stride(0), ld_o=d_o.stride(0),
                     mask=mask, num_candidates=num_candidates, microbatch=microbatch,
                     rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                     num_time_buckets=num_time_buckets, alpha=alpha, dtype=_dtype_code(q),
                     token_types=token_types, rab_type=rab_type, num_types=num_types)
    need = lib().hstu_attention_backward_workspace_size(ctypes.byref(desc))
    ws = workspace(need, q.device) if ws is None else ws.ensure(need)
    if rab_type is not None:
        d_type = torch.empty(num_types * num_types, dtype=torch.float32, device=q.device)
        _check(lib().hstu_attention_backward_typed(
            ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(d_o), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(d_pos), _ptr(d_time), _ptr(d_type), ws.ptr, ws.nbytes,
            _stream_ptr(stream)), "hstu_attention_backward_typed")
        return dq, dk, dv, d_pos, d_time, d_type
    _check(lib().hstu_attention_backward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(d_o),
                                         _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_pos), _ptr(d_time),
                                         ws.ptr, ws.nbytes, _stream_ptr(stream)),
           "hstu_attention_backward")
    return dq, dk, dv, d_pos, d_time


def layer_desc(*, seq_offsets, total_tokens, max_seq_len, timestamps, d_model, num_heads, d_qk,
               d_v, mask=MASK_CAUSAL, num_candidates=0, microbatch=1, rab_pos=None,
               max_pos_dist=0, rab_time=None, num_time_buckets=1, alpha=1.0, ln_eps=1e-5,
               ln_gamma=None, ln_beta=None, dtype=DTYPE_BF16, token_types=None, rab_type=None,
               num_types=0) -> LayerDesc:
    return LayerDesc(
        num_seqs=seq_offsets.numel() - 1, total_tokens=int(total_tokens),
        max_seq_len=int(max_seq_len), seq_offsets=seq_offsets.data_ptr(),
        timestamps=None if timestamps is None else timestamps.data_ptr(), d_model=d_model,
        num_heads=num_heads, d_qk=d_qk, d_v=d_v, mask=mask, num_candidates=num_candidates,
        mfalcon_microbatch=max(1, int(microbatch)),
        rab_pos=None if rab_pos is None else rab_pos.data_ptr(), max_pos_dist=max_pos_dist,
        rab_time=None if rab_time is None else rab_time.data_ptr(),
        num_time_buckets=num_time_buckets, alpha=alpha, ln_eps=ln_eps,
        ln_gamma=None if ln_gamma is None else ln_gamma.data_ptr(),
        ln_beta=None if ln_beta is None else ln_beta.data_ptr(), dtype=dtype,
        token_types=None if token_types is None else token_types.data_ptr(),
        rab_type=None if rab_type is None else rab_type.data_ptr(),
        num_types=int(num_types) if rab_type is not None else 0)


def layer_forward(x, w1, w2, seq_offsets, max_seq_len, timestamps=None, rab_pos=None,
                  rab_time=None, *, num_heads, d_qk, d_v, max_pos_dist=0, num_time_buckets=1,
                  alpha=1.0, mask=MASK_CAUSAL, num_candidates=0, microbatch=128, b1=None,
                  b2=None, ln_eps=1e-5, ln_gamma=None, ln_beta=None, out=None,
                  ws: Optional[Workspace] = None, stream=None, token_types=None, rab_type=None,
                  num_types=0):
    T, d_model = x.shape
    if out is None:
        out = torch.empty_like(x)
    desc = layer_desc(seq_offsets=seq_offsets, total_tokens=T, max_seq_len=max_seq_len,
                      timestamps=timestamps, d_model=d_model, num_heads=num_heads, d_qk=d_qk,
                      d_v=d_v, mask=mask, num_candidates=num_candidates, microbatch=microbatch,
                      rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                      num_time_buckets=num_time_buckets, alpha=alpha, ln_eps=ln_eps,
                      ln_gamma=ln_gamma, ln_beta=ln_beta, dtype=_dtype_code(x),
                      token_types=token_types, rab_type=rab_type, num_types=num_types)
    need = lib().hstu_layer_workspace_size(ctypes.byref(desc))
    ws = workspace(need, x.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_layer_forward(ctypes.byref(desc), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2),
                                    _ptr(b2), _ptr(out), ws.ptr, ws.nbytes, _stream_ptr(stream)),
           "hstu_layer_forward")
    return out


def _layer_call_desc(x_rows_T, seq_offsets, max_seq_len, timestamps, d_model, dtype, **kw):
    return layer_desc(seq_offsets=seq_offsets, total_tokens=x_rows_T, max_seq_len=max_seq_len,
                      timestamps=timestamps, d_model=d_model, dtype=dtype, **kw)


def layer_forward_cached(x, w1, w2, cache, seq_offsets, max_seq_len, timestamps=None,
                         rab_pos=None, rab_time=None, *, num_heads, d_qk, d_v, max_pos_dist=0,
                         num_time_buckets=1, alpha=1.0, num_candidates, microbatch=128, b1=None,
                         b2=None, ln_eps=1e-5, out=None, ws: Optional[Workspace] = None,
                         stream=None):
    """M-FALCON prefill (hstu_layer_forward_cached): the layer forward, keeping its f1 output in
    cache (a [T, 2H(d_qk+d_v)] tensor of x's dtype)."""
    T, d_model = x.shape
    out = torch.empty_like(x) if out is None else out
    desc = _layer_call_desc(T, seq_offsets, max_seq_len, timestamps, d_model, _dtype_code(x),
                            num_heads=num_heads, d_qk=d_qk, d_v=d_v, mask=MASK_MFALCON,
                            num_candidates=num_candidates, microbatch=microbatch,
                            rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                            num_time_buckets=num_time_buckets, alpha=alpha, ln_eps=ln_eps)
    need = lib().hstu_layer_workspace_size(ctypes.byref(desc))
    ws = workspace(need, x.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_layer_forward_cached(ctypes.byref(desc), _ptr(x), _ptr(w1), _ptr(b1),
                                           _ptr(w2), _ptr(b2), _ptr(out), _ptr(cache), ws.ptr,
                                           ws.nbytes, _stream_ptr(stream)),
           "hstu_layer_forward_cached")
    return out


def layer_forward_candidates(x_cand, w1, w2, cache, seq_offsets, total_tokens, max_seq_len,
                             timestamps=None, rab_pos=None, rab_time=None, *, num_heads, d_qk,
                             d_v, max_pos_dist=0, num_time_buckets=1, alpha=1.0, num_candidates,
                             microbatch=128, b1=None, b2=None, ln_eps=1e-5, out=None,
                             ws: Optional[Workspace] = None, stream=None):
    """M-FALCON candidates only (hstu_layer_forward_candidates): x_cand [B m, d_model] ->
    y_cand, reading the history's f1 output from cache."""
    d_model = x_cand.shape[1]
    out = torch.empty_like(x_cand) if out is None else out
    desc = _layer_call_desc(int(total_tokens), seq_offsets, max_seq_len, timestamps, d_model,
                            _dtype_code(x_cand), num_heads=num_heads, d_qk=d_qk, d_v=d_v,
                            mask=MASK_MFALCON, num_candidates=num_candidates,
                            microbatch=microbatch, rab_pos=rab_pos, max_pos_dist=max_pos_dist,
                            rab_time=rab_time, num_time_buckets=num_time_buckets, alpha=alpha,
                            ln_eps=ln_eps)
    need = lib().hstu_layer_candidates_workspace_size(ctypes.byref(desc))
    ws = workspace(need, x_cand.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_layer_forward_candidates(ctypes.byref(desc), _ptr(x_cand), _ptr(w1),
                                               _ptr(b1), _ptr(w2), _ptr(b2), _ptr(out),
                                               _ptr(cache), ws.ptr, ws.nbytes,
                                               _stream_ptr(stream)),
           "hstu_layer_forward_candidates")
    return out


def layer_backward(x, w1, w2, d_y, seq_offsets, max_seq_len, timestamps=None, rab_pos=None,
                   rab_time=None, *, num_heads, d_qk, d_v, max_pos_dist=0, num_time_buckets=1,
                   alpha=1.0, mask=MASK_CAUSAL, num_candidates=0, microbatch=128, b1=None,
                   b2=None, ln_eps=1e-5, ln_gamma=None, ln_beta=None,
                   ws: Optional[Workspace] = None, stream=None):
    """Gradients of Σ d_y ⊙ Y through one layer (hstu_layer_backward): a dict with dx (bf16,
    like x) and the fp32 dw1, db1, dw2, db2, d_rab_pos, d_rab_time, d_ln_gamma, d_ln_beta
    (None where the matching parameter is None)."""
    T, d_model = x.shape
    n1, hv = w1.shape[1], w2.shape[0]
    f32 = dict(dtype=torch.float32, device=x.device)
    out = dict(dx=torch.empty_like(x), dw1=torch.empty((d_model, n1), **f32),
               dw2=torch.empty((hv, d_model), **f32),
               db1=None if b1 is None else torch.empty(n1, **f32),
               db2=None if b2 is None else torch.empty(d_model, **f32),
               d_rab_pos=None if rab_pos is None else torch.empty_like(rab_pos),
               d_rab_time=None if rab_time is None else torch.empty_like(rab_time),
               d_ln_gamma=None if ln_gamma is None else torch.empty(hv, **f32),
               d_ln_beta=None if ln_beta is None else torch.empty(hv, **f32))
    desc = layer_desc(seq_offsets=seq_offsets, total_tokens=T, max_seq_len=max_seq_len,
                      timestamps=timestamps, d_model=d_model, num_heads=num_heads, d_qk=d_qk,
                      d_v=d_v, mask=mask, num_candidates=num_candidates, microbatch=microbatch,
                      rab_pos=rab_pos, max_pos_dist=max_pos_dist, rab_time=rab_time,
                      num_time_buckets=num_time_buckets, alpha=alpha, ln_eps=ln_eps,
                      ln_gamma=ln_gamma, ln_beta=ln_beta, dtype=_dtype_code(x))
    need = lib().hstu_layer_backward_workspace_size(ctypes.byref(desc))
    ws = workspace(need, x.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_layer_backward(
        ctypes.byref(desc), _ptr(x), _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(d_y),
        _ptr(out["dx"]), _ptr(out["dw1"]), _ptr(out["db1"]), _ptr(out["dw2"]), _ptr(out["db2"]),
        _ptr(out["d_rab_pos"]), _ptr(out["d_rab_time"]), _ptr(out["d_ln_gamma"]),
        _ptr(out["d_ln_beta"]), ws.ptr, ws.nbytes, _stream_ptr(stream)), "hstu_layer_backward")
    return out


def stochastic_length(seq_offsets, max_seq_len, u, token_keys, *, sub_len, n_alpha,
                      ws: Optional[Workspace] = None, stream=None):
    """(new_offsets, kept_index) of hstu_stochastic_length: int32 device tensors [B+1] and [T]
    (only the first new_offsets[B] entries of kept_index are meaningful)."""
    B = seq_offsets.numel() - 1
    T = token_keys.numel()
    new_off = torch.empty(B + 1, dtype=torch.int32, device=seq_offsets.device)
    kept = torch.empty(max(T, 1), dtype=torch.int32, device=seq_offsets.device)
    need = lib().hstu_stochastic_length_workspace_size(B, T)
    ws = workspace(need, seq_offsets.device) if ws is None else ws.ensure(need)
    _check(lib().hstu_stochastic_length(_ptr(seq_offsets), B, T, int(max_seq_len), int(sub_len),
                                        float(n_alpha), _ptr(u), _ptr(token_keys), _ptr(new_off),
                                        _ptr(kept), ws.ptr, ws.nbytes, _stream_ptr(stream)),
           "hstu_stochastic_length")
    return new_off, kept


def gather_rows(src: torch.Tensor, index: torch.Tensor, count: Optional[torch.Tensor] = None,
                max_rows: Optional[int] = None, out: Optional[torch.Tensor] = None, stream=None):
    """out[r] = src[index[r]] for r < min(count, max_rows) (hstu_gather_rows); src 1-D or 2-D."""
    n = int(index.numel() if max_rows is None else max_rows)
    row = src.view(src.shape[0], -1)
    if out is None:
        out = torch.zeros((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    o2 = out.view(out.shape[0], -1)
    rb = row.shape[1] * row.element_size()
    _check(lib().hstu_gather_rows(_ptr(row), row.stride(0) * row.element_size(), _ptr(index),
                                  _ptr(count), n, _ptr(o2), o2.stride(0) * o2.element_size(), rb,
                                  _stream_ptr(stream)), "hstu_gather_rows")
    return out


def alibi_tables(m_p: float, m_t: float, max_pos_dist: int, num_time_buckets: int):
    """Host tables (numpy float32) that give the attention the bias -m_p (p_i - p_j) -
    m_t bucket(t_i - t_j) (exact where |p_i - p_j| <= max_pos_dist)."""
    import numpy as np
    pos = np.empty(2 * max_pos_dist + 1, dtype=np.float32)
    tim = np.empty(num_time_buckets, dtype=np.float32)
    _check(lib().hstu_alibi_tables(m_p, m_t, max_pos_dist, num_time_buckets,
                                   pos.ctypes.data_as(ctypes.c_void_p),
                                   tim.ctypes.data_as(ctypes.c_void_p)), "hstu_alibi_tables")
    return pos, tim


def debug_wait_timeout(ws: Workspace, stream=None) -> None:
    """Launch the bounded-wait probe; ws.sync_status() then reports HSTU_ERR_TIMEOUT (5)."""
    _check(lib().hstu_debug_wait_timeout(ws.ptr, ws.nbytes, _stream_ptr(stream)),
           "hstu_debug_wait_timeout")


def debug_time_buckets(dt: torch.Tensor, nb: int, stream=None) -> torch.Tensor:
    out = torch.empty(dt.shape, dtype=torch.int32, device=dt.device)
    _check(lib().hstu_debug_time_buckets(_ptr(dt), dt.numel(), _ptr(out), nb, _stream_ptr(stream)),
           "hstu_debug_time_buckets")
    return out


def debug_bias_index(rule: str, inputs: torch.Tensor, param: int, stream=None) -> torch.Tensor:
    """The attention kernels' bias-table index for each input (see hstu_debug_bias_index):
    inputs is a device int64 tensor [n] for the time rules and [n, 3] for the others."""
    code = BIAS_RULES[rule]
    n = inputs.shape[0]
    out = torch.empty(n, dtype=torch.int32, device=inputs.device)
    _check(lib().hstu_debug_bias_index(code, _ptr(inputs.contiguous()), n, param, _ptr(out),
                                       _stream_ptr(stream)), "hstu_debug_bias_index")
    return out


def jagged_to_padded(values: torch.Tensor, seq_offsets: torch.Tensor, max_len: int,
                     stream=None) -> torch.Tensor:
    B = seq_offsets.numel() - 1
    row_bytes = values.shape[1] * values.element_size()
    out = torch.empty((B, max_len, values.shape[1]), dtype=values.dtype, device=values.device)
    _check(lib().hstu_jagged_padded_copy(_ptr(seq_offsets), B, max_len, _ptr(values),
                                         values.stride(0) * values.element_size(), _ptr(out),
                                         out.stride(1) * out.element_size(), row_bytes, 1,
                                         _stream_ptr(stream)), "hstu_jagged_padded_copy")
    return out


def padded_to_jagged(padded: torch.Tensor, seq_offsets: torch.Tensor, total_tokens: int,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    B, max_len, F = padded.shape
    if out is None:
        out = torch.zeros((total_tokens, F), dtype=padded.dtype, device=padded.device)
    row_bytes = F * padded.element_size()
    _check(lib().hstu_jagged_padded_copy(_ptr(seq_offsets), B, max_len, _ptr(out),
                                         out.stride(0) * out.element_size(), _ptr(padded),
                                         padded.stride(1) * padded.element_size(), row_bytes, 0,
                                         _stream_ptr(stream)), "hstu_jagged_padded_copy")
    return out
