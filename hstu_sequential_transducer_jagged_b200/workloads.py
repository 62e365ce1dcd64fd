"""Seeded synthetic inputs for the HSTU jagged layer and attention.

This module only draws random inputs; it holds none of the method's arithmetic, so both the
CUDA path (through the binding) and the fp64 oracle can consume the very same arrays.

Every workload follows the shapes and distributions that the HSTU pages describe (jagged user
histories of varying length, Exp-distributed gaps between interactions, item/action token
interleaving, M-FALCON candidates appended to a history) with the sizes of five named
configurations:

* ``layer_fp32_b4``          one fp32 layer, 4 users, lengths U{16..128}, d_model 64, H 2, d 32
* ``layer_bf16_b32_geo``     one bf16 layer, 32 users, lengths truncated-geometric (mean 300, max 1024),
                             d_model 256, H 4, d 64
* ``attn_fwdbwd_bf16_b64``   attention forward+backward, 64 users, lengths U{512..2048}, H 8, d 64
* ``stack4_bf16_b8_inter``   4-layer bf16 stack, 8 users, lengths U{2048..8192}, d_model 512, H 8,
                             d 64, interleaved item/action tokens sharing timestamps per pair
* ``mfalcon_bf16_b16``       2-layer ranking inference, 16 users, history 4096 interleaved tokens
                             + 512 candidates (microbatch 128), d_model 512, H 8, d 64

Random streams: one ``numpy.random.SeedSequence([seed, crc32(stream name)])`` per named stream,
so adding a stream never shifts the values of another.  Values are drawn in fp64/fp32 and, for
bf16 workloads, rounded to bf16 with round-to-nearest-even; they are kept as float32 arrays whose
values are exactly representable in bf16.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional

import numpy as np

MASK_CAUSAL = 0
MASK_MFALCON = 1

# p of the truncated geometric on {1..1024} whose truncated mean is 300 (solved numerically).
TRUNC_GEO_P = 0.002729232138824755


def _rng(seed: int, stream: str) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, zlib.crc32(stream.encode())]))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding them."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    rounded = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (rounded.astype(np.uint32) << 16).view(np.float32).reshape(a.shape)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly representable in bf16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


@dataclasses.dataclass
class LayerParams:
    w1: np.ndarray            # [d_model, 2H(d_qk+d_v)]
    w2: np.ndarray            # [H d_v, d_model]
    rab_pos: np.ndarray       # fp32 [2P+1]
    rab_time: np.ndarray      # fp32 [NB]
    b1: Optional[np.ndarray] = None
    b2: Optional[np.ndarray] = None


@dataclasses.dataclass
class Workload:
    name: str
    description: str
    dtype: str                      # "fp32" or "bf16"
    lengths: np.ndarray             # int64 [B]
    seq_offsets: np.ndarray         # int32 [B+1]
    timestamps: np.ndarray          # int64 [T]
    num_heads: int
    d_qk: int
    d_v: int
    max_pos_dist: int               # P
    num_time_buckets: int           # NB
    mask: int = MASK_CAUSAL
    num_candidates: int = 0
    microbatch: int = 0
    alpha: float = 1.0
    ln_eps: float = 1e-5
    d_model: int = 0
    layers: List[LayerParams] = dataclasses.field(default_factory=list)
    x: Optional[np.ndarray] = None          # [T, d_model]
    # attention-only inputs, [T, H*d] row-major
    q: Optional[np.ndarray] = None
    k: Optional[np.ndarray] = None
    v: Optional[np.ndarray] = None
    d_o: Optional[np.ndarray] = None
    rab_pos: Optional[np.ndarray] = None
    rab_time: Optional[np.ndarray] = None

    @property
    def num_seqs(self) -> int:
        return int(self.lengths.shape[0])

    @property
    def total_tokens(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def max_seq_len(self) -> int:
        return int(self.lengths.max()) if self.lengths.size else 0


def offsets_from_lengths(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(np.asarray(lengths, dtype=np.int64), out=off[1:])
    return off.astype(np.int32)


def _gaps(rng: np.random.Generator, n: int, mean_s: float = 600.0) -> np.ndarray:
    return rng.exponential(mean_s, size=n)


def timestamps_plain(rng: np.random.Generator, lengths: np.ndarray) -> np.ndarray:
    """t_0 = 0, t_k = floor(sum of the first k Exp(600 s) gaps), per sequence."""
    out = []
    for L in lengths:
        g = _gaps(rng, int(L))
        g[0] = 0.0
        out.append(np.floor(np.cumsum(g)).astype(np.int64))
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def timestamps_interleaved(rng: np.random.Generator, lengths: np.ndarray) -> np.ndarray:
    """Item token 2k and action token 2k+1 share one timestamp; gaps are drawn per pair."""
    out = []
    for L in lengths:
        pairs = (int(L) + 1) // 2
        g = _gaps(rng, pairs)
        g[0] = 0.0
        tp = np.floor(np.cumsum(g)).astype(np.int64)
        out.append(np.repeat(tp, 2)[: int(L)])
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def _normal(rng, shape, std, bf16: bool) -> np.ndarray:
    a = (rng.standard_normal(size=shape) * std).astype(np.float32)
    return round_to_bf16(a) if bf16 else a


def _layer(seed: int, l: int, d_model: int, H: int, dqk: int, dv: int, P: int, NB: int,
           bf16: bool, table_std: float = 0.02) -> LayerParams:
    n1 = 2 * H * (dqk + dv)
    return LayerParams(
        w1=_normal(_rng(seed, f"w1/{l}"), (d_model, n1), 0.02, bf16),
        w2=_normal(_rng(seed, f"w2/{l}"), (H * dv, d_model), 0.02, bf16),
        rab_pos=_normal(_rng(seed, f"rab_pos/{l}"), (2 * P + 1,), table_std, False),
        rab_time=_normal(_rng(seed, f"rab_time/{l}"), (NB,), table_std, False),
    )


def truncated_geometric(rng: np.random.Generator, n: int, p: float = TRUNC_GEO_P,
                        max_len: int = 1024) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    filled = 0
    while filled < n:
        draw = rng.geometric(p, size=2 * (n - filled) + 8)
        draw = draw[draw <= max_len]
        take = min(len(draw), n - filled)
        out[filled:filled + take] = draw[:take]
        filled += take
    return out


def make_layer_fp32_b4(seed: int = 0) -> Workload:
    B, d_model, H, d, P, NB = 4, 64, 2, 32, 128, 128
    lengths = _rng(seed, "lengths").integers(16, 128, size=B, endpoint=True)
    T = int(lengths.sum())
    return Workload(
        name="layer_fp32_b4",
        description="one fp32 HSTU layer; B=4, L~U{16..128}, d_model=64, H=2, d_qk=d_v=32, P=128, NB=128",
        dtype="fp32", lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
        timestamps=timestamps_plain(_rng(seed, "gaps"), lengths),
        num_heads=H, d_qk=d, d_v=d, max_pos_dist=P, num_time_buckets=NB, d_model=d_model,
        layers=[_layer(seed, 0, d_model, H, d, d, P, NB, bf16=False)],
        x=_normal(_rng(seed, "x"), (T, d_model), 1.0, False))


def make_layer_bf16_b32_geo(seed: int = 0) -> Workload:
    B, d_model, H, d, P, NB = 32, 256, 4, 64, 1024, 128
    lengths = truncated_geometric(_rng(seed, "lengths"), B)
    T = int(lengths.sum())
    return Workload(
        name="layer_bf16_b32_geo",
        description="one bf16 HSTU layer; B=32, L~truncated geometric (mean 300, max 1024), "
                    "d_model=256, H=4, d_qk=d_v=64, P=1024, NB=128",
        dtype="bf16", lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
        timestamps=timestamps_plain(_rng(seed, "gaps"), lengths),
        num_heads=H, d_qk=d, d_v=d, max_pos_dist=P, num_time_buckets=NB, d_model=d_model,
        layers=[_layer(seed, 0, d_model, H, d, d, P, NB, bf16=True)],
        x=_normal(_rng(seed, "x"), (T, d_model), 1.0, True))


def make_attn_fwdbwd_bf16_b64(seed: int = 0, B: int = 64, lo: int = 512, hi: int = 2048) -> Workload:
    H, d, P, NB = 8, 64, 1024, 128
    lengths = _rng(seed, "lengths").integers(lo, hi, size=B, endpoint=True)
    T = int(lengths.sum())
    return Workload(
        name="attn_fwdbwd_bf16_b64",
        description=f"attention-only forward+backward, bf16; B={B}, L~U{{{lo}..{hi}}}, H=8, "
                    "d_qk=d_v=64, P=1024, NB=128, Q/K/V/dO ~ N(0,1)",
        dtype="bf16", lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
        timestamps=timestamps_plain(_rng(seed, "gaps"), lengths),
        num_heads=H, d_qk=d, d_v=d, max_pos_dist=P, num_time_buckets=NB,
        q=_normal(_rng(seed, "q"), (T, H * d), 1.0, True),
        k=_normal(_rng(seed, "k"), (T, H * d), 1.0, True),
        v=_normal(_rng(seed, "v"), (T, H * d), 1.0, True),
        d_o=_normal(_rng(seed, "d_o"), (T, H * d), 1.0, True),
        rab_pos=_normal(_rng(seed, "rab_pos/0"), (2 * P + 1,), 0.02, False),
        rab_time=_normal(_rng(seed, "rab_time/0"), (NB,), 0.02, False))


def make_stack4_bf16_b8_inter(seed: int = 0, B: int = 8, lo: int = 2048, hi: int = 8192,
                              num_layers: int = 4) -> Workload:
    d_model, H, d, P, NB = 512, 8, 64, 1024, 128
    lengths = _rng(seed, "lengths").integers(lo, hi, size=B, endpoint=True)
    T = int(lengths.sum())
    return Workload(
        name="stack4_bf16_b8_inter",
        description=f"{num_layers}-layer bf16 HSTU stack forward; B={B}, L~U{{{lo}..{hi}}}, "
                    "d_model=512, H=8, d_qk=d_v=64, P=1024, NB=128, interleaved item/action "
                    "tokens sharing one timestamp per pair",
        dtype="bf16", lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
        timestamps=timestamps_interleaved(_rng(seed, "gaps"), lengths),
        num_heads=H, d_qk=d, d_v=d, max_pos_dist=P, num_time_buckets=NB, d_model=d_model,
        layers=[_layer(seed, l, d_model, H, d, d, P, NB, bf16=True) for l in range(num_layers)],
        x=_normal(_rng(seed, "x"), (T, d_model), 1.0, True))


def make_mfalcon_bf16_b16(seed: int = 0, B: int = 16, n_hist: int = 4096, m: int = 512,
                          microbatch: int = 128, num_layers: int = 2) -> Workload:
    d_model, H, d, P, NB = 512, 8, 64, 1024, 128
    lengths = np.full(B, n_hist + m, dtype=np.int64)
    hist_ts = timestamps_interleaved(_rng(seed, "gaps"), np.full(B, n_hist, np.int64))
    ts = []
    for b in range(B):
        h = hist_ts[b * n_hist:(b + 1) * n_hist]
        ts.append(np.concatenate([h, np.full(m, h[-1], np.int64)]))
    T = int(lengths.sum())
    return Workload(
        name="mfalcon_bf16_b16",
        description=f"M-FALCON ranking inference, bf16, {num_layers} layers; B={B}, history "
                    f"{n_hist} interleaved tokens + {m} candidates (microbatch {microbatch}), "
                    "d_model=512, H=8, d_qk=d_v=64, P=1024, NB=128",
        dtype="bf16", lengths=lengths, seq_offsets=offsets_from_lengths(lengths),
        timestamps=np.concatenate(ts), num_heads=H, d_qk=d, d_v=d, max_pos_dist=P,
        num_time_buckets=NB, mask=MASK_MFALCON, num_candidates=m, microbatch=microbatch,
        d_model=d_model,
        layers=[_layer(seed, l, d_model, H, d, d, P, NB, bf16=True) for l in range(num_layers)],
        x=_normal(_rng(seed, "x"), (T, d_model), 1.0, True))


WORKLOADS = {
    "layer_fp32_b4": make_layer_fp32_b4,
    "layer_bf16_b32_geo": make_layer_bf16_b32_geo,
    "attn_fwdbwd_bf16_b64": make_attn_fwdbwd_bf16_b64,
    "stack4_bf16_b8_inter": make_stack4_bf16_b8_inter,
    "mfalcon_bf16_b16": make_mfalcon_bf16_b16,
}


def make(name: str, seed: int = 0, **kw) -> Workload:
    return WORKLOADS[name](seed=seed, **kw)


def random_attention_case(seed: int, lengths, H: int, d: int, P: int = 16, NB: int = 16,
                          mask: int = MASK_CAUSAL, num_candidates: int = 0,
                          qkv_std: float = 1.0, table_std: float = 0.5, bf16: bool = True,
                          interleaved: bool = False, gap_mean: float = 600.0) -> Workload:
    """Small attention-only case with large bias tables so that the bias path matters."""
    lengths = np.asarray(lengths, dtype=np.int64)
    T = int(lengths.sum())
    rng_t = _rng(seed, "gaps")
    if interleaved:
        ts = timestamps_interleaved(rng_t, lengths)
    else:
        ts_list = []
        for L in lengths:
            g = rng_t.exponential(gap_mean, size=int(L))
            if L:
                g[0] = 0.0
            ts_list.append(np.floor(np.cumsum(g)).astype(np.int64))
        ts = np.concatenate(ts_list) if ts_list else np.zeros(0, np.int64)
    if mask == MASK_MFALCON and num_candidates > 0:
        # candidates carry the last history timestamp
        off = offsets_from_lengths(lengths)
        for b in range(len(lengths)):
            s, e = int(off[b]), int(off[b + 1])
            n = e - s - num_candidates
            if n > 0:
                ts[s + n:e] = ts[s + n - 1]
    return Workload(
        name="random_attention_case", description="small synthetic attention case",
        dtype="bf16" if bf16 else "fp32", lengths=lengths,
        seq_offsets=offsets_from_lengths(lengths), timestamps=ts, num_heads=H, d_qk=d, d_v=d,
        max_pos_dist=P, num_time_buckets=NB, mask=mask, num_candidates=num_candidates,
        microbatch=128 if mask == MASK_MFALCON else 0,
        q=_normal(_rng(seed, "q"), (T, H * d), qkv_std, bf16),
        k=_normal(_rng(seed, "k"), (T, H * d), qkv_std, bf16),
        v=_normal(_rng(seed, "v"), (T, H * d), qkv_std, bf16),
        d_o=_normal(_rng(seed, "d_o"), (T, H * d), 1.0, bf16),
        rab_pos=_normal(_rng(seed, "rab_pos/0"), (2 * P + 1,), table_std, False),
        rab_time=_normal(_rng(seed, "rab_time/0"), (NB,), table_std, False))


def random_layer_case(seed: int, lengths, d_model: int, H: int, d: int, P: int = 16,
                      NB: int = 16, mask: int = MASK_CAUSAL, num_candidates: int = 0,
                      bf16: bool = True, num_layers: int = 1, w_std: float = 0.05,
                      table_std: float = 0.5) -> Workload:
    lengths = np.asarray(lengths, dtype=np.int64)
    T = int(lengths.sum())
    base = random_attention_case(seed, lengths, H, d, P, NB, mask, num_candidates, bf16=bf16)
    layers = []
    for l in range(num_layers):
        lp = _layer(seed, l, d_model, H, d, d, P, NB, bf16=bf16, table_std=table_std)
        lp.w1 = _normal(_rng(seed, f"w1s/{l}"), lp.w1.shape, w_std, bf16)
        lp.w2 = _normal(_rng(seed, f"w2s/{l}"), lp.w2.shape, w_std, bf16)
        layers.append(lp)
    base.q = base.k = base.v = base.d_o = None
    base.rab_pos = base.rab_time = None
    base.d_model = d_model
    base.layers = layers
    base.x = _normal(_rng(seed, "x"), (T, d_model), 1.0, bf16)
    base.name = "random_layer_case"
    return base
