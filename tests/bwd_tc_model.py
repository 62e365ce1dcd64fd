"""A CPU model of the data movement of csrc/attn_bwd_tc.cu (the tensor-core attention backward).

It restates, in NumPy, what the kernel's threads and asynchronous units do to shared memory and
tensor memory, using the kernel's own address arithmetic:
  * TMA box loads with the 128-byte swizzle (16-byte chunk c of row r stored at c ^ (r mod 8));
  * the operands that tcgen05.mma reads through shared-memory descriptors, decoded with the
    canonical SW128 layouts (K-major: 8-row groups SBO apart; MN-major: 64-element atoms LBO
    apart along M/N and 8-row groups SBO apart along K);
  * tensor-memory operands (packed bf16 pairs, low half = even K index) and accumulators;
  * the epilogue's chunk classes, P / dS formation, and its stores of P^T, (alpha dS)^T and the
    swizzled dS tile; the dQ drain; the bias-gradient runs.
Run over a small case one CTA at a time, it must reproduce the oracle's gradients within the
parity tolerance.  It checks the layout design (which operand lands where); the kernel's parity
on hardware is checked by the GPU tests.  The `knobs` let a test plant a layout mistake and see
the model fail.
"""
import numpy as np

from oracle import hstu_oracle as O
from hstu_sequential_transducer_jagged_b200 import workloads as W

kD, kT, kTileBytes = 64, 128, 128 * 64 * 2


def bf16_bits(a):
    a = np.asarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF).astype(np.uint16)


def bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def swz(addr):
    addr = np.asarray(addr, dtype=np.int64)
    return addr ^ (((addr >> 7) & 7) << 4)


class Smem:
    def __init__(self, nbytes):
        self.b = np.zeros(nbytes, dtype=np.uint8)

    def write_u16(self, addr, vals):  # addr: byte addresses (array), vals: uint16 array
        v = np.asarray(vals, dtype=np.uint16).view(np.uint8).reshape(-1, 2)
        a = np.asarray(addr, dtype=np.int64).reshape(-1)
        self.b[a] = v[:, 0]
        self.b[a + 1] = v[:, 1]

    def read_u16(self, addr):
        a = np.asarray(addr, dtype=np.int64)
        return (self.b[a].astype(np.uint16) | (self.b[a + 1].astype(np.uint16) << 8))


def tma_load_sw128(sm, base, tile_bits):
    """A {64 x R} bf16 box written with the 128-byte swizzle (base 1024-aligned)."""
    R = tile_bits.shape[0]
    r, c = np.meshgrid(np.arange(R), np.arange(64), indexing="ij")
    logical = base + r * 128 + c * 2
    sm.write_u16(swz(logical), tile_bits)


def decode_kmajor(sm, start, MN, SBO):
    """Canonical SW128 K-major operand, K = 16 bf16: element (mn, k)."""
    mn, k = np.meshgrid(np.arange(MN), np.arange(16), indexing="ij")
    logical = start + (mn % 8) * 128 + (mn // 8) * SBO + k * 2
    return bits_to_f32(sm.read_u16(swz(logical)))


def decode_mnmajor(sm, start, MN, LBO, SBO):
    """Canonical SW128 MN-major operand, K = 16: element (mn, k)."""
    mn, k = np.meshgrid(np.arange(MN), np.arange(16), indexing="ij")
    logical = start + (k % 8) * 128 + (k // 8) * SBO + (mn % 64) * 2 + (mn // 64) * LBO
    return bits_to_f32(sm.read_u16(swz(logical)))


class Tmem:
    def __init__(self):
        self.w = np.zeros((128, 512), dtype=np.uint32)

    def f32(self, lanes, col, n):
        return self.w[lanes, col:col + n].view(np.float32)


def mma(tm, dcol, A, B, acc):  # A: M x K, B: N x K, D[m][n] at lanes m, columns dcol + n
    D = (A.astype(np.float64) @ B.astype(np.float64).T).astype(np.float32)
    M, N = D.shape
    cur = tm.w[:M, dcol:dcol + N].view(np.float32)
    out = (cur + D) if acc else D
    tm.w[:M, dcol:dcol + N] = out.astype(np.float32).view(np.uint32)


def tmem_a(tm, acol, M=128):
    """TS A operand, K = 16 bf16 from 8 columns: element k in column acol + k // 2, half k % 2."""
    w = tm.w[:M, acol:acol + 8]
    lo = (w & 0xFFFF).astype(np.uint16)
    hi = (w >> 16).astype(np.uint16)
    A = np.empty((M, 16), dtype=np.float32)
    A[:, 0::2] = bits_to_f32(lo)
    A[:, 1::2] = bits_to_f32(hi)
    return A


def pack(lo, hi):
    return (bf16_bits(lo).astype(np.uint32) | (bf16_bits(hi).astype(np.uint32) << 16))


def time_bucket64(dt, nb):
    return O.time_bucket(np.asarray(dt, dtype=np.int64), nb)


def chunk_class(i0, j0, L, n, P, NB, tq_c, tj, jvalid, tabp, tabt, use_pos=True,
                use_time=True):
    """The epilogue's class of the block of queries i0 .. i0+31 and keys j0 .. j0+31 (as in the
    kernel's chunk_class): ("zero" | "const" | "timeconst" | "general", constant bias, position
    bin, time bucket)."""
    j1 = j0 + 31
    if i0 >= L or j0 >= L or i0 + 31 < j0:
        return "zero", np.float32(0), 0, 0
    if not (i0 >= j1 and i0 + 31 < L and j1 < n):
        return "general", np.float32(0), 0, 0
    tterm, ctidx = np.float32(0), 0
    if use_time:
        tj_lo, tj_hi = tj[jvalid].min(), tj[jvalid].max()
        b_lo = int(time_bucket64(tq_c[:32].min() - tj_hi, NB))
        b_hi = int(time_bucket64(tq_c[:32].max() - tj_lo, NB))
        if b_lo != b_hi:
            return "general", np.float32(0), 0, 0
        ctidx, tterm = b_lo, tabt[b_lo]
    if use_pos:
        if min(i0, n) - j1 < P:
            return "timeconst", np.float32(tterm), 0, ctidx
        return "const", np.float32(tabp[2 * P] + tterm), 2 * P, ctidx
    return "const", np.float32(tterm), 0, ctidx


DEFAULT_KNOBS = dict(ds_swizzle=True, dq_lbo=kTileBytes, split_pc=True, p_col_step=32)


def run(case, fast, knobs=None):
    kn = dict(DEFAULT_KNOBS, **(knobs or {}))
    H = case.num_heads
    T = case.q.shape[0]
    q = bf16_bits(case.q).reshape(T, H, kD)
    k = bf16_bits(case.k).reshape(T, H, kD)
    v = bf16_bits(case.v).reshape(T, H, kD)
    do = bf16_bits(case.d_o).reshape(T, H, kD)
    off = case.seq_offsets
    ts = case.timestamps.astype(np.int64)
    P, NB, alpha = case.max_pos_dist, case.num_time_buckets, np.float32(case.alpha)
    tabp = case.rab_pos.astype(np.float32)
    tabt = case.rab_time.astype(np.float32)
    npos = 2 * P + 1
    bins = np.zeros(npos + NB, dtype=np.float32)
    dq_acc = np.zeros((T, H * kD), dtype=np.float32)
    dk_out = np.zeros((T, H * kD), dtype=np.float32)
    dv_out = np.zeros((T, H * kD), dtype=np.float32)
    # smem layout as in BwdSmem: k, v, q[2], dO[2], ds[2 tiles]
    K_B, V_B, Q_B, DO_B, DS_B = 0, kTileBytes, 2 * kTileBytes, 4 * kTileBytes, 6 * kTileBytes
    sm = Smem(8 * kTileBytes + 4096)
    tm = Tmem()
    kColST, kColDPT, kColDV, kColDK, kColDQ = 0, 128, 256, 320, 384
    # work list: one item per (sequence, 128-row tile); the kernel walks it in reverse
    items = []
    for b in range(len(off) - 1):
        L = int(off[b + 1] - off[b])
        for t in range((L + kT - 1) // kT):
            items.append((b, t, int(off[b]), L))
    items = items[::-1]

    def rows(tensor, r0, head):  # 128 rows from r0 (zero fill past T), one head
        out = np.zeros((kT, kD), dtype=np.uint16)
        n = max(0, min(kT, T - r0))
        if n > 0:
            out[:n] = tensor[r0:r0 + n, head]
        return out

    runs = {"p": [-1, np.float32(0)], "t": [-1, np.float32(0)]}

    def run_add(key, base, idx, val):
        r = runs[key]
        if idx != r[0]:
            if r[0] >= 0:
                bins[base + r[0]] += r[1]
            r[0], r[1] = idx, np.float32(0)
        r[1] = np.float32(r[1] + val)

    for (b, kt, row0, L) in items:
        n = max(L - case.num_candidates, 0) if case.mask == W.MASK_MFALCON else L  # history
        nt = (L + kT - 1) // kT
        for head in range(H):
            tma_load_sw128(sm, K_B, rows(k, row0 + kt * kT, head))
            tma_load_sw128(sm, V_B, rows(v, row0 + kt * kT, head))
            first_item_step = True
            for qt in range(kt, nt):
                r0 = row0 + qt * kT
                st = 0  # stage choice does not matter sequentially
                tma_load_sw128(sm, Q_B, rows(q, r0, head))
                tma_load_sw128(sm, DO_B, rows(do, r0, head))
                tq = np.zeros(kT + 2, dtype=np.int64)
                x0 = r0 & ~1
                nn = max(0, min(130, T - x0))
                tq[:nn] = ts[x0:x0 + nn]
                tq = tq[(r0 & 1):]
                # S^T = K Q^T, dP^T = V dO^T
                for kk in range(4):
                    mma(tm, kColST, decode_kmajor(sm, K_B + kk * 32, 128, 1024),
                        decode_kmajor(sm, Q_B + kk * 32, 128, 1024), kk > 0)
                    mma(tm, kColDPT, decode_kmajor(sm, V_B + kk * 32, 128, 1024),
                        decode_kmajor(sm, DO_B + kk * 32, 128, 1024), kk > 0)
                # epilogue: warps (quad, hq)
                for hq in range(2):
                    for quad in range(4):
                        lanes = quad * 32 + np.arange(32)
                        j0 = kt * kT + quad * 32
                        jrow = j0 + np.arange(32)
                        jvalid = jrow < L
                        pj = np.minimum(jrow, n)
                        tj = np.where(jvalid, ts[np.minimum(row0 + jrow, T - 1)], 0)
                        for ch in range(2):
                            col = 64 * hq + 32 * ch
                            i0 = qt * kT + col
                            tq_c = tq[col:col + 32]
                            cls, cbias, cpidx, ctidx = "general", np.float32(0), 0, 0
                            if fast:
                                cls, cbias, cpidx, ctidx = chunk_class(i0, j0, L, n, P, NB, tq_c,
                                                                       tj, jvalid, tabp, tabt)
                            if cls == "zero":
                                pk = np.zeros((32, 16), dtype=np.uint32)
                                dk_ = np.zeros((32, 16), dtype=np.uint32)
                            else:
                                s = tm.f32(lanes, kColST + col, 32)
                                dp = tm.f32(lanes, kColDPT + col, 32)
                                pv = np.zeros((32, 32), dtype=np.float32)
                                dsa = np.zeros((32, 32), dtype=np.float32)
                                csum = np.zeros(32, dtype=np.float32)
                                for e in range(32):
                                    i = i0 + e
                                    if cls == "const":
                                        bias = np.full(32, cbias, dtype=np.float32)
                                    else:
                                        pi = min(i, n)
                                        d = np.clip(pi - pj, -P, P)
                                        pidx = d + P
                                        bias = np.float32(0) + tabp[pidx]
                                        if cls == "timeconst":
                                            bias = (bias + cbias).astype(np.float32)
                                        else:
                                            bidx = time_bucket64(tq_c[e] - tj, NB)
                                            bias = (bias + tabt[bidx]).astype(np.float32)
                                    x = (alpha * s[:, e] + bias).astype(np.float32)
                                    sg = (np.float32(0.5) * np.tanh(np.float32(0.5) * x) + np.float32(0.5)).astype(np.float32)
                                    p = (x * sg).astype(np.float32)
                                    dsv = (dp[:, e] * sg * (x * (1 - sg) + 1)).astype(np.float32)
                                    if cls == "general":
                                        vis = jvalid & (i < L) & (jrow <= i) & ((jrow < n) | (jrow == i))
                                        p = np.where(vis, p, 0)
                                        dsv = np.where(vis, dsv, 0).astype(np.float32)
                                        for l in range(32):
                                            if vis[l]:
                                                run_add("p", 0, int(pidx[l]), dsv[l])
                                                run_add("t", npos, int(bidx[l]), dsv[l])
                                    else:
                                        if cls == "timeconst":
                                            for l in range(32):
                                                run_add("p", 0, int(pidx[l]), dsv[l])
                                        csum = (csum + dsv).astype(np.float32)
                                    pv[:, e] = p
                                    dsa[:, e] = alpha * dsv
                                if cls == "const":
                                    for l in range(32):
                                        run_add("p", 0, cpidx, csum[l])
                                if cls != "general":
                                    for l in range(32):
                                        run_add("t", npos, ctidx, csum[l])
                                pk = pack(pv[:, 0::2], pv[:, 1::2])
                                dk_ = pack(dsa[:, 0::2], dsa[:, 1::2])
                            # TMEM stores: 16 columns at the chunk's own first columns, 64 hq + 32 ch
                            pcol = kColST + 64 * hq + kn['p_col_step'] * ch
                            tm.w[lanes, pcol:pcol + 16] = pk
                            tm.w[lanes, kColDPT + 64 * hq + 32 * ch:kColDPT + 64 * hq + 32 * ch + 16] = dk_
                            # dS row to shared memory: chunk (4 ch + cc) at (chunk ^ (rr & 7)) * 16
                            rr = quad * 32 + np.arange(32)
                            ds_row = DS_B + hq * kTileBytes + rr * 128
                            for cc in range(4):
                                chunk = 4 * ch + cc
                                words = dk_[:, 4 * cc:4 * cc + 4]  # 4 u32 = 8 bf16 per lane
                                halves = np.stack([words & 0xFFFF, words >> 16], axis=-1).reshape(32, 8).astype(np.uint16)
                                pos = (chunk ^ (rr & 7)) if kn['ds_swizzle'] else np.full(32, chunk)
                                addr = (ds_row + pos * 16)[:, None] + 2 * np.arange(8)[None, :]
                                sm.write_u16(addr, halves)
                # dV += P^T dO, dK += (a dS)^T Q  (TS; B MN-major, LBO = tile bytes)
                for kk in range(8):
                    pc = (32 * (kk >> 1) + 8 * (kk & 1)) if kn['split_pc'] else 8 * kk
                    acc = (not first_item_step) or kk > 0
                    mma(tm, kColDV, tmem_a(tm, kColST + pc),
                        decode_mnmajor(sm, DO_B + kk * 2048, 64, kTileBytes, 1024), acc)
                    mma(tm, kColDK, tmem_a(tm, kColDPT + pc),
                        decode_mnmajor(sm, Q_B + kk * 2048, 64, kTileBytes, 1024), acc)
                # dQ = (a dS) K  (A and B MN-major)
                for kk in range(8):
                    mma(tm, kColDQ, decode_mnmajor(sm, DS_B + kk * 2048, 128, kn['dq_lbo'], 1024),
                        decode_mnmajor(sm, K_B + kk * 2048, 64, kTileBytes, 1024), kk > 0)
                # drain
                dqt = tm.f32(np.arange(128), kColDQ, 64)
                for r in range(128):
                    i = qt * kT + r
                    if i < L:
                        dq_acc[row0 + i, head * kD:(head + 1) * kD] += dqt[r]
                first_item_step = False
            # the item's dV, dK
            dvt, dkt = tm.f32(np.arange(128), kColDV, 64), tm.f32(np.arange(128), kColDK, 64)
            for r in range(128):
                j = kt * kT + r
                if j < L:
                    dv_out[row0 + j, head * kD:(head + 1) * kD] = dvt[r]
                    dk_out[row0 + j, head * kD:(head + 1) * kD] = dkt[r]
    for key, base in (("p", 0), ("t", npos)):
        r = runs[key]
        if r[0] >= 0:
            bins[base + r[0]] += r[1]
    return dq_acc, dk_out, dv_out, bins[:npos], bins[npos:]
