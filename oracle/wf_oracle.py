"""CPU oracle for one Wave Forcing wave round -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import or run this module.  The product path (the CUDA
library and its binding) never calls it, and it shares no code with that path.

Plain, slow, obviously-correct NumPy in fp64 with an explicit visibility mask.
What it follows:

* Chunk-wise causal attention over earlier, cleaner chunks whose denoising is
  not finished ("Wave Forcing: Towards Speed-of-Light Streaming Video
  Generation", arXiv 2611.00859v1, Abstract), i.e. a new chunk conditions on a
  mixed-noise frontier and not only on a clean prior chunk ("Wave Forcing from
  SJTU-DENG Lab: 8 GPUs can't fix a missing sgl-dlab package", first
  paragraph).
* KV-cached chunk-autoregressive generation where the finished chunk's K/V are
  written into the cache ("scope-causal-forcing", "How It Works", steps 1-2);
  the denoising list [1000, 750, 500, 250] ("scope-causal-forcing",
  "Configuration" table) supplies the in-round noise levels.

Readings where the pages are silent (each is a parameter or a stated choice):

* Mask: chunk i sees every cache chunk, the in-round chunks j <= i and all of
  its own tokens (bidirectional inside a chunk); all in-round chunks share the
  same cache window.
* Age order: in-round index 0 is the oldest and cleanest chunk; noise levels
  are metadata that never enter the attention arithmetic.
* 3D RoPE (not on the pages): textbook rotary embedding (Su et al., RoFormer,
  2021) applied per axis to interleaved (even, odd) pairs; pairs split into
  consecutive groups P_t | P_h | P_w; frequency of pair k in a group of P pairs
  is theta^(-k/P); positions are absolute from stream start (t = n*F + f).
  Default split: P_h = P_w = floor((D/2)/3), P_t = D/2 - 2*P_h.
* Ring: slot(n) = n mod S over S pool slots; the cache holds the last Wc
  chunks before the round's oldest in-round chunk n0.
* Scale 1/sqrt(D); rotated Q/K rounded to the storage type (nearest, ties to
  even) from the fp64 rotation; attention itself in fp64.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

KEY_TILE = 128
Q_TILE = 128
Q_PAIR = 256


# --------------------------------------------------------------------------
# rounding to the storage types
# --------------------------------------------------------------------------

def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), kept in fp64.

    bf16 keeps 8 significant bits and the fp32 exponent range: for
    x = m * 2^e (0.5 <= |m| < 1) the spacing of bf16 values is 2^(e-8) for
    normal results and the fixed subnormal spacing 2^-133 below 2^-126.
    Scaling by a power of two and np.rint (ties to even) are exact.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    q_exp = np.maximum(e.astype(np.int64) - 8, -133)
    q = np.ldexp(x, -q_exp)
    r = np.ldexp(np.rint(q), q_exp)
    big = np.abs(r) > 3.3895313892515355e38  # largest finite bf16
    return np.where(big, np.copysign(np.inf, x), r)


def round_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(x, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "f32":
        return round_f32(x)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# token geometry and 3D RoPE
# --------------------------------------------------------------------------

def chunk_len(F: int, fh: int, fw: int) -> int:
    return F * fh * fw


def token_positions(n: int, F: int, fh: int, fw: int):
    """(t, h, w) of every token of global chunk n; tokens are (frame, row, col)."""
    j = np.arange(F * fh * fw)
    f = j // (fh * fw)
    l = j % (fh * fw)
    return n * F + f, l // fw, l % fw


def rope_split(D: int):
    ph = (D // 2) // 3
    return D // 2 - 2 * ph, ph, ph


def rope_angles(t, h, w, pairs, theta: float) -> np.ndarray:
    """Angles [tokens, D/2]: each axis' positions times theta^(-k/P) for its group."""
    cols = []
    for pos, P in zip((t, h, w), pairs):
        if P == 0:
            continue
        k = np.arange(P)
        freq = np.float64(theta) ** (-k / P)
        cols.append(np.asarray(pos, dtype=np.float64)[:, None] * freq[None, :])
    return np.concatenate(cols, axis=1)


def rope_rotate(x, angles) -> np.ndarray:
    """Rotate interleaved pairs of x [tokens, ..., D] by angles [tokens, D/2] (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    a = angles.reshape(angles.shape[0], *([1] * (x.ndim - 2)), angles.shape[1])
    c, s = np.cos(a), np.sin(a)
    ev, od = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = ev * c - od * s
    out[..., 1::2] = ev * s + od * c
    return out


def rope3d_chunk(x, n: int, F: int, fh: int, fw: int, pairs, theta: float) -> np.ndarray:
    """Exact (fp64) 3D RoPE of chunk n's tensor x [C, H, D]."""
    t, h, w = token_positions(n, F, fh, fw)
    return rope_rotate(x, rope_angles(t, h, w, pairs, theta))


# --------------------------------------------------------------------------
# ring cache
# --------------------------------------------------------------------------

def ring_slot(n: int, S: int) -> int:
    return n % S


def cache_window(n0: int, Wc: int):
    """Global indices of the clean cache chunks seen by the round starting at n0."""
    return list(range(max(0, n0 - Wc), n0))


def ring_contents_after(appends, S: int):
    """Simulate appends of global chunk ids into an S-slot ring; slot -> chunk id."""
    slots = [None] * S
    for n in appends:
        slots[ring_slot(n, S)] = n
    return slots


# --------------------------------------------------------------------------
# plan re-derivation (visibility, slots, segments, work list)
# --------------------------------------------------------------------------

MAX_KEY_PARTS = 8     # most parts a unit's key tiles are shared over
MIN_PART_TILES = 8    # fewest key tiles per part in the round's smallest chunk


def key_parts(units_unsplit: int, num_ctas: int, tiles_min: int, split: bool) -> int:
    """Number of parts each unit's key tiles are shared over.  1 without
    `split` (fp32 plans) or with two or more units per bin; otherwise the p
    (at most MAX_KEY_PARTS, each part at least MIN_PART_TILES tiles of the
    smallest chunk) minimising the bin filling ceil(U*p/G) / (U*p/G) plus 1%
    per extra part; ties to fewer parts."""
    best_p, best = 1, None
    for p in range(1, MAX_KEY_PARTS + 1):
        if p > 1 and (not split or units_unsplit >= 2 * num_ctas or tiles_min < MIN_PART_TILES * p):
            break
        up = units_unsplit * p
        score = Fraction(-(-up // num_ctas) * num_ctas, up) + Fraction(p - 1, 100)
        if best is None or score < best:
            best_p, best = p, score
    return best_p


def balance(costs, num_bins: int):
    """Share items with the given costs out over num_bins bins.

    Longest first: the items, ordered by cost (largest first; equal costs keep
    their given order), each go to the bin with the smallest load (the lowest
    bin index on equal loads).  Then, up to 5000 times: take the heaviest bin h
    (lowest index on equal loads) and look at the other bins from the lightest
    (lowest index on equal loads), stopping at the first bin that is not
    lighter than h.  In a bin b, for each item x of h in its order: moving x
    to b gives the larger load max(L_h - c_x, L_b + c_x); for each item y of b
    in its order with c_y < c_x, swapping them gives max(L_h - d, L_b + d),
    d = c_x - c_y.  A change counts if that value is below L_h; the best one
    is the smallest value, ties going to the first found (move of x before
    the swaps of x).  The first bin b offering any change is used: x leaves h
    (and y, for a swap, leaves b); the arriving items are appended to the end
    of their new bin's list.  Stop when no bin offers a change.

    Returns (bins, loads): per bin the list of item indices in order, and
    the bins' total costs."""
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    loads = [0] * num_bins
    bins = [[] for _ in range(num_bins)]
    for i in order:
        c = min(range(num_bins), key=lambda k: (loads[k], k))
        bins[c].append(i)
        loads[c] += costs[i]
    for _ in range(5000):
        h = max(range(num_bins), key=lambda k: (loads[k], -k))
        best = None
        for b in sorted(range(num_bins), key=lambda k: (loads[k], k)):
            if b == h:
                continue
            if loads[b] >= loads[h]:
                break
            for xi, x in enumerate(bins[h]):
                mv = max(loads[h] - costs[x], loads[b] + costs[x])
                if mv < loads[h] and (best is None or mv < best[0]):
                    best = (mv, b, xi, None)
                for yi, y in enumerate(bins[b]):
                    d = costs[x] - costs[y]
                    if d <= 0:
                        continue
                    sw = max(loads[h] - d, loads[b] + d)
                    if sw < loads[h] and (best is None or sw < best[0]):
                        best = (sw, b, xi, yi)
            if best is not None:
                break
        if best is None:
            break
        _, b, xi, yi = best
        x = bins[h].pop(xi)
        loads[h] -= costs[x]
        if yi is not None:
            y = bins[b].pop(yi)
            loads[b] -= costs[y]
            bins[h].append(y)
            loads[h] += costs[y]
        bins[b].append(x)
        loads[b] += costs[x]
    return bins, loads


def plan_round(H, D, fh, fw, F, Wc, R, S, n0, noise_t, num_ctas, split=None):
    """Re-derive the round plan: per-chunk visibility/slots and the LPT work list.
    split: share units' keys over several parts when units are few (default:
    for the 16-bit path, D = 128)."""
    C = F * fh * fw
    wc_eff = min(Wc, n0)
    first = n0 - wc_eff
    chunks = []
    for i in range(R):
        n = n0 + i
        nvis = wc_eff + i + 1
        vis = [first + k for k in range(nvis)]
        s0 = first % S
        len0 = min(nvis, S - s0)
        segs = [(s0 * C, len0 * C), (0, (nvis - len0) * C)]
        tiles = sum(-(-ln // KEY_TILE) for _, ln in segs)
        chunks.append(dict(n=n, slot=n % S, noise=int(noise_t[i]), nvis=nvis,
                           vis_chunks=vis, vis_slots=[v % S for v in vis],
                           keys=nvis * C, segs=segs, key_tiles=tiles))
    pairs = -(-C // Q_PAIR)
    split = (D == 128) if split is None else split
    P = key_parts(R * H * pairs, num_ctas, chunks[0]["key_tiles"], split)
    units = []
    for i in range(R):
        for h in range(H):
            for p in range(pairs):
                rows = min(Q_PAIR, C - Q_PAIR * p)
                live = 1 if rows <= Q_TILE else 2
                n = chunks[i]["key_tiles"]
                for k in range(P):
                    tiles = (k + 1) * n // P - k * n // P
                    slot = ((i * H + h) * pairs + p) * P + k if P > 1 else -1
                    units.append((i, h, p, tiles * (9 + live), k, P, slot))
    units.sort(key=lambda u: (-u[3], -u[0], u[1], u[2], u[4]))
    bins, loads = balance([u[3] for u in units], num_ctas)
    per_cta = [[units[k] for k in b] for b in bins]
    return dict(C=C, wc_eff=wc_eff, first=first, chunks=chunks, units=units,
                per_cta=per_cta, loads=loads, q_pairs=pairs, key_parts=P)


# --------------------------------------------------------------------------
# visibility mask and attention
# --------------------------------------------------------------------------

def logical_key_chunks(wc_eff: int, R: int):
    """Logical key order: cache chunks (oldest first) then in-round chunks 0..R-1.
    Returns (is_cache, in-round index or -1) per key chunk."""
    return [(True, -1)] * wc_eff + [(False, i) for i in range(R)]


def visibility_mask(C: int, wc_eff: int, R: int, q_chunks=None) -> np.ndarray:
    """M[q, k] = 1 iff key chunk is cache or an in-round chunk j <= query chunk i."""
    q_chunk = np.repeat(np.arange(R), C) if q_chunks is None else np.asarray(q_chunks)
    kinfo = logical_key_chunks(wc_eff, R)
    k_is_cache = np.repeat(np.array([c for c, _ in kinfo], dtype=bool), C)
    k_chunk = np.repeat(np.array([i for _, i in kinfo]), C)
    return k_is_cache[None, :] | (k_chunk[None, :] <= q_chunk[:, None])


def attention(q, k, v, mask, scale: float):
    """softmax(q k^T * scale, masked) v in fp64; q [nq,D], k/v [nk,D], mask [nq,nk].
    Returns (O [nq,D], LSE [nq]) with LSE = log sum_k exp(scale * q.k) over visible keys."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = (q @ k.T) * scale
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ v) / l, (m + np.log(l))[:, 0]


def attention_bruteforce(q, k, v, mask, scale: float):
    """Per-query Python loop over visible keys, no max subtraction (tiny inputs only)."""
    nq, D = len(q), len(q[0])
    out = np.zeros((nq, D))
    lse = np.zeros(nq)
    for a in range(nq):
        num = [0.0] * D
        den = 0.0
        for b in range(len(k)):
            if not mask[a][b]:
                continue
            dot = 0.0
            for d in range(D):
                dot += float(q[a][d]) * float(k[b][d])
            w = math.exp(dot * scale)
            den += w
            for d in range(D):
                num[d] += w * float(v[b][d])
        out[a] = [x / den for x in num]
        lse[a] = math.log(den)
    return out, lse


# --------------------------------------------------------------------------
# 8-bit scores: e4m3 codes with per-block scales
# --------------------------------------------------------------------------
# The 8-bit variant of the attention (the B200 counterpart of the 8-bit
# attention backends the Wave Forcing abstract benchmarks against) quantizes
# the rotated Q and K, not V: per (chunk, block of FP8_BLOCK consecutive
# chunk-relative tokens, head) one fp32 scale = amax / 448, and every element
# becomes the e4m3 value nearest x * (448 / amax).  Scores are products of
# the dequantized values (code * scale); P and V stay as in the 16-bit path.

E4M3_MAX = 448.0   # largest finite e4m3 value (1.75 * 2^8)
FP8_BLOCK = 128    # tokens per scale block


def round_e4m3(x) -> np.ndarray:
    """Nearest-even rounding to OCP FP8 E4M3 (sign, 4 exponent bits with bias
    7, 3 mantissa bits; normals from 2^-6, subnormals in steps of 2^-9; no
    infinities), saturating to +-448 as a satfinite conversion does."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, e = np.frexp(a)                       # a = m * 2^e, m in [0.5, 1)
    binade = np.maximum(e - 1, -6)           # subnormals share the 2^-6 binade's step
    step = np.ldexp(1.0, binade - 3)         # 3 mantissa bits
    r = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(r, x)


def fp8_block_quantize(x, C: int):
    """x: [n*C, H, D] values (exact in fp32), n whole chunks of C tokens.

    Per chunk, block b of tokens [b*FP8_BLOCK, min(C, (b+1)*FP8_BLOCK)) and
    head: scale = fp32(amax / 448), inv = fp32(448 / amax), codes =
    round_e4m3(fp32(x * inv)).  Every fp32 operation is a single operation
    rounded to nearest.  A block whose fp32 448 / amax is not finite (amax =
    0, or amax below 448 / FLT_MAX ~ 1.3e-36) is treated as all-zero: scale
    and inv are 1, so its elements round to zero codes (an infinite inv would
    turn every zero into 0 * inf = NaN).  Returns (codes
    [n*C, H, D] as values, scales [n, nblk, H] float64 holding fp32 values).
    """
    x = np.asarray(x, dtype=np.float64)
    T, H, D = x.shape
    n = T // C
    nblk = -(-C // FP8_BLOCK)
    codes = np.zeros_like(x)
    scales = np.zeros((n, nblk, H))
    for c in range(n):
        for b in range(nblk):
            lo, hi = c * C + b * FP8_BLOCK, c * C + min(C, (b + 1) * FP8_BLOCK)
            blk = x[lo:hi].astype(np.float32)                       # [tokens, H, D], exact
            amax = np.abs(blk).max(axis=(0, 2))                      # [H]
            safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
            with np.errstate(over="ignore"):
                inv_raw = (np.float32(E4M3_MAX) / safe).astype(np.float32)
            ok = (amax > 0) & np.isfinite(inv_raw)
            sc = np.where(ok, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
            inv = np.where(ok, inv_raw, np.float32(1.0)).astype(np.float32)
            scales[c, b] = sc
            codes[lo:hi] = round_e4m3((blk * inv[None, :, None]).astype(np.float32))
    return codes, scales


def fp8_dequantize(codes, scales, C: int) -> np.ndarray:
    """codes [n*C, H, D] times the scale of each element's block (exact in fp64)."""
    T, H, D = codes.shape
    tok = np.arange(T)
    sc = scales[tok // C, (tok % C) // FP8_BLOCK]                    # [T, H]
    return codes * sc[:, :, None]


# --------------------------------------------------------------------------
# one wave round
# --------------------------------------------------------------------------

def wave_round(q_raw, k_raw, v_raw, k_cache_raw, v_cache_raw, *, n0, F, fh, fw,
               pairs, theta, dtype, scale=None, rows=None, fp8=False):
    """One wave round for the heads present in the inputs.

    q_raw/k_raw/v_raw: [R, C, H, D] raw in-round tensors (chunk i is global n0+i);
    k_cache_raw/v_cache_raw: [Wc_eff, C, H, D] raw K/V of cache chunks
    n0-Wc_eff .. n0-1 as they were when last appended.
    rows: optional in-round query indices (flat over R*C) to evaluate.
    fp8: scores from block-quantized e4m3 Q and K (see fp8_block_quantize);
    the codes and scales are returned as q8, q_scales, k8 (cache chunks then
    in-round chunks) and k_scales.
    Returns dict with q_rot [R,C,H,D], k_rot [R,C,H,D], k_cache_rot, O [nrows,H,D],
    LSE [nrows,H] -- rotated tensors rounded to ``dtype``.
    """
    R, C, H, D = q_raw.shape
    wc_eff = k_cache_raw.shape[0]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rot = lambda x, n: round_to(rope3d_chunk(x, n, F, fh, fw, pairs, theta), dtype)
    q_rot = np.stack([rot(q_raw[i], n0 + i) for i in range(R)])
    k_rot = np.stack([rot(k_raw[i], n0 + i) for i in range(R)])
    kc_rot = (np.stack([rot(k_cache_raw[c], n0 - wc_eff + c) for c in range(wc_eff)])
              if wc_eff else np.zeros((0, C, H, D)))
    vr = round_to(v_raw, dtype)
    vc = round_to(v_cache_raw, dtype) if wc_eff else np.zeros((0, C, H, D))
    keys = np.concatenate([kc_rot, k_rot]).reshape(-1, H, D)
    vals = np.concatenate([vc, vr]).reshape(-1, H, D)
    rows = np.arange(R * C) if rows is None else np.asarray(rows)
    mask = visibility_mask(C, wc_eff, R, q_chunks=rows // C)
    extra = {}
    qall = q_rot.reshape(-1, H, D)
    if fp8:
        q8, qs = fp8_block_quantize(qall, C)
        k8, ks = fp8_block_quantize(keys, C)
        qall, keys = fp8_dequantize(q8, qs, C), fp8_dequantize(k8, ks, C)
        extra = dict(q8=q8, q_scales=qs, k8=k8, k_scales=ks)
    qf = qall[rows]
    out = np.zeros((len(rows), H, D))
    lse = np.zeros((len(rows), H))
    for h in range(H):
        out[:, h], lse[:, h] = attention(qf[:, h], keys[:, h], vals[:, h], mask, scale)
    return dict(q_rot=q_rot, k_rot=k_rot, k_cache_rot=kc_rot, v=vr, v_cache=vc, O=out, LSE=lse, rows=rows,
                **extra)
