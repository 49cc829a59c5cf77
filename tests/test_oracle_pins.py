"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against hand-derived fixtures, closed forms,
invariants, a brute-force loop, exact rational arithmetic or a library
routine, so that a dropped term, wrong sign, wrong index or transposed operand
anywhere in the oracle fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import wf_oracle as orc
from chunk_causal_attention_block_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- rounding

def _bf16_exact(x: float) -> float:
    """Nearest bf16 (ties to even) by exact rational search over the two neighbours."""
    if x == 0.0:
        return 0.0
    fx = Fraction(x)
    sign = -1 if fx < 0 else 1
    a = abs(fx)
    e = math.floor(math.log2(a)) if a > 0 else 0
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    q = Fraction(2) ** max(e - 7, -133)
    lo = (a // q) * q
    hi = lo + q
    dlo, dhi = a - lo, hi - a
    if dlo < dhi:
        r = lo
    elif dhi < dlo:
        r = hi
    else:
        r = lo if (lo / q) % 2 == 0 else hi
    return sign * float(r)


def test_round_bf16_matches_exact_rationals():
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000),
                         rng.standard_normal(200) * 1e-39])
    got = orc.round_bf16(xs)
    for x, g in zip(xs, got):
        assert g == _bf16_exact(float(x)), x


def test_round_bf16_ties_go_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> even mantissa (1.0)
    assert orc.round_bf16(1.0 + 2.0 ** -8) == 1.0
    # 1 + 3*2^-8 lies halfway between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6
    assert orc.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    # just above the tie rounds up
    assert orc.round_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7
    assert orc.round_bf16(-(1.0 + 2.0 ** -8)) == -1.0
    # bf16-representable values are fixed points
    v = synth.bf16_bits_to_f32(np.arange(0, 0x7F00, 7, dtype=np.uint16)).astype(np.float64)
    assert np.array_equal(orc.round_bf16(v), v)


def test_round_bf16_agrees_with_fp32_path_when_no_double_rounding():
    # values that are exactly fp32: bf16(x) == RNE on the fp32 bit pattern
    rng = np.random.default_rng(2)
    x = rng.standard_normal(20000).astype(np.float32)
    want = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x)).astype(np.float64)
    assert np.array_equal(orc.round_bf16(x.astype(np.float64)), want)


# ---------------------------------------------------------------- RoPE

def test_rope_split_and_positions_golden():
    g = load("rope_cases.json")
    for s in g["splits"]:
        assert list(orc.rope_split(s["D"])) == s["pairs"]
    for c in g["tokens"]:
        pairs = c.get("pairs") or orc.rope_split(c["D"])
        t, h, w = orc.token_positions(c["n"], c["F"], c["fh"], c["fw"])
        j = c["j"]
        assert [t[j], h[j], w[j]] == c["thw"]
        ang = orc.rope_angles(t[j:j + 1], h[j:j + 1], w[j:j + 1], pairs, c["theta"])[0]
        np.testing.assert_allclose(ang, c["angles"], rtol=1e-12, atol=1e-15)


def test_rope_identity_at_origin_and_norm_preserved():
    rng = np.random.default_rng(3)
    D = 64
    pairs = orc.rope_split(D)
    x = rng.standard_normal((48, 2, D))
    # chunk 0, F=1: token 0 is at (0,0,0)
    y = orc.rope3d_chunk(x, 0, 2, 4, 6, pairs, 10000.0)
    np.testing.assert_array_equal(y[0], x[0])
    assert not np.allclose(y[1:], x[1:])
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13)


def test_rope_rotation_direction():
    # (1,0) -> (cos a, sin a); (0,1) -> (-sin a, cos a)
    a = np.array([[0.3, 1.7]])
    x = np.array([[1.0, 0.0, 0.0, 1.0]])
    y = orc.rope_rotate(x, a)
    np.testing.assert_allclose(y[0], [math.cos(0.3), math.sin(0.3), -math.sin(1.7), math.cos(1.7)], rtol=1e-15)


def test_rope_relative_property():
    """<R(p)q, R(p')k> depends only on p - p' per axis."""
    rng = np.random.default_rng(4)
    D = 64
    pairs = orc.rope_split(D)
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)

    def rot(x, t, h, w):
        return orc.rope_rotate(x[None], orc.rope_angles([t], [h], [w], pairs, 10000.0))[0]

    base = rot(q, 5, 2, 3) @ rot(k, 1, 4, 0)
    for dt, dh, dw in [(3, 0, 0), (0, 7, 0), (0, 0, 11), (2, 5, 9)]:
        shifted = rot(q, 5 + dt, 2 + dh, 3 + dw) @ rot(k, 1 + dt, 4 + dh, 0 + dw)
        assert abs(shifted - base) < 1e-11
    # and it does change with the offset between the two tokens
    assert abs(rot(q, 6, 2, 3) @ rot(k, 1, 4, 0) - base) > 1e-3


def test_rope_reduces_to_library_1d_rotary():
    """All pairs on the t axis at h=w=0 is GPT-J style 1-D rotary (transformers)."""
    gptj = pytest.importorskip("transformers.models.gptj.modeling_gptj")
    D, npos = 64, 40
    rng = np.random.default_rng(5)
    x = rng.standard_normal((npos, 1, D))
    pos = np.arange(npos)
    ang = orc.rope_angles(pos, np.zeros(npos), np.zeros(npos), (D // 2, 0, 0), 10000.0)
    ours = orc.rope_rotate(x, ang)
    table = gptj.create_sinusoidal_positions(npos, D).to(torch.float64)  # [pos, D]: sin | cos
    sin, cos = torch.split(table, D // 2, dim=-1)
    sin = torch.repeat_interleave(sin, 2, dim=-1)[None, :, None, :]
    cos = torch.repeat_interleave(cos, 2, dim=-1)[None, :, None, :]
    t = torch.tensor(x)[None]  # [1, pos, 1, D]
    lib = (t * cos) + (gptj.rotate_every_two(t) * sin)
    # the library builds its angles in fp32; compare at that precision
    np.testing.assert_allclose(ours, lib[0].numpy(), atol=2e-4)


# ---------------------------------------------------------------- ring

def test_ring_slot_and_window_after_appends():
    S, Wc, R = 11, 7, 4
    appends = list(range(0, 300))
    for N in (7, 8, 19, 150, 300):
        slots = orc.ring_contents_after(appends[:N], S)
        present = sorted(c for c in slots if c is not None)
        # the ring holds the last min(N, S) chunks
        assert present == list(range(max(0, N - S), N))
        # the logical cache of a round whose oldest in-round chunk is N is the last Wc chunks
        win = orc.cache_window(N, Wc)
        assert win == list(range(max(0, N - Wc), N))
        assert all(slots[orc.ring_slot(n, S)] == n for n in win)
    # eviction victim of the incoming chunk n0+R is the oldest cache chunk n0-Wc
    for n0 in range(Wc, 60):
        assert orc.ring_slot(n0 + R, S) == orc.ring_slot(n0 - Wc, S)


# ---------------------------------------------------------------- plan

def test_plan_golden_cases():
    for c in load("plan_cases.json")["cases"]:
        p = orc.plan_round(c["H"], c["D"], c["fh"], c["fw"], c["F"], c["Wc"], c["R"], c["S"], c["n0"],
                           c["noise_t"], c["num_ctas"])
        assert p["C"] == c["C"] and p["wc_eff"] == c["wc_eff"], c["name"]
        for got, want in zip(p["chunks"], c["chunks"]):
            for key in ("n", "slot", "vis_chunks", "vis_slots", "keys", "key_tiles"):
                assert got[key] == want[key], (c["name"], key)
            assert [list(s) for s in got["segs"]] == want["segs"], c["name"]
        if "per_cta" in c:
            assert [[list(u[:3]) for u in lst] for lst in p["per_cta"]] == c["per_cta"]
            assert p["loads"] == c["loads"]


def test_balance_golden_cases():
    """Hand-derived assignments of the work balancer, one per tie-break and branch."""
    for c in load("balance_cases.json")["cases"]:
        bins, loads = orc.balance(c["costs"], c["num_bins"])
        assert bins == c["bins"], c["name"]
        assert loads == c["loads"], c["name"]


def test_balance_leaves_no_improving_move_or_swap():
    """On random cost lists: the result is a partition of the items, and no move or
    swap between the heaviest bin and a lighter one lowers the heaviest load (the
    refinement's stopping condition, checked by brute force)."""
    rng = np.random.default_rng(7)
    for _ in range(300):
        n = int(rng.integers(0, 14))
        G = int(rng.integers(1, 6))
        costs = [int(x) for x in rng.integers(0, 40, n)]
        bins, loads = orc.balance(costs, G)
        assert sorted(i for b in bins for i in b) == list(range(n))
        assert loads == [sum(costs[i] for i in b) for b in bins]
        top = max(loads)
        for h in range(G):
            if loads[h] != top:
                continue
            for b in range(G):
                if loads[b] >= top:
                    continue
                for x in bins[h]:
                    assert max(top - costs[x], loads[b] + costs[x]) >= top
                    for y in bins[b]:
                        d = costs[x] - costs[y]
                        assert d <= 0 or max(top - d, loads[b] + d) >= top
            break


def test_plan_tile_pairs_match_brute_mask():
    """Key tiles the plan visits per query chunk cover exactly the visible keys."""
    for (C, Wc, R, S, n0) in [(48, 3, 3, 6, 3), (48, 3, 3, 6, 5), (200, 2, 4, 6, 9), (130, 0, 2, 2, 4)]:
        p = orc.plan_round(1, 64, 1, C, 1, Wc, R, S, n0, [0] * R, 4)
        mask = orc.visibility_mask(C, p["wc_eff"], R)
        # physical pool token of each logical key
        kinfo = list(range(n0 - p["wc_eff"], n0)) + list(range(n0, n0 + R))
        phys = np.concatenate([np.arange(C) + (n % S) * C for n in kinfo])
        for i, ch in enumerate(p["chunks"]):
            covered = set()
            for start, ln in ch["segs"]:
                covered |= set(range(start, start + ln))
            want = set(phys[mask[i * C]].tolist())
            assert covered == want
            # every tile of 128 is non-empty and the count matches
            assert ch["key_tiles"] == sum(-(-ln // 128) for _, ln in ch["segs"] if ln)


def _covered_row_tiles(p):
    """Check that the units cover every (chunk, head, query row, key tile) exactly once:
    each row pair's parts partition [0, key_tiles).  Returns the number covered."""
    ranges = {}
    for lst in p["per_cta"]:
        for (i, h, pp, cost, k, P, slot) in lst:
            n = p["chunks"][i]["key_tiles"]
            t0, t1 = k * n // P, (k + 1) * n // P
            rows = min(256, p["C"] - pp * 256)
            assert rows > 0
            assert cost == (t1 - t0) * (9 + (1 if rows <= 128 else 2))
            ranges.setdefault((i, h, pp), []).append((t0, t1, rows))
    total = 0
    for (i, h, pp), rs in ranges.items():
        rs.sort()
        n = p["chunks"][i]["key_tiles"]
        assert rs[0][0] == 0 and rs[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))      # contiguous, no overlap
        total += rs[0][2] * n
    pairs = -(-p["C"] // 256)
    heads = len({h for (_, h, _) in ranges})
    assert len(ranges) == len(p["chunks"]) * heads * pairs                 # every (chunk, head, pair)
    return total


def test_plan_work_list_covers_every_row_once():
    # 12 heads: 912 units on 148 bins, no key split
    p = orc.plan_round(12, 128, 30, 52, 3, 7, 4, 11, 7, [250, 500, 750, 1000], 148)
    assert p["key_parts"] == 1
    assert _covered_row_tiles(p) == sum(p["C"] * 12 * ch["key_tiles"] for ch in p["chunks"])
    assert max(p["loads"]) - min(p["loads"]) <= max(u[3] for u in p["units"])
    # 3 heads: 228 units (< 2 per bin), split in 5 (see the single-chunk case below)
    p = orc.plan_round(3, 128, 30, 52, 3, 7, 4, 11, 7, [250, 500, 750, 1000], 148)
    assert p["key_parts"] == 5
    assert _covered_row_tiles(p) == sum(p["C"] * 3 * ch["key_tiles"] for ch in p["chunks"])
    assert max(p["loads"]) - min(p["loads"]) <= max(u[3] for u in p["units"])


def test_plan_key_split_of_a_single_chunk():
    # 12 heads x 19 row pairs of one 4680-token chunk = 228 units on 148 bins.  Bin filling
    # ceil(228p/148) / (228p/148) + (p-1)/100 for p = 1..8: 1.298, 1.308, 1.102, 1.166, 1.079,
    # 1.132, 1.080, 1.125 -> p = 5 (fewest tiles per part 256/5 >= 8).
    p = orc.plan_round(12, 128, 30, 52, 3, 6, 1, 7, 6, [1000], 148)
    assert p["key_parts"] == 5
    n = p["chunks"][0]["key_tiles"]
    assert n == 256 and _covered_row_tiles(p) == 12 * 4680 * n
    slots = sorted(u[6] for lst in p["per_cta"] for u in lst)
    assert slots == list(range(228 * 5))
    # the 16-bit-only rule: no split for fp32 plans
    assert orc.plan_round(12, 128, 30, 52, 3, 6, 1, 7, 6, [1000], 148, split=False)["key_parts"] == 1


# ---------------------------------------------------------------- mask / attention

def test_mask_golden():
    for c in load("mask_cases.json")["cases"]:
        m = orc.visibility_mask(c["C"], c["wc_eff"], c["R"])
        assert m.astype(int).tolist() == c["mask"]


def test_attention_closed_forms_golden():
    for c in load("attn_cases.json")["cases"]:
        o, lse = orc.attention(np.array(c["q"]), np.array(c["k"]), np.array(c["v"]),
                               np.array(c["mask"], dtype=bool), c["scale"])
        np.testing.assert_allclose(o, c["O"], rtol=1e-14)
        np.testing.assert_allclose(lse, c["LSE"], rtol=1e-14)


def _tiny_round(seed=7, C=6, Wc=2, R=3, H=2, D=8):
    rng = np.random.default_rng(seed)
    nk = (Wc + R) * C
    q = rng.standard_normal((R * C, H, D))
    k = rng.standard_normal((nk, H, D))
    v = rng.standard_normal((nk, H, D))
    return q, k, v, orc.visibility_mask(C, Wc, R)


def test_attention_matches_bruteforce():
    q, k, v, m = _tiny_round()
    for h in range(q.shape[1]):
        o, lse = orc.attention(q[:, h], k[:, h], v[:, h], m, 0.35)
        ob, lb = orc.attention_bruteforce(q[:, h].tolist(), k[:, h].tolist(), v[:, h].tolist(), m.tolist(), 0.35)
        np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, lb, rtol=1e-12)


def test_attention_equal_values_give_that_row():
    q, k, v, m = _tiny_round(8)
    row = np.array([0.5, -1.25, 3.0, 0.0, 2.0, -7.5, 1.0, 0.125])
    v[:] = row
    o, _ = orc.attention(q[:, 0], k[:, 0], v[:, 0], m, 1 / math.sqrt(8))
    np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), rtol=1e-14)


def test_attention_single_visible_key():
    # Wc=0, C=1: chunk 0's only visible key is itself
    q, k, v, m = _tiny_round(9, C=1, Wc=0, R=3)
    o, lse = orc.attention(q[:, 0], k[:, 0], v[:, 0], m, 0.3)
    np.testing.assert_allclose(o[0], v[0, 0], rtol=1e-14)
    assert abs(lse[0] - 0.3 * q[0, 0] @ k[0, 0]) < 1e-13


def test_attention_reduces_to_sdpa_unmasked():
    # Wc=0, R=1: plain bidirectional attention over one chunk
    q, k, v, m = _tiny_round(10, C=9, Wc=0, R=1, D=16)
    assert m.all()
    o, _ = orc.attention(q[:, 0], k[:, 0], v[:, 0], m, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q[:, 0])[None], torch.tensor(k[:, 0])[None], torch.tensor(v[:, 0])[None], scale=0.25)[0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_attention_reduces_to_sdpa_causal():
    # one token per chunk, no cache: token i sees tokens 0..i
    q, k, v, m = _tiny_round(11, C=1, Wc=0, R=7, D=16)
    o, _ = orc.attention(q[:, 0], k[:, 0], v[:, 0], m, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q[:, 0])[None], torch.tensor(k[:, 0])[None], torch.tensor(v[:, 0])[None],
        is_causal=True, scale=0.25)[0]
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_attention_permutation_invariance():
    q, k, v, m = _tiny_round(12, C=5, Wc=2, R=2)
    o, lse = orc.attention(q[:, 1], k[:, 1], v[:, 1], m, 0.4)
    perm = np.random.default_rng(0).permutation(len(k))
    o2, lse2 = orc.attention(q[:, 1], k[perm, 1], v[perm, 1], m[:, perm], 0.4)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)


def test_later_chunks_do_not_affect_earlier_ones():
    C, Wc, R = 4, 2, 3
    q, k, v, m = _tiny_round(13, C=C, Wc=Wc, R=R)
    o, _ = orc.attention(q[:, 0], k[:, 0], v[:, 0], m, 0.4)
    k2, v2 = k.copy(), v.copy()
    k2[(Wc + 1) * C:] += 5.0  # perturb in-round chunks 1, 2
    v2[(Wc + 1) * C:] -= 3.0
    o2, _ = orc.attention(q[:, 0], k2[:, 0], v2[:, 0], m, 0.4)
    np.testing.assert_array_equal(o2[:C], o[:C])       # chunk 0 unchanged, bit for bit
    assert not np.allclose(o2[C:], o[C:])              # chunks 1, 2 do see it


# ---------------------------------------------------------------- whole round

def test_wave_round_against_per_query_bruteforce():
    """End-to-end oracle round on a tiny wave round vs a brute-force restatement."""
    H, D, F, fh, fw, Wc, R, n0 = 2, 8, 1, 2, 3, 2, 2, 5
    C = F * fh * fw
    pairs = (2, 1, 1)
    rng = np.random.default_rng(14)
    q = rng.standard_normal((R, C, H, D))
    k = rng.standard_normal((R, C, H, D))
    v = rng.standard_normal((R, C, H, D))
    kc = rng.standard_normal((Wc, C, H, D))
    vc = rng.standard_normal((Wc, C, H, D))
    out = orc.wave_round(q, k, v, kc, vc, n0=n0, F=F, fh=fh, fw=fw, pairs=pairs, theta=100.0, dtype="f32")
    # brute force: rotate each token from its own (t,h,w) with explicit 2x2 rotations
    def rot_token(x, n, j):
        f, l = divmod(j, fh * fw)
        pos = [n * F + f] * pairs[0] + [l // fw] * pairs[1] + [l % fw] * pairs[2]
        ks = list(range(pairs[0])) + list(range(pairs[1])) + list(range(pairs[2]))
        Ps = [pairs[0]] * pairs[0] + [pairs[1]] * pairs[1] + [pairs[2]] * pairs[2]
        y = np.array(x, dtype=np.float64)
        for m_ in range(D // 2):
            a = pos[m_] * 100.0 ** (-ks[m_] / Ps[m_])
            x0, x1 = x[2 * m_], x[2 * m_ + 1]
            y[2 * m_] = float(np.float32(x0 * math.cos(a) - x1 * math.sin(a)))
            y[2 * m_ + 1] = float(np.float32(x0 * math.sin(a) + x1 * math.cos(a)))
        return y
    keys, vals, kchunk = [], [], []
    for c in range(Wc):
        for j in range(C):
            keys.append([rot_token(kc[c, j, h], n0 - Wc + c, j) for h in range(H)])
            vals.append([vc[c, j, h].astype(np.float32) for h in range(H)])
            kchunk.append(-1)
    for i in range(R):
        for j in range(C):
            keys.append([rot_token(k[i, j, h], n0 + i, j) for h in range(H)])
            vals.append([v[i, j, h].astype(np.float32) for h in range(H)])
            kchunk.append(i)
    for i in range(R):
        for j in range(C):
            for h in range(H):
                qq = rot_token(q[i, j, h], n0 + i, j)
                msk = [[kc_ <= i for kc_ in kchunk]]
                ob, lb = orc.attention_bruteforce([qq], [kk[h] for kk in keys], [vv[h] for vv in vals], msk,
                                                  1 / math.sqrt(D))
                np.testing.assert_allclose(out["O"][i * C + j, h], ob[0], rtol=1e-12, atol=1e-13)
                np.testing.assert_allclose(out["LSE"][i * C + j, h], lb[0], rtol=1e-12)


# ------------------------------------------------------------------ 8-bit scores

def _e4m3_decode(code: int):
    """Value of an E4M3 code from the format's definition (None for NaN)."""
    s, e, m = code >> 7, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return None
    v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
    return -v if s else v


def test_e4m3_codes_are_fixed_points_and_midpoints_go_to_even():
    pos = sorted({_e4m3_decode(c) for c in range(128) if _e4m3_decode(c) is not None})
    assert pos[0] == 0 and pos[1] == Fraction(1, 512) and pos[-1] == 448 and len(pos) == 127
    vals = np.array([float(v) for v in pos])
    assert np.array_equal(orc.round_e4m3(vals), vals)
    assert np.array_equal(orc.round_e4m3(-vals), -vals)
    even = {float(_e4m3_decode(c)): (c & 1) == 0 for c in range(127)}
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = (lo + hi) / 2
        want = float(lo) if even[float(lo)] else float(hi)
        assert orc.round_e4m3(float(mid)) == want, (lo, hi)
        eps = (hi - lo) / 1024
        assert orc.round_e4m3(float(mid - eps)) == float(lo)
        assert orc.round_e4m3(float(mid + eps)) == float(hi)
    # beyond the largest finite value the conversion saturates
    assert np.array_equal(orc.round_e4m3([448.5, 464.0, 480.0, 1e9, -1e9]), [448, 448, 448, 448, -448])


def test_e4m3_rounding_matches_torch_float8():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-14, 9, 200_000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(orc.round_e4m3(x.astype(np.float64)), t)


def test_fp8_block_quantize_hand_case():
    # C = 130 tokens: block 0 = tokens 0..127, block 1 = tokens 128..129 (ragged); 2 heads, D = 4
    C, H, D = 130, 2, 4
    x = np.zeros((C, H, D))
    x[5, 0] = [3.5, -1.0, 0.25, 0.0]          # head 0, block 0: amax 3.5 -> scale 2^-7 exactly
    x[70, 0] = [-2.0, 1.5, 0.0, 0.125]
    x[129, 0] = [0.75, 0.0, 0.0, -0.375]      # head 0, block 1: amax 0.75 -> scale fp32(0.75/448)
    codes, scales = orc.fp8_block_quantize(x, C)
    assert scales.shape == (1, 2, 2)
    assert scales[0, 0, 0] == 2.0 ** -7
    assert scales[0, 0, 1] == 1.0 and scales[0, 1, 1] == 1.0         # all-zero blocks
    assert scales[0, 1, 0] == float(np.float32(0.75) / np.float32(448.0))
    assert np.array_equal(codes[5, 0], [448.0, -128.0, 32.0, 0.0])   # x * 128, all representable
    assert np.array_equal(codes[70, 0], [-256.0, 192.0, 0.0, 16.0])
    assert abs(codes[129, 0, 0]) == 448.0                             # the block max maps to the largest code
    assert codes[129, 0, 3] == orc.round_e4m3(np.float32(-0.375) * (np.float32(448.0) / np.float32(0.75)))
    assert not codes[:, 1].any()
    deq = orc.fp8_dequantize(codes, scales, C)
    assert np.array_equal(deq[5, 0], x[5, 0]) and np.array_equal(deq[70, 0], x[70, 0])


def test_fp8_block_quantize_tiny_block_is_a_zero_block():
    # a block of zeros plus one bf16 subnormal (2^-133): 448 / 2^-133 overflows fp32, so the
    # block takes scale 1 and inv 1 like an all-zero block, and every code is zero -- no NaN
    # from 0 * inf.  A block whose amax (2^-100) keeps 448 / amax finite is quantized as usual.
    C, H, D = 128, 2, 4
    x = np.zeros((C, H, D))
    x[7, 0, 2] = 2.0 ** -133
    x[9, 0, 1] = -2.0 ** -133
    x[3, 1, 0] = 2.0 ** -100
    codes, scales = orc.fp8_block_quantize(x, C)
    assert scales[0, 0, 0] == 1.0 and not np.isnan(codes).any()
    assert np.array_equal(codes[:, 0], np.zeros((C, D)))
    assert scales[0, 0, 1] == float(np.float32(2.0 ** -100) / np.float32(448.0))
    assert codes[3, 1, 0] == 448.0


def test_fp8_dequantized_error_within_half_an_e4m3_step():
    rng = np.random.default_rng(3)
    C = 300
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rng.standard_normal((2 * C, 3, 16)).astype(np.float32))) \
        .astype(np.float64)
    codes, scales = orc.fp8_block_quantize(x, C)
    deq = orc.fp8_dequantize(codes, scales, C)
    tok = np.arange(2 * C)
    sc = scales[tok // C, (tok % C) // orc.FP8_BLOCK][:, :, None]
    # half a step of the binade (relative 2^-4) for normals, 2^-10 * scale in the subnormal range,
    # plus the fp32 roundings of 448 / amax, amax / 448 and x * inv (relative 2^-24 each)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, sc * 2.0 ** -10) * (1 + 2.0 ** -20)
    assert (np.abs(deq - x) <= bound).all()


def test_fp8_round_equals_16_bit_round_when_quantization_is_exact():
    # inputs whose rotated values are e4m3-exact after scaling: a zero angle (n = 0, one token
    # per chunk at position 0) and values that are small multiples of powers of two
    rng = np.random.default_rng(11)
    R, C, H, D = 1, 1, 2, 16
    q = rng.integers(-7, 8, (R, C, H, D)) / 8.0
    k = rng.integers(-7, 8, (R, C, H, D)) / 8.0
    v = rng.standard_normal((R, C, H, D))
    q[0, 0, :, 0] = 1.75
    k[0, 0, :, 0] = 1.75                   # amax 1.75 -> scale 1.75/448 = 2^-8
    kw = dict(n0=0, F=1, fh=1, fw=1, pairs=orc.rope_split(D), theta=10000.0, dtype="f32")
    empty = np.zeros((0, C, H, D))
    a = orc.wave_round(q, k, v, empty, empty, **kw)
    b = orc.wave_round(q, k, v, empty, empty, fp8=True, **kw)
    assert np.array_equal(b["q8"] * 2.0 ** -8, a["q_rot"].reshape(-1, H, D))
    assert np.array_equal(a["O"], b["O"]) and np.array_equal(a["LSE"], b["LSE"])


def test_fp8_block_quantize_matches_a_torch_pipeline():
    # the same definition written with torch: fp32 amax, fp32 448/amax and amax/448, fp32 product,
    # torch's float8_e4m3fn conversion (nearest-even; products stay within its range)
    rng = np.random.default_rng(5)
    C, H, D = 300, 3, 32
    x = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
        (rng.standard_normal((2 * C, H, D)) * np.exp2(rng.integers(-3, 4, (1, H, 1)))).astype(np.float32)))
    codes, scales = orc.fp8_block_quantize(x.astype(np.float64), C)
    t = torch.from_numpy(x.astype(np.float32))
    for c in range(2):
        for b in range(-(-C // 128)):
            lo, hi = c * C + b * 128, c * C + min(C, (b + 1) * 128)
            blk = t[lo:hi]
            amax = blk.abs().amax(dim=(0, 2))
            inv = torch.tensor(448.0, dtype=torch.float32) / amax
            q = (blk * inv[None, :, None]).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            assert np.array_equal(codes[lo:hi], q), (c, b)
            assert np.array_equal(scales[c, b], (amax / torch.tensor(448.0)).to(torch.float64).numpy())
