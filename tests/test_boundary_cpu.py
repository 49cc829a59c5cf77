"""CPU checks of the C ABI: the library loads, exports what the headers
declare, validates arguments on the host, and its planner agrees bit for bit
with the oracle's independent re-derivation of the plan."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

from chunk_causal_attention_block_b200 import wf
from oracle import wf_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def declared_symbols():
    names = []
    for h in ("wf.h", "wf_synth.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(wf_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = wf.lib()
    syms = declared_symbols()
    assert len(syms) >= 10
    assert set(syms) == set(wf.EXPORTS)
    for s in syms:
        assert hasattr(L, s), s
    assert wf.wf_version() == 100
    for code in range(9):
        assert wf.status_string(code).startswith("WF_")


def _desc(**kw):
    base = dict(H=2, D=64, fh=4, fw=6, F=2, Wc=3, R=3, n0=3, noise_t=[250, 500, 750], dtype=wf.WF_F32,
                num_ctas=4)
    base.update(kw)
    args = [base.pop(k) for k in ("H", "D", "fh", "fw", "F", "Wc", "R", "n0", "noise_t")]
    return wf.make_desc(*args, **base)


def _plan(desc):
    n = wf.wf_plan_bytes(desc)
    assert n > 0
    buf = np.zeros(n + 64, dtype=np.uint8)
    off = (-buf.ctypes.data) % 16
    host = buf[off:off + n]
    wf.wf_plan_round(desc, host)
    return host


@pytest.mark.parametrize("kw,code", [
    (dict(H=0), wf.WF_ERR_INVALID_ARG),
    (dict(D=63), wf.WF_ERR_INVALID_ARG),
    (dict(D=96), wf.WF_ERR_UNSUPPORTED),
    (dict(D=64, dtype=wf.WF_BF16), wf.WF_ERR_UNSUPPORTED),
    (dict(R=0), wf.WF_ERR_INVALID_ARG),
    (dict(R=17), wf.WF_ERR_INVALID_ARG),
    (dict(Wc=-1), wf.WF_ERR_INVALID_ARG),
    (dict(S=4), wf.WF_ERR_INVALID_ARG),                       # S < Wc + R
    (dict(noise_t=[500, 250, 750]), wf.WF_ERR_INVALID_ARG),   # an older chunk noisier than a newer one
    (dict(noise_t=[250, 500, 1001]), wf.WF_ERR_INVALID_ARG),
    (dict(pairs=(10, 10, 10)), wf.WF_ERR_INVALID_ARG),         # does not sum to D/2
    (dict(theta=0.0), wf.WF_ERR_INVALID_ARG),
    (dict(n0=-1), wf.WF_ERR_INVALID_ARG),
    (dict(dtype=7), wf.WF_ERR_INVALID_ARG),
    (dict(fh=10000, fw=10000), wf.WF_ERR_CAPACITY),
])
def test_plan_rejects_bad_descriptions(kw, code):
    d = _desc(**kw)
    assert wf.wf_plan_bytes(d) == 0
    buf = np.zeros(1 << 16, dtype=np.uint8)
    with pytest.raises(wf.WfError) as e:
        wf.wf_plan_round(d, buf)
    assert e.value.code == code


def test_plan_rejects_small_or_misaligned_buffers():
    d = _desc()
    n = wf.wf_plan_bytes(d)
    buf = np.zeros(n + 64, dtype=np.uint8)
    off = (-buf.ctypes.data) % 16
    with pytest.raises(wf.WfError) as e:
        wf.wf_plan_round(d, buf[off:off + n - 16])
    assert e.value.code == wf.WF_ERR_WORKSPACE
    with pytest.raises(wf.WfError) as e:
        wf.wf_plan_round(d, buf[off + 4:off + 4 + n])
    assert e.value.code == wf.WF_ERR_ALIGNMENT


def test_entry_points_reject_bad_arguments_before_any_launch():
    host = _plan(_desc())
    fake = 1 << 20  # never dereferenced: validation fails first
    with pytest.raises(wf.WfError) as e:
        wf.wf_rope3d_append(host, fake, fake, fake, fake, fake, fake, None)
    assert e.value.code == wf.WF_ERR_INVALID_ARG
    with pytest.raises(wf.WfError) as e:
        wf.wf_rope3d_append(host, fake, fake + 4, fake, fake, fake, fake, fake)
    assert e.value.code == wf.WF_ERR_ALIGNMENT
    bad = host.copy()
    bad[0] ^= 0xFF
    with pytest.raises(wf.WfError) as e:
        wf.wf_rope3d_append(bad, fake, fake, fake, fake, fake, fake, fake)
    assert e.value.code == wf.WF_ERR_PLAN
    with pytest.raises(wf.WfError) as e:
        wf.wf_chunk_causal_attn(host, fake, fake, fake, fake, fake, None, 0.0, fake, workspace_bytes=16)
    assert e.value.code == wf.WF_ERR_WORKSPACE
    with pytest.raises(wf.WfError) as e:
        wf.wf_chunk_causal_attn(host, fake, fake, fake, fake, fake, None, -1.0, fake, workspace_bytes=4096)
    assert e.value.code == wf.WF_ERR_INVALID_ARG
    assert wf.wf_attn_workspace_bytes(host) >= 256
    assert wf.wf_attn_workspace_bytes(bad) == 0


def test_fp8_entry_points_reject_bad_arguments_before_any_launch():
    f32 = _plan(_desc())
    bf16 = _plan(_desc(D=128, dtype=wf.WF_BF16))
    fake = 1 << 20  # never dereferenced: validation fails first
    cases = [
        (lambda: wf.wf_quantize_fp8(f32, fake, fake, fake, wf.WF_FP8_K), wf.WF_ERR_UNSUPPORTED),
        (lambda: wf.wf_quantize_fp8(bf16, fake, fake, fake, 2), wf.WF_ERR_INVALID_ARG),
        (lambda: wf.wf_quantize_fp8(bf16, fake, fake, None, wf.WF_FP8_Q), wf.WF_ERR_INVALID_ARG),
        (lambda: wf.wf_quantize_fp8(bf16, fake + 8, fake, fake, wf.WF_FP8_Q), wf.WF_ERR_ALIGNMENT),
        (lambda: wf.wf_quantize_fp8(bf16, fake, fake, fake + 2, wf.WF_FP8_Q), wf.WF_ERR_ALIGNMENT),
        (lambda: wf.wf_chunk_causal_attn_fp8(bf16, fake, fake, fake, fake, fake, fake, fake, None, 0.0, fake,
                                             workspace_bytes=16), wf.WF_ERR_WORKSPACE),
        (lambda: wf.wf_chunk_causal_attn_fp8(bf16, fake, fake, fake, fake, None, fake, fake, None, 0.0, fake,
                                             workspace_bytes=4096), wf.WF_ERR_INVALID_ARG),
        (lambda: wf.wf_chunk_causal_attn_fp8(bf16, fake, fake, fake + 2, fake, fake, fake, fake, None, 0.0, fake,
                                             workspace_bytes=4096), wf.WF_ERR_ALIGNMENT),
        (lambda: wf.wf_chunk_causal_attn_fp8(f32, fake, fake, fake, fake, fake, fake, fake, None, 0.0, fake,
                                             workspace_bytes=4096), wf.WF_ERR_UNSUPPORTED),
    ]
    for call, code in cases:
        with pytest.raises(wf.WfError) as e:
            call()
        assert e.value.code == code


def test_fused_rope_entry_points_reject_bad_arguments_before_any_launch():
    f32 = _plan(_desc())
    bf16 = _plan(_desc(D=128, dtype=wf.WF_BF16))
    fake = 1 << 20  # never dereferenced: validation fails first
    cases = [
        (lambda: wf.wf_rope3d_append_kv(bf16, fake, fake, None, fake, fake), wf.WF_ERR_INVALID_ARG),
        (lambda: wf.wf_rope3d_append_kv(bf16, fake, fake, fake, fake + 4, fake), wf.WF_ERR_ALIGNMENT),
        (lambda: wf.wf_chunk_causal_attn_rope(bf16, fake, fake, fake, fake, fake, None, 0.0, fake,
                                              workspace_bytes=16), wf.WF_ERR_WORKSPACE),
        (lambda: wf.wf_chunk_causal_attn_rope(bf16, fake, None, fake, fake, fake, None, 0.0, fake,
                                              workspace_bytes=4096), wf.WF_ERR_INVALID_ARG),
        (lambda: wf.wf_chunk_causal_attn_rope(bf16, fake, fake + 8, fake, fake, fake, None, 0.0, fake,
                                              workspace_bytes=4096), wf.WF_ERR_ALIGNMENT),
        (lambda: wf.wf_chunk_causal_attn_rope(f32, fake, fake, fake, fake, fake, None, 0.0, fake,
                                              workspace_bytes=4096), wf.WF_ERR_UNSUPPORTED),
        (lambda: wf.wf_chunk_causal_attn_rope(bf16, fake, fake, fake, fake, fake, None, -1.0, fake,
                                              workspace_bytes=4096), wf.WF_ERR_INVALID_ARG),
    ]
    for call, code in cases:
        with pytest.raises(wf.WfError) as e:
            call()
        assert e.value.code == code


def test_workspace_size_follows_the_key_split():
    # one 1560-token chunk, 2 heads: 14 units for 148 CTAs -> each unit's keys in 4 parts
    d = wf.make_desc(2, 128, 30, 52, 1, 2, 1, 2, [1000], dtype=wf.WF_BF16, num_ctas=148)
    host = _plan(d)
    p = wf.decode_plan(host)
    assert p["key_parts"] == 4 and p["num_units"] == 56
    assert wf.wf_attn_workspace_bytes(host) == 256 + 56 * 256 * 129 * 4
    fake = 1 << 20
    with pytest.raises(wf.WfError) as e:  # too small for the partial slots: rejected before any launch
        wf.wf_chunk_causal_attn(host, fake, fake, fake, fake, fake, None, 0.0, fake, workspace_bytes=4096)
    assert e.value.code == wf.WF_ERR_WORKSPACE
    with pytest.raises(wf.WfError) as e:  # more than the static scratch of the allocation-free entry point
        wf.wf_chunk_causal_attn_noalloc(host, fake, fake, fake, fake, fake, None, 0.0)
    assert e.value.code == wf.WF_ERR_CAPACITY
    # an unsplit plan needs the status block only
    assert wf.wf_attn_workspace_bytes(_plan(_desc())) == 256


def _compare_plan(host, ref, desc_kw):
    p = wf.decode_plan(host)
    assert p["magic"] == 0x31504657 and p["version"] == 2
    assert p["C"] == ref["C"] and p["wc_eff"] == ref["wc_eff"] and p["first"] == ref["first"]
    for got, want in zip(p["chunks"], ref["chunks"]):
        for key in ("n", "slot", "noise", "nvis", "keys", "key_tiles", "vis_slots"):
            assert got[key] == want[key], key
        assert [tuple(s) for s in got["segs"]] == [tuple(s) for s in want["segs"]]
    assert [[u for u in lst] for lst in p["per_cta"]] == [[tuple(u) for u in lst] for lst in ref["per_cta"]]


PLAN_CASES = [
    dict(H=2, D=64, fh=4, fw=6, F=2, Wc=3, R=3, S=6, n0=3, noise_t=[250, 500, 750], num_ctas=3),
    dict(H=2, D=64, fh=4, fw=6, F=2, Wc=3, R=3, S=6, n0=5, noise_t=[250, 500, 750], num_ctas=5),
    dict(H=12, D=128, fh=30, fw=52, F=3, Wc=6, R=1, S=7, n0=6, noise_t=[1000], num_ctas=148),
    dict(H=12, D=128, fh=30, fw=52, F=3, Wc=7, R=4, S=11, n0=7 + 9, noise_t=[250, 500, 750, 1000], num_ctas=148),
    dict(H=40, D=128, fh=45, fw=80, F=3, Wc=7, R=4, S=11, n0=7 + 199, noise_t=[250, 500, 750, 1000],
         num_ctas=148),
    dict(H=3, D=128, fh=5, fw=7, F=2, Wc=5, R=4, S=13, n0=2, noise_t=[0, 0, 500, 500], num_ctas=7),  # start
    dict(H=1, D=128, fh=1, fw=1, F=1, Wc=0, R=5, S=5, n0=11, noise_t=[0, 1, 2, 3, 4], num_ctas=2),   # C=1
    # the most in-round chunks (16), ring wrapped
    dict(H=1, D=128, fh=6, fw=7, F=1, Wc=3, R=16, S=19, n0=3 + 40, noise_t=[60 * i for i in range(16)],
         num_ctas=148),
    # cache-refresh rounds: the oldest member at t=0 (4-step + refresh, 5-step + refresh), ring wrapped
    dict(H=12, D=128, fh=30, fw=52, F=3, Wc=7, R=5, S=12, n0=7 + 13, noise_t=[0, 250, 500, 750, 1000],
         num_ctas=148),
    dict(H=12, D=128, fh=30, fw=52, F=3, Wc=7, R=6, S=13, n0=7 + 15, noise_t=[0, 200, 400, 600, 800, 1000],
         num_ctas=148),
]


@pytest.mark.parametrize("case", PLAN_CASES)
def test_plan_matches_oracle_rederivation(case):
    kw = dict(case)
    dtype = wf.WF_BF16 if kw["D"] == 128 else wf.WF_F32
    d = wf.make_desc(kw["H"], kw["D"], kw["fh"], kw["fw"], kw["F"], kw["Wc"], kw["R"], kw["n0"], kw["noise_t"],
                     S=kw["S"], dtype=dtype, num_ctas=kw["num_ctas"])
    host = _plan(d)
    ref = orc.plan_round(kw["H"], kw["D"], kw["fh"], kw["fw"], kw["F"], kw["Wc"], kw["R"], kw["S"], kw["n0"],
                         kw["noise_t"], kw["num_ctas"], split=dtype == wf.WF_BF16)
    _compare_plan(host, ref, kw)


def test_plan_golden_cases_through_the_library():
    for c in json.load(open(os.path.join(GOLDEN, "plan_cases.json")))["cases"]:
        dtype = wf.WF_BF16 if c["D"] == 128 else wf.WF_F32
        d = wf.make_desc(c["H"], c["D"], c["fh"], c["fw"], c["F"], c["Wc"], c["R"], c["n0"], c["noise_t"],
                         S=c["S"], dtype=dtype, num_ctas=c["num_ctas"])
        p = wf.decode_plan(_plan(d))
        for got, want in zip(p["chunks"], c["chunks"]):
            assert got["slot"] == want["slot"] and got["keys"] == want["keys"], c["name"]
            assert got["vis_slots"] == want["vis_slots"] and got["key_tiles"] == want["key_tiles"], c["name"]
            assert [list(s) for s in got["segs"]] == want["segs"], c["name"]
        if "per_cta" in c:
            assert [[list(u[:3]) for u in lst] for lst in p["per_cta"]] == c["per_cta"]


def test_balance_golden_cases_through_the_library():
    for c in json.load(open(os.path.join(GOLDEN, "balance_cases.json")))["cases"]:
        assert wf.wf_balance_units(c["costs"], c["num_bins"]) == c["bins"], c["name"]


def test_balance_library_matches_oracle_on_random_lists():
    rng = np.random.default_rng(11)
    for _ in range(400):
        n = int(rng.integers(0, 40))
        G = int(rng.integers(1, 9))
        costs = [int(x) for x in rng.integers(0, int(rng.choice([3, 20, 1000])), n)]
        assert wf.wf_balance_units(costs, G) == orc.balance(costs, G)[0], (costs, G)


@pytest.mark.parametrize("costs,bins", [([1, -1], 2), ([1, 2], 0), ([1], 65537), ([1 << 41], 2)])
def test_balance_rejects_bad_arguments(costs, bins):
    with pytest.raises(wf.WfError) as e:
        wf.wf_balance_units(costs, bins)
    assert e.value.code == wf.WF_ERR_INVALID_ARG


@pytest.mark.parametrize("D,pairs", [(64, (0, 0, 0)), (128, (0, 0, 0)), (64, (11, 11, 10)), (128, (64, 0, 0))])
def test_plan_rope_tables_match_oracle_angles(D, pairs):
    dtype = wf.WF_BF16 if D == 128 else wf.WF_F32
    d = wf.make_desc(2, D, 5, 7, 3, 2, 3, 9, [1, 2, 3], pairs=pairs, theta=10000.0, dtype=dtype, num_ctas=2)
    p = wf.decode_plan(_plan(d))
    Pt, Ph, Pw = (p["Pt"], p["Ph"], p["Pw"])
    if pairs == (0, 0, 0):
        assert (Pt, Ph, Pw) == orc.rope_split(D)
    else:
        assert (Pt, Ph, Pw) == pairs
    # oracle angles for every token of the round's chunks
    for i in range(3):
        t, h, w = orc.token_positions(9 + i, 3, 5, 7)
        ang = orc.rope_angles(t, h, w, (Pt, Ph, Pw), 10000.0)
        f = np.arange(len(t)) // 35
        got_c = np.concatenate([p["rope_t"][0][i * 3 + f], p["rope_h"][0][h], p["rope_w"][0][w]], axis=1)
        got_s = np.concatenate([p["rope_t"][1][i * 3 + f], p["rope_h"][1][h], p["rope_w"][1][w]], axis=1)
        # both sides evaluate cos/sin of the same fp64 angle: at most an ulp or so apart
        tol = 4e-16 * np.maximum(1, np.abs(ang))
        assert np.all(np.abs(got_c - np.cos(ang)) <= tol)
        assert np.all(np.abs(got_s - np.sin(ang)) <= tol)


def test_random_round_shapes_plan_bit_exact_against_the_oracle():
    """Random shapes, positions, ring sizes and CTA counts (split and unsplit work lists)."""
    rng = np.random.default_rng(2024)
    for _ in range(200):  # about one in six draws splits units' keys
        D = int(rng.choice([64, 128]))
        dtype = wf.WF_BF16 if D == 128 else wf.WF_F32
        R = int(rng.integers(1, 7))
        Wc = int(rng.integers(0, 9))
        S = Wc + R + int(rng.integers(0, 4))
        kw = dict(H=int(rng.integers(1, 13)), D=D, fh=int(rng.integers(1, 40)), fw=int(rng.integers(1, 40)),
                  F=int(rng.integers(1, 4)), Wc=Wc, R=R, S=S, n0=int(rng.integers(0, 300)),
                  noise_t=sorted(int(x) for x in rng.integers(0, 1001, R)), num_ctas=int(rng.integers(1, 300)))
        d = wf.make_desc(kw["H"], kw["D"], kw["fh"], kw["fw"], kw["F"], kw["Wc"], kw["R"], kw["n0"], kw["noise_t"],
                         S=kw["S"], dtype=dtype, num_ctas=kw["num_ctas"])
        host = _plan(d)
        ref = orc.plan_round(kw["H"], kw["D"], kw["fh"], kw["fw"], kw["F"], kw["Wc"], kw["R"], kw["S"], kw["n0"],
                             kw["noise_t"], kw["num_ctas"], split=dtype == wf.WF_BF16)
        _compare_plan(host, ref, kw)
        assert wf.decode_plan(host)["key_parts"] == ref["key_parts"], kw


def test_planning_a_round_is_fast_enough_to_overlap_the_previous_one():
    """Host planning must stay far below a round's device time (4 ms for the 1.3B round, 85 ms at 720p)."""
    import time
    cases = [(12, 30, 52, 7, 4, 148, 2.0), (40, 45, 80, 7, 4, 148, 20.0), (12, 30, 52, 6, 1, 148, 2.0)]
    for H, fh, fw, Wc, R, ctas, limit_ms in cases:
        d = wf.make_desc(H, 128, fh, fw, 3, Wc, R, Wc + 40, [250, 500, 750, 1000][:R] if R > 1 else [1000],
                         dtype=wf.WF_BF16, num_ctas=ctas)
        host = _plan(d)
        t0 = time.perf_counter()
        for _ in range(5):
            wf.wf_plan_round(d, host)
        ms = (time.perf_counter() - t0) / 5 * 1e3
        assert ms < limit_ms, (H, fh, fw, R, ms)
