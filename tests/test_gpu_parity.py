"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Bit-exact: device generator vs host generator, plan, RoPE'd Q', pool K'/V
contents.  Within tolerance: attention outputs (bf16: max-abs 2e-2, mean-abs
2e-3, relative RMS 1e-2; fp32: 1e-4 relative per head) and LSE.
"""
import dataclasses

import numpy as np
import pytest
import torch

from chunk_causal_attention_block_b200 import synth, wf
from chunk_causal_attention_block_b200.rollout import CONFIGS, Rollout, RoundConfig
from oracle import wf_oracle as orc
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wf.lib()
    yield


# ------------------------------------------------------------------ generator

@pytest.mark.parametrize("dtype,kscale", [(wf.WF_BF16, False), (wf.WF_F32, False), (wf.WF_BF16, True)])
def test_device_generator_is_bit_identical_to_host(dtype, kscale):
    C, H, D, n_first, nch = 48, 5, 64, 9, 3
    dst = torch.empty(nch * C, H, D, dtype=torch.bfloat16 if dtype == wf.WF_BF16 else torch.float32,
                      device="cuda")
    wf.wf_synth_fill(dst, dtype, 42, synth.TENSOR_K, 3, n_first, nch, C, H, D, kscale=kscale)
    got = dst.float().cpu().numpy().reshape(nch, C, H, D)
    for c in range(nch):
        want = synth.chunk_values(42, synth.TENSOR_K, 3, n_first + c, C, H, D,
                                  "bf16" if dtype == wf.WF_BF16 else "f32", kscale=kscale)
        assert np.array_equal(got[c], want)


# ------------------------------------------------------------------ RoPE / append

@pytest.mark.parametrize("name,heads,rounds", [
    ("tiny_f32", [0, 1], (0, 4)),
    ("wan13b_single", [0, 11], (0,)),
    ("wan13b_round", [3], (0, 7)),
])
def test_rope_append_bit_exact(name, heads, rounds):
    cfg = CONFIGS[name]
    results = {}

    def on_round(ro, r):
        results[r] = gc.check_rope_append(ro, r, heads)

    gc.run_rollout(cfg, rounds, on_round=on_round)
    for r, m in results.items():
        assert all(v == 0 for v in m.values()), (name, r, m)


# ------------------------------------------------------------------ attention

def test_tiny_f32_round_full_oracle():
    cfg = CONFIGS["tiny_f32"]
    errs = []

    def on_round(ro, r):
        e, _ = gc.check_attention(ro, r, [0, 1], np.arange(cfg.R * cfg.C), f"tiny r{r}")
        errs.append(e)

    gc.run_rollout(cfg, (0, 1, 2, 5), on_round=on_round)


def test_tiny_f32_alternate_rope_split():
    cfg = dataclasses.replace(CONFIGS["tiny_f32"], pairs=(11, 11, 10))
    gc.run_rollout(cfg, (0, 3), on_round=lambda ro, r: gc.check_attention(
        ro, r, [0, 1], np.arange(cfg.R * cfg.C), "tiny 11/11/10"))


SMALL_BF16 = [
    # (C not a multiple of 128, two key runs after the ring wraps, several tiles)
    RoundConfig("ragged small", H=2, D=128, fh=10, fw=10, F=3, Wc=3, R=3, noise_t=(250, 500, 750)),
    # empty cache, one in-round chunk: plain bidirectional attention
    RoundConfig("no cache", H=2, D=128, fh=9, fw=13, F=2, Wc=0, R=1, noise_t=(1000,)),
    # one 128-row tile pair with a dead second tile; single key tile runs
    RoundConfig("tiny chunks", H=3, D=128, fh=5, fw=7, F=2, Wc=2, R=4, noise_t=(0, 250, 500, 750)),
    # exactly 256-row chunks: both tiles live, no ragged rows
    RoundConfig("aligned", H=1, D=128, fh=16, fw=16, F=1, Wc=2, R=2, noise_t=(500, 1000)),
    # one token per chunk
    RoundConfig("C=1", H=2, D=128, fh=1, fw=1, F=1, Wc=5, R=4, noise_t=(250, 500, 750, 1000)),
    # the most in-round chunks a round may hold (16), ragged 42-token chunks
    RoundConfig("R=16", H=1, D=128, fh=6, fw=7, F=1, Wc=3, R=16, noise_t=tuple(60 * i for i in range(16))),
    # 14 units for 148 CTAs: every unit's keys split in 4 parts, merged by the combine pass
    RoundConfig("key split", H=2, D=128, fh=30, fw=52, F=1, Wc=2, R=1, noise_t=(1000,)),
]


@pytest.mark.parametrize("cfg", SMALL_BF16, ids=lambda c: c.name)
def test_bf16_small_rounds_all_rows(cfg):
    rows = np.arange(cfg.R * cfg.C)
    heads = list(range(cfg.H))
    gc.run_rollout(cfg, (0, 1, cfg.Wc + cfg.R + 1), on_round=lambda ro, r: gc.check_attention(
        ro, r, heads, rows, f"{cfg.name} r{r}"))


def test_bf16_stream_start_partial_cache():
    cfg = RoundConfig("start", H=2, D=128, fh=10, fw=12, F=2, Wc=5, R=3, noise_t=(250, 500, 750))
    rows = np.arange(cfg.R * cfg.C)
    # first_n0 = 1: one clean chunk, then the window grows round by round
    gc.run_rollout(cfg, (0, 1, 2, 3, 4, 6), first_n0=1, on_round=lambda ro, r: gc.check_attention(
        ro, r, [0, 1], rows, f"start r{r}"))


def test_bf16_work_list_bins_do_not_change_results():
    cfg = SMALL_BF16[0]
    outs = []
    for ctas in (1, 3, 148):
        ro = gc.run_rollout(cfg, (0,), num_ctas=ctas)
        outs.append(ro.out.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("name,heads", [("wan13b_single", [0, 7]), ("wan14b_round", [5, 39])])
def test_bf16_full_size_one_round_sampled(name, heads):
    cfg = CONFIGS[name]
    rows = gc.sample_rows(cfg)
    gc.run_rollout(cfg, (0,), on_round=lambda ro, r: gc.check_attention(ro, r, heads, rows, name))


def test_wan13b_64_round_rollout_sampled():
    cfg = CONFIGS["wan13b_round"]
    rows = gc.sample_rows(cfg, extra=12)
    rope = {}

    def on_round(ro, r):
        gc.check_attention(ro, r, [1, 10], rows, f"wan13b r{r}")
        rope[r] = gc.check_rope_append(ro, r, [10])

    gc.run_rollout(cfg, cfg.check_rounds, on_round=on_round)
    assert all(all(v == 0 for v in m.values()) for m in rope.values()), rope


def test_720p_200_round_rollout_sampled():
    cfg = CONFIGS["p720_rollout"]
    rows = gc.sample_rows(cfg, extra=6)
    gc.run_rollout(cfg, cfg.check_rounds, on_round=lambda ro, r: gc.check_attention(
        ro, r, [17], rows, f"720p r{r}"))


@pytest.mark.parametrize("name,heads", [("wan13b_refresh", [2, 9]), ("wan13b_5step_refresh", [4])])
def test_cache_refresh_rounds_sampled(name, heads):
    """Rounds whose oldest member is the graduating chunk re-run at t=0."""
    cfg = CONFIGS[name]
    rows = gc.sample_rows(cfg, extra=12)
    rope = {}

    def on_round(ro, r):
        gc.check_attention(ro, r, heads, rows, f"{name} r{r}")
        rope[r] = gc.check_rope_append(ro, r, heads[:1])

    gc.run_rollout(cfg, cfg.check_rounds, on_round=on_round)
    assert all(all(v == 0 for v in m.values()) for m in rope.values()), rope


# ------------------------------------------------------------------ invariants and controls

def test_later_chunks_never_touch_earlier_outputs():
    cfg = SMALL_BF16[0]
    ro = gc.run_rollout(cfg, (0,))
    out0 = ro.out.clone()
    C, S = cfg.C, cfg.slots
    n0 = ro.n0_of(0)
    # overwrite the pool slots of in-round chunks 1..R-1 with garbage and rerun attention only
    for i in range(1, cfg.R):
        s = (n0 + i) % S
        ro.k_pool[s * C:(s + 1) * C] = 7.0
        ro.v_pool[s * C:(s + 1) * C] = -3.0
    ro.attend()
    torch.cuda.synchronize()
    assert torch.equal(ro.out[:C], out0[:C])          # chunk 0: bit-identical
    assert not torch.equal(ro.out[C:], out0[C:])      # later chunks see the change


def test_runs_are_deterministic():
    cfg = SMALL_BF16[0]
    a = gc.run_rollout(cfg, (0, 2)).out.clone()
    b = gc.run_rollout(cfg, (0, 2)).out.clone()
    assert torch.equal(a, b)


def test_rescale_path_with_growing_scores():
    """Later key tiles with much larger scores force the lazy O rescale."""
    cfg = RoundConfig("rescale", H=1, D=128, fh=8, fw=16, F=2, Wc=2, R=2, noise_t=(500, 1000))
    ro = Rollout(cfg)
    ro.prefill()
    ro.fill_inputs(ro.n0_of(0), cfg.R, 0)
    ro.k[cfg.C:] *= 6.0  # in-round chunk 1 keys: scores ~6x larger than the cache's
    ro.plan_round(0)
    ro.append()
    ro.attend()
    torch.cuda.synchronize()
    rows = np.arange(cfg.R * cfg.C)

    def boost(k, kc):
        k = k.copy()
        k[1] = orc.round_bf16(k[1] * 6.0)
        return k, kc
    ref = gc.oracle_round(cfg, ro.n0_of(0), ro.first_n0, [0], rows=rows, k_override=boost)
    gc.assert_bf16_close(gc.to_np(ro.out[rows][:, [0]]), ref["O"], "rescale")
    assert ro.device_status()[0] == wf.WF_OK


def test_negative_controls_fail_the_gates():
    cfg = SMALL_BF16[0]
    rows = np.arange(cfg.R * cfg.C)
    ro = gc.run_rollout(cfg, (0,))
    ref = gc.oracle_round(cfg, ro.n0_of(0), ro.first_n0, [0, 1], rows=rows)
    got = gc.to_np(ro.out[rows][:, [0, 1]])
    gc.assert_bf16_close(got, ref["O"], "positive")
    with pytest.raises(AssertionError):
        gc.assert_bf16_close(np.zeros_like(got), ref["O"], "zero output")
    # a round whose oldest chunk is one further on (one-slot-off plan) must not pass
    ref_off = gc.oracle_round(cfg, ro.n0_of(0) + 1, ro.first_n0, [0, 1], rows=rows)
    with pytest.raises(AssertionError):
        gc.assert_bf16_close(got, ref_off["O"], "one slot off")
    # a full (non-causal) mask over the whole pool must not pass either
    q = ref["q_rot"].reshape(-1, 2, cfg.D)
    keys = np.concatenate([ref["k_cache_rot"], ref["k_rot"]]).reshape(-1, 2, cfg.D)
    v_all = np.concatenate([ref["v_cache"], ref["v"]]).reshape(-1, 2, cfg.D)
    full = np.stack([orc.attention(q[:, h], keys[:, h], v_all[:, h], np.ones((len(q), len(keys)), bool),
                                   1 / np.sqrt(cfg.D))[0] for h in range(2)], axis=1)
    with pytest.raises(AssertionError):
        gc.assert_bf16_close(got, full, "no causal mask")


def test_fp32_and_bf16_paths_agree_on_wan_shaped_data():
    """The fp32 CUDA-core kernel and the tensor-core kernel on the same bf16-valued inputs."""
    base = RoundConfig("cross", H=2, D=128, fh=30, fw=52, F=1, Wc=2, R=2, noise_t=(500, 1000))
    f32 = dataclasses.replace(base, dtype=wf.WF_F32)
    a = Rollout(base)
    b = Rollout(f32)
    for ro in (a, b):
        ro.prefill()
    # feed both the bf16 draws (the fp32 rollout gets the same values, exactly)
    a.fill_inputs(a.n0_of(0), base.R, 0)
    b.q.copy_(a.q.float())
    b.k.copy_(a.k.float())
    b.v.copy_(a.v.float())
    for ro in (a, b):
        ro.plan_round(0)
    # the fp32 pool holds fp32-rotated keys; align it with the bf16 pool's values
    a.append()
    b.append()
    b.q_rot.copy_(a.q_rot.float())
    b.k_pool.copy_(a.k_pool.float())
    b.v_pool.copy_(a.v_pool.float())
    a.attend()
    b.attend()
    torch.cuda.synchronize()
    gc.assert_bf16_close(gc.to_np(a.out), gc.to_np(b.out), "fp32 vs bf16 kernels")


# ---------------------------------------------------------------- Q's RoPE inside the attention

FUSED_CASES = SMALL_BF16 + [
    RoundConfig("start", H=2, D=128, fh=10, fw=12, F=2, Wc=5, R=3, noise_t=(250, 500, 750)),
]


def _fused_matches_unfused(cfg, rounds, first_n0=None):
    """The fused path (wf_rope3d_append_kv + wf_chunk_causal_attn_rope from raw Q) against the
    two-call path on the same inputs: O, LSE and the pool bit-identical every round, which also
    shows the in-kernel Q' equals wf_rope3d_append's bit for bit (the MMAs are deterministic)."""
    a = Rollout(cfg, first_n0=first_n0)
    b = Rollout(cfg, first_n0=first_n0, fused_q_rope=True)
    a.prefill()
    b.prefill()
    for r in range(rounds):
        a.run_round(r)
        b.run_round(r)
        torch.cuda.synchronize()
        assert torch.equal(a.out, b.out), f"{cfg.name} round {r}: O"
        assert torch.equal(a.lse, b.lse), f"{cfg.name} round {r}: LSE"
        assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool), f"{cfg.name} round {r}: pool"
    assert b.device_status()[0] == wf.WF_OK
    return a, b


@pytest.mark.parametrize("cfg", FUSED_CASES, ids=lambda c: c.name)
def test_fused_q_rope_bit_identical_to_two_call_path(cfg):
    first = 1 if cfg.name == "start" else None
    _fused_matches_unfused(cfg, cfg.Wc + cfg.R + 2, first_n0=first)


def test_fused_q_rope_full_size_round_against_oracle():
    cfg = CONFIGS["wan13b_round"]
    a, b = _fused_matches_unfused(cfg, 2)
    rows = gc.sample_rows(cfg, extra=8)
    gc.check_attention(b, 1, [4], rows, "fused wan13b r1")
