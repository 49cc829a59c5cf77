"""Shared helpers of the GPU parity tests: oracle inputs drawn on the host
with the same generator the device uses, row sampling and tolerances."""
from __future__ import annotations

import math

import numpy as np
import torch

from chunk_causal_attention_block_b200 import synth, wf
from chunk_causal_attention_block_b200.rollout import RoundConfig, Rollout
from oracle import wf_oracle as orc

# bf16 gates on O (max-abs, mean-abs) plus an internal relative-RMS gate.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
BF16_REL_RMS = 1e-2
F32_REL = 1e-4


def dtype_name(cfg: RoundConfig) -> str:
    return "bf16" if cfg.dtype == wf.WF_BF16 else "f32"


def pairs_of(cfg: RoundConfig):
    return cfg.pairs if any(cfg.pairs) else orc.rope_split(cfg.D)


def raw_chunk(cfg, seed, tensor, tag, n, heads):
    return synth.chunk_values(seed, tensor, tag, n, cfg.C, cfg.H, cfg.D, dtype_name(cfg), heads=heads,
                              kscale=(cfg.kscale and tensor == synth.TENSOR_K)).astype(np.float64)


def oracle_inputs(cfg: RoundConfig, n0: int, first_n0: int, heads, seed=42, k_override=None):
    """Raw (pre-RoPE) arrays of the round with oldest in-round chunk n0, restricted to `heads`."""
    R, Wc = cfg.R, cfg.Wc
    wc_eff = min(Wc, n0)
    tag = synth.kv_tag(n0, n0, first_n0)
    q = np.stack([raw_chunk(cfg, seed, synth.TENSOR_Q, tag, n0 + i, heads) for i in range(R)])
    k = np.stack([raw_chunk(cfg, seed, synth.TENSOR_K, tag, n0 + i, heads) for i in range(R)])
    v = np.stack([raw_chunk(cfg, seed, synth.TENSOR_V, tag, n0 + i, heads) for i in range(R)])
    cache = list(range(n0 - wc_eff, n0))
    shape = (0, cfg.C, len(heads), cfg.D)
    kc = np.stack([raw_chunk(cfg, seed, synth.TENSOR_K, synth.kv_tag(n, n0, first_n0), n, heads)
                   for n in cache]) if cache else np.zeros(shape)
    vc = np.stack([raw_chunk(cfg, seed, synth.TENSOR_V, synth.kv_tag(n, n0, first_n0), n, heads)
                   for n in cache]) if cache else np.zeros(shape)
    if k_override is not None:
        k, kc = k_override(k, kc)
    return q, k, v, kc, vc


def oracle_call(cfg: RoundConfig, n0: int, arrays, rows=None, fp8=False):
    q, k, v, kc, vc = arrays
    return orc.wave_round(q, k, v, kc, vc, n0=n0, F=cfg.F, fh=cfg.fh, fw=cfg.fw, pairs=pairs_of(cfg),
                          theta=cfg.theta, dtype=dtype_name(cfg), rows=rows, fp8=fp8)


def oracle_round(cfg: RoundConfig, n0: int, first_n0: int, heads, rows=None, seed=42, k_override=None, fp8=False):
    """Oracle result of the round with oldest in-round chunk n0, restricted to `heads`."""
    return oracle_call(cfg, n0, oracle_inputs(cfg, n0, first_n0, heads, seed, k_override), rows, fp8)


def sample_rows(cfg: RoundConfig, extra=24, seed=0):
    rng = np.random.default_rng(seed)
    C = cfg.C
    picks = set()
    for i in range(cfg.R):
        for r in (0, 1, 127, 128, 129, 255, 256, C - 129, C - 128, C - 2, C - 1):
            if 0 <= r < C:
                picks.add(i * C + r)
        for r in rng.integers(0, C, extra):
            picks.add(i * C + int(r))
    return np.array(sorted(picks))


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_errors(got: np.ndarray, want: np.ndarray):
    d = np.abs(got - want)
    return dict(max_abs=float(d.max()), mean_abs=float(d.mean()),
                rel_rms=float(np.sqrt((d ** 2).mean() / max((want ** 2).mean(), 1e-300))))


def assert_bf16_close(got, want, what=""):
    e = bf16_errors(got, want)
    assert e["max_abs"] <= BF16_MAX_ABS and e["mean_abs"] <= BF16_MEAN_ABS and e["rel_rms"] <= BF16_REL_RMS, \
        f"{what} {e}"
    return e


def assert_f32_close(got, want, what=""):
    # max |O - O_ref| / max |O_ref| per head
    for h in range(got.shape[1]):
        rel = np.abs(got[:, h] - want[:, h]).max() / np.abs(want[:, h]).max()
        assert rel <= F32_REL, f"{what} head {h}: {rel}"


def run_rollout(cfg: RoundConfig, rounds, first_n0=None, num_ctas=0, seed=42, on_round=None, fp8=False):
    """Prefill, then run rounds 0..max(rounds); call on_round(ro, r) after each listed round."""
    ro = Rollout(cfg, seed=seed, first_n0=first_n0, num_ctas=num_ctas, fp8=fp8)
    ro.prefill()
    last = max(rounds)
    for r in range(last + 1):
        ro.run_round(r)
        if r in rounds and on_round is not None:
            torch.cuda.synchronize()
            on_round(ro, r)
    torch.cuda.synchronize()
    code, detail = ro.device_status()
    assert code == wf.WF_OK, (code, detail)
    return ro


def check_attention(ro: Rollout, r: int, heads, rows, what="", fp8=None):
    cfg = ro.cfg
    fp8 = ro.fp8 if fp8 is None else fp8
    ref = oracle_round(cfg, ro.n0_of(r), ro.first_n0, heads, rows=rows, seed=ro.seed, fp8=fp8)
    got = to_np(ro.out[rows][:, heads])
    if cfg.dtype == wf.WF_BF16:
        e = assert_bf16_close(got, ref["O"], what)
    else:
        assert_f32_close(got, ref["O"], what)
        e = {}
    if ro.lse is not None:
        lse = ro.lse[heads][:, rows].t().cpu().numpy().astype(np.float64)
        tol = 2e-3 if cfg.dtype == wf.WF_BF16 else 1e-5
        np.testing.assert_allclose(lse, ref["LSE"], rtol=0, atol=tol * max(1.0, np.abs(ref["LSE"]).max()))
    return e, ref


def check_rope_append(ro: Rollout, r: int, heads):
    """Bit-exact Q', K' (pool slots of the in-round chunks) and V against the oracle."""
    cfg = ro.cfg
    n0 = ro.n0_of(r)
    ref = oracle_round(cfg, n0, ro.first_n0, heads, rows=np.array([0]), seed=ro.seed)
    C, R, S = cfg.C, cfg.R, cfg.slots
    q_got = to_np(ro.q_rot[:R * C][:, heads]).reshape(R, C, len(heads), cfg.D)
    mism = {"q": int((q_got != ref["q_rot"]).sum())}
    k_pool = ro.k_pool.view(S, C, cfg.H, cfg.D)
    v_pool = ro.v_pool.view(S, C, cfg.H, cfg.D)
    kq = np.stack([to_np(k_pool[(n0 + i) % S][:, heads]) for i in range(R)])
    vq = np.stack([to_np(v_pool[(n0 + i) % S][:, heads]) for i in range(R)])
    mism["k"] = int((kq != ref["k_rot"]).sum())
    mism["v"] = int((vq != ref["v"]).sum())
    wc_eff = min(cfg.Wc, n0)
    kc = np.stack([to_np(k_pool[(n0 - wc_eff + c) % S][:, heads]) for c in range(wc_eff)]) if wc_eff else None
    if wc_eff:
        mism["k_cache"] = int((kc != ref["k_cache_rot"]).sum())
    return mism
