"""A streaming rollout of wave rounds on one GPU, driven through the C ABI.

PyTorch only allocates device memory and supplies the stream; planning,
input generation, RoPE/append and attention all run in libwf.

Round r of a rollout has its oldest in-round chunk at n0 = first_n0 + r.
Before round 0 the ring is prefilled with chunks 0 .. first_n0-1 (clean
history, generator tag -1).  Every round regenerates the in-round chunks'
Q/K/V with tag r (they are re-denoised each round), appends K'/V into their
ring slots and runs the block-causal attention.  The chunk that leaves the
round keeps its K'/V in place as clean cache; the slot of the evicted chunk
n0 - Wc is the one the incoming chunk n0 + R overwrites next round.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import torch

from . import wf


@dataclass
class RoundConfig:
    name: str
    H: int
    D: int
    fh: int
    fw: int
    F: int
    Wc: int
    R: int
    noise_t: Sequence[int]
    dtype: int = wf.WF_BF16
    theta: float = 10000.0
    pairs: tuple = (0, 0, 0)
    kscale: bool = False
    S: int = 0
    rounds: int = 1
    check_rounds: Sequence[int] = field(default_factory=lambda: (0,))

    @property
    def C(self) -> int:
        return self.F * self.fh * self.fw

    @property
    def slots(self) -> int:
        return self.S or (self.Wc + self.R)

    def visible_keys(self):
        return [(self.Wc + i + 1) * self.C for i in range(self.R)]

    def attn_flops(self) -> float:
        """Algorithmic flops of one steady round: 4*D per visible (query, key) pair."""
        return 4.0 * self.D * self.H * self.C * sum(self.visible_keys())

    def rope_bytes(self) -> int:
        """Algorithmic bytes of one RoPE/append pass: read Q,K,V + write Q',K',V."""
        elem = 2 if self.dtype == wf.WF_BF16 else 4
        return 6 * self.R * self.C * self.H * self.D * elem


# The five synthetic wave-round workloads (shapes of the Wan2.1 family).
CONFIGS = {
    "tiny_f32": RoundConfig("tiny fp32 wave round", H=2, D=64, fh=4, fw=6, F=2, Wc=3, R=3,
                            noise_t=(250, 500, 750), dtype=wf.WF_F32),
    "wan13b_single": RoundConfig("Wan2.1-1.3B-shaped single chunk", H=12, D=128, fh=30, fw=52, F=3, Wc=6, R=1,
                                 noise_t=(1000,)),
    "wan13b_round": RoundConfig("Wan2.1-1.3B-shaped 4-step wave round", H=12, D=128, fh=30, fw=52, F=3, Wc=7,
                                R=4, noise_t=(250, 500, 750, 1000), rounds=64, check_rounds=(0, 1, 7, 63)),
    "wan14b_round": RoundConfig("14B-shaped wave round", H=40, D=128, fh=30, fw=52, F=3, Wc=7, R=4,
                                noise_t=(250, 500, 750, 1000), kscale=True),
    "p720_rollout": RoundConfig("720p-shaped long rollout", H=40, D=128, fh=45, fw=80, F=3, Wc=7, R=4,
                                noise_t=(250, 500, 750, 1000), rounds=200, check_rounds=(0, 1, 21, 199)),
}

# Cache-refresh schedules: the round also carries the graduating chunk once
# more at t=0 (the oldest in-round member), so the clean K/V it leaves in its
# ring slot are those of the clean latent.  4-step schedule + refresh (R=5)
# and 5-step schedule + refresh (R=6, steps evenly spaced: the pages print no
# 5-step list).
REFRESH_CONFIGS = {
    "wan13b_refresh": RoundConfig("Wan2.1-1.3B-shaped 4-step round with cache refresh", H=12, D=128, fh=30, fw=52,
                                  F=3, Wc=7, R=5, noise_t=(0, 250, 500, 750, 1000), rounds=16,
                                  check_rounds=(0, 1, 15)),
    "wan13b_5step_refresh": RoundConfig("Wan2.1-1.3B-shaped 5-step round with cache refresh", H=12, D=128, fh=30,
                                        fw=52, F=3, Wc=7, R=6, noise_t=(0, 200, 400, 600, 800, 1000), rounds=16,
                                        check_rounds=(0, 1, 15)),
}
CONFIGS.update(REFRESH_CONFIGS)


class Rollout:
    """Device state of one stream: the K/V ring pool, the round's buffers, plan and workspace."""

    def __init__(self, cfg: RoundConfig, device="cuda", seed: int = 42, first_n0: Optional[int] = None,
                 num_ctas: int = 0, want_lse: bool = True, stream: Optional[torch.cuda.Stream] = None,
                 fp8: bool = False, fused_q_rope: bool = False):
        self.cfg = cfg
        self.device = torch.device(device)
        self.seed = seed
        self.first_n0 = cfg.Wc if first_n0 is None else first_n0
        self.num_ctas = num_ctas
        self.stream = stream or torch.cuda.current_stream(self.device)
        tdt = torch.bfloat16 if cfg.dtype == wf.WF_BF16 else torch.float32
        C, H, D, R, S = cfg.C, cfg.H, cfg.D, cfg.R, cfg.slots
        nq = max(R, 1) * C
        kw = dict(dtype=tdt, device=self.device)
        self.k_pool = torch.zeros(S * C, H, D, **kw)
        self.v_pool = torch.zeros(S * C, H, D, **kw)
        self.q = torch.empty(nq, H, D, **kw)
        self.k = torch.empty(nq, H, D, **kw)
        self.v = torch.empty(nq, H, D, **kw)
        self.q_rot = torch.empty(nq, H, D, **kw)
        self.out = torch.empty(nq, H, D, **kw)
        self.lse = torch.empty(H, nq, dtype=torch.float32, device=self.device) if want_lse else None
        # fused_q_rope: the attention rotates the raw Q itself (wf_chunk_causal_attn_rope)
        # and the append writes only K'/V (wf_rope3d_append_kv)
        if fused_q_rope and (fp8 or cfg.dtype != wf.WF_BF16):
            raise ValueError("the fused Q-RoPE path takes bf16 rounds with 16-bit scores")
        self.fused_q_rope = fused_q_rope
        # 8-bit scores: e4m3 codes of Q' and of the pool's K' with their block scales
        self.fp8 = fp8
        if fp8:
            if cfg.dtype != wf.WF_BF16:
                raise ValueError("the 8-bit score path takes bf16 rounds")
            nblk = -(-C // wf.WF_FP8_BLOCK)
            self.q8 = torch.empty(nq, H, D, dtype=torch.uint8, device=self.device)
            self.q_scales = torch.empty(max(R, 1), nblk, H, dtype=torch.float32, device=self.device)
            self.k8_pool = torch.zeros(S * C, H, D, dtype=torch.uint8, device=self.device)
            self.k_scales = torch.ones(S, nblk, H, dtype=torch.float32, device=self.device)
        self._plan_cap = 0
        self._ensure_plan_capacity(wf.wf_plan_bytes(self.desc(self.first_n0)))
        self.workspace = torch.empty(4096, dtype=torch.uint8, device=self.device)
        wf.wf_attn_workspace_init(self.workspace, self.stream)
        self.round_index = -1

    # ------------------------------------------------------------- planning
    def desc(self, n0: int, R: Optional[int] = None, Wc: Optional[int] = None, noise=None) -> wf.RoundDesc:
        c = self.cfg
        return wf.make_desc(c.H, c.D, c.fh, c.fw, c.F, c.Wc if Wc is None else Wc, c.R if R is None else R, n0,
                            c.noise_t if noise is None else noise, S=c.slots, pairs=c.pairs, theta=c.theta,
                            dtype=c.dtype, num_ctas=self.num_ctas)

    def _ensure_plan_capacity(self, n: int):
        if n <= self._plan_cap:
            return
        self.stream.synchronize()
        self._plan_cap = n
        # two pinned host copies used in turn: planning round r+1 on the host
        # overlaps round r on the device; an event guards each copy's reuse
        self._host_plans = [torch.empty(n, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
        self._plan_events = [torch.cuda.Event() for _ in range(2)]
        self._plan_slot = 0
        self.host_plan = self._host_plans[0]
        self.dev_plan = torch.empty(n, dtype=torch.uint8, device=self.device)

    def _plan(self, d: wf.RoundDesc):
        self._ensure_plan_capacity(wf.wf_plan_bytes(d))
        k = self._plan_slot = 1 - self._plan_slot
        buf = self._host_plans[k]
        self._plan_events[k].synchronize()
        wf.wf_plan_round(d, buf, self.dev_plan, self.stream, host_bytes=buf.numel(), dev_bytes=self.dev_plan.numel())
        self._plan_events[k].record(self.stream)
        self.host_plan = buf
        self._ensure_workspace(wf.wf_attn_workspace_bytes(buf))

    def _ensure_workspace(self, n: int):
        """The attention workspace: a status block, plus partial slots when the plan splits units' keys."""
        if n <= self.workspace.numel():
            return
        self.stream.synchronize()
        self.workspace = torch.empty(n, dtype=torch.uint8, device=self.device)
        wf.wf_attn_workspace_init(self.workspace, self.stream, nbytes=wf.WF_ATTN_STATUS_BYTES)

    # ------------------------------------------------------------- inputs
    def fill_inputs(self, n_first: int, nchunks: int, tag: int):
        c = self.cfg
        for t, dst in ((wf.WF_SYNTH_Q, self.q), (wf.WF_SYNTH_K, self.k), (wf.WF_SYNTH_V, self.v)):
            wf.wf_synth_fill(dst, c.dtype, self.seed, t, tag, n_first, nchunks, c.C, c.H, c.D,
                             kscale=(c.kscale and t == wf.WF_SYNTH_K), stream=self.stream)

    def prefill(self):
        """Write clean history chunks 0 .. first_n0-1 into the ring (tag -1), R at a time."""
        c = self.cfg
        n = 0
        while n < self.first_n0:
            g = min(c.R, self.first_n0 - n)
            self.fill_inputs(n, g, -1)
            self._plan(self.desc(n, R=g, Wc=0, noise=[0] * g))
            wf.wf_rope3d_append_kv(self.host_plan, self.dev_plan, self.k, self.v, self.k_pool, self.v_pool,
                                   self.stream)
            if self.fp8:
                wf.wf_quantize_fp8(self.host_plan, self.k_pool, self.k8_pool, self.k_scales, wf.WF_FP8_K, self.stream)
            n += g
        self.round_index = -1

    # ------------------------------------------------------------- rounds
    def n0_of(self, r: int) -> int:
        return self.first_n0 + r

    def plan_round(self, r: int):
        self._plan(self.desc(self.n0_of(r)))

    def append(self):
        if self.fused_q_rope:
            wf.wf_rope3d_append_kv(self.host_plan, self.dev_plan, self.k, self.v, self.k_pool, self.v_pool,
                                   self.stream)
            return
        wf.wf_rope3d_append(self.host_plan, self.dev_plan, self.q, self.k, self.v, self.q_rot, self.k_pool,
                            self.v_pool, self.stream)
        if self.fp8:
            self.quantize()

    def quantize(self):
        """e4m3 codes and block scales of this round's Q' and of its chunks' K' in the pool."""
        wf.wf_quantize_fp8(self.host_plan, self.q_rot, self.q8, self.q_scales, wf.WF_FP8_Q, self.stream)
        wf.wf_quantize_fp8(self.host_plan, self.k_pool, self.k8_pool, self.k_scales, wf.WF_FP8_K, self.stream)

    def attend(self, scale: float = 0.0):
        if self.fp8:
            wf.wf_chunk_causal_attn_fp8(self.host_plan, self.dev_plan, self.q8, self.q_scales, self.k8_pool,
                                        self.k_scales, self.v_pool, self.out, self.lse, scale, self.workspace,
                                        self.stream)
        elif self.fused_q_rope:
            wf.wf_chunk_causal_attn_rope(self.host_plan, self.dev_plan, self.q, self.k_pool, self.v_pool, self.out,
                                         self.lse, scale, self.workspace, self.stream)
        else:
            wf.wf_chunk_causal_attn(self.host_plan, self.dev_plan, self.q_rot, self.k_pool, self.v_pool, self.out,
                                    self.lse, scale, self.workspace, self.stream)

    def run_round(self, r: int, fill: bool = True):
        """Generate round r's inputs (tag r), plan, RoPE/append, attention."""
        if fill:
            self.fill_inputs(self.n0_of(r), self.cfg.R, r)
        self.plan_round(r)
        self.append()
        self.attend()
        self.round_index = r

    def device_status(self):
        return wf.wf_attn_workspace_status(self.workspace, self.stream)

    # ------------------------------------------------------------- checkpoint / resume
    def checkpoint(self) -> dict:
        """Host copy of the stream state after the last completed round.

        The ring pool is the only state carried between rounds: a round's plan
        is a function of (n0, Wc, R, S) and its inputs are regenerated, so
        resuming is restoring the pool and planning the next round.
        """
        self.stream.synchronize()
        state = {"round": self.round_index, "first_n0": self.first_n0, "seed": self.seed,
                 "k_pool": self.k_pool.cpu(), "v_pool": self.v_pool.cpu()}
        if self.fp8:
            state.update(k8_pool=self.k8_pool.cpu(), k_scales=self.k_scales.cpu())
        return state

    def restore(self, state: dict):
        """Load a checkpoint() taken from a rollout of the same configuration."""
        names = ("k_pool", "v_pool") + (("k8_pool", "k_scales") if self.fp8 else ())
        for name in names:
            if name not in state:
                raise ValueError(f"checkpoint has no {name}")
            src, dst = state[name], getattr(self, name)
            if src.shape != dst.shape or src.dtype != dst.dtype:
                raise ValueError(f"checkpoint {name} is {tuple(src.shape)} {src.dtype}, "
                                 f"this rollout holds {tuple(dst.shape)} {dst.dtype}")
        with torch.cuda.stream(self.stream):
            for name in names:
                getattr(self, name).copy_(state[name], non_blocking=False)
        self.first_n0 = int(state["first_n0"])
        self.seed = int(state["seed"])
        self.round_index = int(state["round"])
        self.stream.synchronize()


def default_scale(cfg: RoundConfig) -> float:
    return 1.0 / math.sqrt(cfg.D)
