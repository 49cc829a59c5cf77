"""Out-of-bounds write check for every kernel, with sentinel guard zones.

A memory checker is not available on the GPUs these tests run on, so this is
the stand-in: every buffer a call writes (Q', O, LSE, the K/V pools, the
attention workspace, the 8-bit codes and scales) is placed between two 4 KB
margins filled with a byte pattern.  After RoPE/append, the attention (bf16,
fp32, 8-bit scores, and a plan that splits units' keys so that the combine
pass runs) and both quantizations, on ragged small rounds over several
rounds, the margins must be intact and the pool slots (and their codes and
scales) of chunks outside the round must be bit-identical to before the call.
Inside the buffers, the outputs are first filled with NaN and must be written
everywhere they should be (no NaN left in Q', O or LSE).
"""
import numpy as np
import pytest
import torch

from chunk_causal_attention_block_b200 import wf
from chunk_causal_attention_block_b200.rollout import CONFIGS, Rollout, RoundConfig

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes on each side


class Guarded:
    """A tensor placed in the middle of a larger byte buffer whose margins hold a pattern."""

    def __init__(self, like: torch.Tensor):
        self.nbytes = like.numel() * like.element_size()
        self.base = torch.empty(MARGIN + self.nbytes + MARGIN, dtype=torch.uint8, device=like.device)
        self.pattern = (torch.arange(MARGIN, dtype=torch.int64, device=like.device) * 37 + 11).remainder(251) \
            .to(torch.uint8)
        self.base[:MARGIN] = self.pattern
        self.base[MARGIN + self.nbytes:] = self.pattern
        mid = self.base[MARGIN:MARGIN + self.nbytes]
        mid.copy_(like.contiguous().view(torch.uint8).reshape(-1))
        self.view = mid.view(like.dtype).view(like.shape)

    def intact(self) -> bool:
        return bool(torch.equal(self.base[:MARGIN], self.pattern)) and \
            bool(torch.equal(self.base[MARGIN + self.nbytes:], self.pattern))


GUARDED = ("q_rot", "out", "lse", "k_pool", "v_pool", "workspace")
GUARDED_FP8 = ("q8", "q_scales", "k8_pool", "k_scales")


def _guard(ro: Rollout):
    names = GUARDED + (GUARDED_FP8 if ro.fp8 else ())
    guards = {}
    for n in names:
        g = Guarded(getattr(ro, n))
        setattr(ro, n, g.view)
        guards[n] = g
    return guards


def _slot_view(ro: Rollout, name: str):
    cfg = ro.cfg
    t = getattr(ro, name)
    if name == "k_scales":
        return t  # [S, nblk, H]
    return t.view(cfg.slots, cfg.C, cfg.H, cfg.D)


def run_guarded(cfg: RoundConfig, rounds: int, fp8=False, first_n0=None):
    ro = Rollout(cfg, fp8=fp8, first_n0=first_n0)
    ro.prefill()
    pools = ("k_pool", "v_pool") + (("k8_pool", "k_scales") if fp8 else ())
    for r in range(rounds):
        ro.fill_inputs(ro.n0_of(r), cfg.R, r)
        ro.plan_round(r)                      # may grow the workspace: guard after planning
        torch.cuda.synchronize()
        guards = _guard(ro)
        for n in ("q_rot", "out", "lse"):
            getattr(ro, n).fill_(float("nan"))
        if fp8:
            ro.q_scales.fill_(float("nan"))
        before = {n: _slot_view(ro, n).clone() for n in pools}
        ro.append()
        ro.attend()
        torch.cuda.synchronize()
        for n, g in guards.items():
            assert g.intact(), f"{cfg.name} round {r}: a write landed outside {n}"
        in_round = {(ro.n0_of(r) + i) % cfg.slots for i in range(cfg.R)}
        for n in pools:
            after = _slot_view(ro, n)
            for s in range(cfg.slots):
                if s not in in_round:
                    assert torch.equal(after[s], before[n][s]), f"{cfg.name} round {r}: {n} slot {s} changed"
        assert not torch.isnan(ro.q_rot.float()).any(), f"{cfg.name} round {r}: Q' not fully written"
        assert not torch.isnan(ro.out.float()).any(), f"{cfg.name} round {r}: O not fully written"
        assert not torch.isnan(ro.lse).any(), f"{cfg.name} round {r}: LSE not fully written"
        if fp8:
            assert not torch.isnan(ro.q_scales).any(), f"{cfg.name} round {r}: Q scales not fully written"
        assert ro.device_status()[0] == wf.WF_OK
    return ro


CASES = [
    RoundConfig("ragged small", H=2, D=128, fh=10, fw=10, F=3, Wc=3, R=3, noise_t=(250, 500, 750)),
    RoundConfig("tiny chunks", H=3, D=128, fh=5, fw=7, F=2, Wc=2, R=4, noise_t=(0, 250, 500, 750)),
    RoundConfig("C=1", H=2, D=128, fh=1, fw=1, F=1, Wc=5, R=4, noise_t=(250, 500, 750, 1000)),
    RoundConfig("key split", H=2, D=128, fh=30, fw=52, F=1, Wc=2, R=1, noise_t=(1000,)),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wf.lib()
    yield


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_bf16_round_writes_stay_inside_their_buffers(cfg):
    run_guarded(cfg, cfg.Wc + cfg.R + 2)


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fp8_round_writes_stay_inside_their_buffers(cfg):
    run_guarded(cfg, cfg.Wc + cfg.R + 2, fp8=True)


def test_fp32_round_writes_stay_inside_their_buffers():
    run_guarded(CONFIGS["tiny_f32"], 5)


def test_stream_start_writes_stay_inside_their_buffers():
    cfg = RoundConfig("start", H=2, D=128, fh=10, fw=12, F=2, Wc=5, R=3, noise_t=(250, 500, 750))
    run_guarded(cfg, 5, first_n0=1)
