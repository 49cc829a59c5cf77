"""The allocation-free attention entry point, through the C ABI.

wf_chunk_causal_attn_noalloc serves callers that cannot call cudaMalloc (for
instance a host that reserves all device memory for its own pool up front):
its scratch is a static device array held by the library.  It runs the same
deterministic kernel on the same plan and buffers as the regular entry point
(which takes a caller workspace), so its O and LSE must be bit-identical to
the regular call's, whichever of the two runs first and on two calls in a row
(the second checks that the shared static scratch, which keeps the previous
call's contents, does not leak into it).

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""
import pytest
import torch

from chunk_causal_attention_block_b200 import wf
from chunk_causal_attention_block_b200.rollout import Rollout, RoundConfig

pytestmark = pytest.mark.gpu


def _noalloc(ro):
    wf.wf_chunk_causal_attn_noalloc(ro.host_plan, ro.dev_plan, ro.q_rot, ro.k_pool, ro.v_pool, ro.out, ro.lse, 0.0,
                                    ro.stream)


def test_noalloc_entry_point_is_bit_identical_to_regular_entry_point():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = RoundConfig("no-alloc", H=2, D=128, fh=10, fw=10, F=3, Wc=3, R=3, noise_t=(250, 500, 750))
    ro = Rollout(cfg)
    ro.prefill()
    for r in range(2):
        ro.run_round(r)  # regular entry point with a caller workspace
        torch.cuda.synchronize()
        want = ro.out.clone()
        want_lse = ro.lse.clone()
        # no-alloc twice in a row after the regular call ...
        for call in range(2):
            ro.out.fill_(float("nan"))
            ro.lse.fill_(float("nan"))
            _noalloc(ro)
            torch.cuda.synchronize()
            assert torch.equal(ro.out, want), f"round {r} no-alloc call {call}: O differs"
            assert torch.equal(ro.lse, want_lse), f"round {r} no-alloc call {call}: LSE differs"
            assert wf.wf_attn_noalloc_status(ro.stream) == (wf.WF_OK, [0, 0, 0, 0]), "no-alloc device status"
        # ... and the regular call again after the no-alloc calls, on the same plan
        ro.out.fill_(float("nan"))
        ro.lse.fill_(float("nan"))
        ro.attend()  # the regular entry point
        torch.cuda.synchronize()
        assert torch.equal(ro.out, want) and torch.equal(ro.lse, want_lse), f"round {r}: regular after no-alloc"
    assert ro.device_status()[0] == wf.WF_OK
