"""The allocation-free attention entry point, through the C ABI.

wf_chunk_causal_attn_noalloc serves callers that cannot call cudaMalloc (for
instance a host that reserves all device memory for its own pool up front):
its scratch is a static device array held by the library.  Two calls in a row
must match the regular entry point, which takes a caller workspace, within the
bf16 gates the other tests use; the second call checks that the shared static
scratch, which keeps the previous call's contents, does not leak into it.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from chunk_causal_attention_block_b200 import wf
from chunk_causal_attention_block_b200.rollout import Rollout, RoundConfig
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


def test_noalloc_entry_point_matches_regular_entry_point_twice():
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
        for call in range(2):
            ro.out.zero_()
            ro.lse.zero_()
            wf.wf_chunk_causal_attn_noalloc(ro.host_plan, ro.dev_plan, ro.q_rot, ro.k_pool, ro.v_pool, ro.out,
                                            ro.lse, 0.0, ro.stream)
            torch.cuda.synchronize()
            gc.assert_bf16_close(gc.to_np(ro.out), gc.to_np(want), f"round {r} call {call}")
            np.testing.assert_allclose(ro.lse.cpu().numpy(), want_lse.cpu().numpy(), rtol=0, atol=1e-5)
    assert ro.device_status()[0] == wf.WF_OK
