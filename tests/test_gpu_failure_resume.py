"""Failure detection and resume on the GPU, through the C ABI.

Failure detection: every wait of the tensor-core attention kernel is bounded
(WF_WAIT_TIMEOUT_MS).  With WF_DEBUG_STALL_FIRST_LOAD=1 the TMA producer of
CTA 0 never issues its first K tile, so that tile's full-barrier is never
armed and the waits on it run out.  The kernel must end, the workspace status
must read WF_ERR_DEVICE_TIMEOUT with block 0, and the context must stay
usable: the next launch, on the same buffers, passes the oracle.  Nothing
faults, traps or hangs; the other CTAs complete normally.

Resume: the ring pool is the whole state carried between rounds.  A rollout
checkpointed after round k and restored into a fresh Rollout continues with
bit-identical outputs to the uninterrupted one.
"""
import numpy as np
import pytest
import torch

from chunk_causal_attention_block_b200 import wf
from chunk_causal_attention_block_b200.rollout import Rollout, RoundConfig
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wf.lib()
    yield


SMALL = RoundConfig("ragged small", H=2, D=128, fh=10, fw=10, F=3, Wc=3, R=3, noise_t=(250, 500, 750))


def test_expired_wait_reports_timeout_and_context_stays_usable(monkeypatch):
    ro = Rollout(SMALL)
    ro.prefill()
    ro.fill_inputs(ro.n0_of(0), SMALL.R, 0)
    ro.plan_round(0)
    ro.append()
    hdr = wf.decode_plan(ro.host_plan)
    assert hdr["per_cta"][0], "CTA 0 must own work for the stall to bite"

    ro.out.fill_(0)
    monkeypatch.setenv("WF_WAIT_TIMEOUT_MS", "100")
    monkeypatch.setenv("WF_DEBUG_STALL_FIRST_LOAD", "1")
    ro.attend()
    code, detail = ro.device_status()
    monkeypatch.delenv("WF_DEBUG_STALL_FIRST_LOAD")
    monkeypatch.delenv("WF_WAIT_TIMEOUT_MS")
    assert code == wf.WF_ERR_DEVICE_TIMEOUT, (code, detail)
    assert detail[0] == wf.WF_ERR_DEVICE_TIMEOUT and detail[2] == 0, detail
    assert torch.cuda.is_available() and torch.cuda.synchronize() is None

    # the same buffers again, status word cleared: a normal, correct launch
    wf.wf_attn_workspace_init(ro.workspace, ro.stream)
    ro.attend()
    torch.cuda.synchronize()
    code, detail = ro.device_status()
    assert code == wf.WF_OK, (code, detail)
    gc.check_attention(ro, 0, [0, 1], np.arange(SMALL.R * SMALL.C), "after timeout")


def test_resume_from_checkpoint_is_bit_identical():
    k, last = 3, 6
    a = Rollout(SMALL)
    a.prefill()
    for r in range(k + 1):
        a.run_round(r)
    state = a.checkpoint()
    want = {}
    for r in range(k + 1, last + 1):
        a.run_round(r)
        torch.cuda.synchronize()
        want[r] = (a.out.clone(), a.lse.clone(), a.k_pool.clone())

    b = Rollout(SMALL)  # fresh device state: zero pool, no prefill
    b.restore(state)
    assert b.round_index == k
    for r in range(k + 1, last + 1):
        b.run_round(r)
        torch.cuda.synchronize()
        out, lse, kp = want[r]
        assert torch.equal(b.out, out), r
        assert torch.equal(b.lse, lse), r
        assert torch.equal(b.k_pool, kp), r
    assert b.device_status()[0] == wf.WF_OK
    gc.check_attention(b, last, [1], gc.sample_rows(SMALL), "resumed")


def test_restore_rejects_a_checkpoint_of_another_shape():
    a = Rollout(SMALL)
    state = a.checkpoint()
    other = RoundConfig("other", H=2, D=128, fh=10, fw=10, F=3, Wc=2, R=3, noise_t=(250, 500, 750))
    b = Rollout(other)
    with pytest.raises(ValueError):
        b.restore(state)
