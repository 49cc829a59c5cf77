"""8-bit score path on the GPU, through the C ABI, against the oracle.

Bit-exact: the e4m3 codes and fp32 block scales of Q' and of the pool's K'
(wf_quantize_fp8) against the oracle's fp8_block_quantize.  Within the bf16
gates (max-abs 2e-2, mean-abs 2e-3, relative RMS 1e-2): the attention of
wf_chunk_causal_attn_fp8 against the oracle evaluated on the same
dequantized codes.  Accuracy of the variant itself: against the exact
(16-bit input) oracle the stated gates still hold and the relative RMS error
stays below 6e-2 (e4m3 keeps 3 mantissa bits: a relative rounding error of at
most 2^-4 per element of Q and K; the oracle alone measures about 3.9e-2 on
these inputs).
"""
import numpy as np
import pytest
import torch

from chunk_causal_attention_block_b200 import wf
from chunk_causal_attention_block_b200.rollout import CONFIGS, RoundConfig
from oracle import wf_oracle as orc
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu

FP8_VS_EXACT_REL_RMS = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wf.lib()
    yield


def _e4m3_values(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def _check_codes(ro, r, heads):
    cfg = ro.cfg
    n0 = ro.n0_of(r)
    ref = gc.oracle_round(cfg, n0, ro.first_n0, heads, rows=np.array([0]), seed=ro.seed, fp8=True)
    C, S, R = cfg.C, cfg.slots, cfg.R
    q8 = _e4m3_values(ro.q8[:R * C][:, heads])
    assert np.array_equal(q8, ref["q8"]), "Q codes"
    assert np.array_equal(ro.q_scales[:R][:, :, heads].cpu().numpy().astype(np.float64), ref["q_scales"]), "Q scales"
    wc_eff = min(cfg.Wc, n0)
    k8 = _e4m3_values(ro.k8_pool.view(S, C, cfg.H, cfg.D)[:, :, heads])
    ks = ro.k_scales[:, :, heads].cpu().numpy().astype(np.float64)
    chunks = list(range(n0 - wc_eff, n0 + R))
    got_k8 = np.concatenate([k8[n % S] for n in chunks])
    got_ks = np.stack([ks[n % S] for n in chunks])
    assert np.array_equal(got_k8, ref["k8"]), "K codes"
    assert np.array_equal(got_ks, ref["k_scales"]), "K scales"


SMALL = [
    RoundConfig("ragged small", H=2, D=128, fh=10, fw=10, F=3, Wc=3, R=3, noise_t=(250, 500, 750)),
    RoundConfig("tiny chunks", H=3, D=128, fh=5, fw=7, F=2, Wc=2, R=4, noise_t=(0, 250, 500, 750)),
    RoundConfig("C=1", H=2, D=128, fh=1, fw=1, F=1, Wc=5, R=4, noise_t=(250, 500, 750, 1000)),
    RoundConfig("no cache", H=2, D=128, fh=9, fw=13, F=2, Wc=0, R=1, noise_t=(1000,)),
    RoundConfig("key split", H=2, D=128, fh=30, fw=52, F=1, Wc=2, R=1, noise_t=(1000,)),
]


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_fp8_codes_bit_exact_and_attention_all_rows(cfg):
    rows = np.arange(cfg.R * cfg.C)
    heads = list(range(cfg.H))

    def on_round(ro, r):
        _check_codes(ro, r, heads)
        gc.check_attention(ro, r, heads, rows, f"{cfg.name} r{r}")

    gc.run_rollout(cfg, (0, 1, cfg.Wc + cfg.R + 1), on_round=on_round, fp8=True)


@pytest.mark.parametrize("name,heads,rounds", [("wan13b_round", [2, 9], (0, 7)), ("wan14b_round", [5, 33], (0,)),
                                               ("wan13b_single", [3], (0,))])
def test_fp8_full_size_sampled(name, heads, rounds):
    cfg = CONFIGS[name]
    rows = gc.sample_rows(cfg, extra=12)

    def on_round(ro, r):
        _check_codes(ro, r, heads[:1])
        gc.check_attention(ro, r, heads, rows, f"{name} r{r}")

    gc.run_rollout(cfg, rounds, on_round=on_round, fp8=True)


def test_fp8_accuracy_against_the_exact_oracle():
    cfg = CONFIGS["wan13b_round"]
    rows = gc.sample_rows(cfg, extra=12)
    errs = []

    def on_round(ro, r):
        ref = gc.oracle_round(cfg, ro.n0_of(r), ro.first_n0, [4], rows=rows, seed=ro.seed)
        got = gc.to_np(ro.out[rows][:, [4]])
        errs.append(gc.bf16_errors(got, ref["O"]))

    gc.run_rollout(cfg, (0,), on_round=on_round, fp8=True)
    e = errs[0]
    assert e["max_abs"] <= 2e-2 and e["mean_abs"] <= 2e-3, e
    assert e["rel_rms"] <= FP8_VS_EXACT_REL_RMS, e


def test_fp8_rollout_resumes_bit_identically():
    cfg = SMALL[0]
    a = gc.run_rollout(cfg, (3,), fp8=True)
    state = a.checkpoint()
    a.run_round(4)
    torch.cuda.synchronize()
    want = a.out.clone()
    from chunk_causal_attention_block_b200.rollout import Rollout
    b = Rollout(cfg, fp8=True)
    b.restore(state)
    b.run_round(4)
    torch.cuda.synchronize()
    assert torch.equal(b.out, want)


def test_fp8_stream_start_and_refresh_round():
    # a stream that starts with one clean chunk (the window grows round by round)
    cfg = SMALL[0]
    rows = np.arange(cfg.R * cfg.C)

    def on_round(ro, r):
        _check_codes(ro, r, [0, 1])
        gc.check_attention(ro, r, [0, 1], rows, f"start r{r}")

    gc.run_rollout(cfg, (0, 1, 2, 4), first_n0=1, on_round=on_round, fp8=True)
    # a cache-refresh round at full size (t = 0 member first)
    ref_cfg = CONFIGS["wan13b_refresh"]
    srows = gc.sample_rows(ref_cfg, extra=8)
    gc.run_rollout(ref_cfg, (0,), on_round=lambda ro, r: gc.check_attention(ro, r, [6], srows, "refresh"), fp8=True)


def test_fp8_720p_long_rollout_sampled():
    # the largest shape over 200 rounds: codes bit-exact and attention within the gates at the checked rounds
    cfg = CONFIGS["p720_rollout"]
    rows = gc.sample_rows(cfg, extra=4)

    def on_round(ro, r):
        _check_codes(ro, r, [29])
        gc.check_attention(ro, r, [29], rows, f"720p fp8 r{r}")

    gc.run_rollout(cfg, cfg.check_rounds, on_round=on_round, fp8=True)


def test_negative_controls_fail_the_gates():
    """Mistakes planted in the oracle (on the CPU) must fail the gates the GPU output passes."""
    from oracle import wf_oracle as orc
    cfg = SMALL[-1]  # the key-split round: 4 parts per unit, merged by the combine pass
    rows = np.arange(cfg.R * cfg.C)
    ro = gc.run_rollout(cfg, (0,), fp8=True)
    assert wf.decode_plan(ro.host_plan)["key_parts"] > 1
    arrays = gc.oracle_inputs(cfg, ro.n0_of(0), ro.first_n0, [0, 1], seed=ro.seed)
    ref = gc.oracle_call(cfg, ro.n0_of(0), arrays, rows, fp8=True)
    got = gc.to_np(ro.out[rows][:, [0, 1]])
    gc.assert_bf16_close(got, ref["O"], "positive")
    H, D, C = 2, cfg.D, cfg.C
    q = orc.fp8_dequantize(ref["q8"], ref["q_scales"], C)
    k = orc.fp8_dequantize(ref["k8"], ref["k_scales"], C)
    v = np.concatenate([ref["v_cache"], ref["v"]]).reshape(-1, H, D)
    mask = orc.visibility_mask(C, min(cfg.Wc, ro.n0_of(0)), cfg.R, q_chunks=rows // C)

    def attend(kk, vv, m):
        return np.stack([orc.attention(q[rows][:, h], kk[:, h], vv[:, h], m, 1 / np.sqrt(D))[0] for h in range(H)],
                        axis=1)

    # the key scales left out (codes read as values times one common scale)
    k_unscaled = ref["k8"] * ref["k_scales"].mean()
    with pytest.raises(AssertionError):
        gc.assert_bf16_close(got, attend(k_unscaled, v, mask), "key scales ignored")
    # one of the parts dropped: only the first three quarters of the keys
    n_keys = k.shape[0]
    keep = np.zeros(n_keys, bool)
    keep[: 3 * n_keys // 4] = True
    with pytest.raises(AssertionError):
        gc.assert_bf16_close(got, attend(k, v, mask & keep[None, :]), "a key part dropped")


def test_fp8_quantize_tiny_and_zero_blocks_bit_exact():
    """Blocks whose 448 / amax overflows fp32 (zeros plus bf16 subnormals) quantize like all-zero
    blocks (scale 1, zero codes, no NaN), next to a normal block and an all-zero one; codes and
    scales bit-exact against the oracle."""
    C, H, D, R = 256, 4, 128, 1
    desc = wf.make_desc(H, D, 1, C, 1, 0, R, 0, [1000], dtype=wf.WF_BF16, num_ctas=2)
    host = wf.host_plan_buffer(desc)
    dev = torch.empty(host.numel(), dtype=torch.uint8, device="cuda")
    wf.wf_plan_round(desc, host, dev)
    x = torch.zeros(R * C, H, D, dtype=torch.float64)
    x[5, 0, 7] = 2.0 ** -133                   # head 0, block 0: one subnormal
    x[200, 0, 3] = -(2.0 ** -126)              # head 0, block 1: amax 2^-126, still overflows
    x[17, 1, 9] = 2.0 ** -100                  # head 1, block 0: tiny but regular
    x[:, 2] = torch.linspace(-3, 3, R * C * D, dtype=torch.float64).reshape(R * C, D)  # head 2: normal
    src = x.to(torch.bfloat16).cuda()          # head 3 stays all-zero
    dst = torch.full((R * C, H, D), 0x7F, dtype=torch.uint8, device="cuda")
    scales = torch.full((R, 2, H), float("nan"), dtype=torch.float32, device="cuda")
    wf.wf_quantize_fp8(host, src, dst, scales, wf.WF_FP8_Q)
    torch.cuda.synchronize()
    codes, ref_scales = orc.fp8_block_quantize(src.float().cpu().numpy().astype(np.float64), C)
    got = _e4m3_values(dst)
    assert not np.isnan(got).any()
    assert np.array_equal(got, codes)
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), ref_scales)
    assert (ref_scales[0, :, 0] == 1.0).all() and not codes[:, 0].any()
