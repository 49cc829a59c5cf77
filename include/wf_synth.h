/*
 * wf_synth.h -- device generator of the synthetic wave-round inputs.
 *
 * Not part of the method: a test and benchmark utility that draws, on the
 * device, the same values as the host generator module (SplitMix64 counter
 * stream with Stafford's Mix13 finaliser, Irwin-Hall(12) of 16-bit halves,
 * optional per-head key scale, bf16 nearest-even or raw fp32).  The host and
 * device draws are bit-identical, which lets full-size inputs be made where
 * they are used.  The pages print no inputs; the seed 42 default is the
 * plugin's base_seed ("scope-causal-forcing", "Configuration" table).
 */
#ifndef WF_SYNTH_H_
#define WF_SYNTH_H_

#include "wf.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Tensor ids of the generator streams. */
#define WF_SYNTH_Q 1
#define WF_SYNTH_K 2
#define WF_SYNTH_V 3

/*
 * Fill dst [nchunks*C, H, D] (dtype WF_BF16 or WF_F32, device memory,
 * 16-byte aligned) with the draws of global chunks n_first .. n_first+nchunks-1
 * of stream (seed, tensor, tag).  kscale != 0 multiplies each head's draws by
 * its fp32 key scale in [0.5, 2) before rounding.  Asynchronous on `stream`.
 * Errors: WF_ERR_INVALID_ARG, WF_ERR_ALIGNMENT, WF_ERR_CUDA.
 */
wf_status wf_synth_fill(void* dst, int32_t dtype, uint64_t seed, int32_t tensor, int64_t tag,
                        int64_t n_first, int32_t nchunks, int32_t C, int32_t H, int32_t D,
                        int32_t kscale, wf_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WF_SYNTH_H_ */
