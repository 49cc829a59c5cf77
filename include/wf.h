/*
 * wf.h -- C ABI of libwf, the chunk-causal attention hot path of one Wave
 * Forcing "wave round" on NVIDIA B200 (sm_100a).
 *
 * A wave round holds R latent chunks at staggered noise levels in one forward
 * pass.  Each chunk's queries attend to a rolling cache of clean chunks, to the
 * earlier (older, cleaner, still partly noisy) chunks of the same round, and to
 * all of their own tokens.  Sources: "Wave Forcing: Towards Speed-of-Light
 * Streaming Video Generation" (arXiv 2611.00859v1), Abstract -- chunk-wise
 * causal attention that reads earlier, cleaner chunks before their denoising
 * is complete, staggered denoising, one output chunk per round; "Wave Forcing
 * from SJTU-DENG Lab: 8 GPUs can't fix a missing sgl-dlab package", first
 * paragraph -- a new chunk conditions on a mixed-noise frontier;
 * "scope-causal-forcing", "How It Works" -- KV-cached chunk generation whose
 * finished chunk's K/V enter the cache.
 *
 * Conventions for every call
 * --------------------------
 * - Notation: H heads, D head_dim, a latent frame of fh x fw tokens, F frames
 *   per chunk, C = F*fh*fw tokens per chunk, Wc cache chunks, R in-round
 *   chunks, S pool slots.  In-round chunk i (0 = oldest = cleanest) is global
 *   chunk n0 + i.  Tokens of a chunk are ordered (frame, row, column).
 * - Tensors are dense, row-major:  new Q/K/V and Q' and O are [R*C, H, D]
 *   (token, head, dim); the K and V pools are [S*C, H, D] where pool token
 *   s*C + j is token j of the chunk held in slot s = n mod S.  Element type is
 *   the plan's dtype (bf16 or fp32) for all of them.
 * - The caller owns every buffer.  The library never allocates or frees
 *   memory and keeps no state between calls except a per-device cache of
 *   kernel attributes (and the static scratch that
 *   wf_chunk_causal_attn_noalloc documents).
 * - Device pointers must be 16-byte aligned; otherwise WF_ERR_ALIGNMENT.
 * - Every call is asynchronous on `stream` (NULL = legacy default stream) and
 *   never synchronises.  Argument errors are detected on the host before any
 *   launch and return a status; launch errors return WF_ERR_CUDA.  Errors that
 *   a running kernel detects (a wait that timed out) are recorded in the
 *   attention workspace and read with wf_attn_workspace_status.
 * - Supported: bf16 with D = 128 (tensor-core path) and fp32 with D = 64 or
 *   128 (fp32 CUDA-core path).  Anything else returns WF_ERR_UNSUPPORTED.
 *   There is no fallback path.
 */
#ifndef WF_H_
#define WF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* wf_stream_t;

typedef enum wf_status {
  WF_OK = 0,
  WF_ERR_INVALID_ARG = 1,    /* bad shape, count, order or NULL pointer */
  WF_ERR_UNSUPPORTED = 2,    /* valid but not built (dtype/head_dim combination) */
  WF_ERR_ALIGNMENT = 3,      /* a device pointer is not 16-byte aligned */
  WF_ERR_CAPACITY = 4,       /* sizes overflow the index types or limits */
  WF_ERR_WORKSPACE = 5,      /* buffer smaller than the size query says */
  WF_ERR_CUDA = 6,           /* a CUDA runtime call or launch failed */
  WF_ERR_DEVICE_TIMEOUT = 7, /* a kernel gave up a bounded wait (see workspace) */
  WF_ERR_PLAN = 8            /* plan blob has the wrong magic/version/size */
} wf_status;

typedef enum wf_dtype { WF_F32 = 0, WF_BF16 = 1 } wf_dtype;

#define WF_MAX_INROUND 16

/* Description of one wave round.  Plain data; copied by wf_plan_round. */
typedef struct wf_round_desc {
  int32_t num_heads;        /* H >= 1 */
  int32_t head_dim;         /* D: 128 for bf16, 64 or 128 for fp32 */
  int32_t frame_h;          /* fh >= 1: token rows of a latent frame */
  int32_t frame_w;          /* fw >= 1: token columns of a latent frame */
  int32_t frames_per_chunk; /* F >= 1 */
  int32_t cache_chunks;     /* Wc >= 0: clean chunks the round sees */
  int32_t inround_chunks;   /* R in [1, WF_MAX_INROUND] */
  int32_t pool_slots;       /* S >= Wc + R; 0 means Wc + R.  Keep it fixed for a stream */
  int64_t n0;               /* global index of the oldest in-round chunk, >= 0 */
  int32_t noise_t[WF_MAX_INROUND]; /* noise level of in-round chunk i, oldest first;
                                      must be non-decreasing and in [0, 1000];
                                      metadata only, it never enters the arithmetic */
  int32_t rope_pairs_t;     /* rotation pairs on the time axis */
  int32_t rope_pairs_h;     /* ... on the row axis */
  int32_t rope_pairs_w;     /* ... on the column axis; the three sum to D/2, or
                               all three 0 for the default split
                               P_h = P_w = floor(D/6), P_t = D/2 - 2*P_h */
  double rope_theta;        /* RoPE base, > 0 (10000 for the Wan shapes) */
  int32_t dtype;            /* wf_dtype of every tensor */
  int32_t num_ctas;         /* attention work-list bins; 0 = SM count of the
                               current device (needs a CUDA device) */
} wf_round_desc;

/*
 * Size in bytes of the plan blob of `desc` (host and device copies have the
 * same size).  Returns 0 if `desc` is invalid.
 */
size_t wf_plan_bytes(const wf_round_desc* desc);

/*
 * wf_plan_round -- per-round visibility, ring-slot and work metadata.
 *
 * Defines which keys each in-round chunk sees (the chunk-wise causal
 * visibility of the arXiv abstract above): chunk i (global n_i = n0 + i) sees
 * cache chunks max(0, n0-Wc) .. n0-1 and in-round chunks n0 .. n_i, all
 * tokens of each.  Chunk n lives in pool slot n mod S; the visible chunks are
 * consecutive, so their pool tokens form at most two contiguous runs, which
 * the plan lists with their 128-key tile counts.  It also holds the fp64
 * cos/sin tables of the round's RoPE angles and the attention work list:
 * units of (chunk, head, 256 query rows) in longest-first order, assigned
 * greedily to `num_ctas` bins and then rebalanced by moves and swaps.  When a
 * bf16 round has fewer than two units per bin (a single chunk), every unit's
 * key tiles are shared out over up to 8 parts (the count that fills the bins
 * best, each part at least 8 tiles); the attention then merges the parts.
 *
 * host_plan: host buffer of >= wf_plan_bytes(desc) bytes, filled on return.
 * dev_plan:  device buffer of the same size, or NULL.  If non-NULL the blob
 *            is copied with cudaMemcpyAsync on `stream`; when host_plan is
 *            pinned the caller must keep it unchanged until that copy is done.
 * Errors: WF_ERR_INVALID_ARG (shape, order of noise levels, S < Wc + R),
 *         WF_ERR_CAPACITY (S*C*H*D or the blob too large), WF_ERR_WORKSPACE
 *         (a buffer too small), WF_ERR_CUDA (copy failed).  Nothing is
 *         written to dev_plan on error.
 */
wf_status wf_plan_round(const wf_round_desc* desc, void* host_plan, size_t host_bytes,
                        void* dev_plan, size_t dev_bytes, wf_stream_t stream);

/*
 * wf_balance_units -- the work balancer wf_plan_round applies to the
 * attention units (its work list is part of the plan), on a given list of
 * item costs.  The pages describe no scheduler: this is the library's own
 * rule, exported so that callers (and tests) can check the assignment.
 *
 * 1. Longest first: items ordered by cost, largest first (equal costs keep
 *    their given order), each go to the bin with the smallest load (lowest
 *    bin index on equal loads).
 * 2. Refinement, at most 5000 times: h = the heaviest bin (lowest index on
 *    equal loads).  Scan the other bins from the lightest (lowest index on
 *    equal loads), stopping at the first that is not lighter than h.  In bin
 *    b, for each item x of h in list order: moving x gives the larger load
 *    max(L_h - c_x, L_b + c_x); then for each item y of b in list order with
 *    c_y < c_x, swapping gives max(L_h - d, L_b + d), d = c_x - c_y.  A change
 *    counts if that value is below L_h; the best is the smallest value, ties
 *    to the first found.  The first bin b that offers any change is taken:
 *    x moves to the end of b's list (and y, for a swap, to the end of h's).
 *    Stop when no bin offers a change.
 *
 * cost:      n item costs, each in [0, 2^40] (host memory).
 * n:         item count in [0, 2^26].
 * bins:      bin count in [1, 65536].
 * bin_start: host int32 [bins + 1] (written): bin b holds items
 *            items[bin_start[b] .. bin_start[b+1]).
 * items:     host int32 [n] (written): item indices (into cost), per bin in
 *            list order.
 * Errors: WF_ERR_INVALID_ARG (counts, a negative cost, NULL).  Host only.
 */
wf_status wf_balance_units(const int64_t* cost, int32_t n, int32_t bins, int32_t* bin_start, int32_t* items);

/*
 * wf_rope3d_append -- 3D rotary embedding of the new Q and K and append of
 * K'/V into the ring pool (the cache write of "scope-causal-forcing", "How It
 * Works", step 2, done for every in-round chunk of the round).
 *
 * For token j of in-round chunk i at position (t, h, w) with t = n_i*F + f,
 * each interleaved pair (x[2m], x[2m+1]) of Q and K is rotated by the angle
 * pos_axis(m) * theta^(-k/P_axis) of its axis group (pairs [0, P_t) on t, the
 * next P_h on h, the last P_w on w; k is the index inside the group).  The
 * rotation is done in fp64 and rounded once (nearest, ties to even) to the
 * storage type.  V is copied unchanged.
 *
 * q, k, v:   device [R*C, H, D] new tensors (read only).
 * q_rot:     device [R*C, H, D] rotated queries (written).
 * k_pool, v_pool: device [S*C, H, D]; the slots of the round's in-round
 *            chunks are overwritten, all other slots are left untouched.
 * host_plan/dev_plan: the plan of this round (dev_plan already holding it on
 *            `stream`).
 * Errors: WF_ERR_PLAN, WF_ERR_INVALID_ARG (NULL), WF_ERR_ALIGNMENT, WF_ERR_CUDA.
 */
wf_status wf_rope3d_append(const void* host_plan, const void* dev_plan,
                           const void* q, const void* k, const void* v,
                           void* q_rot, void* k_pool, void* v_pool, wf_stream_t stream);

/*
 * wf_rope3d_append_kv -- wf_rope3d_append without the queries: rotates the
 * new K and appends K'/V into the pool exactly as wf_rope3d_append does, and
 * neither reads Q nor writes Q'.  Pair it with wf_chunk_causal_attn_rope,
 * which rotates Q itself.  Arguments and errors as wf_rope3d_append.
 */
wf_status wf_rope3d_append_kv(const void* host_plan, const void* dev_plan, const void* k, const void* v,
                              void* k_pool, void* v_pool, wf_stream_t stream);

/* Bytes of attention workspace the plan's kernels need: the 256-byte status
 * block, plus 256 rows x (128 + 1) fp32 per unit when the plan splits units'
 * keys (see wf_plan_round); 0 for an invalid plan. */
size_t wf_attn_workspace_bytes(const void* host_plan);

/*
 * Zero a workspace on `stream` (once, before its first use, and after a
 * reported device error).  The attention kernels only ever set its status
 * word; they never clear it.
 */
wf_status wf_attn_workspace_init(void* workspace, size_t workspace_bytes, wf_stream_t stream);

/*
 * Read the status word of a workspace: synchronises `stream`, then returns
 * WF_OK or the error a kernel recorded (WF_ERR_DEVICE_TIMEOUT).  When
 * `detail` is non-NULL it receives 4 int32 (code, where, block, thread).
 */
wf_status wf_attn_workspace_status(const void* workspace, wf_stream_t stream, int32_t* detail);

/*
 * wf_chunk_causal_attn -- block-causal attention forward of one wave round
 * (the chunk-wise causal attention of the arXiv abstract above).
 *
 * For every head h and in-round chunk i:
 *   O_i = softmax(Q'_i K'_V(i)^T * scale) V_V(i),
 * V(i) = the visible chunks of the plan (cache chunks and in-round chunks
 * 0..i, full attention inside a chunk).  Keys of chunks not visible to i are
 * never read.  bf16: products on tensor cores with fp32 accumulation, P
 * rounded to bf16 before the PV product, O rounded once to bf16.  fp32: all
 * arithmetic in fp32 on CUDA cores.
 *
 * q_rot:  device [R*C, H, D] (the output of wf_rope3d_append).
 * k_pool, v_pool: device [S*C, H, D] ring pool holding every visible chunk.
 *         Every slot must hold finite values (zero a new pool once): the last
 *         128-key tile of a visible run may extend into the next slot, whose
 *         keys are masked out of the softmax (weight exactly 0) but still
 *         enter the P*V product, where 0 * inf or 0 * NaN would be NaN.
 * out:    device [R*C, H, D] (written).
 * lse:    device fp32 [H, R*C] (natural-log sum of exp of scaled scores), or NULL.
 * softmax_scale: 0 means 1/sqrt(D).
 * workspace: device buffer of >= wf_attn_workspace_bytes(host_plan) bytes,
 *            zeroed once by wf_attn_workspace_init.  Calls that overlap on
 *            the GPU may share one workspace unless the plan splits units'
 *            keys: their partial rows live there until the combine pass (a
 *            second kernel on `stream`) has merged them.
 * Errors: WF_ERR_PLAN, WF_ERR_INVALID_ARG, WF_ERR_ALIGNMENT,
 *         WF_ERR_UNSUPPORTED, WF_ERR_WORKSPACE, WF_ERR_CUDA.
 */
wf_status wf_chunk_causal_attn(const void* host_plan, const void* dev_plan,
                               const void* q_rot, const void* k_pool, const void* v_pool,
                               void* out, float* lse, float softmax_scale,
                               void* workspace, size_t workspace_bytes, wf_stream_t stream);

/*
 * wf_chunk_causal_attn_rope -- wf_chunk_causal_attn from the round's raw
 * (not yet rotated) queries: the attention kernel applies Q's 3D RoPE itself,
 * on each unit's query tiles in shared memory, with the same fp64 rotation and
 * single rounding to bf16 as wf_rope3d_append, so O and LSE are bit-identical
 * to wf_rope3d_append followed by wf_chunk_causal_attn.  This saves writing
 * and re-reading Q' (a third of the RoPE/append traffic) and the Q' buffer.
 *
 * q:      device [R*C, H, D] raw queries (read only).
 * The pool must already hold this round's K'/V (wf_rope3d_append_kv).  All
 * other arguments and the errors are those of wf_chunk_causal_attn; bf16
 * plans with D = 128 only (else WF_ERR_UNSUPPORTED).
 */
wf_status wf_chunk_causal_attn_rope(const void* host_plan, const void* dev_plan, const void* q,
                                    const void* k_pool, const void* v_pool, void* out, float* lse,
                                    float softmax_scale, void* workspace, size_t workspace_bytes,
                                    wf_stream_t stream);

/*
 * wf_chunk_causal_attn_noalloc -- wf_chunk_causal_attn for callers that cannot
 * allocate device memory.  The pages have no counterpart: this is an
 * integration aid of this library, not part of the method.
 *
 * Some callers cannot call cudaMalloc: a serving engine or plugin host that
 * reserves all of a GPU's memory for its own pool when it starts and forbids
 * side allocations, or code that runs where allocating is not allowed.  This
 * call takes the same inputs and outputs as wf_chunk_causal_attn but no
 * workspace: the attention's scratch (its 256-byte status block) lives in a
 * 4096-byte array in device memory that the library reserves on every GPU it
 * is loaded on and keeps until the process exits.
 *
 * - The first call on a device looks up that array's device address (with the
 *   device current) and caches it; make that first call before any stream
 *   capture.  The call itself allocates nothing.
 * - Each call zeroes the status block on `stream` before launching.  A wait
 *   that times out is recorded there but is not returned by this call (it
 *   returns once the kernel is queued); wf_attn_noalloc_status reads it.
 * - Every call shares the one array: calls that overlap on the GPU (different
 *   streams, not ordered) race on it.
 * Errors: as wf_chunk_causal_attn, plus WF_ERR_CAPACITY if the plan's
 * workspace need exceeds the 4096-byte array and WF_ERR_CUDA if the address
 * look-up or the zeroing fails.
 */
wf_status wf_chunk_causal_attn_noalloc(const void* host_plan, const void* dev_plan,
                                       const void* q_rot, const void* k_pool, const void* v_pool,
                                       void* out, float* lse, float softmax_scale, wf_stream_t stream);

/*
 * wf_attn_noalloc_status -- the device status of the last
 * wf_chunk_causal_attn_noalloc call on the current device, read from the
 * library's static status block as wf_attn_workspace_status reads a
 * workspace: synchronises `stream` (the stream of that call), then returns
 * WF_OK or the error a kernel recorded (WF_ERR_DEVICE_TIMEOUT); `detail`, when
 * non-NULL, receives 4 int32 (code, where, block, thread).  Before any
 * no-alloc call on the device the block is all zero (WF_OK).
 * Errors: WF_ERR_CUDA if the synchronisation, the address look-up or the copy
 * fails.
 */
wf_status wf_attn_noalloc_status(wf_stream_t stream, int32_t* detail);

/*
 * 8-bit scores.  The Wave Forcing abstract (arXiv 2611.00859v1) measures its
 * system with 8-bit attention backends; these two calls are this library's
 * B200 counterpart: Q' and K' as OCP FP8 E4M3 codes with one fp32 scale per
 * block, scores on the tensor cores' e4m3 path (kind::f8f6f4), P and V in
 * bf16 as in wf_chunk_causal_attn.
 *
 * Blocks are WF_FP8_BLOCK consecutive tokens of one chunk (chunk-relative,
 * the last one ragged: nblk = ceil(C / WF_FP8_BLOCK) per chunk) times one
 * head.  scale = amax / 448 and inv = 448 / amax in fp32 (both 1 for a
 * block whose 448 / amax is not finite: amax 0, or below 448 / FLT_MAX, about
 * 1.3e-36, whose codes are then all zero); each element becomes the e4m3
 * value nearest x * inv (one
 * fp32 product, then the nearest-even conversion that saturates at +-448),
 * and is read back as code * scale.
 */
#define WF_FP8_BLOCK 128
typedef enum wf_fp8_which { WF_FP8_Q = 0, WF_FP8_K = 1 } wf_fp8_which;

/*
 * wf_quantize_fp8 -- e4m3 codes and block scales of the round's rotated
 * queries (WF_FP8_Q) or of the in-round chunks' rotated keys in the pool
 * (WF_FP8_K).  Run it after wf_rope3d_append of the same round; the cache
 * chunks keep the codes written in their last in-round round.
 *
 * WF_FP8_Q: src = q_rot [R*C, H, D] bf16; dst8 = [R*C, H, D] bytes;
 *           scales = [R, nblk, H] fp32.
 * WF_FP8_K: src = k_pool [S*C, H, D] bf16; dst8 = [S*C, H, D] bytes (only the
 *           in-round slots are written); scales = [S, nblk, H] fp32 (only the
 *           in-round slots' rows).
 * Requires a bf16 plan with D = 128; pointers 16-byte aligned (scales 4).
 * Errors: WF_ERR_INVALID_ARG, WF_ERR_PLAN, WF_ERR_ALIGNMENT,
 *         WF_ERR_UNSUPPORTED, WF_ERR_CUDA.
 */
wf_status wf_quantize_fp8(const void* host_plan, const void* src, void* dst8, float* scales, int32_t which,
                          wf_stream_t stream);

/*
 * wf_chunk_causal_attn_fp8 -- wf_chunk_causal_attn with the scores computed
 * from the e4m3 codes: S = (q8 k8^T) * q_scale * k_scale per (query block,
 * key block), then the same online softmax, bf16 P and PV with bf16 V.  The
 * key tiles are the chunks' scale blocks (each visible chunk is walked on
 * its own, nblk tiles, the last one ragged).
 *
 * q8, q_scales: from wf_quantize_fp8(WF_FP8_Q); k8_pool, k_scales: from
 * wf_quantize_fp8(WF_FP8_K) over the stream so far; v_pool, out, lse,
 * softmax_scale, workspace as in wf_chunk_causal_attn.
 * Errors: as wf_chunk_causal_attn (bf16 plans with D = 128 only).
 */
wf_status wf_chunk_causal_attn_fp8(const void* host_plan, const void* dev_plan, const void* q8,
                                   const float* q_scales, const void* k8_pool, const float* k_scales,
                                   const void* v_pool, void* out, float* lse, float softmax_scale,
                                   void* workspace, size_t workspace_bytes, wf_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char* wf_status_string(wf_status status);

/* Library ABI version (major * 100 + minor). */
int32_t wf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WF_H_ */
