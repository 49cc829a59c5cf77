// wf_chunk_causal_attn: argument checks and dispatch, the fp32 CUDA-core
// kernel, and the attention workspace helpers.
//
// The fp32 path serves the fp32 tiny round (head_dim 64) and fp32 checks at
// head_dim 128.  It keeps every product and sum in fp32 (no TF32), because a
// 1e-4 relative bound on O is beyond TF32 tensor-core products.  One block
// covers 128/TPR query rows of one (chunk, head); each row is split over
// TPR = D/32 threads holding 32 dims of q and of the accumulator, whose
// partial dot products are summed with warp shuffles.  K/V tiles of 32 keys
// are staged in shared memory and the online softmax is updated once per
// tile.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>

#include "wf.h"
#include "wf_plan.h"

namespace wf {
wf_status launch_attn_sm100(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q_rot, const void* k_pool,
                            const void* v_pool, void* out, float* lse, float scale, void* workspace,
                            uint64_t timeout_ns, cudaStream_t stream);
wf_status launch_attn_sm100_rope_q(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q_raw,
                                   const void* k_pool, const void* v_pool, void* out, float* lse, float scale,
                                   void* workspace, uint64_t timeout_ns, cudaStream_t stream);
wf_status launch_attn_sm100_fp8(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q8, const float* q_scales,
                                const void* k8_pool, const float* k_scales, const void* v_pool, void* out, float* lse,
                                float scale, void* workspace, uint64_t timeout_ns, cudaStream_t stream);
}

namespace {

constexpr int kF32Keys = 32;

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  float* out;
  float* lse;
  int32_t H, C, rc;
  float scale;
  int32_t seg_start[WF_MAX_INROUND][2];
  int32_t seg_len[WF_MAX_INROUND][2];
};

template <int D>
__global__ void __launch_bounds__(128) attn_f32_kernel(const F32Params p) {
  constexpr int TPR = D / 32;
  constexpr int ROWS = 128 / TPR;
  __shared__ float ks[kF32Keys][D];
  __shared__ float vs[kF32Keys][D];
  const int i = blockIdx.z, h = blockIdx.y;
  const int r = threadIdx.x / TPR, part = threadIdx.x % TPR;
  const int row = blockIdx.x * ROWS + r;
  const bool valid_row = row < p.C;
  const int64_t qtok = int64_t(i) * p.C + row;
  float q[32], o[32];
#pragma unroll
  for (int d = 0; d < 32; ++d) {
    q[d] = valid_row ? p.q[(qtok * p.H + h) * D + part * 32 + d] : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int seg = 0; seg < 2; ++seg) {
    const int32_t start = p.seg_start[i][seg], len = p.seg_len[i][seg];
    for (int t0 = 0; t0 < len; t0 += kF32Keys) {
      const int nk = min(kF32Keys, len - t0);
      for (int x = threadIdx.x; x < kF32Keys * D; x += blockDim.x) {
        const int kk = x / D, d = x % D;
        float kv = 0.f, vv = 0.f;
        if (kk < nk) {
          const int64_t off = (int64_t(start + t0 + kk) * p.H + h) * D + d;
          kv = p.k[off];
          vv = p.v[off];
        }
        ks[kk][d] = kv;
        vs[kk][d] = vv;
      }
      __syncthreads();
      float s[kF32Keys];
      float mt = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kF32Keys; ++kk) {
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < 32; ++d) acc = fmaf(q[d], ks[kk][part * 32 + d], acc);
#pragma unroll
        for (int off = 1; off < TPR; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        s[kk] = kk < nk ? acc * p.scale : -INFINITY;
        mt = fmaxf(mt, s[kk]);
      }
      const float m_new = fmaxf(m, mt);
      const float corr = expf(m - m_new);
      l *= corr;
#pragma unroll
      for (int d = 0; d < 32; ++d) o[d] *= corr;
#pragma unroll
      for (int kk = 0; kk < kF32Keys; ++kk) {
        const float pk = expf(s[kk] - m_new);
        l += pk;
#pragma unroll
        for (int d = 0; d < 32; ++d) o[d] = fmaf(pk, vs[kk][part * 32 + d], o[d]);
      }
      m = m_new;
      __syncthreads();
    }
  }
  if (!valid_row) return;
  const float inv = 1.f / l;
#pragma unroll
  for (int d = 0; d < 32; ++d) p.out[(qtok * p.H + h) * D + part * 32 + d] = o[d] * inv;
  if (p.lse && part == 0) p.lse[int64_t(h) * p.rc + qtok] = m + logf(l);
}

bool misaligned(const void* ptr) { return reinterpret_cast<uintptr_t>(ptr) % 16 != 0; }

// Units whose keys the plan split into parts leave normalised partial O and
// LSE rows in the workspace; this pass merges the parts of every (chunk,
// head, row pair): LSE = log sum_k exp(LSE_k), O = sum_k exp(LSE_k - LSE) O_k.
// One warp per row, four dims per lane; a block covers 8 rows of one pair.
struct CombineParams {
  const float* part_o;    // [units][256][128]
  const float* part_lse;  // [units][256]
  __nv_bfloat16* out;
  float* lse;
  int32_t H, C, q_pairs, parts, rc;
};

__global__ void __launch_bounds__(256) attn_combine_kernel(const CombineParams p) {
  const int g = blockIdx.x;  // (chunk, head, row pair); its parts are slots g*parts .. g*parts+parts-1
  const int pair = g % p.q_pairs, ih = g / p.q_pairs, h = ih % p.H, i = ih / p.H;
  const int rows = min(256, p.C - pair * 256);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * 8 + warp;
  if (r < rows) {
    const float lk = lane < p.parts ? p.part_lse[(int64_t(g) * p.parts + lane) * 256 + r] : -INFINITY;
    float mx = lk;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float w = lane < p.parts ? expf(lk - mx) : 0.f;
    float wsum = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < p.parts; ++k) {
      const float wk = __shfl_sync(0xffffffffu, w, k);
      const float4 o = reinterpret_cast<const float4*>(p.part_o + ((int64_t(g) * p.parts + k) * 256 + r) * 128)[lane];
      acc.x = fmaf(wk, o.x, acc.x);
      acc.y = fmaf(wk, o.y, acc.y);
      acc.z = fmaf(wk, o.z, acc.z);
      acc.w = fmaf(wk, o.w, acc.w);
    }
    const float inv = 1.0f / wsum;
    const int64_t tok = int64_t(i) * p.C + pair * 256 + r;
    uint2 packed;
    packed.x = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.x * inv))) |
               (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.y * inv))) << 16);
    packed.y = uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.z * inv))) |
               (uint32_t(__bfloat16_as_ushort(__float2bfloat16_rn(acc.w * inv))) << 16);
    reinterpret_cast<uint2*>(p.out + (tok * p.H + h) * 128)[lane] = packed;
    if (lane == 0 && p.lse) p.lse[int64_t(h) * p.rc + tok] = mx + logf(wsum);
  }
}

// Parts per unit of a plan (1: nothing to combine).
int32_t key_parts(const wf_plan_hdr* h, const void* host_plan) {
  if (h->num_units == 0) return 1;
  const wf_plan_unit* u =
      reinterpret_cast<const wf_plan_unit*>(static_cast<const uint8_t*>(host_plan) + h->off_units);
  return u[0].parts;
}

wf_status launch_combine(const wf_plan_hdr* h, const void* host_plan, void* workspace, void* out, float* lse,
                         cudaStream_t stream) {
  const int32_t parts = key_parts(h, host_plan);
  if (parts <= 1) return WF_OK;
  CombineParams c{};
  c.part_o = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) + WF_ATTN_STATUS_BYTES);
  c.part_lse = c.part_o + int64_t(h->num_units) * 256 * 128;
  c.out = static_cast<__nv_bfloat16*>(out);
  c.lse = lse;
  c.H = h->H;
  c.C = h->C;
  c.q_pairs = h->q_pairs;
  c.parts = parts;
  c.rc = h->R * h->C;
  const int64_t groups = int64_t(h->num_units) / parts;
  if (groups > 0x7FFFFFFF) return WF_ERR_CAPACITY;
  attn_combine_kernel<<<dim3(unsigned(groups), 32), 256, 0, stream>>>(c);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

// Limit of every bounded wait in the tensor-core kernel (WF_WAIT_TIMEOUT_MS,
// default 2000 ms), read at each launch.
uint64_t wait_timeout_ns() {
  const char* env = std::getenv("WF_WAIT_TIMEOUT_MS");
  long ms = env ? std::atol(env) : 2000;
  if (ms < 1) ms = 1;
  return uint64_t(ms) * 1000000ull;
}

}  // namespace

extern "C" size_t wf_attn_workspace_bytes(const void* host_plan) {
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (!h || h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return 0;
  if (key_parts(h, host_plan) <= 1) return WF_ATTN_STATUS_BYTES;
  return WF_ATTN_STATUS_BYTES + size_t(h->num_units) * 256 * (128 + 1) * sizeof(float);
}

extern "C" wf_status wf_attn_workspace_init(void* workspace, size_t workspace_bytes, wf_stream_t stream) {
  if (!workspace || workspace_bytes < WF_ATTN_STATUS_BYTES) return WF_ERR_WORKSPACE;
  if (misaligned(workspace)) return WF_ERR_ALIGNMENT;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? WF_OK
             : WF_ERR_CUDA;
}

extern "C" wf_status wf_attn_workspace_status(const void* workspace, wf_stream_t stream, int32_t* detail) {
  if (!workspace) return WF_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return WF_ERR_CUDA;
  wf_dev_status st;
  if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return WF_ERR_CUDA;
  if (detail) {
    detail[0] = st.code;
    detail[1] = st.where;
    detail[2] = st.block;
    detail[3] = st.thread;
  }
  return st.code == 0 ? WF_OK : static_cast<wf_status>(st.code);
}

extern "C" wf_status wf_chunk_causal_attn(const void* host_plan, const void* dev_plan, const void* q_rot,
                                          const void* k_pool, const void* v_pool, void* out, float* lse,
                                          float softmax_scale, void* workspace, size_t workspace_bytes,
                                          wf_stream_t stream) {
  if (!host_plan || !dev_plan || !q_rot || !k_pool || !v_pool || !out || !workspace) return WF_ERR_INVALID_ARG;
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return WF_ERR_PLAN;
  if (misaligned(dev_plan) || misaligned(q_rot) || misaligned(k_pool) || misaligned(v_pool) || misaligned(out) ||
      misaligned(workspace) || (reinterpret_cast<uintptr_t>(lse) % 4))
    return WF_ERR_ALIGNMENT;
  if (workspace_bytes < wf_attn_workspace_bytes(host_plan)) return WF_ERR_WORKSPACE;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return WF_ERR_INVALID_ARG;
  const float scale = softmax_scale == 0.f ? float(1.0 / std::sqrt(double(h->D))) : softmax_scale;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint8_t* dp = static_cast<const uint8_t*>(dev_plan);

  if (h->dtype == WF_BF16) {
    if (h->D != 128) return WF_ERR_UNSUPPORTED;
    const wf_status st =
        wf::launch_attn_sm100(h, dp, q_rot, k_pool, v_pool, out, lse, scale, workspace, wait_timeout_ns(), s);
    return st == WF_OK ? launch_combine(h, host_plan, workspace, out, lse, s) : st;
  }
  if (h->dtype != WF_F32 || (h->D != 64 && h->D != 128)) return WF_ERR_UNSUPPORTED;
  F32Params p{};
  p.q = static_cast<const float*>(q_rot);
  p.k = static_cast<const float*>(k_pool);
  p.v = static_cast<const float*>(v_pool);
  p.out = static_cast<float*>(out);
  p.lse = lse;
  p.H = h->H;
  p.C = h->C;
  p.rc = h->R * h->C;
  p.scale = scale;
  const wf_plan_chunk* ch =
      reinterpret_cast<const wf_plan_chunk*>(static_cast<const uint8_t*>(host_plan) + h->off_chunks);
  for (int i = 0; i < h->R; ++i)
    for (int sgi = 0; sgi < 2; ++sgi) {
      p.seg_start[i][sgi] = ch[i].seg_start[sgi];
      p.seg_len[i][sgi] = ch[i].seg_len[sgi];
    }
  const int rows = h->D == 64 ? 64 : 32;
  dim3 grid((h->C + rows - 1) / rows, h->H, h->R);
  if (grid.y > 65535 || grid.z > 65535) return WF_ERR_CAPACITY;
  if (h->D == 64)
    attn_f32_kernel<64><<<grid, 128, 0, s>>>(p);
  else
    attn_f32_kernel<128><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}

extern "C" wf_status wf_chunk_causal_attn_rope(const void* host_plan, const void* dev_plan, const void* q,
                                               const void* k_pool, const void* v_pool, void* out, float* lse,
                                               float softmax_scale, void* workspace, size_t workspace_bytes,
                                               wf_stream_t stream) {
  if (!host_plan || !dev_plan || !q || !k_pool || !v_pool || !out || !workspace) return WF_ERR_INVALID_ARG;
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return WF_ERR_PLAN;
  if (misaligned(dev_plan) || misaligned(q) || misaligned(k_pool) || misaligned(v_pool) || misaligned(out) ||
      misaligned(workspace) || (reinterpret_cast<uintptr_t>(lse) % 4))
    return WF_ERR_ALIGNMENT;
  if (workspace_bytes < wf_attn_workspace_bytes(host_plan)) return WF_ERR_WORKSPACE;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return WF_ERR_INVALID_ARG;
  if (h->dtype != WF_BF16 || h->D != 128) return WF_ERR_UNSUPPORTED;
  const float scale = softmax_scale == 0.f ? float(1.0 / std::sqrt(double(h->D))) : softmax_scale;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const wf_status st = wf::launch_attn_sm100_rope_q(h, static_cast<const uint8_t*>(dev_plan), q, k_pool, v_pool, out,
                                                    lse, scale, workspace, wait_timeout_ns(), s);
  return st == WF_OK ? launch_combine(h, host_plan, workspace, out, lse, s) : st;
}

extern "C" wf_status wf_chunk_causal_attn_fp8(const void* host_plan, const void* dev_plan, const void* q8,
                                              const float* q_scales, const void* k8_pool, const float* k_scales,
                                              const void* v_pool, void* out, float* lse, float softmax_scale,
                                              void* workspace, size_t workspace_bytes, wf_stream_t stream) {
  if (!host_plan || !dev_plan || !q8 || !q_scales || !k8_pool || !k_scales || !v_pool || !out || !workspace)
    return WF_ERR_INVALID_ARG;
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return WF_ERR_PLAN;
  if (misaligned(dev_plan) || misaligned(q8) || misaligned(k8_pool) || misaligned(v_pool) || misaligned(out) ||
      misaligned(workspace) || (reinterpret_cast<uintptr_t>(lse) % 4) ||
      (reinterpret_cast<uintptr_t>(q_scales) % 4) || (reinterpret_cast<uintptr_t>(k_scales) % 4))
    return WF_ERR_ALIGNMENT;
  if (workspace_bytes < wf_attn_workspace_bytes(host_plan)) return WF_ERR_WORKSPACE;
  if (!(softmax_scale >= 0.f) || !std::isfinite(softmax_scale)) return WF_ERR_INVALID_ARG;
  if (h->dtype != WF_BF16 || h->D != 128) return WF_ERR_UNSUPPORTED;
  const float scale = softmax_scale == 0.f ? float(1.0 / std::sqrt(double(h->D))) : softmax_scale;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const wf_status st = wf::launch_attn_sm100_fp8(h, static_cast<const uint8_t*>(dev_plan), q8, q_scales, k8_pool,
                                                 k_scales, v_pool, out, lse, scale, workspace, wait_timeout_ns(), s);
  return st == WF_OK ? launch_combine(h, host_plan, workspace, out, lse, s) : st;
}
