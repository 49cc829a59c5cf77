// wf_quantize_fp8: e4m3 codes and per-block fp32 scales of the round's
// rotated Q (all in-round chunks) or of the in-round chunks' rotated K in
// the ring pool.
//
// One CTA per (block of WF_FP8_BLOCK chunk-relative tokens, head, in-round
// chunk).  Sixteen threads share a token's 256-byte bf16 row (one 16-byte
// vector each), so every warp load covers two whole rows; a CTA of 256
// threads takes sixteen rows per pass and keeps its eight passes in
// registers while the block's absolute maximum is reduced, then writes the
// codes (8 bytes per thread per row) and the block scale.  Four CTAs per SM
// (64 registers, a few bytes spilled) keep more loads in flight than the
// two that 87 registers allowed: 93 -> 69 us for Q and K of the 4-chunk
// round.
//   scale = amax / 448 and inv = 448 / amax (fp32, nearest; both 1 for an
//           all-zero block)
//   code  = e4m3(x * inv): one fp32 product, then the nearest-even
//           conversion that saturates at +-448.  (A product instead of a
//           division by scale: the correctly rounded division made the
//           kernel instruction-bound.)
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "wf.h"
#include "wf_plan.h"

namespace {

constexpr int kRowsPerPass = 16;
constexpr int kPasses = WF_FP8_BLOCK / kRowsPerPass;
static_assert(kPasses * kRowsPerPass == WF_FP8_BLOCK, "block rows");

struct QuantParams {
  const uint4* src;  // bf16 rows [tokens, H, 128]: 16 vectors of 8 values per row
  uint2* dst;        // e4m3 rows [tokens, H, 128]: 16 groups of 8 bytes per row
  float* scales;     // [chunks, nblk, H]
  int32_t H, C, nblk;
  // chunk index in src/dst/scales of in-round chunk i: i for Q, its ring slot
  // (first + i) mod S for K
  int32_t first, S;
};

__device__ __forceinline__ float abs_max8(const uint4& v, float m) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(p[k]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return m;
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d, float inv) {
  const uint32_t qa = __nv_cvt_float_to_fp8(__fmul_rn(a, inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t qb = __nv_cvt_float_to_fp8(__fmul_rn(b, inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t qc = __nv_cvt_float_to_fp8(__fmul_rn(c, inv), __NV_SATFINITE, __NV_E4M3);
  const uint32_t qd = __nv_cvt_float_to_fp8(__fmul_rn(d, inv), __NV_SATFINITE, __NV_E4M3);
  return qa | (qb << 8) | (qc << 16) | (qd << 24);  // lowest address = lowest dim
}

__global__ void __launch_bounds__(256, 4) fp8_quant_kernel(const QuantParams p) {
  __shared__ float warp_max[8];
  const int b = blockIdx.x, h = blockIdx.y;
  const int32_t chunk = (p.first + int32_t(blockIdx.z)) % p.S;
  const int part = threadIdx.x & 15, r0 = threadIdx.x >> 4;
  const int rows = min(WF_FP8_BLOCK, p.C - b * WF_FP8_BLOCK);
  const int64_t tok0 = int64_t(chunk) * p.C + int64_t(b) * WF_FP8_BLOCK;
  uint4 v[kPasses];
  float amax = 0.f;
#pragma unroll
  for (int s = 0; s < kPasses; ++s) {
    const int r = s * kRowsPerPass + r0;
    v[s] = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      v[s] = __ldcs(p.src + ((tok0 + r) * p.H + h) * 16 + part);
      amax = abs_max8(v[s], amax);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);
  // a block whose 448 / amax is not finite (amax 0 or below 448 / FLT_MAX) is
  // an all-zero block: scale 1, inv 1 (an infinite inv would give 0 * inf = NaN)
  const float inv_raw = __fdiv_rn(448.0f, amax);
  const bool regular = amax > 0.f && isfinite(inv_raw);
  const float scale = regular ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float inv = regular ? inv_raw : 1.0f;
#pragma unroll
  for (int s = 0; s < kPasses; ++s) {
    const int r = s * kRowsPerPass + r0;
    if (r < rows) {
      const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&v[s]);
      const float2 f0 = __bfloat1622float2(x[0]), f1 = __bfloat1622float2(x[1]);
      const float2 f2 = __bfloat1622float2(x[2]), f3 = __bfloat1622float2(x[3]);
      uint2 q;
      q.x = e4m3x4(f0.x, f0.y, f1.x, f1.y, inv);
      q.y = e4m3x4(f2.x, f2.y, f3.x, f3.y, inv);
      p.dst[((tok0 + r) * p.H + h) * 16 + part] = q;
    }
  }
  if (threadIdx.x == 0) p.scales[(int64_t(chunk) * p.nblk + b) * p.H + h] = scale;
}

bool misaligned(const void* ptr, uintptr_t a) { return reinterpret_cast<uintptr_t>(ptr) % a != 0; }

}  // namespace

extern "C" wf_status wf_quantize_fp8(const void* host_plan, const void* src, void* dst8, float* scales,
                                     int32_t which, wf_stream_t stream) {
  if (!host_plan || !src || !dst8 || !scales) return WF_ERR_INVALID_ARG;
  if (which != WF_FP8_Q && which != WF_FP8_K) return WF_ERR_INVALID_ARG;
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return WF_ERR_PLAN;
  if (h->dtype != WF_BF16 || h->D != 128) return WF_ERR_UNSUPPORTED;
  if (misaligned(src, 16) || misaligned(dst8, 16) || misaligned(scales, 4)) return WF_ERR_ALIGNMENT;
  QuantParams p{};
  p.src = static_cast<const uint4*>(src);
  p.dst = static_cast<uint2*>(dst8);
  p.scales = scales;
  p.H = h->H;
  p.C = h->C;
  p.nblk = (h->C + WF_FP8_BLOCK - 1) / WF_FP8_BLOCK;
  const wf_plan_chunk* ch =
      reinterpret_cast<const wf_plan_chunk*>(static_cast<const uint8_t*>(host_plan) + h->off_chunks);
  // in-round chunks sit in consecutive ring slots
  p.first = which == WF_FP8_Q ? 0 : ch[0].slot;
  p.S = which == WF_FP8_Q ? h->R : h->S;
  if (h->H > 65535 || h->R > 65535) return WF_ERR_CAPACITY;
  const dim3 grid(unsigned(p.nblk), unsigned(h->H), unsigned(h->R));
  fp8_quant_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}
