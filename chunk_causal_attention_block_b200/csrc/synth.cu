// Device side of the synthetic input generator (test/benchmark utility).
// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) with Stafford's Mix13
// finaliser; element e of a stream consumes outputs 3e..3e+2, whose twelve
// 16-bit halves form an Irwin-Hall(12) draw that is exact in fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "wf_synth.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kTensorMul = 0xD1B54A32D192ED03ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, int32_t tensor, int64_t tag) {
  const uint64_t k0 = mix64(seed * kGolden);
  const uint64_t k1 = mix64(k0 ^ (uint64_t(int64_t(tensor)) * kTensorMul));
  return mix64(k1 ^ (uint64_t(tag) * kGolden));
}

__device__ __forceinline__ float irwin_hall12(uint64_t key, uint64_t e) {
  int32_t acc = 0;
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const uint64_t w = mix64(key + (3 * e + m + 1) * kGolden);
    acc += int32_t(w & 0xFFFF) + int32_t((w >> 16) & 0xFFFF) + int32_t((w >> 32) & 0xFFFF) +
           int32_t((w >> 48) & 0xFFFF);
  }
  return __int2float_rn(acc + 6 - 6 * 65536) * (1.0f / 65536.0f);
}

template <bool kBf16>
__global__ void synth_kernel(void* dst, uint64_t key, uint64_t kscale_key, int kscale, uint64_t e_base,
                             int64_t count, int32_t H, int32_t D) {
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= count) return;
  float z = irwin_hall12(key, e_base + uint64_t(idx));
  if (kscale) {
    const int32_t h = int32_t((idx / D) % H);
    const uint64_t x = mix64(kscale_key + (uint64_t(h) + 1) * kGolden) & 0xFFFF;
    const float s = __int2float_rn(int32_t(65536 + 3 * x)) * (1.0f / 131072.0f);
    z = __fmul_rn(z, s);
  }
  if (kBf16)
    static_cast<__nv_bfloat16*>(dst)[idx] = __float2bfloat16_rn(z);
  else
    static_cast<float*>(dst)[idx] = z;
}

}  // namespace

extern "C" wf_status wf_synth_fill(void* dst, int32_t dtype, uint64_t seed, int32_t tensor, int64_t tag,
                                   int64_t n_first, int32_t nchunks, int32_t C, int32_t H, int32_t D,
                                   int32_t kscale, wf_stream_t stream) {
  if (!dst || nchunks < 0 || C < 1 || H < 1 || D < 1 || n_first < 0) return WF_ERR_INVALID_ARG;
  if (dtype != WF_BF16 && dtype != WF_F32) return WF_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dst) % 16) return WF_ERR_ALIGNMENT;
  const int64_t count = int64_t(nchunks) * C * H * D;
  if (count == 0) return WF_OK;
  const uint64_t e_base = uint64_t(n_first) * uint64_t(C) * uint64_t(H) * uint64_t(D);
  const uint64_t key = stream_key(seed, tensor, tag);
  const uint64_t kkey = stream_key(seed, 4, 0);
  const int threads = 256;
  const int64_t blocks = (count + threads - 1) / threads;
  if (blocks > 0x7FFFFFFF) return WF_ERR_CAPACITY;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WF_BF16)
    synth_kernel<true><<<unsigned(blocks), threads, 0, s>>>(dst, key, kkey, kscale, e_base, count, H, D);
  else
    synth_kernel<false><<<unsigned(blocks), threads, 0, s>>>(dst, key, kkey, kscale, e_base, count, H, D);
  return cudaGetLastError() == cudaSuccess ? WF_OK : WF_ERR_CUDA;
}
