// Device arithmetic of the 3D rotary embedding shared by the RoPE/append
// kernel and the attention variant that rotates Q itself: the fp64 rotation
// of one interleaved pair, the (cos, sin) lookup in the plan's per-axis
// tables, and the once-only rounding of the fp64 result to the storage type.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace {

// (cos, sin) of pair m of a token at time row `trow` of the t table (i * F + f),
// row hh and column ww: pairs [0, Pt) turn with t, the next Ph with h, the last
// Pw with w; each table row holds its axis group's pairs.
__device__ __forceinline__ double2 rope_cos_sin(const double2* tab_t, const double2* tab_h, const double2* tab_w,
                                                int32_t Pt, int32_t Ph, int32_t Pw, uint32_t trow, uint32_t hh,
                                                uint32_t ww, int32_t m) {
  const double2* e;
  if (m < Pt)
    e = tab_t + int64_t(trow) * Pt + m;
  else if (m < Pt + Ph)
    e = tab_h + int64_t(hh) * Ph + (m - Pt);
  else
    e = tab_w + int64_t(ww) * Pw + (m - Pt - Ph);
  return __ldg(e);
}

// x rounded once, to nearest even, to bf16: the conversion instruction rounds
// from fp64 directly (cvt.rn.bf16.f64).
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double x) { return __bfloat16_as_ushort(__double2bfloat16(x)); }

__device__ __forceinline__ void rotate_pair(double x, double y, double2 cs, double& xr, double& yr) {
  // same operation order as a plain fp64 evaluation of x*c - y*s, x*s + y*c
  xr = __dsub_rn(__dmul_rn(x, cs.x), __dmul_rn(y, cs.y));
  yr = __dadd_rn(__dmul_rn(x, cs.y), __dmul_rn(y, cs.x));
}

template <typename T>
struct Pack;

template <>
struct Pack<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ static void unpack(const uint4& v, double* out) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p[i]);
      out[2 * i] = f.x;
      out[2 * i + 1] = f.y;
    }
  }
  __device__ static uint4 pack(const double* in) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = uint32_t(f64_to_bf16_bits(in[2 * i])) | (uint32_t(f64_to_bf16_bits(in[2 * i + 1])) << 16);
    return v;
  }
};

template <>
struct Pack<float> {
  static constexpr int kElems = 4;
  __device__ static void unpack(const uint4& v, double* out) {
    const float* p = reinterpret_cast<const float*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = p[i];
  }
  __device__ static uint4 pack(const double* in) {
    uint4 v;
    float* p = reinterpret_cast<float*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = __double2float_rn(in[i]);
    return v;
  }
};

// One interleaved bf16 pair (packed in a 32-bit word, lower address = even
// element) rotated by (cos, sin) in fp64 and rounded once to bf16.
__device__ __forceinline__ uint32_t rope_pair_bf16(uint32_t word, double2 cs) {
  const float2 xy = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&word));
  double xr, yr;
  rotate_pair(double(xy.x), double(xy.y), cs, xr, yr);
  return uint32_t(f64_to_bf16_bits(xr)) | (uint32_t(f64_to_bf16_bits(yr)) << 16);
}

}  // namespace
