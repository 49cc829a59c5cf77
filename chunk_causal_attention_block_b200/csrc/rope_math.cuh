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

// x rounded toward zero to fp32 with the last bit set when that lost anything
// ("round to odd"); rounding that to bf16 to nearest-even then equals direct
// nearest-even rounding of x (Boldo and Melquiond, "Emulation of FMA and
// correctly rounded sums: proved algorithms using rounding to odd", IEEE TC
// 2008: rounding to odd in a format with at least two more bits makes the
// second rounding correct).
__device__ __forceinline__ float f64_to_f32_round_odd(double x) {
  float r = __double2float_rz(x);
  if (double(r) != x) r = __int_as_float(__float_as_int(r) | 1);
  return r;
}

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
    __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = __floats2bfloat162_rn(f64_to_f32_round_odd(in[2 * i]), f64_to_f32_round_odd(in[2 * i + 1]));
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
  const __nv_bfloat162 r = __floats2bfloat162_rn(f64_to_f32_round_odd(xr), f64_to_f32_round_odd(yr));
  return *reinterpret_cast<const uint32_t*>(&r);
}

}  // namespace
