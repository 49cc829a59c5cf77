// wf_rope3d_append: 3D rotary embedding of the round's new Q and K, fused
// with the append of K'/V into the ring pool (and wf_rope3d_append_kv, the
// same without the queries).
//
// HBM-bound in bytes, but the bit-exact fp64 rotation makes it instruction-
// and conversion-heavy: per (token, head) row it reads Q, K, V and writes Q',
// K', V (6 * D * elem bytes).  Each thread moves one 16-byte vector of each
// tensor; a warp covers consecutive vectors, so every load and store is a
// fully coalesced 512-byte run.  Index decoding uses exact multiply-shift
// reciprocals instead of integer division.  The rotation runs in fp64 from
// the plan's fp64 cos/sin tables (L1-resident, a few KB) and is rounded once
// to the storage type (rope_math.cuh): for bf16 by the direct fp64 -> bf16
// conversion, one conversion per element instead of the two of an fp64 ->
// fp32 round-to-odd step and its exactness test (57.9 against 62.0 us for
// the 4-chunk round's launch under ncu; the conversion pipe was the limit).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "wf.h"
#include "rope_math.cuh"
#include "wf_plan.h"

namespace {

// n / d for 0 <= n < 2^31 by a multiply and a shift: with k = 32 + ceil(log2 d)
// and m = ceil(2^k / d), n*m / 2^k exceeds n/d by less than 1/(2d), which
// cannot carry past the next integer, so the quotient is exact.
struct FastDiv {
  uint64_t m;
  uint32_t k, d;
};

FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((uint64_t(1) << l) < d) ++l;
  FastDiv f;
  f.k = 32 + l;
  f.m = uint64_t((((unsigned __int128)1 << f.k) + d - 1) / d);
  f.d = d;
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return uint32_t((uint64_t(n) * f.m) >> f.k);  // n < 2^31, m < 2^33: no overflow
}

struct RopeParams {
  int32_t H, D, fh, fw, F, C, R, Pt, Ph, Pw;
  FastDiv div_vpr, div_H, div_C, div_fhw, div_fw;
  int32_t slot[WF_MAX_INROUND];
  const double2* tab_t;  // [R*F][Pt]
  const double2* tab_h;  // [fh][Ph]
  const double2* tab_w;  // [fw][Pw]
  int64_t nvec;          // vectors in the new tensors
};

// Rotate and store one 16-byte vector of Q (kWithQ) and K, and copy V, given
// its flat index e in the [R*C, H, D] tensors.
template <typename T, bool kWithQ>
__device__ __forceinline__ void rope_vector(const RopeParams& p, uint32_t e, const uint4& qv, const uint4& kv,
                                            const uint4& vv, uint4* __restrict__ q_rot, uint4* __restrict__ k_pool,
                                            uint4* __restrict__ v_pool) {
  constexpr int E = Pack<T>::kElems;
  const uint32_t row = fdiv(e, p.div_vpr);                   // token * H + head
  const uint32_t vin = e - row * p.div_vpr.d;
  const uint32_t token = fdiv(row, p.div_H);
  const uint32_t head = row - token * uint32_t(p.H);
  const uint32_t i = fdiv(token, p.div_C);                   // in-round chunk
  const uint32_t j = token - i * uint32_t(p.C);              // token inside the chunk
  const uint32_t f = fdiv(j, p.div_fhw);
  const uint32_t l = j - f * p.div_fhw.d;
  const uint32_t hh = fdiv(l, p.div_fw);
  const uint32_t ww = l - hh * uint32_t(p.fw);
  double qd[E], kd[E];
  if (kWithQ) Pack<T>::unpack(qv, qd);
  Pack<T>::unpack(kv, kd);
#pragma unroll
  for (int u = 0; u < E / 2; ++u) {
    const int32_t m = int32_t(vin) * (E / 2) + u;  // pair index in [0, D/2)
    const double2 cs = rope_cos_sin(p.tab_t, p.tab_h, p.tab_w, p.Pt, p.Ph, p.Pw, i * p.F + f, hh, ww, m);
    if (kWithQ) rotate_pair(qd[2 * u], qd[2 * u + 1], cs, qd[2 * u], qd[2 * u + 1]);
    rotate_pair(kd[2 * u], kd[2 * u + 1], cs, kd[2 * u], kd[2 * u + 1]);
  }
  const int64_t dst = ((int64_t(p.slot[i]) * p.C + j) * p.H + head) * p.div_vpr.d + vin;
  if (kWithQ) __stcs(q_rot + e, Pack<T>::pack(qd));
  __stcs(k_pool + dst, Pack<T>::pack(kd));
  __stcs(v_pool + dst, vv);
}

constexpr int kRopeThreads = 256;

// One 16-byte vector of each tensor per thread, a block per 256 vectors
// (62 registers: four blocks per SM).  Measured slower on the 4-chunk round,
// against 72 us for the kernel of the time: a grid-stride loop that keeps 3-5
// further steps' loads in flight through cp.async into shared memory (85-98
// us), half vectors per thread at 6 or 8 blocks per SM (82 us, issue-bound at
// 75% issue activity), and converting bf16 -> fp64 or testing a round-to-odd
// step's exactness with integer operations instead of conversions (83-91 us).
template <typename T, bool kWithQ>
__global__ void __launch_bounds__(kRopeThreads)
    rope3d_append_kernel(RopeParams p, const uint4* __restrict__ q, const uint4* __restrict__ k,
                         const uint4* __restrict__ v, uint4* __restrict__ q_rot, uint4* __restrict__ k_pool,
                         uint4* __restrict__ v_pool) {
  const int64_t e = int64_t(blockIdx.x) * kRopeThreads + threadIdx.x;
  if (e >= p.nvec) return;
  const uint4 qv = kWithQ ? __ldcs(q + e) : make_uint4(0, 0, 0, 0);
  const uint4 kv = __ldcs(k + e), vv = __ldcs(v + e);
  rope_vector<T, kWithQ>(p, uint32_t(e), qv, kv, vv, q_rot, k_pool, v_pool);
}

bool misaligned(const void* ptr) { return reinterpret_cast<uintptr_t>(ptr) % 16 != 0; }


// Shared by the two entry points; q / q_rot are null for the K/V-only append.
wf_status rope_append(const void* host_plan, const void* dev_plan, const void* q, const void* k, const void* v,
                      void* q_rot, void* k_pool, void* v_pool, wf_stream_t stream) {
  const bool with_q = q != nullptr;
  const wf_plan_hdr* h = static_cast<const wf_plan_hdr*>(host_plan);
  if (h->magic != WF_PLAN_MAGIC || h->version != WF_PLAN_VERSION) return WF_ERR_PLAN;
  if (misaligned(dev_plan) || (with_q && (misaligned(q) || misaligned(q_rot))) || misaligned(k) || misaligned(v) ||
      misaligned(k_pool) || misaligned(v_pool))
    return WF_ERR_ALIGNMENT;
  const int elem = h->dtype == WF_BF16 ? 2 : 4;
  if ((h->D * elem) % 16 != 0) return WF_ERR_UNSUPPORTED;

  RopeParams p{};
  p.H = h->H; p.D = h->D; p.fh = h->fh; p.fw = h->fw; p.F = h->F; p.C = h->C; p.R = h->R;
  p.Pt = h->Pt; p.Ph = h->Ph; p.Pw = h->Pw;
  const wf_plan_chunk* ch = reinterpret_cast<const wf_plan_chunk*>(static_cast<const uint8_t*>(host_plan) + h->off_chunks);
  for (int i = 0; i < h->R; ++i) p.slot[i] = ch[i].slot;
  const uint8_t* dp = static_cast<const uint8_t*>(dev_plan);
  p.tab_t = reinterpret_cast<const double2*>(dp + h->off_rope_t);
  p.tab_h = reinterpret_cast<const double2*>(dp + h->off_rope_h);
  p.tab_w = reinterpret_cast<const double2*>(dp + h->off_rope_w);
  p.nvec = int64_t(h->R) * h->C * h->H * h->D * elem / 16;
  if (p.nvec == 0) return WF_OK;
  if (p.nvec >= (int64_t(1) << 31)) return WF_ERR_CAPACITY;  // the divisions assume indices < 2^31
  p.div_vpr = make_fastdiv(uint32_t(h->D * elem / 16));
  p.div_H = make_fastdiv(uint32_t(h->H));
  p.div_C = make_fastdiv(uint32_t(h->C));
  p.div_fhw = make_fastdiv(uint32_t(h->fh * h->fw));
  p.div_fw = make_fastdiv(uint32_t(h->fw));

  const int64_t nblocks = (p.nvec + kRopeThreads - 1) / kRopeThreads;
  if (nblocks > 0x7FFFFFFF) return WF_ERR_CAPACITY;
  const unsigned blocks = unsigned(nblocks);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint4* q4 = static_cast<const uint4*>(q);
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  uint4* qr4 = static_cast<uint4*>(q_rot);
  uint4* kp4 = static_cast<uint4*>(k_pool);
  uint4* vp4 = static_cast<uint4*>(v_pool);
  const bool bf16 = h->dtype == WF_BF16;
  if (with_q && bf16)
    rope3d_append_kernel<__nv_bfloat16, true><<<blocks, kRopeThreads, 0, s>>>(p, q4, k4, v4, qr4, kp4, vp4);
  else if (with_q)
    rope3d_append_kernel<float, true><<<blocks, kRopeThreads, 0, s>>>(p, q4, k4, v4, qr4, kp4, vp4);
  else if (bf16)
    rope3d_append_kernel<__nv_bfloat16, false><<<blocks, kRopeThreads, 0, s>>>(p, q4, k4, v4, qr4, kp4, vp4);
  else
    rope3d_append_kernel<float, false><<<blocks, kRopeThreads, 0, s>>>(p, q4, k4, v4, qr4, kp4, vp4);
  if (cudaGetLastError() != cudaSuccess) return WF_ERR_CUDA;
  return WF_OK;
}

}  // namespace

extern "C" wf_status wf_rope3d_append(const void* host_plan, const void* dev_plan, const void* q, const void* k,
                                      const void* v, void* q_rot, void* k_pool, void* v_pool,
                                      wf_stream_t stream) {
  if (!host_plan || !dev_plan || !q || !k || !v || !q_rot || !k_pool || !v_pool) return WF_ERR_INVALID_ARG;
  return rope_append(host_plan, dev_plan, q, k, v, q_rot, k_pool, v_pool, stream);
}

extern "C" wf_status wf_rope3d_append_kv(const void* host_plan, const void* dev_plan, const void* k, const void* v,
                                         void* k_pool, void* v_pool, wf_stream_t stream) {
  if (!host_plan || !dev_plan || !k || !v || !k_pool || !v_pool) return WF_ERR_INVALID_ARG;
  return rope_append(host_plan, dev_plan, nullptr, k, v, nullptr, k_pool, v_pool, stream);
}
