// Block-causal flash-attention forward of one wave round on B200 tensor
// cores (tcgen05 + TMEM + TMA), bf16 in/out, head_dim 128.
//
// Persistent kernel, one CTA per SM, each CTA working through the plan's
// list of units (chunk i, head h, 256 query rows = two 128-row tiles).  The
// visible keys of chunk i are the plan's one or two contiguous pool runs,
// walked in 128-key tiles; tiles of chunks that chunk i may not see are never
// loaded.  Only the last tile of a run can be ragged; its extra columns are
// masked to -inf.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for query tile 0 (thread = one TMEM lane = one row)
//   warps 4-7  softmax for query tile 1
//   warp  8    tcgen05.mma issue (lane 0) and TMEM allocation (whole warp)
//   warp  9    TMA producer (lane 0); warps 10-11 idle
// The block launches at 168 registers per thread (the most that three warps
// per SM sub-partition allow); the control warpgroup then gives registers
// back (setmaxnreg.dec to 56) and the softmax warpgroups take them
// (setmaxnreg.inc to 224): 2*128*224 + 128*56 = 384*168.
// TMEM (512 columns x 128 lanes x 32 bit):
//   S_t = Q_t K^T at columns [128t, 128t+128), fp32; P_t (bf16 pairs) is
//   written over the first 64 of them; O_t at [256+128t, 256+128t+128).
// Shared memory: Q_0, Q_1 (32 KB each) and a ring of kStages 32 KB K/V tiles,
// all 128-byte-swizzled, K-major for Q and K, MN-major for V.
//
// Per key tile j the MMA thread issues, in order,
//   PV_0(j-1) .. S_0(j) .. PV_1(j-1) .. S_1(j)
// so the commit that announces S_t(j) also covers PV_t(j-1): when a softmax
// thread sees S_t(j) it owns O_t and may rescale it in place.  Online
// softmax in the log2 domain with a lazily updated reference max: O is only
// rescaled when a row's max grows by more than 8 (a factor 256), so P stays
// below 256 and the fp32 sums stay exact enough; the final O / l uses the
// same reference, so the result is unchanged.
//
// The kFp8 instantiation computes the scores from e4m3 codes: Q and K tiles
// are 128 rows x 128 bytes (one TMA box each), S_t is four kind::f8f6f4 MMAs
// of 32 K elements, and the key tiles are the chunks' 128-token scale blocks
// (each visible chunk walked on its own, its last tile ragged), so that the
// softmax scales a tile's scores by one factor, q_scale * k_scale.  P, V, O
// and everything else are as in the bf16 instantiation.
//
// Every mbarrier wait is bounded by a time limit; on expiry the CTA records
// WF_ERR_DEVICE_TIMEOUT in the workspace status word, stops issuing work,
// drains what it issued and frees its TMEM before returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstddef>
#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "rope_math.cuh"
#include "sm100_ptx.cuh"
#include "wf.h"
#include "wf_plan.h"

namespace wf {
namespace {

constexpr int kThreads = 384;
constexpr uint32_t kSoftmaxRegs = 224;
constexpr uint32_t kControlRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs == kThreads * 168, "register split must match launch");
constexpr int kTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 tile
constexpr int kHalfBytes = kTileBytes / 2; // one 64-column (128-byte) half
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, 1);
// 8-bit scores: Q and K tiles of 128 tokens x 128 e4m3 codes (one 128-byte row each)
constexpr uint32_t kIdescQK8 = idesc_e4m3_f32(128, 128);
constexpr int kTile8Bytes = 128 * 128;

struct Params {
  const wf_plan_chunk* chunks;
  const wf_plan_unit* units;
  const int32_t* cta_off;
  __nv_bfloat16* out;
  float* lse;
  wf_dev_status* status;
  int32_t H, C;
  int32_t rc;            // R * C, the LSE row stride
  float scale_log2;      // softmax scale * log2(e)
  uint64_t timeout_ns;
  int32_t stall_first_load;  // test hook: CTA 0 never issues its first K tile
  // 8-bit scores only
  const float* q_scales;     // [R, nblk, H]
  const float* k_scales;     // [S, nblk, H]
  int32_t S, nblk;           // pool slots; scale blocks (= key tiles) per chunk
  // split units: normalised partial O [slot][256][128] and LSE [slot][256]
  float* part_o;
  float* part_lse;
  // Q's RoPE in the kernel: the device plan (token grid, fp64 (cos, sin) tables).
  // Read from the plan rather than passed here: a larger parameter block made
  // ptxas spill in the softmax.
  const wf_plan_hdr* plan;
};

// Token grid and table offsets for the in-kernel Q rotation, copied from the
// plan into shared memory (re-read there each row: held in registers across
// the loop they pushed the 56-register control warps into spills).
struct RopeConsts {
  uint32_t fw, fhw, F;
  int32_t Pt, Ph, Pw;
  uint32_t off_t, off_h, off_w;
};

// Shared-memory and barrier layout.  The kRopeQ instantiation (Q's RoPE done
// in the kernel) double-buffers Q so that the next unit's tile can be rotated
// while the current unit runs, and keeps three K/V stages to stay within
// 227 KB; the others hold one Q buffer and four K/V stages.
template <bool kRopeQ>
struct Layout {
  static constexpr int kQBufs = kRopeQ ? 2 : 1;
  static constexpr int kStages = kRopeQ ? 3 : 4;
  static constexpr int kQFull = 0;                             // + buffer: Q ready for the MMAs
  static constexpr int kQEmpty = kQFull + kQBufs;              // + buffer: last S MMA of its unit done
  static constexpr int kQRaw = kQEmpty + kQBufs;               // + buffer: raw Q landed (kRopeQ)
  static constexpr int kSFull = kQRaw + (kRopeQ ? kQBufs : 0);  // + t
  static constexpr int kPFull = kSFull + 2;                    // + t
  static constexpr int kOFull = kPFull + 2;                    // + t
  static constexpr int kMmaDone = kOFull + 2;
  static constexpr int kKVFull = kMmaDone + 1;                 // + stage
  static constexpr int kKVEmpty = kKVFull + kStages;           // + stage
  static constexpr int kNumBars = kKVEmpty + kStages;
  static constexpr int kTiles = 2 * kQBufs + kStages;          // 32 KB tiles: Q buffers, then K/V stages
  static constexpr int kSmemBytes = 1024 + kTiles * kTileBytes + 256;
  static_assert(8 * kNumBars + 8 + sizeof(RopeConsts) <= 256, "barrier block");
  static_assert(kSmemBytes <= 232448, "shared memory per block");
};

struct Shared {
  uint8_t* base;  // Q buffers (two tiles each), then the K/V stages; 1024-aligned
  uint64_t* bars;
  uint32_t* tmem_slot;
  int32_t* abort_flag;
  RopeConsts* rope;
};

template <bool kRopeQ>
__device__ __forceinline__ uint8_t* q_tile(const Shared& s, int buf, int t) {
  return s.base + (2 * buf + t) * kTileBytes;
}
template <bool kRopeQ>
__device__ __forceinline__ uint8_t* kv_tile(const Shared& s, int st) {
  return s.base + (2 * Layout<kRopeQ>::kQBufs + st) * kTileBytes;
}

template <bool kRopeQ>
__device__ __forceinline__ Shared carve_smem(uint8_t* raw) {
  Shared s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.base = base;
  uint8_t* tail = base + Layout<kRopeQ>::kTiles * kTileBytes;
  s.bars = reinterpret_cast<uint64_t*>(tail);
  s.tmem_slot = reinterpret_cast<uint32_t*>(tail + 8 * Layout<kRopeQ>::kNumBars);
  s.abort_flag = reinterpret_cast<int32_t*>(tail + 8 * Layout<kRopeQ>::kNumBars + 4);
  s.rope = reinterpret_cast<RopeConsts*>(tail + 8 * Layout<kRopeQ>::kNumBars + 8);
  return s;
}

// Bounded wait.  Returns false if this CTA is aborting (the wait expired here
// or in another role); the first expiry records the status word.
__device__ __forceinline__ bool wait_bar(const Shared& sh, const Params& p, int bar, uint32_t parity, int where) {
  const uint32_t addr = smem_u32(sh.bars + bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(addr, parity)) return true;
    if (*reinterpret_cast<volatile int32_t*>(sh.abort_flag)) return false;
    if (global_timer_ns() - t0 > p.timeout_ns) {
      *reinterpret_cast<volatile int32_t*>(sh.abort_flag) = 1;
      if (atomicCAS(&p.status->code, 0, int32_t(WF_ERR_DEVICE_TIMEOUT)) == 0) {
        p.status->where = where;
        p.status->block = int32_t(blockIdx.x);
        p.status->thread = int32_t(threadIdx.x);
        __threadfence();
      }
      return false;
    }
  }
}

// Key tile j of chunk c: pool token of its first key and the number of valid keys.
__device__ __forceinline__ void key_tile(const wf_plan_chunk& c, int j, int32_t& tok, int32_t& valid) {
  // selects, not a dynamic index: keeps the record in registers
  const bool first = j < c.seg_tiles[0];
  const int t = first ? j : j - c.seg_tiles[0];
  tok = (first ? c.seg_start[0] : c.seg_start[1]) + t * 128;
  const int32_t left = (first ? c.seg_len[0] : c.seg_len[1]) - t * 128;
  valid = left < 128 ? left : 128;
}

// 8-bit path: the key tiles are the chunks' scale blocks.  Tile j of a unit
// whose oldest visible chunk sits in slot first_slot is block `blk` of
// visible chunk j / nblk.
__device__ __forceinline__ void key_tile_fp8(const Params& p, int first_slot, int j, int32_t& tok, int32_t& valid,
                                             int32_t& slot, int32_t& blk) {
  const int v = j / p.nblk;
  blk = j - v * p.nblk;
  slot = first_slot + v;  // v < nvis <= S
  if (slot >= p.S) slot -= p.S;
  tok = slot * p.C + blk * 128;
  const int32_t left = p.C - blk * 128;
  valid = left < 128 ? left : 128;
}

// Visible chunks are the consecutive global indices n - nvis + 1 .. n.
__device__ __forceinline__ int first_visible_slot(const Params& p, const wf_plan_chunk* rec) {
  const int64_t n = __ldg(&rec->n);
  const int32_t nvis = __ldg(&rec->nvis);
  return int((n - nvis + 1) % p.S);
}

// Key tiles [t0, t1) of a unit: its part of the chunk's n tiles.
__device__ __forceinline__ void unit_tile_range(const wf_plan_unit& unit, int n, int& t0, int& t1) {
  t0 = unit.part * n / unit.parts;
  t1 = (unit.part + 1) * n / unit.parts;
}

template <bool kFp8>
__device__ __forceinline__ int unit_key_tiles(const Params& p, const wf_plan_chunk* rec) {
  if constexpr (kFp8)
    return __ldg(&rec->nvis) * p.nblk;
  else
    return __ldg(&rec->key_tiles);
}

__device__ __forceinline__ wf_plan_chunk load_chunk(const wf_plan_chunk* p) {
  wf_plan_chunk c;
  c.seg_start[0] = __ldg(&p->seg_start[0]);
  c.seg_start[1] = __ldg(&p->seg_start[1]);
  c.seg_len[0] = __ldg(&p->seg_len[0]);
  c.seg_len[1] = __ldg(&p->seg_len[1]);
  c.seg_tiles[0] = __ldg(&p->seg_tiles[0]);
  c.seg_tiles[1] = __ldg(&p->seg_tiles[1]);
  c.key_tiles = __ldg(&p->key_tiles);
  return c;
}

// ---------------------------------------------------------------- roles

// TMA loads of one unit's query tiles into Q buffer `buf`, completing on `bar`
// (the raw tiles when the kernel rotates Q itself).
template <bool kFp8, bool kRopeQ>
__device__ __forceinline__ void load_q(const Shared& sh, const CUtensorMap* tm_q, const wf_plan_unit& unit, int C,
                                       int buf, uint32_t bar) {
  const int32_t row0 = unit.chunk * C + unit.pair * 256;
  const bool live1 = C - unit.pair * 256 > 128;
  uint8_t* q0 = q_tile<kRopeQ>(sh, buf, 0);
  uint8_t* q1 = q_tile<kRopeQ>(sh, buf, 1);
  if constexpr (kFp8) {
    mbar_arrive_expect_tx(bar, live1 ? 2 * kTile8Bytes : kTile8Bytes);
    tma_load_3d(smem_u32(q0), tm_q, bar, 0, unit.head, row0);
    if (live1) tma_load_3d(smem_u32(q1), tm_q, bar, 0, unit.head, row0 + 128);
  } else {
    mbar_arrive_expect_tx(bar, live1 ? 2 * kTileBytes : kTileBytes);
    tma_load_3d(smem_u32(q0), tm_q, bar, 0, unit.head, row0);
    tma_load_3d(smem_u32(q0 + kHalfBytes), tm_q, bar, 64, unit.head, row0);
    if (live1) {
      tma_load_3d(smem_u32(q1), tm_q, bar, 0, unit.head, row0 + 128);
      tma_load_3d(smem_u32(q1 + kHalfBytes), tm_q, bar, 64, unit.head, row0 + 128);
    }
  }
}

template <bool kFp8, bool kRopeQ>
__device__ __forceinline__ void producer(const Shared& sh, const Params& p, const CUtensorMap* tm_q,
                                         const CUtensorMap* tm_k, const CUtensorMap* tm_v, int u0, int u1) {
  using L = Layout<kRopeQ>;
  constexpr int kQB = L::kQBufs;
  int kv_it = 0;
  int q_it = 0;  // Q loads issued
  bool ok = true;
  // Q load of unit u into buffer q_it % kQB, once the unit that last used
  // that buffer has issued its final score MMA.
  auto issue_q = [&](int u) -> bool {
    const int buf = q_it % kQB;
    if (q_it >= kQB && !wait_bar(sh, p, L::kQEmpty + buf, ((q_it / kQB) - 1) & 1, 1)) return false;
    const uint32_t bar = smem_u32(sh.bars + (kRopeQ ? L::kQRaw : L::kQFull) + buf);
    load_q<kFp8, kRopeQ>(sh, tm_q, p.units[u], p.C, buf, bar);
    ++q_it;
    return true;
  };
  if (kRopeQ && u0 < u1 && !issue_q(u0)) ok = false;
  for (int u = u0; u < u1 && ok; ++u) {
    const wf_plan_unit unit = p.units[u];
    const wf_plan_chunk c = load_chunk(p.chunks + unit.chunk);
    if (!kRopeQ && !issue_q(u)) { ok = false; break; }
    const int first_slot = kFp8 ? first_visible_slot(p, p.chunks + unit.chunk) : 0;
    int t0, t1;
    unit_tile_range(unit, unit_key_tiles<kFp8>(p, p.chunks + unit.chunk), t0, t1);
    // with two Q buffers the next unit's tile is loaded once this unit's
    // first key tiles are in flight (so the buffer it reuses is surely free
    // soon), leaving the rotation the rest of this unit to finish
    const int q_next_at = t0 + (t1 - t0 < L::kStages ? t1 - t0 : L::kStages);
    for (int j = t0; j < t1; ++j) {
      if (kRopeQ && j == q_next_at && u + 1 < u1 && !issue_q(u + 1)) { ok = false; break; }
      int32_t tok, valid;
      if constexpr (kFp8) {
        int32_t slot, blk;
        key_tile_fp8(p, first_slot, j, tok, valid, slot, blk);
      } else {
        key_tile(c, j, tok, valid);
      }
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const int st = kv_it % L::kStages;
        if (p.stall_first_load && blockIdx.x == 0 && kv_it == 0) {
          // failure-detection test: this fill's barrier is never armed, so
          // the MMA thread's bounded wait on it must expire
          ++kv_it;
          continue;
        }
        if (!wait_bar(sh, p, L::kKVEmpty + st, ((kv_it / L::kStages) & 1) ^ 1, 2)) { ok = false; break; }
        const uint32_t bar = smem_u32(sh.bars + L::kKVFull + st);
        const CUtensorMap* tm = kv == 0 ? tm_k : tm_v;
        uint8_t* dst = kv_tile<kRopeQ>(sh, st);
        if (kFp8 && kv == 0) {  // e4m3 K: one 128-byte-wide box
          mbar_arrive_expect_tx(bar, kTile8Bytes);
          tma_load_3d(smem_u32(dst), tm, bar, 0, unit.head, tok);
        } else {
          mbar_arrive_expect_tx(bar, kTileBytes);
          tma_load_3d(smem_u32(dst), tm, bar, 0, unit.head, tok);
          tma_load_3d(smem_u32(dst + kHalfBytes), tm, bar, 64, unit.head, tok);
        }
        ++kv_it;
      }
      if (!ok) break;
    }
    if (ok && kRopeQ && q_next_at >= t1 && u + 1 < u1 && !issue_q(u + 1)) ok = false;
  }
  // Drain: the CTA must not exit with bulk copies still landing in its smem.
  if (!ok) {
    for (int s = 0; s < L::kStages; ++s) {
      if (kv_it <= s) continue;
      const int last_fill = (kv_it - 1 - s) / L::kStages;  // fill count - 1 of stage s
      const uint32_t addr = smem_u32(sh.bars + L::kKVFull + s);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(addr, uint32_t(last_fill) & 1) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int b = 0; b < kQB; ++b) {
      if (q_it <= b) continue;
      const int last_fill = (q_it - 1 - b) / kQB;
      const uint32_t addr = smem_u32(sh.bars + (kRopeQ ? L::kQRaw : L::kQFull) + b);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(addr, uint32_t(last_fill) & 1) && global_timer_ns() - t0 < p.timeout_ns) {
      }
    }
  }
}

// kRopeQ: warps 10-11 rotate each unit's raw query tiles in place, in fp64
// from the plan's tables, rounding once to bf16 exactly as wf_rope3d_append
// does, then hand the buffer to the MMA thread.  In the 128-byte-swizzled
// tile, row r's 16-byte chunk c of a 64-column half sits at chunk c ^ (r % 8);
// an interleaved pair never straddles a chunk.  Rows past the chunk's end are
// left as loaded (their outputs are never stored).
__device__ __forceinline__ void rope_q_role(const Shared& sh, const Params& p, int u0, int u1) {
  using L = Layout<true>;
  const int th = threadIdx.x - 320;  // 0..63
  // 64 threads stride over a tile's 128 rows x 16 chunks: each thread keeps
  // chunk column cc (dims 8cc..8cc+7, pairs 4cc..4cc+3) on every fourth row
  const int cc = th & 15;
  const uint32_t q_base = smem_u32(q_tile<true>(sh, 0, 0)) + (cc >> 3) * kHalfBytes;
  const uint32_t rc_addr = smem_u32(sh.rope);
  const uint8_t* plan = reinterpret_cast<const uint8_t*>(p.plan);
  int q_it = 0;
  for (int u = u0; u < u1; ++u, ++q_it) {
    const int buf = q_it % L::kQBufs;
    if (!__all_sync(0xffffffffu, wait_bar(sh, p, L::kQRaw + buf, (q_it / L::kQBufs) & 1, 30))) return;
    const int32_t chunk = p.units[u].chunk, pair = p.units[u].pair;
    for (int t = 0; t < 2; ++t) {
      const int rows_here = p.C - pair * 256 - 128 * t;
      if (rows_here <= 0) break;
      const uint32_t tile = q_base + uint32_t(2 * buf + t) * kTileBytes;
#pragma unroll 1
      for (int row = th >> 4; row < 128 && row < rows_here; row += 4) {
        const uint32_t addr = tile + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
        const uint32_t fw = ld_shared_u32(rc_addr + offsetof(RopeConsts, fw));
        const uint32_t fhw = ld_shared_u32(rc_addr + offsetof(RopeConsts, fhw));
        const uint32_t q = uint32_t(pair * 256 + 128 * t + row);  // token inside the chunk
        const uint32_t f = q / fhw, l = q - f * fhw;
        const uint32_t hh = l / fw, ww = l - hh * fw;
        const uint32_t trow = uint32_t(chunk) * ld_shared_u32(rc_addr + offsetof(RopeConsts, F)) + f;
        uint32_t w[4];
        ld_shared_v4(addr, w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int32_t m = 4 * cc + k;
          const int32_t Pt = int32_t(ld_shared_u32(rc_addr + offsetof(RopeConsts, Pt)));
          const int32_t Ph = int32_t(ld_shared_u32(rc_addr + offsetof(RopeConsts, Ph)));
          const double2* tab;
          if (m < Pt) {
            tab = reinterpret_cast<const double2*>(plan + ld_shared_u32(rc_addr + offsetof(RopeConsts, off_t))) +
                  int64_t(trow) * Pt + m;
          } else if (m < Pt + Ph) {
            tab = reinterpret_cast<const double2*>(plan + ld_shared_u32(rc_addr + offsetof(RopeConsts, off_h))) +
                  int64_t(hh) * Ph + (m - Pt);
          } else {
            const int32_t Pw = int32_t(ld_shared_u32(rc_addr + offsetof(RopeConsts, Pw)));
            tab = reinterpret_cast<const double2*>(plan + ld_shared_u32(rc_addr + offsetof(RopeConsts, off_w))) +
                  int64_t(ww) * Pw + (m - Pt - Ph);
          }
          w[k] = rope_pair_bf16(w[k], __ldg(tab));
        }
        st_shared_v4(addr, w[0], w[1], w[2], w[3]);
      }
    }
    // make the rotated tile visible to the tensor cores (async proxy)
    fence_proxy_async_smem();
    mbar_arrive(smem_u32(sh.bars + L::kQFull + buf));
  }
}

// The descriptor's start-address field holds (address >> 4) in its low 14
// bits; every offset below stays inside one tile, so adding (offset >> 4) to
// a base descriptor moves its start address without touching other fields.
// MMA issue is fully unrolled with every per-slice descriptor offset an
// immediate: a single thread issues the MMAs, and per-MMA address arithmetic
// in a loop made issue (about 100 cycles per MMA) slower than the tensor core
// (64 cycles per 128x128x16 MMA).  Offsets are in 16-byte units and stay
// inside one tile, so they never carry out of the start-address field.
template <int kk>
struct SliceOff {
  // K-major, 128-byte swizzle: 16-element K slices are 32 bytes apart inside
  // a 64-element half; the second half starts 16 KB later.
  static constexpr uint32_t kKMajor = uint32_t(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
  // V is MN-major (head_dim contiguous): 16 keys = 2 KB further on; the two
  // 64-column halves are 16 KB apart (leading byte offset), 8-key groups 1 KB
  // apart (stride byte offset).
  static constexpr uint32_t kMNMajor = uint32_t((kk * 2048) >> 4);
};

template <int kk>
__device__ __forceinline__ void issue_s_slice(uint32_t s_tmem, uint64_t qd, uint64_t kd) {
  mma_ss_off<SliceOff<kk>::kKMajor, SliceOff<kk>::kKMajor>(s_tmem, qd, kd, kIdescQK, kk > 0 ? 1u : 0u);
  if constexpr (kk < 7) issue_s_slice<kk + 1>(s_tmem, qd, kd);
}

template <int kk>
__device__ __forceinline__ void issue_pv_slice(uint32_t o_tmem, uint32_t p_tmem, uint64_t vd, uint32_t acc0) {
  // P_t holds 2 bf16 per TMEM column: 16 keys = 8 columns
  mma_ts_off<kk * 8, SliceOff<kk>::kMNMajor>(o_tmem, p_tmem, vd, kIdescPV, kk > 0 ? 1u : acc0);
  if constexpr (kk < 7) issue_pv_slice<kk + 1>(o_tmem, p_tmem, vd, acc0);
}

__device__ __forceinline__ uint64_t kmajor_desc(const uint8_t* tile) { return smem_desc_sw128(smem_u32(tile), 16, 1024); }
__device__ __forceinline__ uint64_t mnmajor_desc(const uint8_t* tile) {
  return smem_desc_sw128(smem_u32(tile), kHalfBytes, 1024);
}

// e4m3 scores: four 32-element K slices, 32 bytes apart inside the 128-byte rows.
template <int kk>
__device__ __forceinline__ void issue_s8_slice(uint32_t s_tmem, uint64_t qd, uint64_t kd) {
  mma_f8_ss_off<kk * 2, kk * 2>(s_tmem, qd, kd, kIdescQK8, kk > 0 ? 1u : 0u);
  if constexpr (kk < 3) issue_s8_slice<kk + 1>(s_tmem, qd, kd);
}

template <bool kFp8>
__device__ __forceinline__ void issue_s(uint32_t s_tmem, uint64_t qd, const uint8_t* k) {
  if constexpr (kFp8)
    issue_s8_slice<0>(s_tmem, qd, kmajor_desc(k));
  else
    issue_s_slice<0>(s_tmem, qd, kmajor_desc(k));
}

__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, const uint8_t* v, bool accumulate) {
  issue_pv_slice<0>(o_tmem, p_tmem, mnmajor_desc(v), accumulate ? 1u : 0u);
}

template <bool kFp8, bool kRopeQ>
__device__ __forceinline__ void mma_issuer(const Shared& sh, const Params& p, uint32_t tmem, int u0, int u1) {
  using L = Layout<kRopeQ>;
  int kv_it = 0, q_it = 0;
  int p_cnt[2] = {0, 0};
  bool ok = true;
  const uint32_t s_tm[2] = {tmem + 0, tmem + 128};
  const uint32_t o_tm[2] = {tmem + 256, tmem + 384};
  for (int u = u0; u < u1 && ok; ++u) {
    const wf_plan_unit unit = p.units[u];
    int t0, t1;
    unit_tile_range(unit, unit_key_tiles<kFp8>(p, p.chunks + unit.chunk), t0, t1);
    const int n = t1 - t0;  // key tiles of this unit
    const bool live1 = p.C - unit.pair * 256 > 128;
    const int qbuf = q_it % L::kQBufs;
    if (!wait_bar(sh, p, L::kQFull + qbuf, (q_it / L::kQBufs) & 1, 10)) { ok = false; break; }
    ++q_it;
    const uint64_t qd0 = kmajor_desc(q_tile<kRopeQ>(sh, qbuf, 0)), qd1 = kmajor_desc(q_tile<kRopeQ>(sh, qbuf, 1));
    tc_fence_after();
    int kst = kv_it % L::kStages;
    if (!wait_bar(sh, p, L::kKVFull + kst, (kv_it / L::kStages) & 1, 11)) { ok = false; break; }
    ++kv_it;
    tc_fence_after();
    issue_s<kFp8>(s_tm[0], qd0, kv_tile<kRopeQ>(sh, kst));
    mma_commit(smem_u32(sh.bars + L::kSFull + 0));
    if (live1) {
      issue_s<kFp8>(s_tm[1], qd1, kv_tile<kRopeQ>(sh, kst));
      mma_commit(smem_u32(sh.bars + L::kSFull + 1));
    }
    mma_commit(smem_u32(sh.bars + L::kKVEmpty + kst));
    if (n == 1) mma_commit(smem_u32(sh.bars + L::kQEmpty + qbuf));
    for (int j = 0; j < n; ++j) {
      const int vst = kv_it % L::kStages;
      if (!wait_bar(sh, p, L::kKVFull + vst, (kv_it / L::kStages) & 1, 12)) { ok = false; break; }
      ++kv_it;
      const bool more = j + 1 < n;
      if (more) {
        kst = kv_it % L::kStages;
        if (!wait_bar(sh, p, L::kKVFull + kst, (kv_it / L::kStages) & 1, 13)) { ok = false; break; }
        ++kv_it;
      }
      // tile 0
      if (!wait_bar(sh, p, L::kPFull + 0, p_cnt[0] & 1, 14)) { ok = false; break; }
      ++p_cnt[0];
      tc_fence_after();
      issue_pv(o_tm[0], s_tm[0], kv_tile<kRopeQ>(sh, vst), j > 0);
      if (more) {
        issue_s<kFp8>(s_tm[0], qd0, kv_tile<kRopeQ>(sh, kst));
        mma_commit(smem_u32(sh.bars + L::kSFull + 0));
      } else {
        mma_commit(smem_u32(sh.bars + L::kOFull + 0));
      }
      // tile 1
      if (live1) {
        if (!wait_bar(sh, p, L::kPFull + 1, p_cnt[1] & 1, 15)) { ok = false; break; }
        ++p_cnt[1];
        tc_fence_after();
        issue_pv(o_tm[1], s_tm[1], kv_tile<kRopeQ>(sh, vst), j > 0);
        if (more) {
          issue_s<kFp8>(s_tm[1], qd1, kv_tile<kRopeQ>(sh, kst));
          mma_commit(smem_u32(sh.bars + L::kSFull + 1));
        } else {
          mma_commit(smem_u32(sh.bars + L::kOFull + 1));
        }
      }
      mma_commit(smem_u32(sh.bars + L::kKVEmpty + vst));
      if (more) mma_commit(smem_u32(sh.bars + L::kKVEmpty + kst));
      if (j + 2 == n) mma_commit(smem_u32(sh.bars + L::kQEmpty + qbuf));
    }
  }
  // all issued MMAs complete before TMEM is released
  mma_commit(smem_u32(sh.bars + L::kMmaDone));
  const uint32_t addr = smem_u32(sh.bars + L::kMmaDone);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(addr, 0) && global_timer_ns() - t0 < p.timeout_ns) {
  }
}

// exp2 of one row's 128 scores (scaled by sl2, minus the reference max m_ref)
// stored as bf16 pairs into TMEM at s_tm; returns the row sum of the fp32
// values.  Every exp2 runs on MUFU (masked columns hold -inf and give +0).
// Moving a share of them to an FMA-pipe polynomial (a cubic on the fraction
// plus an exponent add) measured slower at every share tried: 1/8, 1/4 and
// 3/8 of the pairs gave 1058, 1052 and 1003 against 1124 TFLOP/s.  Four
// independent partial sums keep the row sum off one serial chain.
__device__ __forceinline__ float exp_to_p(const float (&s)[128], float sl2, float m_ref, uint32_t s_tm) {
  const float2 sl2x2 = make_float2(sl2, sl2);
  const float2 negm2 = make_float2(-m_ref, -m_ref);
  float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint32_t pk[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int pi = 16 * q4 + x;
      const float2 v = __ffma2_rn(make_float2(s[2 * pi], s[2 * pi + 1]), sl2x2, negm2);
      const float2 pr = make_float2(fast_exp2(v.x), fast_exp2(v.y));
      ls[x & 3] = __fadd2_rn(ls[x & 3], pr);
      pk[x] = pack_bf16x2(pr.x, pr.y);
    }
    tmem_st16(s_tm + 16 * q4, pk);
  }
  const float2 l01 = __fadd2_rn(ls[0], ls[1]), l23 = __fadd2_rn(ls[2], ls[3]);
  const float2 lt = __fadd2_rn(l01, l23);
  return lt.x + lt.y;
}

template <bool kFp8, bool kRopeQ>
__device__ __forceinline__ void softmax_role(const Shared& sh, const Params& p, uint32_t tmem, int t, int u0, int u1) {
  using L = Layout<kRopeQ>;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int row_in_tile = (warp % 4) * 32 + lane;
  const uint32_t lane_off = uint32_t((warp % 4) * 32) << 16;
  const uint32_t s_tm = tmem + lane_off + uint32_t(128 * t);
  const uint32_t o_tm = tmem + lane_off + uint32_t(256 + 128 * t);
  int s_cnt = 0, o_cnt = 0;
  for (int u = u0; u < u1; ++u) {
    const wf_plan_unit unit = p.units[u];
    const int rows_here = p.C - unit.pair * 256 - 128 * t;
    if (rows_here <= 0) continue;  // dead tile: the MMA thread skips it too
    const wf_plan_chunk c = load_chunk(p.chunks + unit.chunk);
    // scores -> log2 units: softmax scale * log2(e), times the query block's
    // scale on the 8-bit path (the key block's scale is applied per tile)
    float sl2_unit = p.scale_log2;
    int first_slot = 0;
    if constexpr (kFp8) {
      first_slot = first_visible_slot(p, p.chunks + unit.chunk);
      sl2_unit *= __ldg(p.q_scales + (int64_t(unit.chunk) * p.nblk + 2 * unit.pair + t) * p.H + unit.head);
    }
    int t0, t1;
    unit_tile_range(unit, unit_key_tiles<kFp8>(p, p.chunks + unit.chunk), t0, t1);
    float m_ref = -INFINITY;  // reference max (log2 units)
    float l = 0.f;
    for (int j = t0; j < t1; ++j) {
      int32_t tok, valid;
      float sl2 = sl2_unit;
      if constexpr (kFp8) {
        int32_t slot, blk;
        key_tile_fp8(p, first_slot, j, tok, valid, slot, blk);
        sl2 *= __ldg(p.k_scales + (int64_t(slot) * p.nblk + blk) * p.H + unit.head);
      } else {
        key_tile(c, j, tok, valid);
      }
      // warp-uniform: the TMEM loads and stores below are warp-collective
      if (!__all_sync(0xffffffffu, wait_bar(sh, p, L::kSFull + t, s_cnt & 1, 20 + t))) return;
      ++s_cnt;
      tc_fence_after();
      float s[128];
      float mxs[8];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t r[32];
        tmem_ld32(s_tm + 32 * q4, r);
#pragma unroll
        for (int x = 0; x < 32; ++x) s[32 * q4 + x] = __uint_as_float(r[x]);
      }
      tmem_wait_ld();
      if (valid < 128) {
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x >= valid) s[x] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) mxs[c] = fmaxf(s[c], s[c + 8]);
#pragma unroll
      for (int x = 16; x < 128; x += 16) {
#pragma unroll
        for (int c = 0; c < 8; ++c) mxs[c] = max3f(mxs[c], s[x + c], s[x + 8 + c]);
      }
      const float mx = fmaxf(max3f(mxs[0], mxs[1], mxs[2]), max3f(mxs[3], max3f(mxs[4], mxs[5], mxs[6]), mxs[7]));
      const float m_new = fmaxf(m_ref, mx * sl2);
      if (j == t0) {
        m_ref = m_new;
      } else {
        const bool need = m_new > m_ref + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t r[32];
            tmem_ld32(o_tm + 32 * q4, r);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
            tmem_st32(o_tm + 32 * q4, r);
          }
          tmem_wait_st();
          if (need) {
            l *= alpha;
            m_ref = m_new;
          }
        }
      }
      // P = exp2(s * sl2 - m_ref) into TMEM over S's first 64 columns
      l += exp_to_p(s, sl2, m_ref, s_tm);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(sh.bars + L::kPFull + t));
    }
    // epilogue: O / l -> bf16 rows of this tile (a part of a split unit:
    // fp32 rows and the LSE into its partial slot, merged by the combine pass)
    if (!__all_sync(0xffffffffu, wait_bar(sh, p, L::kOFull + t, o_cnt & 1, 24 + t))) return;
    ++o_cnt;
    tc_fence_after();
    const float inv_l = 1.0f / l;
    const int32_t qtok = unit.chunk * p.C + unit.pair * 256 + 128 * t + row_in_tile;
    const bool store = row_in_tile < rows_here;
    const float lse_row = (m_ref + __log2f(l)) * 0.69314718055994531f;
    if (unit.parts > 1) {
      const int64_t prow = int64_t(unit.slot) * 256 + 128 * t + row_in_tile;
      float4* pdst = reinterpret_cast<float4*>(p.part_o + prow * 128);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t r[32];
        tmem_ld32(o_tm + 32 * q4, r);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            pdst[8 * q4 + v] = make_float4(__uint_as_float(r[4 * v]) * inv_l, __uint_as_float(r[4 * v + 1]) * inv_l,
                                           __uint_as_float(r[4 * v + 2]) * inv_l, __uint_as_float(r[4 * v + 3]) * inv_l);
        }
      }
      if (store) p.part_lse[prow] = lse_row;
      continue;
    }
    uint4* dst = reinterpret_cast<uint4*>(p.out + (int64_t(qtok) * p.H + unit.head) * 128);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t r[32];
      tmem_ld32(o_tm + 32 * q4, r);
      tmem_wait_ld();
      if (store) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) * inv_l, __uint_as_float(r[8 * v + 1]) * inv_l);
          w.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) * inv_l, __uint_as_float(r[8 * v + 3]) * inv_l);
          w.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) * inv_l, __uint_as_float(r[8 * v + 5]) * inv_l);
          w.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) * inv_l, __uint_as_float(r[8 * v + 7]) * inv_l);
          dst[4 * q4 + v] = w;
        }
      }
    }
    if (store && p.lse) p.lse[int64_t(unit.head) * p.rc + qtok] = lse_row;
  }
}

template <bool kFp8, bool kRopeQ>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using L = Layout<kRopeQ>;
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve_smem<kRopeQ>(smem_raw);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (warp == 9 && lane == 0) {
    for (int b = 0; b < L::kNumBars; ++b) {
      uint32_t count = 1;
      if (b == L::kPFull || b == L::kPFull + 1) count = 128;  // the tile's softmax threads
      if (kRopeQ && b >= L::kQFull && b < L::kQFull + L::kQBufs) count = 64;  // the rotation threads
      mbar_init(smem_u32(sh.bars + b), count);
    }
    *sh.abort_flag = 0;
    if (kRopeQ) {
      RopeConsts rc;
      rc.fw = uint32_t(p.plan->fw);
      rc.fhw = uint32_t(p.plan->fh) * rc.fw;
      rc.F = uint32_t(p.plan->F);
      rc.Pt = p.plan->Pt;
      rc.Ph = p.plan->Ph;
      rc.Pw = p.plan->Pw;
      rc.off_t = uint32_t(p.plan->off_rope_t);
      rc.off_h = uint32_t(p.plan->off_rope_h);
      rc.off_w = uint32_t(p.plan->off_rope_w);
      *sh.rope = rc;
    }
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(sh.tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sh.tmem_slot;
  const int u0 = __ldg(p.cta_off + blockIdx.x);
  const int u1 = __ldg(p.cta_off + blockIdx.x + 1);

  if (warp < 8) {
    regs_increase<kSoftmaxRegs>();
    softmax_role<kFp8, kRopeQ>(sh, p, tmem, warp / 4, u0, u1);
  } else {
    regs_decrease<kControlRegs>();
    if (warp == 8) {
      if (lane == 0) mma_issuer<kFp8, kRopeQ>(sh, p, tmem, u0, u1);
      __syncwarp();
    } else if (warp == 9) {
      if (lane == 0) producer<kFp8, kRopeQ>(sh, p, &tm_q, &tm_k, &tm_v, u0, u1);
    } else if (kRopeQ) {
      rope_q_role(sh, p, u0, u1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host

// WF_VERBOSE=1 in the environment prints the failing CUDA step to stderr.
bool report(const char* step, int err) {
  static const int verbose = [] {
    const char* v = std::getenv("WF_VERBOSE");
    return v && v[0] == '1';
  }();
  if (verbose) std::fprintf(stderr, "[libwf] %s failed: error %d\n", step, err);
  return false;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess) {
      report("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", int(e) * 1000 + int(q));
      return nullptr;
    }
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [tokens, H, 128] viewed as 3-D (dim, head, token).  bf16: box = 64 dims x 1
// head x 128 tokens (128 bytes wide, loaded as two halves); e4m3 codes: box =
// all 128 dims (128 bytes) x 1 head x 128 tokens.
bool make_tmap(CUtensorMap* tm, const void* base, int64_t tokens, int32_t H, bool bytes) {
  auto encode = get_encode();
  if (!encode) return false;
  const cuuint64_t elem = bytes ? 1 : 2;
  cuuint64_t dims[3] = {128, cuuint64_t(H), cuuint64_t(tokens)};
  cuuint64_t strides[2] = {128 * elem, cuuint64_t(H) * 128 * elem};
  cuuint32_t box[3] = {bytes ? 128u : 64u, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(tm, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? true : report("cuTensorMapEncodeTiled", int(r));
}

template <bool kFp8, bool kRopeQ>
wf_status launch(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q, const float* q_scales,
                 const void* k_pool, const float* k_scales, const void* v_pool, void* out, float* lse, float scale,
                 void* workspace, uint64_t timeout_ns, cudaStream_t stream) {
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WF_ERR_CUDA;
  if (dev < 0 || dev >= 64) return WF_ERR_UNSUPPORTED;
  if (!attr_done[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(attn_fwd_sm100<kFp8, kRopeQ>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<kRopeQ>::kSmemBytes);
    if (e != cudaSuccess) {
      report(cudaGetErrorString(e), int(e));
      cudaGetLastError();
      return WF_ERR_CUDA;
    }
    attr_done[dev] = 1;
  }
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, int64_t(h->R) * h->C, h->H, kFp8) ||
      !make_tmap(&tk, k_pool, int64_t(h->S) * h->C, h->H, kFp8) ||
      !make_tmap(&tv, v_pool, int64_t(h->S) * h->C, h->H, false))
    return WF_ERR_CUDA;
  Params p{};
  p.chunks = reinterpret_cast<const wf_plan_chunk*>(dev_plan + h->off_chunks);
  p.units = reinterpret_cast<const wf_plan_unit*>(dev_plan + h->off_units);
  p.cta_off = reinterpret_cast<const int32_t*>(dev_plan + h->off_cta);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = static_cast<wf_dev_status*>(workspace);
  p.H = h->H;
  p.C = h->C;
  p.rc = h->R * h->C;
  p.scale_log2 = float(double(scale) * 1.4426950408889634);
  p.timeout_ns = timeout_ns;
  const char* stall = std::getenv("WF_DEBUG_STALL_FIRST_LOAD");
  p.stall_first_load = (stall && stall[0] == '1') ? 1 : 0;
  p.q_scales = q_scales;
  p.k_scales = k_scales;
  p.S = h->S;
  p.nblk = (h->C + 127) / 128;
  // partial slots after the status block (used only by split units)
  p.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + WF_ATTN_STATUS_BYTES);
  p.part_lse = p.part_o + int64_t(h->num_units) * 256 * 128;
  p.plan = reinterpret_cast<const wf_plan_hdr*>(dev_plan);
  attn_fwd_sm100<kFp8, kRopeQ><<<h->num_ctas, kThreads, Layout<kRopeQ>::kSmemBytes, stream>>>(tq, tk, tv, p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    report(cudaGetErrorString(e), int(e));
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, attn_fwd_sm100<kFp8, kRopeQ>) == cudaSuccess) {
      char msg[256];
      std::snprintf(msg, sizeof(msg), "attributes: regs %d, max threads %d, static smem %zu, max dyn smem %d",
                    fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes, fa.maxDynamicSharedSizeBytes);
      report(msg, 0);
    }
    return WF_ERR_CUDA;
  }
  return WF_OK;
}

}  // namespace

// Launch the tcgen05 path; arguments were validated by the caller.
wf_status launch_attn_sm100(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q_rot, const void* k_pool,
                            const void* v_pool, void* out, float* lse, float scale, void* workspace,
                            uint64_t timeout_ns, cudaStream_t stream) {
  return launch<false, false>(h, dev_plan, q_rot, nullptr, k_pool, nullptr, v_pool, out, lse, scale, workspace,
                              timeout_ns, stream);
}

// The same from the raw (not yet rotated) queries: the kernel applies Q's RoPE.
wf_status launch_attn_sm100_rope_q(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q_raw,
                                   const void* k_pool, const void* v_pool, void* out, float* lse, float scale,
                                   void* workspace, uint64_t timeout_ns, cudaStream_t stream) {
  return launch<false, true>(h, dev_plan, q_raw, nullptr, k_pool, nullptr, v_pool, out, lse, scale, workspace,
                             timeout_ns, stream);
}

// The same with e4m3 Q and K codes and their block scales.
wf_status launch_attn_sm100_fp8(const wf_plan_hdr* h, const uint8_t* dev_plan, const void* q8, const float* q_scales,
                                const void* k8_pool, const float* k_scales, const void* v_pool, void* out, float* lse,
                                float scale, void* workspace, uint64_t timeout_ns, cudaStream_t stream) {
  return launch<true, false>(h, dev_plan, q8, q_scales, k8_pool, k_scales, v_pool, out, lse, scale, workspace,
                             timeout_ns, stream);
}

}  // namespace wf
