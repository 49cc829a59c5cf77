// Internal layout of the plan blob written by wf_plan_round and read by the
// kernels (device copy) and launchers (host copy).  Both copies are the same
// bytes.  Offsets below are fixed; the Python binding mirrors them.
#pragma once

#include <stddef.h>
#include <stdint.h>

#define WF_PLAN_MAGIC 0x31504657u  // "WFP1" little-endian
#define WF_PLAN_VERSION 2u
#define WF_KEY_TILE 128            // keys per attention tile
#define WF_Q_TILE 128              // query rows per tensor-core tile
#define WF_Q_PAIR 256              // query rows per attention work unit (two tiles)

// One in-round chunk.  Its visible chunks are consecutive global indices
// first .. n, i.e. consecutive ring slots, which occupy at most two
// contiguous runs ("segments") of pool tokens.
struct wf_plan_chunk {
  int64_t n;             // global chunk index n0 + i
  int32_t slot;          // n mod S
  int32_t noise;         // noise level (metadata)
  int32_t nvis;          // number of visible chunks
  int32_t keys;          // nvis * C
  int32_t seg_start[2];  // first pool token of each run
  int32_t seg_len[2];    // tokens in each run (second may be 0)
  int32_t seg_tiles[2];  // ceil(seg_len / WF_KEY_TILE)
  int32_t key_tiles;     // seg_tiles[0] + seg_tiles[1]
  int32_t frame_base;    // index of this chunk's first frame in the t table (i * F)
};
static_assert(sizeof(wf_plan_chunk) == 56, "chunk record layout");

// One attention work unit: query rows [pair*256, min(C, pair*256+256)) of
// in-round chunk `chunk`, head `head`, against part `part` of `parts` equal
// shares of the chunk's key tiles (tiles [part*n/parts, (part+1)*n/parts),
// n the kernel's tile count; parts = 1: all of them).  A split unit writes
// its normalised partial O and LSE to partial slot `slot` of the attention
// workspace and a combine pass merges the parts (slot = -1 when parts = 1).
// cost = its key tiles * (9 + live 128-row tiles): a unit's time is
// dominated by its per-key-tile pipeline latency.
struct wf_plan_unit {
  int32_t chunk, head, pair, cost;
  int32_t part, parts, slot, pad;
};
static_assert(sizeof(wf_plan_unit) == 32, "unit record layout");

#define WF_MAX_KEY_PARTS 8        // most parts a unit's keys are split into
#define WF_MIN_PART_TILES 8       // fewest 128-key tiles a part may hold

struct wf_plan_hdr {
  uint32_t magic;        // 0
  uint32_t version;      // 4
  uint64_t total_bytes;  // 8
  int32_t H, D, fh, fw;  // 16
  int32_t F, C, Wc, wc_eff;  // 32
  int32_t R, S, dtype, Pt;   // 48
  int32_t Ph, Pw, num_ctas, num_units;  // 64
  int32_t q_pairs, q_tiles, max_key_tiles, max_nvis;  // 80
  int64_t n0, first;     // 96
  double theta;          // 112
  uint64_t off_chunks;   // 120: wf_plan_chunk[R]
  uint64_t off_vis;      // 128: int32[R][Wc + R] visible slots (-1 padded)
  uint64_t off_rope_t;   // 136: double2 (cos, sin) [R*F][Pt]
  uint64_t off_rope_h;   // 144: double2 [fh][Ph]
  uint64_t off_rope_w;   // 152: double2 [fw][Pw]
  uint64_t off_units;    // 160: wf_plan_unit[num_units], CTA-major
  uint64_t off_cta;      // 168: int32[num_ctas + 1] unit offsets per CTA
  int32_t noise_t[16];   // 176
};                       // 240
static_assert(sizeof(wf_plan_hdr) == 240, "header layout");
static_assert(offsetof(wf_plan_hdr, n0) == 96, "header layout");
static_assert(offsetof(wf_plan_hdr, off_chunks) == 120, "header layout");

#define WF_ATTN_STATUS_BYTES 256  // status word block at the start of the workspace
// After it, for plans with split units: partial O [slots][256 rows][128] fp32,
// then partial LSE [slots][256 rows] fp32 (slots = number of units).

// Device-side status record at the start of an attention workspace.
struct wf_dev_status {
  int32_t code;    // 0 = ok, else a wf_status value
  int32_t where;   // which wait gave up
  int32_t block;
  int32_t thread;
};
