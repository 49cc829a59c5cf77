// Host planner of a wave round: visibility, ring slots, RoPE tables and the
// attention work list.  Pure integer/fp64 host code plus one optional
// cudaMemcpyAsync of the finished blob.
//
// Visibility follows the chunk-wise causal attention of "Wave Forcing:
// Towards Speed-of-Light Streaming Video Generation" (arXiv 2611.00859v1,
// Abstract): an in-round chunk reads the clean cache and the earlier, cleaner
// in-round chunks, plus itself.  The ring and the RoPE layout are this
// library's stated choices (slot = n mod S; interleaved pairs split t|h|w,
// frequency theta^(-k/P) per axis group).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <queue>
#include <vector>

#include "wf.h"
#include "wf_plan.h"

namespace {

struct Geometry {
  int32_t H, D, fh, fw, F, C, Wc, wc_eff, R, S, dtype, Pt, Ph, Pw, G;
  int64_t n0, first;
  double theta;
  int32_t q_pairs, q_tiles, parts;
  int64_t num_units;
  uint64_t off_chunks, off_vis, off_rope_t, off_rope_h, off_rope_w, off_units, off_cta, total;
};

uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Validate `desc` and lay out the blob.  `need_device` controls whether
// num_ctas == 0 may query the current device.
wf_status geometry(const wf_round_desc* d, Geometry* g, bool query_device) {
  if (!d) return WF_ERR_INVALID_ARG;
  std::memset(g, 0, sizeof(*g));
  if (d->num_heads < 1 || d->num_heads > 4096) return WF_ERR_INVALID_ARG;
  if (d->head_dim < 2 || d->head_dim % 2 || d->head_dim > 1024) return WF_ERR_INVALID_ARG;
  if (d->frame_h < 1 || d->frame_w < 1 || d->frames_per_chunk < 1) return WF_ERR_INVALID_ARG;
  if (d->cache_chunks < 0 || d->inround_chunks < 1 || d->inround_chunks > WF_MAX_INROUND)
    return WF_ERR_INVALID_ARG;
  if (d->n0 < 0 || d->n0 > (int64_t(1) << 40)) return WF_ERR_INVALID_ARG;
  if (d->dtype != WF_F32 && d->dtype != WF_BF16) return WF_ERR_INVALID_ARG;
  if (!(d->rope_theta > 0.0) || !std::isfinite(d->rope_theta)) return WF_ERR_INVALID_ARG;
  if (d->num_ctas < 0 || d->num_ctas > 65536) return WF_ERR_INVALID_ARG;
  if (d->dtype == WF_BF16 && d->head_dim != 128) return WF_ERR_UNSUPPORTED;
  if (d->dtype == WF_F32 && d->head_dim != 64 && d->head_dim != 128) return WF_ERR_UNSUPPORTED;

  const int64_t C = int64_t(d->frames_per_chunk) * d->frame_h * d->frame_w;
  if (C > (int64_t(1) << 24)) return WF_ERR_CAPACITY;
  const int64_t S = d->pool_slots ? d->pool_slots : int64_t(d->cache_chunks) + d->inround_chunks;
  if (d->pool_slots < 0 || S < int64_t(d->cache_chunks) + d->inround_chunks) return WF_ERR_INVALID_ARG;
  if (S * C >= (int64_t(1) << 31)) return WF_ERR_CAPACITY;
  if (S * C * d->num_heads * d->head_dim >= (int64_t(1) << 40)) return WF_ERR_CAPACITY;

  for (int i = 0; i < d->inround_chunks; ++i) {
    if (d->noise_t[i] < 0 || d->noise_t[i] > 1000) return WF_ERR_INVALID_ARG;
    // older in-round chunks are cleaner: an earlier chunk may not be noisier
    if (i > 0 && d->noise_t[i - 1] > d->noise_t[i]) return WF_ERR_INVALID_ARG;
  }
  int32_t Pt = d->rope_pairs_t, Ph = d->rope_pairs_h, Pw = d->rope_pairs_w;
  if (Pt == 0 && Ph == 0 && Pw == 0) {
    Ph = Pw = (d->head_dim / 2) / 3;
    Pt = d->head_dim / 2 - 2 * Ph;
  }
  if (Pt < 0 || Ph < 0 || Pw < 0 || Pt + Ph + Pw != d->head_dim / 2) return WF_ERR_INVALID_ARG;

  int32_t G = d->num_ctas;
  if (G == 0) {
    if (!query_device) return WF_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
      cudaGetLastError();
      return WF_ERR_CUDA;
    }
    G = sms;
  }

  g->H = d->num_heads; g->D = d->head_dim; g->fh = d->frame_h; g->fw = d->frame_w;
  g->F = d->frames_per_chunk; g->C = int32_t(C); g->Wc = d->cache_chunks;
  g->R = d->inround_chunks; g->S = int32_t(S); g->dtype = d->dtype;
  g->Pt = Pt; g->Ph = Ph; g->Pw = Pw; g->G = G; g->n0 = d->n0; g->theta = d->rope_theta;
  g->wc_eff = int32_t(std::min<int64_t>(d->cache_chunks, d->n0));
  g->first = d->n0 - g->wc_eff;
  g->q_pairs = int32_t(ceil_div(C, WF_Q_PAIR));
  g->q_tiles = int32_t(ceil_div(C, WF_Q_TILE));
  // Key split: when the round has fewer than two units per bin (a single
  // chunk), each unit's key tiles are shared out over `parts` units, the
  // count whose bin filling ceil(U*p/G) / (U*p/G) plus 1% per extra part is
  // smallest (ties: fewer parts), with at least WF_MIN_PART_TILES tiles per
  // part in the round's smallest chunk.  bf16 plans only.  With two or more
  // units per bin the longest-first assignment and its refinement balance
  // the bins without it.
  const int64_t pairs_all = int64_t(g->R) * g->H * g->q_pairs;
  {
    const int64_t nvis0 = g->wc_eff + 1;  // chunk 0 sees the fewest keys
    const int64_t s0 = g->first % S, len0 = std::min<int64_t>(nvis0, S - s0);
    const int64_t tiles0 = ceil_div(len0 * C, WF_KEY_TILE) + ceil_div((nvis0 - len0) * C, WF_KEY_TILE);
    int32_t best_p = 1;
    int64_t best_a = 0;
    for (int32_t p = 1; p <= WF_MAX_KEY_PARTS; ++p) {
      if (p > 1 && (d->dtype != WF_BF16 || pairs_all >= 2 * int64_t(G) ||
                    tiles0 < int64_t(WF_MIN_PART_TILES) * p))
        break;
      // score(p) = A_p / (100 U p) with A_p = 100 ceil(U p / G) G + (p - 1) U p
      const int64_t up = pairs_all * p;
      const int64_t a = 100 * ceil_div(up, G) * G + int64_t(p - 1) * up;
      if (p == 1 || a * best_p < best_a * p) {
        best_p = p;
        best_a = a;
      }
    }
    g->parts = best_p;
  }
  g->num_units = pairs_all * g->parts;
  if (g->num_units > (int64_t(1) << 26)) return WF_ERR_CAPACITY;

  uint64_t off = sizeof(wf_plan_hdr);
  off = align_up(off, 16); g->off_chunks = off; off += sizeof(wf_plan_chunk) * g->R;
  off = align_up(off, 16); g->off_vis = off; off += sizeof(int32_t) * g->R * (g->Wc + g->R);
  off = align_up(off, 16); g->off_rope_t = off; off += 16ull * g->R * g->F * Pt;
  off = align_up(off, 16); g->off_rope_h = off; off += 16ull * g->fh * Ph;
  off = align_up(off, 16); g->off_rope_w = off; off += 16ull * g->fw * Pw;
  off = align_up(off, 16); g->off_units = off; off += sizeof(wf_plan_unit) * g->num_units;
  off = align_up(off, 16); g->off_cta = off; off += sizeof(int32_t) * (uint64_t(G) + 1);
  g->total = align_up(off, 256);
  if (g->total > (uint64_t(1) << 31)) return WF_ERR_CAPACITY;
  return WF_OK;
}

void fill_rope(double* dst, int64_t npos, const int64_t* pos, int32_t P, double theta) {
  for (int64_t r = 0; r < npos; ++r) {
    for (int32_t k = 0; k < P; ++k) {
      const double freq = std::pow(theta, -double(k) / double(P));
      const double ang = double(pos[r]) * freq;
      dst[2 * (r * P + k)] = std::cos(ang);
      dst[2 * (r * P + k) + 1] = std::sin(ang);
    }
  }
}

// Work balancer.  Longest first: items ordered by cost (largest first,
// equal costs in their given order) each go to the least-loaded bin (lowest
// index on ties).  Refinement: with ~6 large units per bin the greedy start
// leaves the heaviest bin ~10% above the mean, so repeatedly move one item out
// of the heaviest bin h (lowest index on ties), or swap it for a lighter one,
// choosing the change that leaves the two bins' larger load smallest, from the
// lightest bin (lowest index on ties) that offers any change lowering L_h.
// Ties keep the first candidate in bin order, item order, move before swap;
// arriving items go to the end of their new bin.  Right after the greedy start
// no move can lower L_h (the last item placed in a bin is its smallest and was
// placed when that bin was the lightest), so moves only follow swaps.
void balance(const std::vector<int64_t>& cost, int32_t G, std::vector<std::vector<int32_t>>& bins) {
  const int32_t n = int32_t(cost.size());
  std::vector<int32_t> order(n);
  for (int32_t i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int32_t a, int32_t b) { return cost[a] > cost[b]; });
  using Bin = std::pair<int64_t, int32_t>;  // (load, index): min-heap pops lowest load, then index
  std::priority_queue<Bin, std::vector<Bin>, std::greater<Bin>> heap;
  for (int32_t c = 0; c < G; ++c) heap.push({0, c});
  bins.assign(size_t(G), {});
  std::vector<int64_t> load(G, 0);
  for (int32_t i : order) {
    const Bin b = heap.top();
    heap.pop();
    bins[b.second].push_back(i);
    load[b.second] += cost[i];
    heap.push({load[b.second], b.second});
  }
  std::vector<int32_t> by_load(G);
  for (int iter = 0; iter < 5000; ++iter) {
    int32_t h = 0;
    for (int32_t c = 1; c < G; ++c)
      if (load[c] > load[h]) h = c;
    for (int32_t c = 0; c < G; ++c) by_load[c] = c;
    std::stable_sort(by_load.begin(), by_load.end(), [&](int32_t a, int32_t b) { return load[a] < load[b]; });
    int64_t best = -1;
    int32_t best_b = -1, best_x = -1, best_y = -1;
    for (int32_t b : by_load) {
      if (b == h) continue;
      if (load[b] >= load[h]) break;
      for (int32_t xi = 0; xi < int32_t(bins[h].size()); ++xi) {
        const int64_t x = cost[bins[h][xi]];
        const int64_t mv = std::max(load[h] - x, load[b] + x);
        if (mv < load[h] && (best < 0 || mv < best)) {
          best = mv; best_b = b; best_x = xi; best_y = -1;
        }
        for (int32_t yi = 0; yi < int32_t(bins[b].size()); ++yi) {
          const int64_t d = x - cost[bins[b][yi]];
          if (d <= 0) continue;
          const int64_t sw = std::max(load[h] - d, load[b] + d);
          if (sw < load[h] && (best < 0 || sw < best)) {
            best = sw; best_b = b; best_x = xi; best_y = yi;
          }
        }
      }
      if (best >= 0) break;
    }
    if (best < 0) break;
    const int32_t x = bins[h][best_x];
    bins[h].erase(bins[h].begin() + best_x);
    load[h] -= cost[x];
    if (best_y >= 0) {
      const int32_t y = bins[best_b][best_y];
      bins[best_b].erase(bins[best_b].begin() + best_y);
      load[best_b] -= cost[y];
      bins[h].push_back(y);
      load[h] += cost[y];
    }
    bins[best_b].push_back(x);
    load[best_b] += cost[x];
  }
}

}  // namespace

extern "C" size_t wf_plan_bytes(const wf_round_desc* desc) {
  Geometry g;
  if (geometry(desc, &g, true) != WF_OK) return 0;
  return size_t(g.total);
}

extern "C" wf_status wf_plan_round(const wf_round_desc* desc, void* host_plan, size_t host_bytes,
                                   void* dev_plan, size_t dev_bytes, wf_stream_t stream) {
  Geometry g;
  wf_status st = geometry(desc, &g, true);
  if (st != WF_OK) return st;
  if (!host_plan) return WF_ERR_INVALID_ARG;
  if (host_bytes < g.total || (dev_plan && dev_bytes < g.total)) return WF_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(host_plan) % 16 || reinterpret_cast<uintptr_t>(dev_plan) % 16)
    return WF_ERR_ALIGNMENT;

  uint8_t* base = static_cast<uint8_t*>(host_plan);
  std::memset(base, 0, g.total);
  wf_plan_hdr* h = reinterpret_cast<wf_plan_hdr*>(base);
  h->magic = WF_PLAN_MAGIC; h->version = WF_PLAN_VERSION; h->total_bytes = g.total;
  h->H = g.H; h->D = g.D; h->fh = g.fh; h->fw = g.fw; h->F = g.F; h->C = g.C;
  h->Wc = g.Wc; h->wc_eff = g.wc_eff; h->R = g.R; h->S = g.S; h->dtype = g.dtype;
  h->Pt = g.Pt; h->Ph = g.Ph; h->Pw = g.Pw; h->num_ctas = g.G; h->num_units = int32_t(g.num_units);
  h->q_pairs = g.q_pairs; h->q_tiles = g.q_tiles; h->n0 = g.n0; h->first = g.first;
  h->theta = g.theta;
  h->off_chunks = g.off_chunks; h->off_vis = g.off_vis; h->off_rope_t = g.off_rope_t;
  h->off_rope_h = g.off_rope_h; h->off_rope_w = g.off_rope_w; h->off_units = g.off_units;
  h->off_cta = g.off_cta;
  for (int i = 0; i < g.R; ++i) h->noise_t[i] = desc->noise_t[i];

  // per-chunk visibility: consecutive chunks first .. n_i -> consecutive slots
  wf_plan_chunk* ch = reinterpret_cast<wf_plan_chunk*>(base + g.off_chunks);
  int32_t* vis = reinterpret_cast<int32_t*>(base + g.off_vis);
  int32_t max_tiles = 0, max_nvis = 0;
  for (int i = 0; i < g.R; ++i) {
    wf_plan_chunk& c = ch[i];
    c.n = g.n0 + i;
    c.slot = int32_t(c.n % g.S);
    c.noise = desc->noise_t[i];
    c.nvis = g.wc_eff + i + 1;
    c.keys = c.nvis * g.C;
    const int32_t s0 = int32_t(g.first % g.S);
    const int32_t len0 = std::min(c.nvis, g.S - s0);
    c.seg_start[0] = s0 * g.C; c.seg_len[0] = len0 * g.C;
    c.seg_start[1] = 0;        c.seg_len[1] = (c.nvis - len0) * g.C;
    c.seg_tiles[0] = int32_t(ceil_div(c.seg_len[0], WF_KEY_TILE));
    c.seg_tiles[1] = int32_t(ceil_div(c.seg_len[1], WF_KEY_TILE));
    c.key_tiles = c.seg_tiles[0] + c.seg_tiles[1];
    c.frame_base = i * g.F;
    int32_t* row = vis + int64_t(i) * (g.Wc + g.R);
    for (int k = 0; k < g.Wc + g.R; ++k)
      row[k] = k < c.nvis ? int32_t((g.first + k) % g.S) : -1;
    max_tiles = std::max(max_tiles, c.key_tiles);
    max_nvis = std::max(max_nvis, c.nvis);
  }
  h->max_key_tiles = max_tiles;
  h->max_nvis = max_nvis;

  // RoPE tables: time positions of the round's frames, then rows, then columns
  {
    std::vector<int64_t> pos(size_t(g.R) * g.F);
    for (int i = 0; i < g.R; ++i)
      for (int f = 0; f < g.F; ++f) pos[size_t(i) * g.F + f] = (g.n0 + i) * g.F + f;
    fill_rope(reinterpret_cast<double*>(base + g.off_rope_t), int64_t(pos.size()), pos.data(), g.Pt, g.theta);
    std::vector<int64_t> rows(g.fh), cols(g.fw);
    for (int r = 0; r < g.fh; ++r) rows[r] = r;
    for (int c = 0; c < g.fw; ++c) cols[c] = c;
    fill_rope(reinterpret_cast<double*>(base + g.off_rope_h), g.fh, rows.data(), g.Ph, g.theta);
    fill_rope(reinterpret_cast<double*>(base + g.off_rope_w), g.fw, cols.data(), g.Pw, g.theta);
  }

  // attention work list: longest first, then greedy to the least-loaded bin
  {
    std::vector<wf_plan_unit> units;
    units.reserve(size_t(g.num_units));
    for (int i = 0; i < g.R; ++i)
      for (int hh = 0; hh < g.H; ++hh)
        for (int p = 0; p < g.q_pairs; ++p) {
          const int32_t rows = std::min(WF_Q_PAIR, g.C - WF_Q_PAIR * p);
          const int32_t live = rows <= WF_Q_TILE ? 1 : 2;
          // A unit's time is set by its per-key-tile pipeline latency, which
          // a second live query tile only lengthens by about a tenth (its
          // softmax overlaps the first tile's MMAs): weight 11 for two live
          // tiles, 10 for one.
          const int32_t n = ch[i].key_tiles, P = g.parts;
          for (int32_t k = 0; k < P; ++k) {
            const int32_t tiles = (k + 1) * n / P - k * n / P;
            const int32_t slot = P > 1 ? ((i * g.H + hh) * g.q_pairs + p) * P + k : -1;
            units.push_back({i, hh, p, tiles * (9 + live), k, P, slot, 0});
          }
        }
    std::sort(units.begin(), units.end(), [](const wf_plan_unit& a, const wf_plan_unit& b) {
      if (a.cost != b.cost) return a.cost > b.cost;
      if (a.chunk != b.chunk) return a.chunk > b.chunk;
      if (a.head != b.head) return a.head < b.head;
      if (a.pair != b.pair) return a.pair < b.pair;
      return a.part < b.part;
    });
    std::vector<int64_t> cost(units.size());
    for (size_t u = 0; u < units.size(); ++u) cost[u] = units[u].cost;
    std::vector<std::vector<int32_t>> bins;
    balance(cost, g.G, bins);
    int32_t* cta = reinterpret_cast<int32_t*>(base + g.off_cta);
    wf_plan_unit* out = reinterpret_cast<wf_plan_unit*>(base + g.off_units);
    cta[0] = 0;
    for (int32_t c = 0; c < g.G; ++c) {
      cta[c + 1] = cta[c] + int32_t(bins[c].size());
      for (size_t k = 0; k < bins[c].size(); ++k) out[cta[c] + k] = units[size_t(bins[c][k])];
    }
  }

  if (dev_plan) {
    if (cudaMemcpyAsync(dev_plan, host_plan, g.total, cudaMemcpyHostToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
      cudaGetLastError();
      return WF_ERR_CUDA;
    }
  }
  return WF_OK;
}

extern "C" wf_status wf_balance_units(const int64_t* cost, int32_t n, int32_t bins, int32_t* bin_start,
                                      int32_t* items) {
  if (n < 0 || bins < 1 || bins > 65536 || n > (int32_t(1) << 26)) return WF_ERR_INVALID_ARG;
  if (!bin_start || (n > 0 && (!cost || !items))) return WF_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i)
    if (cost[i] < 0 || cost[i] > (int64_t(1) << 40)) return WF_ERR_INVALID_ARG;
  std::vector<int64_t> c(cost, cost + n);
  std::vector<std::vector<int32_t>> out;
  balance(c, bins, out);
  bin_start[0] = 0;
  for (int32_t b = 0; b < bins; ++b) {
    bin_start[b + 1] = bin_start[b] + int32_t(out[b].size());
    for (size_t k = 0; k < out[b].size(); ++k) items[bin_start[b] + int32_t(k)] = out[b][k];
  }
  return WF_OK;
}

extern "C" const char* wf_status_string(wf_status s) {
  switch (s) {
    case WF_OK: return "WF_OK";
    case WF_ERR_INVALID_ARG: return "WF_ERR_INVALID_ARG: invalid argument";
    case WF_ERR_UNSUPPORTED: return "WF_ERR_UNSUPPORTED: dtype/head_dim combination not built";
    case WF_ERR_ALIGNMENT: return "WF_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case WF_ERR_CAPACITY: return "WF_ERR_CAPACITY: sizes exceed supported limits";
    case WF_ERR_WORKSPACE: return "WF_ERR_WORKSPACE: buffer too small";
    case WF_ERR_CUDA: return "WF_ERR_CUDA: CUDA call or launch failed";
    case WF_ERR_DEVICE_TIMEOUT: return "WF_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
    case WF_ERR_PLAN: return "WF_ERR_PLAN: plan blob is not a valid wf plan";
  }
  return "WF_ERR_UNKNOWN";
}

extern "C" int32_t wf_version(void) { return 100; }
