// Internal definitions shared by the kernels and the host side of
// libmla_b200.so: schedule / workspace layouts and the scheduler's
// position arithmetic (compiled for both host and device so the host
// planner and the device scheduler are the same code).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/mla.h"

#define MLA_HD __host__ __device__ __forceinline__

namespace mla {

// ---------------------------------------------------------------------------
// schedule buffer (int32 words)
//   header[kHeaderInts]
//   worker[num_workers][kWorkerInts] : tile_begin, page_begin, tile_end,
//                                      page_end, first_split, 0, 0, 0
//   tile[num_tiles][kTileInts]       : n_pages, cost_prefix, n_splits, slot_base
// A worker covers the (tile, page) units from (tile_begin, page_begin) up to
// but excluding (tile_end, page_end) in lexicographic order.
// ---------------------------------------------------------------------------
constexpr int kHeaderInts = 16;
constexpr int kWorkerInts = 8;
constexpr int kTileInts = 4;
constexpr int32_t kSchedMagic = 0x4d4c4131;  // "MLA1"
// Cost of one piece beyond its pages, in page units: loading the 128x576
// query tile and writing the 128x512 result cost about as much as two pages.
constexpr int kPieceOverhead = 2;

enum HeaderField {
  H_MAGIC = 0, H_WORKERS, H_TILES, H_TILES_PER_REQ, H_TOTAL_COST, H_MAX_SLOTS, H_STATUS,
  H_BATCH, H_SQ, H_HEADS, H_CAUSAL, H_MAX_PAGES
};
enum WorkerField { W_TILE_BEGIN = 0, W_PAGE_BEGIN, W_TILE_END, W_PAGE_END, W_FIRST_SPLIT };
enum TileField { T_PAGES = 0, T_PREFIX, T_SPLITS, T_SLOT_BASE };

// device status bits (sticky)
constexpr int32_t kStatusTimeout = 1;
constexpr int32_t kStatusBadSeqlen = 2;
constexpr int32_t kStatusBadPage = 4;
constexpr int32_t kStatusWorkspace = 8;
constexpr int32_t kStatusBadInput = 16;   // a cache value the decode cannot represent (V outside fp16)

// ---------------------------------------------------------------------------
// workspace: [256 B status][max_slots x 128 x 512 fp32 O][max_slots x 128 fp32 lse]
// ---------------------------------------------------------------------------
constexpr size_t kStatusBytes = 256;
constexpr size_t kSlotOFloats = size_t(MLA_TILE_ROWS) * MLA_D_V;

MLA_HD int num_workers_for(int num_sms) { return num_sms >= 2 ? num_sms / 2 : 1; }
MLA_HD int max_slots_for(int workers) { return 2 * workers; }
constexpr size_t kSlotBytes = kSlotOFloats * 4 + MLA_TILE_ROWS * 4;   // O + lse of one slot

MLA_HD int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct ShapeInfo {
  int batch, s_q, heads, causal, max_pages, tiles_per_req;
};

// Keys visible to query token i of a request holding t cached tokens.
MLA_HD int visible_len(int t, int s_q, int i, int causal) {
  int L = causal ? t - s_q + i + 1 : t;
  return L < 0 ? 0 : L;
}

// Pages a tile must walk: the largest visible length among its rows
// (rows are (query token, head) pairs, row = i*h + head).
MLA_HD int tile_pages(const ShapeInfo& s, int t, int qt) {
  int rows = s.s_q * s.heads;
  int last = qt * MLA_TILE_ROWS + MLA_TILE_ROWS;
  if (last > rows) last = rows;
  int i_last = (last - 1) / s.heads;
  int L = visible_len(t, s.s_q, i_last, s.causal);
  return (L + MLA_PAGE_SIZE - 1) / MLA_PAGE_SIZE;
}

MLA_HD int tile_cost(int pages) { return pages > 0 ? pages + kPieceOverhead : 0; }
// Last index i in [0, n) with a[i*stride] <= x (a non-decreasing); -1 if none.
MLA_HD int last_le(const int32_t* a, int stride, int n, int64_t x) {
  int lo = 0, hi = n;  // answer in [lo-1, hi-1]
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (int64_t(a[size_t(mid) * stride]) <= x) lo = mid + 1; else hi = mid;
  }
  return lo - 1;
}

// Lexicographic (tile, page) key.
MLA_HD int64_t tp_key(int tile, int page) { return (int64_t(tile) << 32) | uint32_t(page); }

// Extra cost, in page units, of a tile finished through fp32 partials: its
// pieces' 128x512 fp32 writes and reads and the combine launch.  The
// scheduler cuts tiles only when the whole-tile assignment's longest worker
// exceeds the even share by more than this.  (Measured on B200: 64 equal
// 64-page tiles over 74 SM pairs run faster whole, 1 tile per worker, than
// cut to the even share of 57 units.)
constexpr int kSplitOverhead = 12;

// Whole-tile assignment: worker w of We takes the tiles whose cost prefix
// lies in [total*w/We, total*(w+1)/We).  prefix[T*stride] is tile T's
// exclusive cost prefix (non-decreasing); the range is [*tb, *te).
MLA_HD void whole_tile_range(const int32_t* prefix, int stride, int num_tiles, int64_t total, int64_t We, int w,
                             int* tb, int* te) {
  if (w >= We) { *tb = *te = num_tiles; return; }
  const int64_t x0 = total * w / We, x1 = total * (w + 1) / We;
  *tb = last_le(prefix, stride, num_tiles, x0 - 1) + 1;
  *te = w + 1 < We ? last_le(prefix, stride, num_tiles, x1 - 1) + 1 : num_tiles;
}

MLA_HD int64_t prefix_at(const int32_t* prefix, int stride, int num_tiles, int64_t total, int T) {
  return T < num_tiles ? int64_t(prefix[size_t(T) * stride]) : total;
}

}  // namespace mla
