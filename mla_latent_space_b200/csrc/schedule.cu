// Split-KV scheduler (FlashMLA-2 newsletter page, "Architectural Analysis":
// sequence partitions are balanced across SMs so that a batch mixing short
// and very long requests has no straggler).
//
// The work of a decode step is a list of 128-row tiles (request r, row block
// qt), each walking ceil(visible/64) KV pages.  Costing every tile as
// pages + kPieceOverhead and laying the tiles end to end gives a line of
// total cost C; worker w takes the units whose cost position lies in
// [C*w/W, C*(w+1)/W).  A position inside a tile's overhead maps to the start
// of that tile, so no worker gets an empty piece of a tile.  A tile cut by k
// worker boundaries is computed in k+1 pieces whose partial results the
// combine kernel merges.  This replaces the pages' radix-sorted block
// scheduler with a prefix sum and binary searches: the same balance for a
// contiguous assignment, and every step is parallel.
//
// Cutting a tile costs its pieces' fp32 partials and the combine, so the
// scheduler first prices the whole-tile assignment (worker boundaries moved
// to tile starts, whole_tile_range) and keeps it when its longest worker is
// within kSplitOverhead of the even share: batches of similar lengths then
// run without partials, jagged ones are cut.
#include <cuda_runtime.h>

#include "kernel_util.cuh"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

MLA_HD int clamp_seqlen(int t, int max_pages, int32_t* flag) {
  int cap = max_pages * MLA_PAGE_SIZE;
  if (t < 0) { *flag |= kStatusBadSeqlen; return 0; }
  if (t > cap) { *flag |= kStatusBadSeqlen; return cap; }
  return t;
}

// (tile, page) where cost position x starts.
MLA_HD void map_position(const int32_t* tiles, int num_tiles, int64_t x, int* tile, int* page) {
  int T = last_le(tiles + T_PREFIX, kTileInts, num_tiles, x);
  int64_t pg = x - int64_t(tiles[size_t(T) * kTileInts + T_PREFIX]) - kPieceOverhead;
  *tile = T;
  *page = pg > 0 ? int(pg) : 0;
}

// First worker whose start key is >= key.
MLA_HD int first_worker_ge(const int32_t* workers, int W, int64_t key) {
  int lo = 0, hi = W;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    const int32_t* wm = workers + size_t(mid) * kWorkerInts;
    if (tp_key(wm[W_TILE_BEGIN], wm[W_PAGE_BEGIN]) < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

MLA_HD void fill_header(int32_t* hdr, const ShapeInfo& s, int W, int num_tiles) {
  for (int i = 0; i < kHeaderInts; ++i) hdr[i] = 0;
  hdr[H_MAGIC] = kSchedMagic;
  hdr[H_WORKERS] = W;
  hdr[H_TILES] = num_tiles;
  hdr[H_TILES_PER_REQ] = s.tiles_per_req;
  hdr[H_BATCH] = s.batch;
  hdr[H_SQ] = s.s_q;
  hdr[H_HEADS] = s.heads;
  hdr[H_CAUSAL] = s.causal;
  hdr[H_MAX_PAGES] = s.max_pages;
}

// Worker w's start position.  Only min(W, total) workers get work, so the
// start positions floor(total*w/W_eff) are strictly increasing and an
// interior page boundary is never shared by two workers; the remaining
// workers start (and end) at (num_tiles, 0).
MLA_HD void worker_start(const int32_t* tiles, int num_tiles, int64_t total, int w, int W,
                         int* tile, int* page) {
  const int64_t We = total < W ? total : W;
  if (w >= We) { *tile = num_tiles; *page = 0; return; }
  map_position(tiles, num_tiles, total * w / We, tile, page);
}

// ---- device scheduler ------------------------------------------------------
// One CTA.  The tile costs, their prefix and the worker start keys live in
// shared memory, so that the binary searches of the position mapping (a few
// dozen dependent lookups) never wait on global memory; only the results go
// out.  Schedules too large for shared memory take the same steps on the
// global copies (schedule_kernel_global).
constexpr int kSchedThreads = 256;
constexpr int kSchedWarps = kSchedThreads / 32;
constexpr size_t kSchedSmemMax = 200 * 1024;

// Block-wide exclusive scan of one int64 per thread (warp shuffles, then the
// warp totals); returns the block total.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* warp_tot, int64_t* excl) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int64_t u = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += u;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  int64_t base = 0, total = 0;
#pragma unroll
  for (int k = 0; k < kSchedWarps; ++k) {
    const int64_t t = warp_tot[k];
    base += k < warp ? t : 0;
    total += t;
  }
  *excl = base + inc - v;
  __syncthreads();   // warp_tot may be reused by the next scan
  return total;
}

// Block-wide maximum of one int64 per thread.
__device__ int64_t block_max(int64_t v, int64_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const int64_t u = __shfl_xor_sync(0xffffffffu, v, off);
    v = u > v ? u : v;
  }
  if (lane == 0) warp_tot[warp] = v;
  __syncthreads();
  int64_t m = 0;
#pragma unroll
  for (int k = 0; k < kSchedWarps; ++k) m = warp_tot[k] > m ? warp_tot[k] : m;
  __syncthreads();
  return m;
}

// First index in [0, W) whose key is >= key (keys non-decreasing).
__device__ __forceinline__ int first_key_ge(const int64_t* keys, int W, int64_t key) {
  int lo = 0, hi = W;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (keys[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Shared-memory layout: pages[num_tiles], prefix[num_tiles] (int32), then
// wkey[W] (int64, 8-byte aligned).
MLA_HD size_t sched_smem_bytes(int num_tiles, int W) {
  return ((size_t(num_tiles) * 8 + 7) & ~size_t(7)) + size_t(W) * 8;
}

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(const int32_t* __restrict__ seqlens, ShapeInfo s, int W, int32_t* __restrict__ sched) {
  // the decode kernel behind this one (a programmatic dependent) may start
  // its prologue now; it reads the schedule only after this grid completes
  ptx::griddep_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int64_t warp_tot[kSchedWarps];
  __shared__ int32_t flag_sh;
  const int tid = threadIdx.x;
  const int num_tiles = s.batch * s.tiles_per_req;
  int32_t* pages_sm = reinterpret_cast<int32_t*>(smem);
  int32_t* prefix_sm = pages_sm + num_tiles;
  int64_t* wkey = reinterpret_cast<int64_t*>(smem + ((size_t(num_tiles) * 8 + 7) & ~size_t(7)));
  int32_t* hdr = sched;
  int32_t* workers = sched + kHeaderInts;
  int32_t* tiles = workers + size_t(W) * kWorkerInts;
  if (tid == 0) flag_sh = 0;
  __syncthreads();

  // 1-2: tile pages, costs and their exclusive prefix (contiguous chunks)
  const int chunk = (num_tiles + kSchedThreads - 1) / kSchedThreads;
  const int t0 = min(num_tiles, tid * chunk), t1 = min(num_tiles, t0 + chunk);
  int32_t flag = 0;
  int64_t local = 0;
  for (int T = t0; T < t1; ++T) {
    const int r = T / s.tiles_per_req, qt = T % s.tiles_per_req;
    const int t = clamp_seqlen(seqlens[r], s.max_pages, &flag);
    const int pages = tile_pages(s, t, qt);
    pages_sm[T] = pages;
    local += tile_cost(pages);
  }
  if (flag) atomicOr(&flag_sh, flag);
  int64_t excl;
  const int64_t total = block_exclusive_scan(local, warp_tot, &excl);
  for (int T = t0; T < t1; ++T) {
    prefix_sm[T] = int32_t(excl);
    tiles[size_t(T) * kTileInts + T_PAGES] = pages_sm[T];
    tiles[size_t(T) * kTileInts + T_PREFIX] = int32_t(excl);
    excl += tile_cost(pages_sm[T]);
  }
  __syncthreads();

  // whole tiles or cut tiles: the whole-tile assignment's longest worker
  const int64_t We = total < W ? total : W;
  int64_t mw = 0;
  for (int w = tid; w < We; w += kSchedThreads) {
    int tb, te;
    whole_tile_range(prefix_sm, 1, num_tiles, total, We, w, &tb, &te);
    const int64_t c = prefix_at(prefix_sm, 1, num_tiles, total, te) - prefix_at(prefix_sm, 1, num_tiles, total, tb);
    mw = c > mw ? c : mw;
  }
  mw = block_max(mw, warp_tot);
  const bool whole = We > 0 && mw <= (total + We - 1) / We + kSplitOverhead;
  if (whole) {
    for (int w = tid; w < W; w += kSchedThreads) {
      int tb, te;
      whole_tile_range(prefix_sm, 1, num_tiles, total, We, w, &tb, &te);
      int32_t* wm = workers + size_t(w) * kWorkerInts;
      wm[W_TILE_BEGIN] = tb;
      wm[W_PAGE_BEGIN] = 0;
      wm[W_TILE_END] = te;
      wm[W_PAGE_END] = 0;
      for (int k = W_FIRST_SPLIT; k < kWorkerInts; ++k) wm[k] = 0;
    }
    for (int T = t0; T < t1; ++T) {
      tiles[size_t(T) * kTileInts + T_SPLITS] = pages_sm[T] > 0 ? 1 : 0;
      tiles[size_t(T) * kTileInts + T_SLOT_BASE] = 0;
    }
    if (tid == 0) {
      fill_header(hdr, s, W, num_tiles);
      hdr[H_TOTAL_COST] = int32_t(total);
      hdr[H_MAX_SLOTS] = 0;
      hdr[H_STATUS] = flag_sh;
    }
    return;
  }

  // 3: worker start positions (only min(W, total) workers get work)
  for (int w = tid; w < W; w += kSchedThreads) {
    int tile = num_tiles, page = 0;
    if (w < We) {
      const int64_t x = total * w / We;
      tile = last_le(prefix_sm, 1, num_tiles, x);
      const int64_t pg = x - int64_t(prefix_sm[tile]) - kPieceOverhead;
      page = pg > 0 ? int(pg) : 0;
    }
    wkey[w] = tp_key(tile, page);
  }
  __syncthreads();
  for (int w = tid; w < W; w += kSchedThreads) {
    const int64_t k0 = wkey[w];
    const int64_t k1 = w + 1 < W ? wkey[w + 1] : tp_key(num_tiles, 0);
    int32_t* wm = workers + size_t(w) * kWorkerInts;
    wm[W_TILE_BEGIN] = int32_t(k0 >> 32);
    wm[W_PAGE_BEGIN] = int32_t(uint32_t(k0));
    wm[W_TILE_END] = int32_t(k1 >> 32);
    wm[W_PAGE_END] = int32_t(uint32_t(k1));
    int first = 0;
    if (uint32_t(k0) > 0) first = w - first_key_ge(wkey, W, tp_key(int32_t(k0 >> 32), 1)) + 1;
    wm[W_FIRST_SPLIT] = first;
    for (int k = W_FIRST_SPLIT + 1; k < kWorkerInts; ++k) wm[k] = 0;
  }

  // 4-5: pieces per tile and the base of their partial slots
  int64_t slots = 0;
  for (int T = t0; T < t1; ++T) {
    int n = 0;
    if (pages_sm[T] > 0)
      n = 1 + first_key_ge(wkey, W, tp_key(T + 1, 0)) - first_key_ge(wkey, W, tp_key(T, 1));
    tiles[size_t(T) * kTileInts + T_SPLITS] = n;
    slots += n > 1 ? n : 0;
  }
  int64_t sexcl;
  const int64_t slot_total = block_exclusive_scan(slots, warp_tot, &sexcl);
  for (int T = t0; T < t1; ++T) {
    const int n = tiles[size_t(T) * kTileInts + T_SPLITS];
    tiles[size_t(T) * kTileInts + T_SLOT_BASE] = int32_t(sexcl);
    sexcl += n > 1 ? n : 0;
  }
  if (tid == 0) {
    fill_header(hdr, s, W, num_tiles);
    hdr[H_TOTAL_COST] = int32_t(total);
    hdr[H_MAX_SLOTS] = int32_t(slot_total);
    hdr[H_STATUS] = flag_sh;
  }
}

}  // namespace

// Sequential form of schedule_kernel (identical results): the host planner,
// and the device fallback for oversized schedules.
MLA_HD void plan_schedule_seq(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched) {
  const int num_tiles = s.batch * s.tiles_per_req;
  int32_t* hdr = sched;
  int32_t* workers = sched + kHeaderInts;
  int32_t* tiles = workers + size_t(W) * kWorkerInts;
  int32_t flag = 0;
  int64_t total = 0;
  for (int T = 0; T < num_tiles; ++T) {
    int r = T / s.tiles_per_req, qt = T % s.tiles_per_req;
    int t = clamp_seqlen(seqlens[r], s.max_pages, &flag);
    int pages = tile_pages(s, t, qt);
    tiles[size_t(T) * kTileInts + T_PAGES] = pages;
    tiles[size_t(T) * kTileInts + T_PREFIX] = int32_t(total);
    total += tile_cost(pages);
  }
  {
    const int64_t We = total < W ? total : W;
    const int32_t* prefix = tiles + T_PREFIX;
    int64_t mw = 0;
    for (int w = 0; w < We; ++w) {
      int tb, te;
      whole_tile_range(prefix, kTileInts, num_tiles, total, We, w, &tb, &te);
      const int64_t c = prefix_at(prefix, kTileInts, num_tiles, total, te) -
                        prefix_at(prefix, kTileInts, num_tiles, total, tb);
      mw = c > mw ? c : mw;
    }
    if (We > 0 && mw <= (total + We - 1) / We + kSplitOverhead) {
      for (int w = 0; w < W; ++w) {
        int tb, te;
        whole_tile_range(prefix, kTileInts, num_tiles, total, We, w, &tb, &te);
        int32_t* wm = workers + size_t(w) * kWorkerInts;
        wm[W_TILE_BEGIN] = tb;
        wm[W_PAGE_BEGIN] = 0;
        wm[W_TILE_END] = te;
        wm[W_PAGE_END] = 0;
        for (int k = W_FIRST_SPLIT; k < kWorkerInts; ++k) wm[k] = 0;
      }
      for (int T = 0; T < num_tiles; ++T) {
        tiles[size_t(T) * kTileInts + T_SPLITS] = tiles[size_t(T) * kTileInts + T_PAGES] > 0 ? 1 : 0;
        tiles[size_t(T) * kTileInts + T_SLOT_BASE] = 0;
      }
      fill_header(hdr, s, W, num_tiles);
      hdr[H_TOTAL_COST] = int32_t(total);
      hdr[H_MAX_SLOTS] = 0;
      hdr[H_STATUS] = flag;
      return;
    }
  }
  for (int w = 0; w < W; ++w) {
    int tile, page;
    worker_start(tiles, num_tiles, total, w, W, &tile, &page);
    int32_t* wm = workers + size_t(w) * kWorkerInts;
    wm[W_TILE_BEGIN] = tile;
    wm[W_PAGE_BEGIN] = page;
    for (int k = W_FIRST_SPLIT; k < kWorkerInts; ++k) wm[k] = 0;
  }
  for (int w = 0; w < W; ++w) {
    int32_t* wm = workers + size_t(w) * kWorkerInts;
    if (w + 1 < W) {
      wm[W_TILE_END] = workers[size_t(w + 1) * kWorkerInts + W_TILE_BEGIN];
      wm[W_PAGE_END] = workers[size_t(w + 1) * kWorkerInts + W_PAGE_BEGIN];
    } else {
      wm[W_TILE_END] = num_tiles;
      wm[W_PAGE_END] = 0;
    }
    if (wm[W_PAGE_BEGIN] > 0) {
      int lo = first_worker_ge(workers, W, tp_key(wm[W_TILE_BEGIN], 1));
      wm[W_FIRST_SPLIT] = w - lo + 1;
    }
  }
  int64_t slots = 0;
  for (int T = 0; T < num_tiles; ++T) {
    int32_t* tm = tiles + size_t(T) * kTileInts;
    int n = 0;
    if (tm[T_PAGES] > 0) {
      int lo = first_worker_ge(workers, W, tp_key(T, 1));
      int hi = first_worker_ge(workers, W, tp_key(T + 1, 0));
      n = 1 + (hi - lo);
    }
    tm[T_SPLITS] = n;
    tm[T_SLOT_BASE] = int32_t(slots);
    slots += n > 1 ? n : 0;
  }
  fill_header(hdr, s, W, num_tiles);
  hdr[H_TOTAL_COST] = int32_t(total);
  hdr[H_MAX_SLOTS] = int32_t(slots);
  hdr[H_STATUS] = flag;
}

void plan_schedule_host(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched) {
  plan_schedule_seq(seqlens, s, W, sched);
}

namespace {
// Schedules whose tables do not fit in shared memory: one thread runs the
// sequential planner on the global copies (slow, but only for batches of
// tens of thousands of tiles).
__global__ void schedule_kernel_global(const int32_t* seqlens, ShapeInfo s, int W, int32_t* sched) {
  ptx::griddep_launch_dependents();   // as in schedule_kernel
  if (threadIdx.x == 0 && blockIdx.x == 0) plan_schedule_seq(seqlens, s, W, sched);
}
}  // namespace

namespace {
// Whole-tile variant of schedule_kernel, for the no-allocation entry point:
// worker w starts at the first tile whose cost prefix is >= total*w/W_eff,
// so worker boundaries fall on tile starts, no tile is split and no partial
// slot is ever used.  Same schedule format (every split count is 1, or 0 for
// a tile with no visible key), so the decode and combine kernels run on it
// unchanged.  The balance is coarser than schedule_kernel's: a worker's share
// is rounded to whole tiles.  Invalid lengths are flagged in the schedule
// header and in *status.
__global__ void __launch_bounds__(kSchedThreads)
schedule_whole_tiles_kernel(const int32_t* __restrict__ seqlens, ShapeInfo s, int W, int32_t* __restrict__ sched,
                            int32_t* __restrict__ status) {
  ptx::griddep_launch_dependents();   // as in schedule_kernel
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int64_t warp_tot[kSchedWarps];
  __shared__ int32_t flag_sh;
  const int tid = threadIdx.x;
  const int num_tiles = s.batch * s.tiles_per_req;
  int32_t* pages_sm = reinterpret_cast<int32_t*>(smem);
  int32_t* prefix_sm = pages_sm + num_tiles;
  int32_t* hdr = sched;
  int32_t* workers = sched + kHeaderInts;
  int32_t* tiles = workers + size_t(W) * kWorkerInts;
  if (tid == 0) flag_sh = 0;
  __syncthreads();

  const int chunk = (num_tiles + kSchedThreads - 1) / kSchedThreads;
  const int t0 = min(num_tiles, tid * chunk), t1 = min(num_tiles, t0 + chunk);
  int32_t flag = 0;
  int64_t local = 0;
  for (int T = t0; T < t1; ++T) {
    const int r = T / s.tiles_per_req, qt = T % s.tiles_per_req;
    const int pages = tile_pages(s, clamp_seqlen(seqlens[r], s.max_pages, &flag), qt);
    pages_sm[T] = pages;
    local += tile_cost(pages);
  }
  if (flag) atomicOr(&flag_sh, flag);
  int64_t excl;
  const int64_t total = block_exclusive_scan(local, warp_tot, &excl);
  for (int T = t0; T < t1; ++T) {
    prefix_sm[T] = int32_t(excl);
    int32_t* tm = tiles + size_t(T) * kTileInts;
    tm[T_PAGES] = pages_sm[T];
    tm[T_PREFIX] = int32_t(excl);
    tm[T_SPLITS] = pages_sm[T] > 0 ? 1 : 0;
    tm[T_SLOT_BASE] = 0;
    excl += tile_cost(pages_sm[T]);
  }
  __syncthreads();

  const int64_t We = total < W ? total : W;
  for (int w = tid; w < W; w += kSchedThreads) {
    int32_t* wm = workers + size_t(w) * kWorkerInts;
    int tb = num_tiles, te = num_tiles;
    if (w < We) {
      // first tile with prefix >= x (prefix non-decreasing)
      const int64_t x = total * w / We, x1 = total * (w + 1) / We;
      tb = last_le(prefix_sm, 1, num_tiles, x - 1) + 1;
      te = w + 1 < We ? last_le(prefix_sm, 1, num_tiles, x1 - 1) + 1 : num_tiles;
    }
    wm[W_TILE_BEGIN] = tb;
    wm[W_PAGE_BEGIN] = 0;
    wm[W_TILE_END] = te;
    wm[W_PAGE_END] = 0;
    for (int k = W_FIRST_SPLIT; k < kWorkerInts; ++k) wm[k] = 0;
  }
  if (tid == 0) {
    fill_header(hdr, s, W, num_tiles);
    hdr[H_TOTAL_COST] = int32_t(total);
    hdr[H_MAX_SLOTS] = 0;
    hdr[H_STATUS] = flag_sh;
    if (flag_sh) atomicOr(status, flag_sh);
  }
}
}  // namespace

// Shared-memory bytes the whole-tile scheduler needs (0 when it cannot run).
size_t schedule_whole_tiles_smem(int num_tiles) {
  const size_t b = size_t(num_tiles) * 8;
  return b <= kSchedSmemMax ? b : 0;
}

cudaError_t launch_schedule_whole_tiles(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched,
                                        int32_t* status, cudaStream_t stream) {
  const size_t smem = schedule_whole_tiles_smem(s.batch * s.tiles_per_req);
  if (smem == 0 && s.batch * s.tiles_per_req > 0) return cudaErrorInvalidValue;   // over the shared-memory budget
  if (smem > 48 * 1024 &&
      !ensure_smem_attr(reinterpret_cast<const void*>(&schedule_whole_tiles_kernel), int(kSchedSmemMax)))
    return cudaErrorInvalidValue;
  schedule_whole_tiles_kernel<<<1, kSchedThreads, smem, stream>>>(seqlens, s, W, sched, status);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched,
                            cudaStream_t stream) {
  const size_t smem = sched_smem_bytes(s.batch * s.tiles_per_req, W);
  if (smem <= kSchedSmemMax) {
    if (smem > 48 * 1024 &&
        !ensure_smem_attr(reinterpret_cast<const void*>(&schedule_kernel), int(kSchedSmemMax)))
      return cudaErrorInvalidValue;
    schedule_kernel<<<1, kSchedThreads, smem, stream>>>(seqlens, s, W, sched);
  } else {
    schedule_kernel_global<<<1, 32, 0, stream>>>(seqlens, s, W, sched);
  }
  return cudaGetLastError();
}

}  // namespace mla
