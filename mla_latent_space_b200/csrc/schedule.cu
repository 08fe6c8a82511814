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
#include <cuda_runtime.h>

#include "common.cuh"

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

constexpr int kSchedThreads = 1024;

// Block-wide exclusive scan of one int64 per thread; returns the total.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* buf, int64_t* excl) {
  int tid = threadIdx.x;
  buf[tid] = v;
  __syncthreads();
  for (int off = 1; off < kSchedThreads; off <<= 1) {
    int64_t add = tid >= off ? buf[tid - off] : 0;
    __syncthreads();
    buf[tid] += add;
    __syncthreads();
  }
  *excl = buf[tid] - v;
  int64_t total = buf[kSchedThreads - 1];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(const int32_t* __restrict__ seqlens, ShapeInfo s, int W, int32_t* __restrict__ sched) {
  __shared__ int64_t buf[kSchedThreads];
  __shared__ int32_t flag_sh;
  int tid = threadIdx.x;
  const int num_tiles = s.batch * s.tiles_per_req;
  int32_t* hdr = sched;
  int32_t* workers = sched + kHeaderInts;
  int32_t* tiles = workers + size_t(W) * kWorkerInts;
  if (tid == 0) flag_sh = 0;
  __syncthreads();

  // 1-2: tile pages, costs and their exclusive prefix
  const int chunk = (num_tiles + kSchedThreads - 1) / kSchedThreads;
  const int t0 = tid * chunk, t1 = min(num_tiles, t0 + chunk);
  int32_t flag = 0;
  int64_t local = 0;
  for (int T = t0; T < t1; ++T) {
    int r = T / s.tiles_per_req, qt = T % s.tiles_per_req;
    int t = clamp_seqlen(seqlens[r], s.max_pages, &flag);
    int pages = tile_pages(s, t, qt);
    tiles[size_t(T) * kTileInts + T_PAGES] = pages;
    local += tile_cost(pages);
  }
  if (flag) atomicOr(&flag_sh, flag);
  int64_t excl;
  const int64_t total = block_exclusive_scan(local, buf, &excl);
  for (int T = t0; T < t1; ++T) {
    tiles[size_t(T) * kTileInts + T_PREFIX] = int32_t(excl);
    excl += tile_cost(tiles[size_t(T) * kTileInts + T_PAGES]);
  }
  __syncthreads();

  // 3: worker start positions (end = next worker's start)
  for (int w = tid; w < W; w += kSchedThreads) {
    int tile, page;
    worker_start(tiles, num_tiles, total, w, W, &tile, &page);
    int32_t* wm = workers + size_t(w) * kWorkerInts;
    wm[W_TILE_BEGIN] = tile;
    wm[W_PAGE_BEGIN] = page;
    for (int k = W_FIRST_SPLIT; k < kWorkerInts; ++k) wm[k] = 0;
  }
  __syncthreads();
  for (int w = tid; w < W; w += kSchedThreads) {
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

  // 4-5: pieces per tile and the base of their partial slots
  int64_t slots = 0;
  for (int T = t0; T < t1; ++T) {
    int32_t* tm = tiles + size_t(T) * kTileInts;
    int n = 0;
    if (tm[T_PAGES] > 0) {
      int lo = first_worker_ge(workers, W, tp_key(T, 1));
      int hi = first_worker_ge(workers, W, tp_key(T + 1, 0));
      n = 1 + (hi - lo);
    }
    tm[T_SPLITS] = n;
    slots += n > 1 ? n : 0;
  }
  int64_t sexcl;
  const int64_t slot_total = block_exclusive_scan(slots, buf, &sexcl);
  for (int T = t0; T < t1; ++T) {
    int32_t* tm = tiles + size_t(T) * kTileInts;
    tm[T_SLOT_BASE] = int32_t(sexcl);
    sexcl += tm[T_SPLITS] > 1 ? tm[T_SPLITS] : 0;
  }
  if (tid == 0) {
    fill_header(hdr, s, W, num_tiles);
    hdr[H_TOTAL_COST] = int32_t(total);
    hdr[H_MAX_SLOTS] = int32_t(slot_total);
    hdr[H_STATUS] = flag_sh;
  }
}

}  // namespace

// Sequential host copy of schedule_kernel (identical results).
void plan_schedule_host(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched) {
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

cudaError_t launch_schedule(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched,
                            cudaStream_t stream) {
  schedule_kernel<<<1, kSchedThreads, 0, stream>>>(seqlens, s, W, sched);
  return cudaGetLastError();
}

}  // namespace mla
