// Device helpers shared by the decode and combine kernels: schedule walking,
// output / partial-slot addressing and element conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"

namespace mla {

// Raises a kernel's dynamic shared-memory limit on the CURRENT device, once
// per (kernel, device): the attribute is per device, so a process that
// launches on several GPUs sets it on each of them.  Returns false when the
// runtime refuses it.  Device ordinals at or above 64 are set on every call.
inline bool ensure_smem_attr(const void* fn, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  constexpr int kFns = 16;
  static std::mutex mu;
  static const void* fns[kFns] = {};
  static uint64_t done[kFns] = {};
  std::lock_guard<std::mutex> lock(mu);
  int i = 0;
  while (i < kFns && fns[i] != nullptr && fns[i] != fn) ++i;
  if (i < kFns && fns[i] == fn && dev < 64 && ((done[i] >> dev) & 1u)) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (i < kFns && dev < 64) {
    fns[i] = fn;
    done[i] |= uint64_t(1) << dev;
  }
  return true;
}

struct SchedView {
  const int32_t* hdr;
  const int32_t* workers;
  const int32_t* tiles;
  int W, num_tiles, tiles_per_req, batch, s_q, heads, causal, max_pages;

  __device__ __forceinline__ explicit SchedView(const void* p) {
    hdr = static_cast<const int32_t*>(p);
    W = hdr[H_WORKERS];
    num_tiles = hdr[H_TILES];
    tiles_per_req = hdr[H_TILES_PER_REQ];
    batch = hdr[H_BATCH];
    s_q = hdr[H_SQ];
    heads = hdr[H_HEADS];
    causal = hdr[H_CAUSAL];
    max_pages = hdr[H_MAX_PAGES];
    workers = hdr + kHeaderInts;
    tiles = workers + size_t(W) * kWorkerInts;
  }
  __device__ __forceinline__ int tile_pages(int T) const { return tiles[size_t(T) * kTileInts + T_PAGES]; }
  __device__ __forceinline__ int tile_splits(int T) const { return tiles[size_t(T) * kTileInts + T_SPLITS]; }
  __device__ __forceinline__ int tile_slot_base(int T) const { return tiles[size_t(T) * kTileInts + T_SLOT_BASE]; }
};

// One piece of a worker's range: pages [p0, p1) of tile T, split index `split`.
struct Piece {
  int T, p0, p1, split;
};

// Iterates the pieces of worker w in order.  Usage:
//   PieceIter it(sv, w); Piece pc; while (it.next(&pc)) {...}
struct PieceIter {
  const SchedView& sv;
  int tb, pb, te, pe, fs, T;
  __device__ __forceinline__ PieceIter(const SchedView& s, int w) : sv(s) {
    const int32_t* wm = s.workers + size_t(w) * kWorkerInts;
    tb = wm[W_TILE_BEGIN]; pb = wm[W_PAGE_BEGIN];
    te = wm[W_TILE_END]; pe = wm[W_PAGE_END]; fs = wm[W_FIRST_SPLIT];
    T = tb;
  }
  __device__ __forceinline__ bool next(Piece* pc) {
    while (T <= te && T < sv.num_tiles) {
      int pages = sv.tile_pages(T);
      int p0 = T == tb ? pb : 0;
      int p1 = T == te ? pe : pages;
      if (p1 > pages) p1 = pages;
      int split = T == tb ? fs : 0;
      int cur = T++;
      if (p0 < p1) { *pc = Piece{cur, p0, p1, split}; return true; }
    }
    return false;
  }
};

// Partial-slot regions are laid out for `cap` slots, the capacity the host
// derives from the workspace size (so decode and combine agree on it).
__device__ __forceinline__ float* ws_partial_o(void* ws, int cap, int slot) {
  (void)cap;
  return reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes) + size_t(slot) * kSlotOFloats;
}
__device__ __forceinline__ float* ws_partial_lse(void* ws, int cap, int slot) {
  return reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes) + size_t(cap) * kSlotOFloats +
         size_t(slot) * MLA_TILE_ROWS;
}
__device__ __forceinline__ int32_t* ws_status(void* ws) { return static_cast<int32_t*>(ws); }

__device__ __forceinline__ void flag_status(void* ws, int32_t bits) { atomicOr(ws_status(ws), bits); }

__device__ __forceinline__ float e4m3_to_float(uint8_t b) {
  __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(b), __NV_E4M3);
  return __half2float(__half(hr));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

}  // namespace mla
