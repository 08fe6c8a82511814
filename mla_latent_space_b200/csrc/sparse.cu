// Token-level sparse decode over the paged latent cache (the FlashMLA product
// page lists token-level sparse attention for decoding): query token (r, i)
// attends, with all its heads, to the cache rows at the positions listed in
// indices[r][i][0..topk); positions outside [0, t_r) are skipped and a
// position listed twice is two keys.
//
// This version composes two B200 kernels.  A gather kernel compacts each
// query token's valid rows, in list order, into its own run of scratch pages
// of the cache's own format (a plain HBM-bound copy: 16-byte loads and
// stores, many in flight per thread; for the FP8 cache the e4m3 latent part,
// the bf16 RoPE part and the per-token scale of each row).  The tcgen05 decode kernel then runs over the scratch pages as a
// dense batch of b*s single-query requests with an identity block table.
// The rows cross HBM three times (read, write, read back) where a fused
// producer would read them once.
#include <cuda_runtime.h>

#include "kernel_util.cuh"

namespace mla {

namespace {

constexpr int kGatherThreads = 256;        // index slots per CTA
// FP8 page: 64 x 512 e4m3 latent bytes, then 64 x 64 bf16 RoPE values
constexpr int kFp8LatBytes = MLA_PAGE_SIZE * MLA_D_V;
constexpr int kFp8PageBytes = kFp8LatBytes + MLA_PAGE_SIZE * MLA_D_ROPE * 2;

// 16-byte chunks per cache row: BF16 72 (1152 bytes); FP8 32 latent + 8 RoPE
template <bool kFp8>
constexpr int row_chunks() {
  return kFp8 ? (MLA_D_V + MLA_D_ROPE * 2) / 16 : MLA_D_QK * 2 / 16;
}

// Byte offset of 16-byte chunk `ch` of row `slot` of page `page`.
template <bool kFp8>
__device__ __forceinline__ size_t chunk_offset(uint32_t page, uint32_t slot, int ch) {
  if constexpr (kFp8) {
    return ch < MLA_D_V / 16 ? size_t(page) * kFp8PageBytes + slot * MLA_D_V + 16 * ch
                             : size_t(page) * kFp8PageBytes + kFp8LatBytes + slot * (MLA_D_ROPE * 2) +
                                   16 * (ch - MLA_D_V / 16);
  } else {
    return (size_t(page) * MLA_PAGE_SIZE + slot) * (2 * MLA_D_QK) + 16 * ch;
  }
}

// Is list entry j of request r usable: inside the request's tokens and on a
// valid page?  Sets *bad_page for a listed position whose page id is out of
// range (the entry is then skipped).
__device__ __forceinline__ bool usable(int j, int t, const int32_t* bt_row, int num_pages, bool* bad_page,
                                       int* page) {
  if (j < 0 || j >= t) return false;
  const int p = bt_row[j / MLA_PAGE_SIZE];
  if (p < 0 || p >= num_pages) {
    *bad_page = true;
    return false;
  }
  *page = p;
  return true;
}

// grid (b*s query tokens, ceil(topk / 256) chunks of the list), 256 threads.
template <bool kFp8>
__global__ void __launch_bounds__(kGatherThreads)
    sparse_gather_kernel(const int32_t* __restrict__ indices, int topk, const int32_t* __restrict__ seqlens,
                         int s_q, const int32_t* __restrict__ block_table, int max_pages, int num_pages,
                         const uint8_t* __restrict__ pool, const float* __restrict__ kv_scale,
                         uint8_t* __restrict__ scratch, float* __restrict__ vscale, int vpages,
                         int32_t* __restrict__ vseqlens, int32_t* __restrict__ vbt, void* status_ws) {
  constexpr int kRowChunks = row_chunks<kFp8>();
  __shared__ int warp_sum[kGatherThreads / 32];
  __shared__ int s_base, s_total;
  __shared__ uint32_t src_row[kGatherThreads];   // pool row (page * 64 + slot) of each compacted entry
  const int v = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = v / s_q;
  int t = seqlens[r];
  const int cap = max_pages * MLA_PAGE_SIZE;
  if (t < 0 || t > cap) {
    if (c == 0 && tid == 0) flag_status(status_ws, kStatusBadSeqlen);
    t = t < 0 ? 0 : cap;
  }
  const int32_t* list = indices + size_t(v) * topk;
  const int32_t* bt_row = block_table + size_t(r) * max_pages;
  bool bad = false;
  int page = 0;

  // usable entries before this chunk (c == 0 also counts the whole list for
  // the request's length)
  const int upto = c == 0 ? topk : c * kGatherThreads;
  int before = 0, total = 0;
  for (int k = tid; k < upto; k += kGatherThreads) {
    const bool u = usable(list[k], t, bt_row, num_pages, &bad, &page);
    if (k < c * kGatherThreads) before += u;
    total += u;
  }
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (lane == 0) warp_sum[warp] = before;
  __syncthreads();
  if (tid == 0) {
    int b = 0;
    for (int w = 0; w < kGatherThreads / 32; ++w) b += warp_sum[w];
    s_base = b;
  }
  __syncthreads();
  if (lane == 0) warp_sum[warp] = total;
  __syncthreads();
  if (tid == 0) {
    int b = 0;
    for (int w = 0; w < kGatherThreads / 32; ++w) b += warp_sum[w];
    s_total = b;
  }
  __syncthreads();
  const int base = s_base;

  // this chunk's entries: compact the usable ones in list order
  const int k = c * kGatherThreads + tid;
  int pg = 0;
  const bool u = k < topk && usable(list[k], t, bt_row, num_pages, &bad, &pg);
  const unsigned m = __ballot_sync(0xffffffffu, u);
  const int in_warp = __popc(m & ((1u << lane) - 1u));
  __syncthreads();
  if (lane == 0) warp_sum[warp] = __popc(m);
  __syncthreads();
  int pre = 0;
  for (int w = 0; w < warp; ++w) pre += warp_sum[w];
  const int local = pre + in_warp;
  if (u) src_row[local] = uint32_t(pg) * MLA_PAGE_SIZE + uint32_t(list[k] % MLA_PAGE_SIZE);
  int n = 0;
  for (int w = 0; w < kGatherThreads / 32; ++w) n += warp_sum[w];
  if (bad) flag_status(status_ws, kStatusBadPage);
  if (c == 0) {
    if (tid == 0) vseqlens[v] = s_total;
    for (int p = tid; p < vpages; p += kGatherThreads) vbt[size_t(v) * vpages + p] = v * vpages + p;
  }
  __syncthreads();

  // copy the n compacted rows (16-byte chunks spread over the CTA, eight
  // loads in flight per thread) to rows base .. base+n-1 of this query
  // token's scratch pages
  const uint32_t vrow0 = uint32_t(v) * uint32_t(vpages) * MLA_PAGE_SIZE + uint32_t(base);
  if constexpr (kFp8) {
    if (tid < n) {
      const uint32_t vr = vrow0 + uint32_t(tid);
      vscale[vr] = kv_scale[src_row[tid]];
    }
  }
  const int work = n * kRowChunks;
  for (int w0 = tid; w0 < work; w0 += 8 * kGatherThreads) {
    uint4 val[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int w = w0 + e * kGatherThreads;
      if (w < work) {
        const int row = w / kRowChunks, ch = w % kRowChunks;
        const uint32_t sr = src_row[row];
        val[e] = __ldg(reinterpret_cast<const uint4*>(
            pool + chunk_offset<kFp8>(sr / MLA_PAGE_SIZE, sr % MLA_PAGE_SIZE, ch)));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int w = w0 + e * kGatherThreads;
      if (w < work) {
        const int row = w / kRowChunks, ch = w % kRowChunks;
        const uint32_t vr = vrow0 + uint32_t(row);
        *reinterpret_cast<uint4*>(scratch + chunk_offset<kFp8>(vr / MLA_PAGE_SIZE, vr % MLA_PAGE_SIZE, ch)) = val[e];
      }
    }
  }
}

}  // namespace

cudaError_t launch_sparse_gather(const int32_t* indices, int topk, const int32_t* seqlens, int batch, int s_q,
                                 const int32_t* block_table, int max_pages, int num_pages, const void* pool,
                                 const float* kv_scale, void* scratch, float* vscale, int vpages, int32_t* vseqlens,
                                 int32_t* vbt, void* status_ws, bool fp8, cudaStream_t stream) {
  const dim3 grid(unsigned(batch * s_q), unsigned((topk + kGatherThreads - 1) / kGatherThreads));
  if (fp8)
    sparse_gather_kernel<true><<<grid, kGatherThreads, 0, stream>>>(
        indices, topk, seqlens, s_q, block_table, max_pages, num_pages, static_cast<const uint8_t*>(pool), kv_scale,
        static_cast<uint8_t*>(scratch), vscale, vpages, vseqlens, vbt, status_ws);
  else
    sparse_gather_kernel<false><<<grid, kGatherThreads, 0, stream>>>(
        indices, topk, seqlens, s_q, block_table, max_pages, num_pages, static_cast<const uint8_t*>(pool), nullptr,
        static_cast<uint8_t*>(scratch), nullptr, vpages, vseqlens, vbt, status_ws);
  return cudaGetLastError();
}

}  // namespace mla
