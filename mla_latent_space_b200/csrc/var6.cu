// MLAvar6+ split attention for speculative steps ("MLA Cost Analysis &
// Regime Guide", section "MLAvar6+ Design"): each request's o = t - n older
// tokens stay in latent form, its n newest are held as decompressed per-head
// keys (d = 128, plus the RoPE part of their cache rows) and values.  One
// softmax covers both.  Because softmax attention over a union of keys is
// the log-sum-exp merge of the attentions over the parts, the step runs as:
//
//   1. old lengths t - n (var6_old_len_kernel);
//   2. the latent decode over the old tokens (schedule, tcgen05 decode,
//      combine) and the output decompression of its result (the projection
//      kernel), giving O_old [b, s, h, d] and lse_old.  Both intermediates
//      travel as two bf16 terms (hi + lo, fp32-accurate), so the step adds
//      no rounding of its own to the decode's;
//   3. var6_new_kernel: attention of each (request, head)'s s query rows
//      over its n decompressed tokens, merged with (O_old, lse_old).
//
// With n >= s every old token is visible to every query row of a causal
// step, so the latent part needs no mask; the causal mask falls on the new
// tokens only.  Step 3 reads n * h * (2d + p) values per request against
// 2 (d + p) FLOPs each per query row: bandwidth-bound at decode sizes, so it
// is a plain SIMT kernel (one CTA per (request, head), one warp per query
// row, online softmax over 32-token chunks staged in shared memory).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "kernel_util.cuh"

namespace mla {

namespace {

constexpr int kVarThreads = 128;
constexpr int kVarWarps = kVarThreads / 32;
constexpr int kMaxRowsPerWarp = 8;               // s_q <= 32 (query rows per warp, at most)
constexpr int kChunk = 32;                       // new tokens per stage

__global__ void var6_old_len_kernel(const int32_t* __restrict__ seqlens, int batch, int n_new, int cap,
                                    int32_t* __restrict__ old_len) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < batch) {
    int t = seqlens[r];
    t = t < 0 ? 0 : (t > cap ? cap : t);
    old_len[r] = t > n_new ? t - n_new : 0;
  }
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// grid (batch, heads), 128 threads.  RPW: query rows per warp, the
// smallest power of two >= ceil(s_q / 4), so that no row loop issues work
// for rows that do not exist.
template <bool kFp8, int RPW>
__global__ void __launch_bounds__(kVarThreads, 4)
    var6_new_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k_new,
                    const uint16_t* __restrict__ v_new, const uint8_t* __restrict__ pool,
                    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens,
                    const uint16_t* __restrict__ o_old, const uint16_t* __restrict__ o_old_lo,
                    const float* __restrict__ lse_old, int s_q, int heads,
                    int n_new, int max_pages, int num_pages, int causal, float scale, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, void* status_ws) {
  constexpr int kQ = MLA_D_HEAD + MLA_D_ROPE;   // 192
  __shared__ float qs[32][kQ];                         // the request's query rows of this head
  __shared__ uint32_t ks[kChunk][kQ / 2 + 1];          // keys [k_new | RoPE part] as bf16 pairs, padded
  __shared__ __align__(16) uint32_t vs[kChunk][MLA_D_HEAD / 2];   // values as bf16 pairs
  __shared__ int pos_s[kChunk];                        // token positions; -1 if absent
  const int r = blockIdx.x, hd = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cap = max_pages * MLA_PAGE_SIZE;
  int t = seqlens[r];
  t = t < 0 ? 0 : (t > cap ? cap : t);

  // query rows of this (request, head): s_q x 192, as 16-byte pieces (24
  // per row), every load of a thread issued before its stores
  {
    constexpr int kPer = 32 * (kQ / 8) / kVarThreads;   // 6
    uint4 w[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + kVarThreads * u, i = e / (kQ / 8), c = e % (kQ / 8);
      if (i < s_q) w[u] = *reinterpret_cast<const uint4*>(q + ((size_t(r) * s_q + i) * heads + hd) * kQ + 8 * c);
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + kVarThreads * u, i = e / (kQ / 8), c = e % (kQ / 8);
      if (i < s_q) {
        float* d = &qs[i][8 * c];
        d[0] = bf16_lo(w[u].x); d[1] = bf16_hi(w[u].x); d[2] = bf16_lo(w[u].y); d[3] = bf16_hi(w[u].y);
        d[4] = bf16_lo(w[u].z); d[5] = bf16_hi(w[u].z); d[6] = bf16_lo(w[u].w); d[7] = bf16_hi(w[u].w);
      }
    }
  }

  float m_run[RPW], l_run[RPW], acc[RPW][4];
#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    m_run[k] = -INFINITY;
    l_run[k] = 0.f;
    acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;
  }
  bool bad_page = false;
  const float scale_log2 = scale * 1.4426950408889634f;

  for (int m0 = 0; m0 < n_new; m0 += kChunk) {
    __syncthreads();   // the previous chunk has been used; (first pass) the query rows are in
    // positions and the RoPE parts of this chunk's tokens
    if (tid < kChunk) {
      const int m = m0 + tid;
      int p = m < n_new ? t - n_new + m : -1;
      if (p >= 0) {
        const int pg = block_table[size_t(r) * max_pages + p / MLA_PAGE_SIZE];
        if (pg < 0 || pg >= num_pages) {
          bad_page = true;
          p = -1;
        }
      }
      pos_s[tid] = p;
    }
    __syncthreads();
    // keys and values: 16-byte pieces (40 per token), zeros for absent
    // tokens; every load of a thread issued before its stores
    constexpr int kPieces = MLA_D_HEAD / 8 * 2 + MLA_D_ROPE / 8;   // 40
    constexpr int kPer = kChunk * kPieces / kVarThreads;           // 10
    uint4 wv[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + kVarThreads * u;
      const int tok = e / kPieces, c = e % kPieces;
      const int p = pos_s[tok];
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (p >= 0) {
        const int m = m0 + tok;
        if (c < MLA_D_HEAD / 8) {
          w = *reinterpret_cast<const uint4*>(k_new + ((size_t(r) * n_new + m) * heads + hd) * MLA_D_HEAD + 8 * c);
        } else if (c < MLA_D_HEAD / 4) {
          w = *reinterpret_cast<const uint4*>(v_new + ((size_t(r) * n_new + m) * heads + hd) * MLA_D_HEAD +
                                              8 * (c - MLA_D_HEAD / 8));
        } else {
          const int pg = block_table[size_t(r) * max_pages + p / MLA_PAGE_SIZE], slot = p % MLA_PAGE_SIZE;
          const uint8_t* rope = kFp8 ? pool + size_t(pg) * (MLA_PAGE_SIZE * (MLA_D_V + 2 * MLA_D_ROPE)) +
                                           MLA_PAGE_SIZE * MLA_D_V + slot * (2 * MLA_D_ROPE)
                                     : pool + (size_t(pg) * MLA_PAGE_SIZE + slot) * (2 * MLA_D_QK) + 2 * MLA_D_V;
          w = *reinterpret_cast<const uint4*>(rope + 16 * (c - MLA_D_HEAD / 4));
        }
      }
      wv[u] = w;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + kVarThreads * u;
      const int tok = e / kPieces, c = e % kPieces;
      const uint4 w = wv[u];
      if (c < MLA_D_HEAD / 8) {
        uint32_t* dst = &ks[tok][4 * c];
        dst[0] = w.x; dst[1] = w.y; dst[2] = w.z; dst[3] = w.w;
      } else if (c < MLA_D_HEAD / 4) {
        *reinterpret_cast<uint4*>(&vs[tok][4 * (c - MLA_D_HEAD / 8)]) = w;
      } else {
        uint32_t* dst = &ks[tok][MLA_D_HEAD / 2 + 4 * (c - MLA_D_HEAD / 4)];
        dst[0] = w.x; dst[1] = w.y; dst[2] = w.z; dst[3] = w.w;
      }
    }
    __syncthreads();
    // lane = token of the chunk; warp = query rows warp, warp + 4, ...:
    // every key word read from shared memory serves all of the warp's rows
    const int p = pos_s[lane];
    const int nrows = s_q > warp ? (s_q - warp + kVarWarps - 1) / kVarWarps : 0;
    float xs[RPW];
#pragma unroll
    for (int k = 0; k < RPW; ++k) xs[k] = 0.f;
#pragma unroll 4
    for (int c = 0; c < kQ / 2; ++c) {
      const uint32_t kw = ks[lane][c];
      const float k0 = bf16_lo(kw), k1 = bf16_hi(kw);
#pragma unroll
      for (int k = 0; k < RPW; ++k)
        if (k < nrows) {
          const float2 qv = *reinterpret_cast<const float2*>(&qs[warp + kVarWarps * k][2 * c]);
          xs[k] = fmaf(qv.x, k0, fmaf(qv.y, k1, xs[k]));
        }
    }
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int i = warp + kVarWarps * k;
      if (i >= s_q) break;
      const int vis = causal ? t - s_q + i + 1 : t;
      float x = xs[k];
      const bool ok = p >= 0 && p < vis;
      x = ok ? x * scale_log2 : -INFINITY;
      float mx = x;
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_run[k], mx);
      if (m_new == -INFINITY) continue;   // nothing visible yet in this row
      const float alpha = exp2f(m_run[k] - m_new);
      const float pr = ok ? exp2f(x - m_new) : 0.f;
      float ps = pr;
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l_run[k] = l_run[k] * alpha + ps;
      m_run[k] = m_new;
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[k][c] *= alpha;
      for (int j = 0; j < kChunk; ++j) {
        const float pj = __shfl_sync(0xffffffffu, pr, j);
        const uint2 v2 = *reinterpret_cast<const uint2*>(&vs[j][2 * lane]);
        acc[k][0] = fmaf(pj, bf16_lo(v2.x), acc[k][0]);
        acc[k][1] = fmaf(pj, bf16_hi(v2.x), acc[k][1]);
        acc[k][2] = fmaf(pj, bf16_lo(v2.y), acc[k][2]);
        acc[k][3] = fmaf(pj, bf16_hi(v2.y), acc[k][3]);
      }
    }
  }
  if (bad_page) flag_status(status_ws, kStatusBadPage);

  // merge with the old tokens' result: L = ln(e^lse_old + e^lse_new)
#pragma unroll
  for (int k = 0; k < RPW; ++k) {
    const int i = warp + kVarWarps * k;
    if (i >= s_q) break;
    const size_t row = (size_t(r) * s_q + i) * heads + hd;
    const float lo = lse_old[row];
    const float ln = l_run[k] > 0.f ? m_run[k] / 1.4426950408889634f + logf(l_run[k]) : -INFINITY;
    const float mm = fmaxf(lo, ln);
    float L = -INFINITY, wo = 0.f, wn = 0.f;
    if (mm > -INFINITY) {
      const float so = expf(lo - mm), sn = expf(ln - mm);
      L = mm + logf(so + sn);
      wo = so / (so + sn);
      wn = sn / (so + sn);
    }
    // the old part arrives as two bf16 terms, hi + lo (fp32-accurate)
    const uint2 ob = *reinterpret_cast<const uint2*>(o_old + row * MLA_D_HEAD + 4 * lane);
    const uint2 ol = *reinterpret_cast<const uint2*>(o_old_lo + row * MLA_D_HEAD + 4 * lane);
    const float inv = l_run[k] > 0.f ? 1.f / l_run[k] : 0.f;
    const float a0 = bf16_lo(ob.x) + bf16_lo(ol.x), a1 = bf16_hi(ob.x) + bf16_hi(ol.x);
    const float a2 = bf16_lo(ob.y) + bf16_lo(ol.y), a3 = bf16_hi(ob.y) + bf16_hi(ol.y);
    const float o0 = wo * a0 + wn * acc[k][0] * inv, o1 = wo * a1 + wn * acc[k][1] * inv;
    const float o2 = wo * a2 + wn * acc[k][2] * inv, o3 = wo * a3 + wn * acc[k][3] * inv;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + row * MLA_D_HEAD + 4 * lane);
    dst[0] = __floats2bfloat162_rn(o0, o1);
    dst[1] = __floats2bfloat162_rn(o2, o3);
    if (lane == 0) lse[row] = L;
  }
}

}  // namespace

cudaError_t launch_var6_old_len(const int32_t* seqlens, int batch, int n_new, int max_pages, int32_t* old_len,
                                cudaStream_t stream) {
  var6_old_len_kernel<<<(batch + 127) / 128, 128, 0, stream>>>(seqlens, batch, n_new, max_pages * MLA_PAGE_SIZE,
                                                               old_len);
  return cudaGetLastError();
}

cudaError_t launch_var6_new(const void* q, const void* k_new, const void* v_new, const void* pool, bool fp8,
                            const int32_t* block_table, const int32_t* seqlens, const void* o_old,
                            const void* o_old_lo, const float* lse_old, int batch, int s_q, int heads, int n_new,
                            int max_pages, int num_pages, int causal, float scale, void* out, float* lse,
                            void* status_ws, cudaStream_t stream) {
  const dim3 grid = dim3(unsigned(batch), unsigned(heads), 1u);
  const uint16_t* qq = static_cast<const uint16_t*>(q);
  const uint16_t* kk = static_cast<const uint16_t*>(k_new);
  const uint16_t* vv = static_cast<const uint16_t*>(v_new);
  const uint8_t* pp = static_cast<const uint8_t*>(pool);
  const uint16_t* oo = static_cast<const uint16_t*>(o_old);
  const uint16_t* ool = static_cast<const uint16_t*>(o_old_lo);
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out);
  auto go = [&](auto fp8_tag, auto rpw_tag) {
    var6_new_kernel<decltype(fp8_tag)::value, decltype(rpw_tag)::value><<<grid, kVarThreads, 0, stream>>>(
        qq, kk, vv, pp, block_table, seqlens, oo, ool, lse_old, s_q, heads, n_new, max_pages, num_pages, causal,
        scale, dst, lse, status_ws);
  };
  auto by_rows = [&](auto fp8_tag) {
    const int rpw = (s_q + kVarWarps - 1) / kVarWarps;
    if (rpw <= 1) go(fp8_tag, std::integral_constant<int, 1>{});
    else if (rpw <= 2) go(fp8_tag, std::integral_constant<int, 2>{});
    else if (rpw <= 4) go(fp8_tag, std::integral_constant<int, 4>{});
    else go(fp8_tag, std::integral_constant<int, kMaxRowsPerWarp>{});
  };
  if (fp8) by_rows(std::true_type{});
  else by_rows(std::false_type{});
  return cudaGetLastError();
}

}  // namespace mla
