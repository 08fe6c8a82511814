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
// tokens only.  Step 3 is a small attention per (request, head): M = s <= 32
// query rows against n tokens, K = d + p = 192 and N = d = 128.  M is below
// the smallest tcgen05 tile (64 rows) and n may be as small as s, so it runs
// on warp-level tensor-core MMAs (mma.sync m16n8k16): one CTA per (request,
// head), the CTA staging 32-token chunks and every warp computing the
// chunk's scores and softmax, then the product with its own quarter of the
// value dimensions; the result is merged at the end with the old part.  Q.K^T is bf16 x bf16 exactly as stored; P.V takes P as two bf16
// terms (hi + lo) against the bf16 values, so no value is converted and P
// keeps about 16 significant bits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>


#include "kernel_util.cuh"

namespace mla {

namespace {

constexpr int kVarThreads = 128;
constexpr int kVarWarps = kVarThreads / 32;
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

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) . B (16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2_bf16(float x, float y) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack2_bf16(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Shared memory (bf16 rows padded by 8 elements so that the 8 rows of an
// ldmatrix block fall in different banks).
constexpr int kKStride = MLA_D_HEAD + MLA_D_ROPE + 8;   // 200: one key row [k_new | RoPE]
constexpr int kVStride = MLA_D_HEAD + 8;                // 136: one value row
constexpr int kQStride = kKStride;                      // one query row [q_nope | q_pe]
struct Var6Smem {
  __nv_bfloat16 q[16][kQStride];
  __nv_bfloat16 k[kChunk][kKStride];
  __nv_bfloat16 v[kChunk][kVStride];
  int pos[kChunk];                                      // token position, -1 if absent
};

// grid (batch, heads), 128 threads.  For each 16-row tile of the s_q query
// rows, the CTA stages 32-token chunks (all threads, 16-byte pieces); every
// warp computes the chunk's S = Q.K^T (12 k-steps x 4 n-tiles; the four
// warps compute the same S, which is cheap next to staging it, and so keep
// identical softmax statistics without exchanging them), masks it, runs the
// online softmax in log2 units, and accumulates O += P_hi.V + P_lo.V for its
// own 32 of the 128 value dimensions.  The result is merged with
// (O_old, lse_old) at the end.
template <bool kFp8>
__global__ void __launch_bounds__(kVarThreads, 4)
    var6_new_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k_new,
                    const uint16_t* __restrict__ v_new, const uint8_t* __restrict__ pool,
                    const int32_t* __restrict__ block_table, const int32_t* __restrict__ seqlens,
                    const uint16_t* __restrict__ o_old, const uint16_t* __restrict__ o_old_lo,
                    const float* __restrict__ lse_old, int s_q, int heads,
                    int n_new, int max_pages, int num_pages, int causal, float scale, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, void* status_ws) {
  __shared__ __align__(16) Var6Smem sm;
  constexpr int kQ = MLA_D_HEAD + MLA_D_ROPE;   // 192
  constexpr int kPieces = MLA_D_HEAD / 8 * 2 + MLA_D_ROPE / 8;   // 16-byte pieces per token: 40
  constexpr int kPer = kChunk * kPieces / kVarThreads;           // per thread per chunk: 10
  const int r = blockIdx.x, hd = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, tq = lane & 3;       // mma fragment row group / column pair
  const int mi = lane >> 3, mr = lane & 7;      // ldmatrix: this lane's matrix and row
  const int dw = 32 * warp;                     // this warp's value dimensions dw .. dw+31
  const int cap = max_pages * MLA_PAGE_SIZE;
  int t = seqlens[r];
  t = t < 0 ? 0 : (t > cap ? cap : t);
  const float scale_log2 = scale * 1.4426950408889634f;
  bool bad_page = false;

  for (int m0 = 0; m0 < s_q; m0 += 16) {
    // ---- the tile's query rows (zeros past s_q)
    for (int e = tid; e < 16 * (kQ / 8); e += kVarThreads) {
      const int i = e / (kQ / 8), c = e % (kQ / 8);
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (m0 + i < s_q) w = *reinterpret_cast<const uint4*>(q + ((size_t(r) * s_q + m0 + i) * heads + hd) * kQ + 8 * c);
      *reinterpret_cast<uint4*>(&sm.q[i][8 * c]) = w;
    }

    float o[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    int vis[2];   // visible length of this thread's rows g, g + 8 (-1 past s_q)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = m0 + g + 8 * h;
      vis[h] = i >= s_q ? -1 : (causal ? t - s_q + i + 1 : t);
    }

    for (int tok0 = 0; tok0 < n_new; tok0 += kChunk) {
      __syncthreads();   // the previous chunk (or tile) has been read
      if (tid < kChunk) {
        const int m = tok0 + tid;
        int ps = m < n_new ? t - n_new + m : -1;
        if (ps >= 0) {
          const int pg = block_table[size_t(r) * max_pages + ps / MLA_PAGE_SIZE];
          if (pg < 0 || pg >= num_pages) {
            bad_page = true;
            ps = -1;
          }
        }
        sm.pos[tid] = ps;
      }
      __syncthreads();
      // ---- stage the chunk: every load of a thread before its stores
      uint4 wv[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int e = tid + kVarThreads * u, tok = e / kPieces, pc = e % kPieces;
        const int ps = sm.pos[tok];
        wv[u] = make_uint4(0u, 0u, 0u, 0u);
        if (ps >= 0) {
          const int m = tok0 + tok;
          if (pc < MLA_D_HEAD / 8) {
            wv[u] = *reinterpret_cast<const uint4*>(k_new + ((size_t(r) * n_new + m) * heads + hd) * MLA_D_HEAD + 8 * pc);
          } else if (pc < MLA_D_HEAD / 4) {
            wv[u] = *reinterpret_cast<const uint4*>(v_new + ((size_t(r) * n_new + m) * heads + hd) * MLA_D_HEAD +
                                                    8 * (pc - MLA_D_HEAD / 8));
          } else {
            const int pg = block_table[size_t(r) * max_pages + ps / MLA_PAGE_SIZE], slot = ps % MLA_PAGE_SIZE;
            const uint8_t* rope = kFp8 ? pool + size_t(pg) * (MLA_PAGE_SIZE * (MLA_D_V + 2 * MLA_D_ROPE)) +
                                             MLA_PAGE_SIZE * MLA_D_V + slot * (2 * MLA_D_ROPE)
                                       : pool + (size_t(pg) * MLA_PAGE_SIZE + slot) * (2 * MLA_D_QK) + 2 * MLA_D_V;
            wv[u] = *reinterpret_cast<const uint4*>(rope + 16 * (pc - MLA_D_HEAD / 4));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int e = tid + kVarThreads * u, tok = e / kPieces, pc = e % kPieces;
        if (pc < MLA_D_HEAD / 8)
          *reinterpret_cast<uint4*>(&sm.k[tok][8 * pc]) = wv[u];
        else if (pc < MLA_D_HEAD / 4)
          *reinterpret_cast<uint4*>(&sm.v[tok][8 * (pc - MLA_D_HEAD / 8)]) = wv[u];
        else
          *reinterpret_cast<uint4*>(&sm.k[tok][MLA_D_HEAD + 8 * (pc - MLA_D_HEAD / 4)]) = wv[u];
      }
      __syncthreads();

      // ---- S = Q . K^T: 16 rows x 32 tokens (4 n-tiles of 8)
      float sacc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < kQ / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(smem_addr(&sm.q[mr + 8 * (mi & 1)][16 * ks + 8 * (mi >> 1)]), a);
#pragma unroll
        for (int jp = 0; jp < 2; ++jp) {   // n-tiles 2jp, 2jp+1
          uint32_t b[4];
          ldsm_x4(smem_addr(&sm.k[16 * jp + 8 * (mi >> 1) + mr][16 * ks + 8 * (mi & 1)]), b);
          mma_16816(sacc[2 * jp], a, b[0], b[1]);
          mma_16816(sacc[2 * jp + 1], a, b[2], b[3]);
        }
      }

      // ---- mask, online softmax (log2 units); thread rows g and g + 8
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = e >> 1, ps = sm.pos[8 * j + 2 * tq + (e & 1)];
          const bool ok = ps >= 0 && ps < vis[h];
          sacc[j][e] = ok ? sacc[j][e] * scale_log2 : -INFINITY;
          mx[h] = fmaxf(mx[h], sacc[j][e]);
        }
      float alpha[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float mn = fmaxf(mrow[h], mx[h]);
        alpha[h] = mn == -INFINITY ? 1.f : exp2f(mrow[h] - mn);   // 0 on the first visible chunk
        mrow[h] = mn;
      }
      float psum[2] = {0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = e >> 1;
          const float pv = sacc[j][e] == -INFINITY ? 0.f : exp2f(sacc[j][e] - mrow[h]);
          sacc[j][e] = pv;
          psum[h] += pv;
        }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 1);
        psum[h] += __shfl_xor_sync(0xffffffffu, psum[h], 2);
        lrow[h] = lrow[h] * alpha[h] + psum[h];
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        o[j][0] *= alpha[0];
        o[j][1] *= alpha[0];
        o[j][2] *= alpha[1];
        o[j][3] *= alpha[1];
      }

      // ---- O[:, dw .. dw+31] += P . V, P as bf16 hi + lo (the S fragments
      // of n-tiles 2kk, 2kk+1 are the A fragment of token k-step kk)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t ahi[4], alo[4];
#pragma unroll
        for (int q2 = 0; q2 < 4; ++q2) {
          const int j = 2 * kk + (q2 >> 1), e0 = 2 * (q2 & 1);
          const float x0 = sacc[j][e0], x1 = sacc[j][e0 + 1];
          ahi[q2] = pack2_bf16(x0, x1);
          const float2 hf = unpack2_bf16(ahi[q2]);
          alo[q2] = pack2_bf16(x0 - hf.x, x1 - hf.y);
        }
#pragma unroll
        for (int np = 0; np < 2; ++np) {   // dims dw + 16np .. +15: n-tiles 2np, 2np+1
          uint32_t b[4];
          ldsm_x4_t(smem_addr(&sm.v[16 * kk + 8 * (mi & 1) + mr][dw + 16 * np + 8 * (mi >> 1)]), b);
          mma_16816(o[2 * np], ahi, b[0], b[1]);
          mma_16816(o[2 * np], alo, b[0], b[1]);
          mma_16816(o[2 * np + 1], ahi, b[2], b[3]);
          mma_16816(o[2 * np + 1], alo, b[2], b[3]);
        }
      }
    }

    // ---- merge with the old part: thread (g, tq) holds rows g, g + 8 and
    // dims dw + 8j + 2tq, +1 (j < 4)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row_i = m0 + g + 8 * h;
      if (row_i >= s_q) continue;
      const float ln = lrow[h] > 0.f ? (mrow[h] + log2f(lrow[h])) * 0.69314718055994531f : -INFINITY;
      const float inv = lrow[h] > 0.f ? 1.f / lrow[h] : 0.f;
      const size_t row = (size_t(r) * s_q + row_i) * heads + hd;
      const float lo = lse_old[row];
      const float mm = fmaxf(lo, ln);
      float L = -INFINITY, wo = 0.f, wn = 0.f;
      if (mm > -INFINITY) {
        const float so = expf(lo - mm), sn = expf(ln - mm);
        L = mm + logf(so + sn);
        wo = so / (so + sn);
        wn = sn / (so + sn);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = dw + 8 * j + 2 * tq;
        // the old part arrives as two bf16 terms, hi + lo (fp32-accurate)
        const uint32_t ob = *reinterpret_cast<const uint32_t*>(o_old + row * MLA_D_HEAD + d);
        const uint32_t ol = *reinterpret_cast<const uint32_t*>(o_old_lo + row * MLA_D_HEAD + d);
        const float a0 = bf16_lo(ob) + bf16_lo(ol), a1 = bf16_hi(ob) + bf16_hi(ol);
        *reinterpret_cast<uint32_t*>(out + row * MLA_D_HEAD + d) =
            pack2_bf16(wo * a0 + wn * o[j][2 * h] * inv, wo * a1 + wn * o[j][2 * h + 1] * inv);
      }
      if (warp == 0 && tq == 0) lse[row] = L;
    }
    __syncthreads();   // every warp is done with the query tile before the next one is staged
  }
  if (bad_page) flag_status(status_ws, kStatusBadPage);
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
  if (fp8)
    var6_new_kernel<true><<<grid, kVarThreads, 0, stream>>>(qq, kk, vv, pp, block_table, seqlens, oo, ool, lse_old,
                                                            s_q, heads, n_new, max_pages, num_pages, causal, scale,
                                                            dst, lse, status_ws);
  else
    var6_new_kernel<false><<<grid, kVarThreads, 0, stream>>>(qq, kk, vv, pp, block_table, seqlens, oo, ool, lse_old,
                                                             s_q, heads, n_new, max_pages, num_pages, causal, scale,
                                                             dst, lse, status_ws);
  return cudaGetLastError();
}

}  // namespace mla
