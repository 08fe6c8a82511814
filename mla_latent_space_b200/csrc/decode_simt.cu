// Plain SIMT decode kernel: the same latent-space decode as the tcgen05
// kernel ("MLA Cost Analysis & Regime Guide", section "Absorption Trick":
// scores against the 576-d cache rows, values = their first 512 entries),
// computed with fp32 FMAs and an online softmax over 32-token chunks.  It
// exists to check the host plumbing, the schedule and the combine against
// the oracle independently of the tensor-core kernel; it is only reachable
// through the debug entry point mla_decode_fwd_simt.
//
// Grid: (workers, 8).  blockIdx.y picks 16 of a tile's 128 rows.
#include "kernel_util.cuh"

namespace mla {

namespace {

constexpr int kRows = 16;       // rows per CTA
constexpr int kChunk = 32;      // tokens per chunk
constexpr int kThreads = 256;
constexpr int kKStride = MLA_D_QK + 1;  // padded smem row (bank spread)

struct SimtSmem {
  float q[kRows][MLA_D_QK];
  float k[kChunk][kKStride];
  float p[kRows][kChunk];
  float alpha[kRows];
  float m[kRows];
  float l[kRows];
  int len[kRows];
};

__global__ void __launch_bounds__(kThreads)
decode_simt_kernel(const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kv,
                   const float* __restrict__ kv_scale, const int32_t* __restrict__ block_table,
                   const int32_t* __restrict__ seqlens, float scale, const void* __restrict__ sched,
                   void* ws, __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int num_pages,
                   int fp8, int cap_slots) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  const SchedView sv(sched);
  const int tid = threadIdx.x;
  const int rows_total = sv.s_q * sv.heads;
  const int orow = tid / 16;           // row this thread accumulates
  const int olane = tid % 16;          // dims olane + 16*c
  for (int w = blockIdx.x; w < sv.W; w += gridDim.x) {
  PieceIter it(sv, w);
  Piece pc;
  while (it.next(&pc)) {
    const int r = pc.T / sv.tiles_per_req, qt = pc.T % sv.tiles_per_req;
    const int row0 = qt * MLA_TILE_ROWS + blockIdx.y * kRows;
    int t = seqlens[r];
    t = max(0, min(t, sv.max_pages * MLA_PAGE_SIZE));
    if (row0 >= rows_total) continue;   // uniform for the CTA
    for (int idx = tid; idx < kRows * MLA_D_QK; idx += kThreads) {
      int i = idx / MLA_D_QK, d = idx % MLA_D_QK, rho = row0 + i;
      float v = 0.f;
      if (rho < rows_total) v = __bfloat162float(q[(size_t(r) * rows_total + rho) * MLA_D_QK + d]);
      sm.q[i][d] = v;
    }
    if (tid < kRows) {
      int rho = row0 + tid;
      sm.len[tid] = rho < rows_total ? visible_len(t, sv.s_q, rho / sv.heads, sv.causal) : 0;
      sm.m[tid] = -INFINITY;
      sm.l[tid] = 0.f;
    }
    float acc[MLA_D_V / 16];
#pragma unroll
    for (int c = 0; c < MLA_D_V / 16; ++c) acc[c] = 0.f;
    __syncthreads();

    for (int pg = pc.p0; pg < pc.p1; ++pg) {
      int page = block_table[size_t(r) * sv.max_pages + pg];
      if (page < 0 || page >= num_pages) {
        if (tid == 0) flag_status(ws, kStatusBadPage);
        continue;
      }
      for (int half = 0; half < MLA_PAGE_SIZE / kChunk; ++half) {
        const int j0 = pg * MLA_PAGE_SIZE + half * kChunk;
        // load 32 cache rows as fp32; rows at or past t are zero (their
        // bytes may be anything, and 0 * NaN would poison the sum)
        for (int idx = tid; idx < kChunk * MLA_D_QK; idx += kThreads) {
          int j = idx / MLA_D_QK, d = idx % MLA_D_QK;
          int tok = half * kChunk + j;
          float v = 0.f;
          if (j0 + j < t) {
            if (!fp8) {
              const uint16_t* pb = reinterpret_cast<const uint16_t*>(kv) + size_t(page) * MLA_PAGE_SIZE * MLA_D_QK;
              v = bf16_bits_to_float(pb[size_t(tok) * MLA_D_QK + d]);
            } else {
              const uint8_t* pb = kv + size_t(page) * (MLA_PAGE_SIZE * MLA_D_V + MLA_PAGE_SIZE * 64 * 2);
              if (d < MLA_D_V) {
                v = e4m3_to_float(pb[size_t(tok) * MLA_D_V + d]) * kv_scale[size_t(page) * MLA_PAGE_SIZE + tok];
              } else {
                const uint16_t* rope = reinterpret_cast<const uint16_t*>(pb + MLA_PAGE_SIZE * MLA_D_V);
                v = bf16_bits_to_float(rope[size_t(tok) * 64 + (d - MLA_D_V)]);
              }
            }
          }
          sm.k[j][d] = v;
        }
        __syncthreads();
        // scores
        for (int e = tid; e < kRows * kChunk; e += kThreads) {
          int i = e / kChunk, j = e % kChunk;
          float s = 0.f;
#pragma unroll 8
          for (int d = 0; d < MLA_D_QK; ++d) s = fmaf(sm.q[i][d], sm.k[j][d], s);
          s *= scale;
          sm.p[i][j] = (j0 + j < sm.len[i]) ? s : -INFINITY;
        }
        __syncthreads();
        // online softmax: 16 threads per row, 2 tokens each
        {
          int i = tid / 16, l16 = tid % 16;
          float s0 = sm.p[i][l16], s1 = sm.p[i][l16 + 16];
          float mx = fmaxf(s0, s1);
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          float m_old = sm.m[i];
          float m_new = fmaxf(m_old, mx);
          float alpha = 1.f, p0 = 0.f, p1 = 0.f;
          if (m_new != -INFINITY) {
            alpha = __expf(m_old - m_new);
            p0 = __expf(s0 - m_new);
            p1 = __expf(s1 - m_new);
          }
          float ps = p0 + p1;
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
          __syncwarp();
          sm.p[i][l16] = p0;
          sm.p[i][l16 + 16] = p1;
          if (l16 == 0) {
            sm.alpha[i] = alpha;
            sm.m[i] = m_new;
            sm.l[i] = sm.l[i] * alpha + ps;
          }
        }
        __syncthreads();
        {
          float a = sm.alpha[orow];
#pragma unroll
          for (int c = 0; c < MLA_D_V / 16; ++c) acc[c] *= a;
          for (int j = 0; j < kChunk; ++j) {
            float pj = sm.p[orow][j];
#pragma unroll
            for (int c = 0; c < MLA_D_V / 16; ++c) acc[c] = fmaf(pj, sm.k[j][olane + 16 * c], acc[c]);
          }
        }
        __syncthreads();
      }
    }
    // epilogue
    const int rho = row0 + orow;
    if (rho < rows_total) {
      float l = sm.l[orow], m = sm.m[orow];
      float inv = l > 0.f ? 1.f / l : 0.f;
      float lse_v = l > 0.f ? m + logf(l) : -INFINITY;
      const int lane = blockIdx.y * kRows + orow;
      if (sv.tile_splits(pc.T) == 1) {
        __nv_bfloat16* o = out + (size_t(r) * rows_total + rho) * MLA_D_V;
#pragma unroll
        for (int c = 0; c < MLA_D_V / 16; ++c) o[olane + 16 * c] = __float2bfloat16_rn(acc[c] * inv);
        if (olane == 0) lse[size_t(r) * rows_total + rho] = lse_v;
      } else {
        int slot = sv.tile_slot_base(pc.T) + pc.split;
        if (slot < cap_slots) {
          float* o = ws_partial_o(ws, cap_slots, slot) + size_t(lane) * MLA_D_V;
#pragma unroll
          for (int c = 0; c < MLA_D_V / 16; ++c) o[olane + 16 * c] = acc[c] * inv;
          if (olane == 0) ws_partial_lse(ws, cap_slots, slot)[lane] = lse_v;
        } else if (olane == 0) {
          flag_status(ws, kStatusWorkspace);
        }
      }
    }
    __syncthreads();
  }
  }
}

}  // namespace

size_t simt_smem_bytes() { return sizeof(SimtSmem); }

cudaError_t launch_decode_simt(const void* q, const void* kv, const float* kv_scale, const int32_t* block_table,
                               const int32_t* seqlens, float scale, const void* sched, void* ws, void* out,
                               float* lse, int num_pages, int fp8, int cap_slots, int grid_ctas,
                               cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem);
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(grid_ctas, MLA_TILE_ROWS / kRows);
  decode_simt_kernel<<<grid, kThreads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(kv), kv_scale, block_table, seqlens, scale,
      sched, ws, static_cast<__nv_bfloat16*>(out), lse, num_pages, fp8, cap_slots);
  return cudaGetLastError();
}

}  // namespace mla
