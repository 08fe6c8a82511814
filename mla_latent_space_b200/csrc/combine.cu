// Log-sum-exp merge of split pieces (the combine step of split-KV decode).
// Piece i of a row carries its normalised partial output O_i and its lse_i;
// the row's result is L = ln sum_i e^{lse_i} and O = sum_i e^{lse_i - L} O_i.
// Tiles that no worker touched (no visible key) get O = 0 and lse = -inf.
// With out_lo, O is written as two bf16 terms (out + out_lo).
//
// One warp per row, (tile, 16 row blocks) CTAs of 8 warps: the lanes read
// the pieces' lse values at once and reduce max and sum with shuffles; then
// each lane streams its 16 fp32 values of one piece at a time (four float4
// loads in flight per lane).  At most 64 registers a thread, so that four
// CTAs share an SM and every row of a typical batch is in flight in about
// one wave: the kernel is bound by how many loads are outstanding.
#include "decode_launch.cuh"
#include "kernel_util.cuh"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

constexpr int kWarps = 8;
constexpr int kRowBlocks = MLA_TILE_ROWS / kWarps;   // 16

__global__ void __launch_bounds__(kWarps * 32, 4)
combine_kernel(const void* __restrict__ sched, const void* __restrict__ ws_c, __nv_bfloat16* __restrict__ out,
               __nv_bfloat16* __restrict__ out_lo, float* __restrict__ lse, int cap_slots) {
  ptx::griddep_wait();   // launched programmatically behind the decode kernel
  const SchedView sv(sched);
  void* ws = const_cast<void*>(ws_c);
  const int T = blockIdx.x;
  const int n = sv.tile_splits(T);
  if (n == 1) return;
  const int r = T / sv.tiles_per_req, qt = T % sv.tiles_per_req;
  const int rows_total = sv.s_q * sv.heads;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int row = blockIdx.y * kWarps + warp;
  const int rho = qt * MLA_TILE_ROWS + row;
  if (rho >= rows_total) return;
  const int base = n > 1 ? sv.tile_slot_base(T) : 0;
  if (n > 1 && base + n > cap_slots) {
    if (lane == 0) flag_status(ws, kStatusWorkspace);
    return;
  }
  __nv_bfloat16* o = out + (size_t(r) * rows_total + rho) * MLA_D_V;
  __nv_bfloat16* ol = out_lo != nullptr ? out_lo + (size_t(r) * rows_total + rho) * MLA_D_V : nullptr;
  if (n == 0) {
    reinterpret_cast<uint4*>(o)[lane * 2] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(o)[lane * 2 + 1] = make_uint4(0, 0, 0, 0);
    if (ol != nullptr) {
      reinterpret_cast<uint4*>(ol)[lane * 2] = make_uint4(0, 0, 0, 0);
      reinterpret_cast<uint4*>(ol)[lane * 2 + 1] = make_uint4(0, 0, 0, 0);
    }
    if (lane == 0) lse[size_t(r) * rows_total + rho] = -INFINITY;
    return;
  }
  // the first piece's values do not depend on the weights: their loads go
  // out before the lse reduction so that the two latencies overlap
  float4 v0[MLA_D_V / 128];
  {
    const float4* src = reinterpret_cast<const float4*>(ws_partial_o(ws, cap_slots, base) + size_t(row) * MLA_D_V);
#pragma unroll
    for (int c = 0; c < MLA_D_V / 128; ++c) v0[c] = __ldcs(src + lane + 32 * c);
  }
  float mx = -INFINITY;
  for (int i = lane; i < n; i += 32) mx = fmaxf(mx, ws_partial_lse(ws, cap_slots, base + i)[row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  if (mx != -INFINITY)
    for (int i = lane; i < n; i += 32) sum += __expf(ws_partial_lse(ws, cap_slots, base + i)[row] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float L = (mx == -INFINITY || sum <= 0.f) ? -INFINITY : mx + logf(sum);
  float4 acc[MLA_D_V / 128];
#pragma unroll
  for (int c = 0; c < MLA_D_V / 128; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (L != -INFINITY) {
    for (int i = 0; i < n; ++i) {
      const float w = __expf(ws_partial_lse(ws, cap_slots, base + i)[row] - L);
      float4 v[MLA_D_V / 128];
      if (i == 0) {
#pragma unroll
        for (int c = 0; c < MLA_D_V / 128; ++c) v[c] = v0[c];
      } else {
        const float4* src =
            reinterpret_cast<const float4*>(ws_partial_o(ws, cap_slots, base + i) + size_t(row) * MLA_D_V);
#pragma unroll
        for (int c = 0; c < MLA_D_V / 128; ++c) v[c] = __ldcs(src + lane + 32 * c);
      }
      if (w == 0.f) continue;
#pragma unroll
      for (int c = 0; c < MLA_D_V / 128; ++c) {
        acc[c].x = fmaf(w, v[c].x, acc[c].x);
        acc[c].y = fmaf(w, v[c].y, acc[c].y);
        acc[c].z = fmaf(w, v[c].z, acc[c].z);
        acc[c].w = fmaf(w, v[c].w, acc[c].w);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < MLA_D_V / 128; ++c) {
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(acc[c].x, acc[c].y);
    const __nv_bfloat162 h23 = __floats2bfloat162_rn(acc[c].z, acc[c].w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&h01);
    pk.y = *reinterpret_cast<const uint32_t*>(&h23);
    reinterpret_cast<uint2*>(o)[lane + 32 * c] = pk;
    if (ol != nullptr) {   // second term: bf16 of what the first one dropped
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      const __nv_bfloat162 l01 = __floats2bfloat162_rn(acc[c].x - f01.x, acc[c].y - f01.y);
      const __nv_bfloat162 l23 = __floats2bfloat162_rn(acc[c].z - f23.x, acc[c].w - f23.y);
      pk.x = *reinterpret_cast<const uint32_t*>(&l01);
      pk.y = *reinterpret_cast<const uint32_t*>(&l23);
      reinterpret_cast<uint2*>(ol)[lane + 32 * c] = pk;
    }
  }
  if (lane == 0) lse[size_t(r) * rows_total + rho] = L;
}

}  // namespace

cudaError_t launch_combine(const void* sched, const void* ws, void* out, float* lse, int num_tiles,
                           int cap_slots, cudaStream_t stream, void* out_lo) {
  if (num_tiles == 0) return cudaSuccess;
  // programmatic dependent launch behind the decode kernel (the kernel waits
  // for it before reading anything)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_tiles, kRowBlocks);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, combine_kernel, sched, ws, static_cast<__nv_bfloat16*>(out),
                                           static_cast<__nv_bfloat16*>(out_lo), lse, cap_slots);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace mla
