// Per-head projections on either side of the latent decode, for B200
// (sm_100a).  "MLA Cost Analysis & Regime Guide", section "Absorption
// Trick": the key up-projection is folded into the query before the
// attention, and the latent output is decompressed by a separate GEMM after
// it.  With d = 128 head dims and p = 64 RoPE dims:
//
//   absorb      Qz[r, j, c]       = sum_n q[r, j, n] * Wk[j, c, n]     c < 512, n < d
//               Qz[r, j, 512 + e] = q[r, j, d + e]                    e < p (copied)
//   decompress  out[r, j, v]      = sum_c O[r, j, c] * Wkvb2[j, v, c]  v < d, c < 512
//
// Both are computed as D = X_j . W_j^T on the 5th-generation tensor core:
// A is 128 activation rows of head j (K-major, rows of the activation
// tensor), B is a 128-row slice of head j's weight (K-major, which is the
// weight's own layout), and D = 128 rows x 128 output features sits in fp32
// TMEM, one row per TMEM lane, so an epilogue thread holds consecutive
// features of its row and writes them 16 bytes at a time.  Rows past the end
// of a small decode batch (64 rows at b = 64) are zeros read from outside the
// tensor: the MMA does them for free and the epilogue skips them.  The
// weights dominate the bytes
// (16.8 MB per projection at h = 128, against 2-8 MB of activations at
// decode batch sizes), so the kernel is HBM-bound and is written for
// streaming, as a persistent kernel with one CTA per SM, each taking an
// equal contiguous range of the units (128 rows x 128 features of one head;
// feature tile fastest, so consecutive units share their activation rows
// and read consecutive weight slices):
//   warp 0     TMA producer: 64-column K chunks of the weight slice and of
//              the activation rows (128-byte swizzle boxes, 16 KB each)
//              through a 4-stage ring that runs on across units;
//   warp 1     MMA issuer (one thread): 4 MMAs (M = N = 128, K = 16) per
//              chunk into one of two TMEM accumulators;
//   warps 2-5  epilogue: accumulator -> bf16 -> one of two staging tiles
//              [row][feature] in 128-byte swizzle atoms -> two TMA stores
//              per unit (they clip the rows past the end of the batch).  Before their first unit they
//              copy the absorbed query's RoPE part for the CTA's units, so
//              those scattered row loads overlap the first TMA loads.
// Two accumulators and two staging tiles let a unit's epilogue and store
// overlap the next unit's loads and MMAs, so each SM keeps its loads in
// flight from its first unit to its last.
//
// Every wait is bounded: a wait that runs out raises a CTA-wide abort flag
// and a status bit (when the caller passed a status word); every role then
// leaves its loop, the producer waits (bounded) for the copies it issued,
// the MMA issuer for its MMAs, and TMEM is freed before the CTA returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "kernel_util.cuh"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

using namespace ptx;

constexpr int kProjThreads = 192;              // producer warp, MMA warp, 4 epilogue warps
constexpr int kTileM = 128;                    // output features per unit (TMEM lanes)
constexpr int kTileN = 128;                    // activation rows per unit (TMEM columns)
constexpr int kRing = 4;                       // K-chunk stages
constexpr uint32_t kChunk = 128u * 64u * 2u;   // 128 rows x 64 bf16: one 128-byte swizzle box
constexpr uint32_t kStage = 2 * kChunk;        // weight chunk + activation chunk
constexpr uint32_t kStaging = uint32_t(kTileN) * kTileM * 2;   // one bf16 output tile (two 64-feature boxes)
constexpr uint32_t kStagingBox = kStaging / 2;
constexpr uint32_t kOffStaging = kRing * kStage;
constexpr uint32_t kProjSmem = kOffStaging + 2 * kStaging + 1024;   // + alignment slack
constexpr uint64_t kProjTimeoutNs = 2000000000ull;
// kind::f16: bf16 A and B, fp32 D, both K-major, M = kTileN rows, N = kTileM features
constexpr uint32_t kIdescProj =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t(kTileM) >> 3) << 17) | ((uint32_t(kTileN) >> 4) << 24);
static_assert(kProjSmem <= 232448, "shared memory");

struct ProjArgs {
  int w_rows_per_head;   // weight rows of one head: absorb 512, decompress 128
  int x_cols_per_head;   // columns of one head in an activation row: absorb d+p, decompress 512
  int o_cols_per_head;   // columns of one head in an output row: absorb 576, decompress d
  int rows, heads;
  int n_tiles, m_tiles;  // units = m_tiles x n_tiles x heads, feature tile fastest
  const uint8_t* rope_src;   // absorb: q, whose RoPE part is copied through; else null
  uint8_t* rope_dst;         // absorb: Qz
  int32_t* status;           // optional sticky status word
  __nv_bfloat16* o_lo;       // two-term decompress: bf16 of what the bf16 output dropped
};

struct Unit {
  int r0, m0, head;
};

__device__ __forceinline__ Unit unit_of(const ProjArgs& a, int u) {
  Unit x;
  x.m0 = (u % a.m_tiles) * kTileM;
  const int rest = u / a.m_tiles;
  x.r0 = (rest % a.n_tiles) * kTileN;
  x.head = rest / a.n_tiles;
  return x;
}

// Copies the RoPE part of query row r of head `head` (128 bytes) from q to
// Qz; `v` holds it in between.
__device__ __forceinline__ void rope_load(const ProjArgs& a, int r, int head, uint4 (&v)[8]) {
  const size_t row = size_t(r) * a.heads + head;
  const uint8_t* src = a.rope_src + row * (2 * (MLA_D_HEAD + MLA_D_ROPE)) + 2 * MLA_D_HEAD;
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = ld_global_nc_v4(src + 16 * k);
}
__device__ __forceinline__ void rope_store(const ProjArgs& a, int r, int head, const uint4 (&v)[8]) {
  const size_t row = size_t(r) * a.heads + head;
  uint4* dst = reinterpret_cast<uint4*>(a.rope_dst + row * (2 * MLA_D_QK) + 2 * MLA_D_V);
#pragma unroll
  for (int k = 0; k < 8; ++k) dst[k] = v[k];
}

// 2-D tiled store from this CTA's shared memory (bulk group; elements
// outside the tensor are not written).
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(tmap)), "r"(src), "r"(c0), "r"(c1)
               : "memory");
}

// Shared-memory descriptor of a K-major operand in 128-byte swizzle atoms
// (8 rows x 128 bytes, atoms 1024 bytes apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return uint64_t((addr >> 4) & 0x3FFF) | (uint64_t(16 >> 4) << 16) | (uint64_t(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

// Bounded phase wait.  Gives up when another role raised the abort flag, or
// after kProjTimeoutNs, in which case it raises the flag and the status bit.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* status) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (globaltimer() - t0 > kProjTimeoutNs) {
      *abort = 1;
      if (status != nullptr) atomicOr(status, kStatusTimeout);
      return false;
    }
  }
  return true;
}

// KC: number of 64-wide K chunks (absorb: d/64 = 2, decompress: 512/64 = 8).
// kTwo: the activation comes as two bf16 terms (xmap + x2map, which carry an
// fp32-accurate input) and the output goes out as two: D = (X + X2) . W^T is
// one accumulation over 2 KC chunks (the weight chunks read twice), written
// as o = bf16(D) through omap and o_lo = bf16(D - o) with plain stores.
template <int KC, bool kTwo>
__global__ void __launch_bounds__(kProjThreads, 1)
    proj_sm100_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap x2map, const __grid_constant__ CUtensorMap omap,
                      const ProjArgs a) {
  constexpr int KT = kTwo ? 2 * KC : KC;   // K chunks per unit
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kRing];
  __shared__ __align__(8) uint64_t empty[kRing];
  __shared__ __align__(8) uint64_t acc_full[2];
  __shared__ __align__(8) uint64_t acc_empty[2];
  __shared__ __align__(8) uint64_t mma_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  volatile int* abort = &abort_flag;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's units: [ub, ue), an equal share of all units
  const int units = a.n_tiles * a.m_tiles * a.heads;
  const int per = units / int(gridDim.x), extra = units % int(gridDim.x), b = int(blockIdx.x);
  const int ub = b * per + (b < extra ? b : extra), ue = ub + per + (b < extra ? 1 : 0);

  if (tid == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 128);
    }
    mbar_init(smem_u32(&mma_drain), 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&wmap);
    tma_prefetch_desc(&xmap);
    if (kTwo) tma_prefetch_desc(&x2map);
    tma_prefetch_desc(&omap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 2 * kTileN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // launched as a programmatic dependent: the set-up above overlapped the
  // previous kernel; its results are visible once this returns.  A kernel
  // after this one may begin its own set-up now (it waits the same way).
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // ---- TMA producer
    if (elect_one()) {
      int g = 0;   // chunks issued
      for (int u = ub; u < ue && !*abort; ++u) {
        const Unit x = unit_of(a, u);
        const int wy = x.head * a.w_rows_per_head + x.m0, xx = x.head * a.x_cols_per_head;
        bool go = true;
        for (int kc = 0; kc < KT; ++kc, ++g) {
          const int s = g % kRing;
          const int fill = g / kRing;   // earlier fills of stage s
          if (fill > 0 && !wait_bounded(smem_u32(&empty[s]), uint32_t((fill - 1) & 1), abort, a.status)) {
            go = false;
            break;
          }
          const uint32_t st = base + uint32_t(s) * kStage;
          const int kw = kc % KC;   // the weight chunk (read twice in two-term mode)
          mbar_arrive_expect_tx(smem_u32(&full[s]), kStage);
          tma_load_2d(st, &wmap, 64 * kw, wy, smem_u32(&full[s]));
          tma_load_2d(st + kChunk, (kTwo && kc >= KC) ? &x2map : &xmap, xx + 64 * kw, x.r0, smem_u32(&full[s]));
        }
        if (!go) break;
      }
      // every copy issued has landed before the CTA may leave (the waits
      // below give up only after their own time limit, not on abort)
      for (int s = 0; s < kRing && s < g; ++s) {
        const int n = (g - s + kRing - 1) / kRing;   // fills of stage s
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(smem_u32(&full[s]), uint32_t((n - 1) & 1)))
          if (globaltimer() - t0 > kProjTimeoutNs) break;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMA issuer
    if (elect_one()) {
      int g = 0;
      for (int u = ub, i = 0; u < ue; ++u, ++i) {
        const int acc = i & 1, use = i >> 1;   // earlier uses of this accumulator
        if (use > 0 && !wait_bounded(smem_u32(&acc_empty[acc]), uint32_t((use - 1) & 1), abort, a.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(acc * kTileN);
        bool go = true;
        for (int kc = 0; kc < KT; ++kc, ++g) {
          const int s = g % kRing;
          if (!wait_bounded(smem_u32(&full[s]), uint32_t((g / kRing) & 1), abort, a.status)) {
            go = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + uint32_t(s) * kStage;
          const uint64_t ad = sw128_desc(st + kChunk), bd = sw128_desc(st);   // A: rows, B: weight
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_ss(d, ad + 2u * k, bd + 2u * k, kIdescProj, (kc | k) != 0 ? 1u : 0u);
          mma_commit(smem_u32(&empty[s]));
        }
        if (!go) break;
        mma_commit(smem_u32(&acc_full[acc]));
      }
      // every MMA issued has completed before TMEM is freed
      mma_commit(smem_u32(&mma_drain));
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(&mma_drain), 0))
        if (globaltimer() - t0 > kProjTimeoutNs) break;
    }
    __syncwarp();
  } else {
    // ---- epilogue: thread (warp w, lane l) owns row 32 (w % 4) + l of the
    // unit, its TMEM lane, and writes its 128 features
    const int et = tid - 64;   // 0..127
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    // absorb: the RoPE part of the query rows of this CTA's units of the
    // first feature tile, one row per thread, two units' loads in flight
    if (a.rope_src != nullptr) {
      const int u0 = (ub + a.m_tiles - 1) / a.m_tiles * a.m_tiles;   // first unit with m0 == 0
      for (int u = u0; u < ue; u += 2 * a.m_tiles) {
        uint4 v0[8], v1[8];
        const Unit x0 = unit_of(a, u);
        const bool has1 = u + a.m_tiles < ue;
        const Unit x1 = unit_of(a, has1 ? u + a.m_tiles : u);
        const bool in0 = x0.r0 + et < a.rows, in1 = has1 && x1.r0 + et < a.rows;
        if (in0) rope_load(a, x0.r0 + et, x0.head, v0);
        if (in1) rope_load(a, x1.r0 + et, x1.head, v1);
        if (in0) rope_store(a, x0.r0 + et, x0.head, v0);
        if (in1) rope_store(a, x1.r0 + et, x1.head, v1);
      }
    }
    for (int u = ub, i = 0; u < ue; ++u, ++i) {
      const Unit x = unit_of(a, u);
      const int acc = i & 1, use = i >> 1;
      bool ok = wait_bounded(smem_u32(&acc_full[acc]), uint32_t(use & 1), abort, a.status);
      tc_fence_after();
      // staging tile `acc` was last read by the store issued two units ago
      if (et == 0) bulk_wait_group_read<1>();
      if (!named_bar_and(1, 128, ok)) break;
      const uint32_t stg = base + kOffStaging + uint32_t(acc) * kStaging;
      // a warp whose 32 rows all lie past the end of the batch has nothing to write
      if (x.r0 + quarter * 32 < a.rows) {
        const uint32_t taddr = tmem + uint32_t(acc * kTileN) + (uint32_t(quarter * 32) << 16);
        const uint32_t sw = uint32_t(row & 7);
#pragma unroll 1
        for (int j = 0; j < kTileM / 32; ++j) {
          uint32_t v[32];
          tmem_ld32(taddr + 32u * uint32_t(j), v);
          tmem_wait_ld();
          // features 32j .. 32j+31: four 16-byte chunks of box j / 2
          const uint32_t rowaddr = stg + uint32_t(j >> 1) * kStagingBox + uint32_t(row) * 128u;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4], wl[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float f0 = __uint_as_float(v[8 * c + 2 * k]), f1 = __uint_as_float(v[8 * c + 2 * k + 1]);
              const __nv_bfloat162 pr = __floats2bfloat162_rn(f0, f1);
              w[k] = *reinterpret_cast<const uint32_t*>(&pr);
              if constexpr (kTwo) {
                const float2 h = __bfloat1622float2(pr);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(f0 - h.x, f1 - h.y);
                wl[k] = *reinterpret_cast<const uint32_t*>(&lo);
              }
            }
            const uint32_t chunk = uint32_t(4 * (j & 1) + c);
            st_shared_v4(rowaddr + ((chunk ^ sw) << 4), w[0], w[1], w[2], w[3]);
            if constexpr (kTwo) {
              if (x.r0 + row < a.rows) {
                __nv_bfloat16* dst = a.o_lo + (size_t(x.r0 + row) * a.heads * a.o_cols_per_head +
                                               size_t(x.head) * a.o_cols_per_head + x.m0 + 32 * j + 8 * c);
                *reinterpret_cast<uint4*>(dst) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[acc]));   // the MMA issuer may reuse the accumulator
      fence_proxy_async_cta();
      named_bar_sync(1, 128);
      if (et == 0) {
        tma_store_2d(&omap, stg, x.head * a.o_cols_per_head + x.m0, x.r0);
        tma_store_2d(&omap, stg + kStagingBox, x.head * a.o_cols_per_head + x.m0 + 64, x.r0);
        bulk_commit_group();
      }
    }
    if (et == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kTileN);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 proj_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D bf16 tensor map: `inner` contiguous columns, `outer` rows `stride`
// bytes apart, boxes of 64 columns x 128 rows in 128-byte swizzle atoms
// (the operand tiles and the output staging boxes).
bool make_map(CUtensorMap* map, const void* p, uint64_t inner, uint64_t outer, uint64_t stride) {
  auto fn = proj_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(p), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int proj_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
  return n;
}

template <int KC, bool kTwo>
int launch_proj(const CUtensorMap& w, const CUtensorMap& x, const CUtensorMap& x2, const CUtensorMap& o, ProjArgs a,
                cudaStream_t stream) {
  if (!ensure_smem_attr(reinterpret_cast<const void*>(&proj_sm100_kernel<KC, kTwo>), int(kProjSmem)))
    return MLA_ERR_CUDA;
  const int sms = proj_num_sms();
  if (sms < 0) return MLA_ERR_CUDA;
  a.n_tiles = (a.rows + kTileN - 1) / kTileN;
  const long long units = (long long)a.n_tiles * a.m_tiles * a.heads;
  if (units >= (1ll << 31)) return MLA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(units < sms ? units : sms));
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = kProjSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, proj_sm100_kernel<KC, kTwo>, w, x, x2, o, a);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

// Host entry points behind mla_absorb_q / mla_decompress_o: arguments are
// already validated (rows >= 1, 1 <= heads <= 65535, 16-byte aligned).
int launch_absorb_q(int rows, int heads, const void* q, const void* w_k, void* qz, int32_t* status,
                    cudaStream_t stream) {
  CUtensorMap w, x, o;
  const uint64_t h = uint64_t(heads), R = uint64_t(rows);
  if (!make_map(&w, w_k, MLA_D_HEAD, h * MLA_D_V, 2 * MLA_D_HEAD)) return MLA_ERR_CUDA;
  if (!make_map(&x, q, h * (MLA_D_HEAD + MLA_D_ROPE), R, 2 * h * (MLA_D_HEAD + MLA_D_ROPE))) return MLA_ERR_CUDA;
  if (!make_map(&o, qz, h * MLA_D_QK, R, 2 * h * MLA_D_QK)) return MLA_ERR_CUDA;
  ProjArgs a;
  a.w_rows_per_head = MLA_D_V;
  a.x_cols_per_head = MLA_D_HEAD + MLA_D_ROPE;
  a.o_cols_per_head = MLA_D_QK;
  a.rows = rows;
  a.heads = heads;
  a.rope_src = static_cast<const uint8_t*>(q);
  a.rope_dst = static_cast<uint8_t*>(qz);
  a.status = status;
  a.o_lo = nullptr;
  a.m_tiles = MLA_D_V / kTileM;
  return launch_proj<MLA_D_HEAD / 64, false>(w, x, x, o, a, stream);
}

// o_lat_lo / out_lo: both null (one-term bf16 decompression), or both set
// (two-term: the input is o_lat + o_lat_lo, the output out + out_lo).
int launch_decompress_o(int rows, int heads, const void* o_lat, const void* w_kvb2, void* out, int32_t* status,
                        cudaStream_t stream, const void* o_lat_lo, void* out_lo) {
  CUtensorMap w, x, x2, o;
  const uint64_t h = uint64_t(heads), R = uint64_t(rows);
  const bool two = o_lat_lo != nullptr;
  if (two != (out_lo != nullptr)) return MLA_ERR_INVALID_ARG;
  if (!make_map(&w, w_kvb2, MLA_D_V, h * MLA_D_HEAD, 2 * MLA_D_V)) return MLA_ERR_CUDA;
  if (!make_map(&x, o_lat, h * MLA_D_V, R, 2 * h * MLA_D_V)) return MLA_ERR_CUDA;
  if (two && !make_map(&x2, o_lat_lo, h * MLA_D_V, R, 2 * h * MLA_D_V)) return MLA_ERR_CUDA;
  if (!make_map(&o, out, h * MLA_D_HEAD, R, 2 * h * MLA_D_HEAD)) return MLA_ERR_CUDA;
  ProjArgs a;
  a.w_rows_per_head = MLA_D_HEAD;
  a.x_cols_per_head = MLA_D_V;
  a.o_cols_per_head = MLA_D_HEAD;
  a.rows = rows;
  a.heads = heads;
  a.rope_src = nullptr;
  a.rope_dst = nullptr;
  a.status = status;
  a.o_lo = static_cast<__nv_bfloat16*>(out_lo);
  a.m_tiles = MLA_D_HEAD / kTileM;
  return two ? launch_proj<MLA_D_V / 64, true>(w, x, x2, o, a, stream)
             : launch_proj<MLA_D_V / 64, false>(w, x, x, o, a, stream);
}

}  // namespace mla
