// tcgen05 decode kernel for B200 (sm_100a): MLA decode in absorbed latent
// space ("MLA Cost Analysis & Regime Guide", section "Absorption Trick":
// S = scale * Qz . C^T over the 576-d cache rows, O = softmax(S) . C[:, :512]).
//
// Why a CTA pair.  One tile is 128 (query token, head) rows.  Its fp32
// output accumulator, 128 x 512, is exactly the 256 KB of tensor memory
// (TMEM) of one SM, and its query block, 128 x 576 bf16 = 144 KB, does not
// fit beside a useful KV ring in shared memory.  So the work of a tile is
// split by role across the two SMs of a 2-CTA cluster, each doing
// full-width (M = 128) MMAs and no math twice:
//
//   CTA 0 ("score"): the query rows live in its TMEM (288 columns) as the A
//     operand of S = Q . C^T.  Keys are taken two pages (128 tokens) at a
//     time, because an N=64 MMA runs at about half the tensor core's rate
//     and N=128 at full rate.  One TMA warp streams the query rows and then
//     each 2-page block through an 11-deep ring of 16 KB stages (one 64-column
//     box of both pages, 128-byte swizzle) and bulk-prefetches later pages
//     into L2.  One thread issues 36 MMAs of M=128, N=128, K=16 per block
//     into a 128-column TMEM accumulator.  Two warpgroups run the online
//     softmax, one page each (thread = row), exchanging the row max and sum
//     through shared memory; the running max is lazy (it moves only when a
//     block's max exceeds it by 8 in log2 units, so P <= 256 fits fp16).
//     They write P (fp16, in the output CTA's swizzled layout) and per-row
//     rescale factors to a staging buffer, which one thread ships to the
//     output CTA with a single bulk copy over distributed shared memory.
//   CTA 1 ("output"): O (128 x 512 fp32) fills its TMEM.  Its own TMA warp
//     streams each page's 512 value columns (8 boxes, 128-byte swizzle, which
//     is the N-major operand layout) through a 3-deep ring; eight converter
//     warps rewrite each landed stage in place from bf16 to fp16 (exact in
//     fp16's normal range).  Each SM ingests at most ~60 GB/s, so both CTAs
//     keep ~190 KB of loads in flight.  One thread issues
//     O += P . V (M=128, N=256, K=16, twice per 16 tokens) page by page; a
//     warpgroup applies the rare rescales to O between blocks and writes the
//     normalised result at the end of a piece.
//
// P is fp16 rather than bf16 because rounding P to bf16 alone costs about
// 1e-3 of relative L1 error in O; fp16 keeps it near 2e-4.  The MMA needs
// both operands of one type, hence the fp16 copy of V.
//
// FP8 cache (kFp8): the score CTA's ring carries the cache's e4m3 latent
// columns as they are, and the latent scores run as kind::f8f6f4 MMAs
// against a two-part e4m3 copy of the query (hi + lo with a per-row
// power-of-two scale, which reproduces the bf16 query); the RoPE part
// stays a bf16 MMA.  The output CTA expands each page's e4m3 values, times
// their per-token scales, to fp16 in place.
//
// Every wait is bounded: a wait that runs out sets a status bit in the
// workspace, tells the peer CTA to stop, and the kernel drains its
// in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "decode_launch.cuh"
#include "kernel_util.cuh"
#include "sm100_ptx.cuh"

namespace mla {

namespace {

using namespace ptx;

// Score CTA ring.  BF16 cache: 5 stages of 32 KB, each two 64-column boxes
// of both pages (the ninth box, the RoPE columns, alone in the fifth), so
// the QK issuer waits once per 8 MMAs: each wait in the issuing thread idles
// the tensor pipe, whose queue holds only a few MMAs.  FP8 cache: 6 stages
// of 16 KB (query, e4m3 and RoPE stages; 10 measured no faster).
constexpr int NZ = 5;
constexpr int NZ8 = 6;
constexpr int kNZMax = 6;
// P page slots (output CTA): slot 0 takes page 0 of a block with the block's
// rescale factors and row sums, slot 1 its page 1.  Each is refilled as soon
// as its own page's PVs completed, so the next block's page 0 crosses over
// while this block's page 1 is multiplied.
constexpr int NX = 2;
constexpr int NV = 3;   // V page stages (output CTA): its own TMA ring
// Per-block PV completion barriers for the correction warpgroup.  It may lag
// the MMAs by up to three blocks (a block's P arrives once PV of block - 2
// completed), so a ring of four keeps every parity wait unambiguous.
constexpr int NB = 4;
// L2 bulk-prefetch distance in pages (0 disables the prefetch).
#ifndef MLA_PREFETCH_PAGES
#define MLA_PREFETCH_PAGES 0
#endif
constexpr int kPrefetchPages = MLA_PREFETCH_PAGES;
constexpr int kThreads = 512;
constexpr uint32_t kBox = 8192;                       // 64 rows x 128 B
constexpr uint32_t kZStage = 2 * kBox;                // one 64-column box of both pages (128 rows)
constexpr uint32_t kPageBytes = 9 * kBox;             // 64 tokens x 576 bf16
constexpr uint32_t kVStage = 8 * kBox;                // 64 tokens x 512 fp16
constexpr uint32_t kPPage = 128 * 64 * 2;             // 128 rows x 64 fp16 (one page of P)
constexpr uint32_t kMetaBytes = 1024;                 // alpha[128], l[128]
constexpr uint32_t kPSlot0 = kPPage + kMetaBytes;     // page 0 and the block's meta
constexpr uint32_t kPStage = kPSlot0 + kPPage;        // both slots; also the score CTA's staging
constexpr uint32_t kTmemS = 384;                      // S accumulator: columns 384..511
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kEvRescale = 1, kEvEnd = 2;        // correction events (Bars::ev_type)        // a wait gives up after 2 s
constexpr float kLazyMax = 8.0f;                      // log2 units
constexpr int kConvThreads = 256;                     // output-CTA converter warps (conv_rank)
constexpr int kSmThreads = 256;                       // score-CTA warps 4..11
constexpr uint32_t kSoftmaxBar = 1;                   // named barrier of the softmax warps
constexpr uint32_t kConvBar = 2;                      // named barrier of a CTA's converter warps
constexpr uint32_t kFp8PageBytes = 64 * 512 + 64 * 64 * 2;   // 64x512 e4m3, then 64x64 bf16 RoPE
constexpr uint32_t kTmemSLat = 256;                   // FP8 cache: latent-part scores, columns 256..383
constexpr uint32_t kTmemQLo = 128;                    // FP8 cache: the query's e4m3 lo part, columns 128..255

struct Bars {
  // score CTA (FP8 cache: also the query RoPE buffer)
  uint64_t z_full[kNZMax], z_empty[kNZMax], s_full, s_empty, q_ready, x_free[NX];
  uint64_t qpe_full, qpe_empty;
  uint64_t never;   // test hook: a barrier nothing arrives on (Params::test_stall)
  // output CTA
  uint64_t v_loaded[NV], v_full[NV], pv_done[NV], p_full[NX], corr_go, corr_done, pv_blk[NB], o_free;
  // correction events, from the PV issuer warp to the correction warpgroup:
  // a block's rescale factors (O must be rescaled before its PVs) or, at the
  // end of a piece, its row sums (normalise and store O)
  uint32_t ev_type, ev_blk;
  alignas(16) float ev_val[128];
  // both
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort;
};

constexpr uint32_t kOffData = 1024;
// score CTA.  BF16 cache: ring | P staging | exchange.  FP8 cache: ring |
// query RoPE columns (128 rows x 64, one 16 KB stage) | P staging |
// exchange | per-token scales of the block's two pages | half-row maxima of
// the query.
template <bool kFp8>
struct LayS {
  static constexpr int nz = kFp8 ? NZ8 : NZ;
  static constexpr uint32_t zbytes = kFp8 ? kZStage : 2 * kZStage;   // bytes per ring stage
  static constexpr uint32_t z = kOffData;
  static constexpr uint32_t qpe = z + nz * zbytes;
  static constexpr uint32_t stage = qpe + (kFp8 ? kZStage : 0u);
  static constexpr uint32_t xchg = stage + kPStage;               // row max / sum exchange
  static constexpr uint32_t scales = xchg + 4 * 128 * 4;           // FP8: 2 x 64 fp32
  static constexpr uint32_t qam = scales + (kFp8 ? 2 * 64 * 4 : 0u);   // FP8: 2 x 128 fp32 half-row maxima
  static constexpr uint32_t end = qam + (kFp8 ? 2 * 128 * 4 : 0u);
};
constexpr uint32_t kSmemS = LayS<false>::end > LayS<true>::end ? LayS<false>::end : LayS<true>::end;
// output CTA
constexpr uint32_t kOffV = kOffData;
constexpr uint32_t kOffP = kOffV + NV * kVStage;              // P + meta block stages
constexpr uint32_t kSmemO = kOffP + kPStage;
constexpr uint32_t kSmemBytes = (kSmemS > kSmemO ? kSmemS : kSmemO) + 1024;  // + alignment slack
static_assert(sizeof(Bars) <= kOffData, "barrier block");
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kPSlot0 % 1024 == 0 && kPStage % 1024 == 0 && kZStage % 1024 == 0,
              "swizzle atoms need 1024-byte alignment");
static_assert(LayS<true>::qpe % 1024 == 0 && LayS<true>::stage % 1024 == 0, "align");

// Instruction descriptors (kind::f16, fp32 accumulate, M = 128).
//   QK: A = Q bf16 (TMEM), B = cache rows bf16 K-major, N = 128
//   PV: A = P fp16 K-major (smem), B = V fp16 N-major (smem), N = 256
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) | ((256u >> 3) << 17) |
                              ((128u >> 4) << 24);
//   FP8 cache, latent part (kind::f8f6f4): A = the query's e4m3 hi or lo part
//   (TMEM), B = the cache's e4m3 rows K-major, N = 128
constexpr uint32_t kIdescQK8 = (1u << 4) | (0u << 7) | (0u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory matrix descriptor, 128-byte swizzle.  lbo / sbo in bytes.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((addr >> 4) & 0x3FFF) | (uint64_t((lbo >> 4) & 0x3FFF) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

struct Params {
  const uint16_t* q;
  const uint8_t* kv;
  const float* kv_scale;   // FP8 cache: per-token scales [pages][64]
  const int32_t* block_table;
  const int32_t* seqlens;
  const void* sched;
  void* ws;
  __nv_bfloat16* out;
  __nv_bfloat16* out_lo;   // optional: out_lo = bf16(O - out), so out + out_lo carries O to ~2^-17
  float* lse;
  float scale_log2;   // softmax_scale * log2(e)
  int num_pages;
  int cap_slots;
  int q_rows;         // batch * s_q * heads
  int test_stall;     // test hook, 0 in every product call (see the QK issuer)
};


struct Ctl {
  volatile int32_t* abort;
  uint32_t peer_abort;
  void* ws;
};

__device__ __noinline__ void trip(const Ctl& c) {
  *c.abort = 1;
  st_cluster_u32(c.peer_abort, 1);
  flag_status(c.ws, kStatusTimeout);
}

// Bounded wait on an mbarrier phase; false when this CTA is aborting.
// kCluster selects cluster-scope acquire (barriers the peer CTA arrives on).
// kSpin polls with test_wait (no suspension: for the single threads that
// feed the tensor core and the copy engine); otherwise try_wait, which lets
// the hardware suspend a waiting warp between polls.
template <bool kCluster = false, bool kSpin = false>
__device__ __forceinline__ bool bwait(const Ctl& c, uint32_t bar, uint32_t parity) {
  auto try_once = [&] {
    if (kSpin) return kCluster ? mbar_test_wait_cluster(bar, parity) : mbar_test_wait(bar, parity);
    return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity);
  };
  if (try_once()) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (try_once()) return true;
    if ((n & 15) == 0) {
      if (*c.abort) return false;
      if (globaltimer() - t0 > kTimeoutNs) {
        trip(c);
        return false;
      }
    }
  }
}

// Pipeline-driver wait: a spinning bwait.
template <bool kCluster = false>
__device__ __forceinline__ bool swait(const Ctl& c, uint32_t bar, uint32_t parity) {
  return bwait<kCluster, true>(c, bar, parity);
}

// Warp-uniform bounded wait: lane 0 polls, the warp follows its verdict.
// __syncwarp orders the other lanes' later accesses after lane 0's acquire.
template <bool kCluster = false>
__device__ __forceinline__ bool wwait(const Ctl& c, uint32_t bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = bwait<kCluster>(c, bar, parity);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  return ok;
}

// Issuer-warp bounded wait: every lane polls without suspending (each lane
// holds its own acquire) and the warp leaves together.
template <bool kCluster = false>
__device__ __forceinline__ bool ewait(const Ctl& c, uint32_t bar, uint32_t parity) {
  auto once = [&] { return kCluster ? mbar_test_wait_cluster(bar, parity) : mbar_test_wait(bar, parity); };
  if (__all_sync(0xffffffffu, once())) return true;
  const bool lead = (threadIdx.x & 31) == 0;
  const uint64_t t0 = lead ? globaltimer() : 0ull;
  for (uint32_t n = 1;; ++n) {
    if (__all_sync(0xffffffffu, once())) return true;
    if ((n & 15) == 0) {
      const int stop = __shfl_sync(0xffffffffu, lead ? (*c.abort ? 1 : (globaltimer() - t0 > kTimeoutNs ? 2 : 0)) : 0, 0);
      if (stop != 0) {
        if (stop == 2 && lead) trip(c);
        return false;
      }
    }
  }
}

// Softmax-group bounded wait: the group's first thread polls, the named
// barrier hands its verdict (and, through the barrier, its acquire) to the
// other 255 threads, and the group decides together (a thread leaving alone
// would strand the others at the group's named barrier).  `carried` is the
// poller's verdict on an earlier wait the group did not wait for.
__device__ __forceinline__ bool gwait(const Ctl& c, uint32_t bar, uint32_t parity, bool poller, bool carried = true) {
  bool ok = true;
  if (poller) ok = carried && bwait(c, bar, parity);
  return named_bar_and(kSoftmaxBar, kSmThreads, ok);
}

// Bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (globaltimer() - t0 > kTimeoutNs) return;
  }
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two e4m3 bytes (low byte first) -> two fp16 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return uint32_t(h.x) | (uint32_t(h.y) << 16);
}

// The same, times a per-token scale (fp16 product, one rounding).
__device__ __forceinline__ uint32_t e4m3x2_scaled(uint32_t two, __half2 scale) {
  const uint32_t w = e4m3x2_to_f16x2(two);
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&w), scale);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Running max of |h| over fp16 pairs, NaN-propagating: a converted V value
// that left fp16's finite range (a bf16 value of magnitude 65520 or more, an
// infinite or NaN input, an FP8 value times a scale above the range) leaves
// an infinity or a NaN here.
__device__ __forceinline__ void track_absmax(__half2& acc, uint32_t w) {
  acc = __hmax2_nan(acc, __habs2(*reinterpret_cast<const __half2*>(&w)));
}

__device__ __forceinline__ bool absmax_finite(__half2 acc) {
  const float2 f = __half22float2(acc);
  return f.x <= 65504.f && f.y <= 65504.f;   // false for inf and NaN
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f8f6f4 (the FP8 cache's latent scores).
__device__ __forceinline__ void mma_ts_f8(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// 16 consecutive 32-bit columns of this thread's lane (32x32b shape).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Largest |value| of the two bf16 values of w.
__device__ __forceinline__ float bf16_abs_max(uint32_t w) {
  return fmaxf(fabsf(__uint_as_float(w << 16)), fabsf(__uint_as_float(w & 0xFFFF0000u)));
}

// e with am / 2^e <= 448 (e4m3's largest finite value), the smallest such
// but at least -126, so that 2^-e stays finite (a row that small loses
// nothing that matters: its values still land in e4m3's range); 0 for
// am = 0 or a non-finite am (its NaN or infinity then reaches S as is).
// frexpf gives the estimate; the loops correct it by at most a few steps
// (at most 126 for a subnormal am) and always end.
__device__ __forceinline__ int pow2_scale_exp(float am) {
  if (!(am > 0.f) || !(am <= 3.402823466e38f)) return 0;
  int e = 0;
  frexpf(am * (1.f / 448.f), &e);   // am / 448 = m 2^e, 0.5 <= m < 1
  while (ldexpf(am, -e) > 448.f) ++e;
  while (e > -126 && ldexpf(am, -(e - 1)) <= 448.f) --e;
  return e < -126 ? -126 : e;
}

// Four bf16 values (w01, w23, low half first) times `inv` (a power of two)
// as e4m3 hi = RNE(x) and lo = RNE(x - hi), four bytes each, value 4k+j in
// byte j.  x - hi is exact in fp32.
__device__ __forceinline__ void split_e4m3x4(uint32_t w01, uint32_t w23, float inv, uint32_t* hi, uint32_t* lo) {
  const float2 a = make_float2(__uint_as_float(w01 << 16) * inv, __uint_as_float(w01 & 0xFFFF0000u) * inv);
  const float2 b = make_float2(__uint_as_float(w23 << 16) * inv, __uint_as_float(w23 & 0xFFFF0000u) * inv);
  const __nv_fp8x2_storage_t ha = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hb = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
  const float2 fa = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(ha, __NV_E4M3)));
  const float2 fb = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(hb, __NV_E4M3)));
  const __nv_fp8x2_storage_t la = __nv_cvt_float2_to_fp8x2(make_float2(a.x - fa.x, a.y - fa.y), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t lb = __nv_cvt_float2_to_fp8x2(make_float2(b.x - fb.x, b.y - fb.y), __NV_SATFINITE, __NV_E4M3);
  *hi = uint32_t(ha) | (uint32_t(hb) << 16);
  *lo = uint32_t(la) | (uint32_t(lb) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// (a, b) -> bf16 pairs hi = (bf16(a), bf16(b)) and lo = bf16 of the
// remainders (a - hi_a, b - hi_b; exact in fp32).
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t* hi, uint32_t* lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  *hi = *reinterpret_cast<const uint32_t*>(&h);
  *lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// BF16 cache: V chunks per converter thread loaded together before their
// stores (decode launch at b=64, h=128, t=4096: 116.7 us one at a time,
// 111.4 us in groups of 4, 112.6 us with 8, 117.8 us with 16).
constexpr int kConvGroup = 4;

// Output CTA: the eight converter warps (-1 for other warps).  None shares a
// scheduler sub-partition (warp % 4) with the PV issuer (warp 1): their
// bursts of shared-memory loads would delay the issuer's barrier polls.
__device__ __forceinline__ int conv_rank(int warp) {
  switch (warp) {
    case 2: return 0;
    case 3: return 1;
    case 8: return 2;
    case 10: return 3;
    case 11: return 4;
    case 12: return 5;
    case 14: return 6;
    case 15: return 7;
    default: return -1;
  }
}

// Calls f(piece) for every piece of every worker this cluster owns; stops
// when f returns false.  Returns true when every call returned true.
template <class F>
__device__ __forceinline__ bool each_piece(const SchedView& sv, F&& f) {
  const int ncl = int(nclusters_x());
  for (int w = int(cluster_id_x()); w < sv.W; w += ncl) {
    PieceIter it(sv, w);
    Piece pc;
    while (it.next(&pc))
      if (!f(pc)) return false;
  }
  return true;
}

__device__ __forceinline__ int clamp_len(int t, const SchedView& sv) {
  return max(0, min(t, sv.max_pages * MLA_PAGE_SIZE));
}

// kFp8: the cache pages hold e4m3 latent values with per-token scales and a
// bf16 RoPE part (pool_map covers the e4m3 bytes, rope_map the RoPE values);
// otherwise pool_map covers bf16 rows and rope_map is not used.
template <bool kFp8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_sm100_kernel(const __grid_constant__ CUtensorMap pool_map, const __grid_constant__ CUtensorMap q_map,
                    const __grid_constant__ CUtensorMap rope_map, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  Bars* bars = reinterpret_cast<Bars*>(gbase);
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();

  if (tid == 0) {
    // FP8 cache: a ring stage is refilled once the softmax and the issuer
    // have each released it (see the issuer)
    for (int s = 0; s < kNZMax; ++s) {
      mbar_init(bar(bars->z_full[s]), 1);
      mbar_init(bar(bars->z_empty[s]), kFp8 ? 2 : 1);
    }
    mbar_init(bar(bars->s_full), 1);
    mbar_init(bar(bars->s_empty), kSmThreads);
    mbar_init(bar(bars->q_ready), kSmThreads);
    for (int s = 0; s < NX; ++s) {
      mbar_init(bar(bars->x_free[s]), 1);
      mbar_init(bar(bars->p_full[s]), 1);
    }
    mbar_init(bar(bars->corr_go), 32);
    mbar_init(bar(bars->corr_done), 128);
    for (int s = 0; s < NV; ++s) {
      mbar_init(bar(bars->v_loaded[s]), 1);
      mbar_init(bar(bars->v_full[s]), kConvThreads);
      mbar_init(bar(bars->pv_done[s]), 1);
    }
    for (int s = 0; s < NB; ++s) mbar_init(bar(bars->pv_blk[s]), 1);
    mbar_init(bar(bars->qpe_full), 1);
    mbar_init(bar(bars->qpe_empty), 1);
    mbar_init(bar(bars->never), 1);
    mbar_init(bar(bars->o_free), 128);
    mbar_init(bar(bars->mma_done), 1);
    bars->abort = 0;
    fence_mbar_init();
    // the output CTA arms its P slots for their first bulk copies
    if (rank == 1) {
      mbar_arrive_expect_tx(bar(bars->p_full[0]), kPSlot0);
      mbar_arrive_expect_tx(bar(bars->p_full[1]), kPPage);
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&pool_map);
    if (rank == 0) tma_prefetch_desc(&q_map);
    if (kFp8 && rank == 0) tma_prefetch_desc(&rope_map);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  cluster_sync();
  // everything above overlaps the scheduler kernel still running before us
  // (programmatic dependent launch); its schedule is read from here on
  griddep_wait();
  griddep_launch_dependents();
  const SchedView sv(p.sched);
  const int rows_total = sv.s_q * sv.heads;

  Ctl ctl{&bars->abort, mapa(smem_u32(&bars->abort), rank ^ 1u), p.ws};

  if (rank == 0) {
    // ======================= score CTA =======================
    using L = LayS<kFp8>;
    constexpr int nz = L::nz;
    if (warp == 0) {
      // ---- TMA producer warp (one lane issues).  BF16 cache: 9 query
      // stages per piece, then 9 per 2-page block.  FP8 cache: 8 query
      // stages (latent columns) plus the query RoPE columns into their own
      // buffer per piece, then per block one RoPE stage (bf16) and 4 e4m3
      // stages of 128 latent columns.  A block's page ids are read one block
      // ahead, so their load latency hides behind the previous block's
      // stages.
      {
        const bool leader = elect_one();
        uint32_t zc = 0, pieces = 0;
        auto page_of = [&](int r, int j) {
          int page = p.block_table[size_t(r) * sv.max_pages + j];
          return (page < 0 || page >= p.num_pages) ? -1 : page;
        };
        auto stage = [&](uint32_t tx, uint32_t* dst) -> bool {
          const uint32_t s = zc % nz, ph = (zc / nz) & 1u;
          if (!ewait(ctl, bar(bars->z_empty[s]), ph ^ 1u)) return false;
          if (leader) {
            mbar_arrive_expect_tx(bar(bars->z_full[s]), tx);
          }
          *dst = sbase + L::z + s * L::zbytes;
          return true;
        };
        each_piece(sv, [&](const Piece& pc) {
          const int r = pc.T / sv.tiles_per_req, qt = pc.T % sv.tiles_per_req;
          const int row0 = r * rows_total + qt * MLA_TILE_ROWS;
          int npa = page_of(r, pc.p0), npb = pc.p0 + 1 < pc.p1 ? page_of(r, pc.p0 + 1) : 0;
          if (leader)
            prefetch_l2_bulk(p.q + size_t(row0) * MLA_D_QK,
                             uint32_t(min(MLA_TILE_ROWS, p.q_rows - row0)) * MLA_D_QK * 2);
          // query boxes: FP8 cache one per stage (8), BF16 cache two per
          // stage (9 in 5 stages)
          constexpr int nqs = kFp8 ? 8 : 5, qbs = kFp8 ? 1 : 2;
          for (int q = 0; q < nqs; ++q, ++zc) {
            const int nb = kFp8 ? 1 : (q < 4 ? 2 : 1);
            uint32_t dst;
            if (!stage(uint32_t(nb) * kZStage, &dst)) return false;
            const uint32_t fb = bar(bars->z_full[zc % nz]);
            if (leader) {
              for (int k = 0; k < nb; ++k) {
                const int c = qbs * q + k;
                tma_load_2d(dst + uint32_t(k) * kZStage, &q_map, 64 * c, row0, fb);
                tma_load_2d(dst + uint32_t(k) * kZStage + kBox, &q_map, 64 * c, row0 + 64, fb);
              }
            }
            __syncwarp();
          }
          if constexpr (kFp8) {
            // the RoPE MMAs of the previous piece must be done with the buffer
            if (!ewait(ctl, bar(bars->qpe_empty), (pieces & 1u) ^ 1u)) return false;
            const uint32_t fb = bar(bars->qpe_full);
            if (leader) {
              mbar_arrive_expect_tx(fb, kZStage);
              tma_load_2d(sbase + L::qpe, &q_map, MLA_D_V, row0, fb);
              tma_load_2d(sbase + L::qpe + kBox, &q_map, MLA_D_V, row0 + 64, fb);
            }
            __syncwarp();
          }
          ++pieces;
          for (int j = pc.p0; j < pc.p1; j += 2) {
            const bool two = j + 1 < pc.p1;
            if constexpr (!kFp8) {
              for (int u = 0; u < 2; ++u)
                if (kPrefetchPages > 0 && j + u + kPrefetchPages < pc.p1) {
                  const int pg = page_of(r, j + u + kPrefetchPages);
                  if (pg >= 0 && leader) prefetch_l2_bulk(p.kv + size_t(pg) * kPageBytes, kPageBytes);
                }
            }
            int pa = npa, pb = two ? npb : 0;
            if (j + 2 < pc.p1) {
              npa = page_of(r, j + 2);
              npb = j + 3 < pc.p1 ? page_of(r, j + 3) : 0;
            }
            if ((pa < 0 || pb < 0) && leader) flag_status(p.ws, kStatusBadPage);
            pa = max(pa, 0);     // any valid page; the consumers mask every token of it
            pb = max(pb, 0);
            if constexpr (kFp8) {
              uint32_t dst;
              if (!stage(two ? kZStage : kBox, &dst)) return false;
              uint32_t fb = bar(bars->z_full[zc % nz]);
              if (leader) {
                tma_load_3d(dst, &rope_map, 0, 0, pa, fb);
                if (two) tma_load_3d(dst + kBox, &rope_map, 0, 0, pb, fb);
              }
              __syncwarp();
              ++zc;
              for (int c = 0; c < 4; ++c, ++zc) {
                if (!stage(two ? kZStage : kBox, &dst)) return false;
                fb = bar(bars->z_full[zc % nz]);
                if (leader) {
                  tma_load_3d(dst, &pool_map, 128 * c, 0, pa, fb);
                  if (two) tma_load_3d(dst + kBox, &pool_map, 128 * c, 0, pb, fb);
                }
                __syncwarp();
              }
            } else {
              // stage q: boxes 2q and 2q + 1 (box 8 alone), each both pages
              for (int q = 0; q < 5; ++q, ++zc) {
                const int nb = q < 4 ? 2 : 1;
                uint32_t dst;
                if (!stage(uint32_t(nb) * (two ? kZStage : kBox), &dst)) return false;
                const uint32_t fb = bar(bars->z_full[zc % nz]);
                if (leader) {
                  for (int k = 0; k < nb; ++k) {
                    const int c = 2 * q + k;
                    tma_load_3d(dst + uint32_t(k) * kZStage, &pool_map, 64 * c, 0, pa, fb);
                    if (two) tma_load_3d(dst + uint32_t(k) * kZStage + kBox, &pool_map, 64 * c, 0, pb, fb);
                  }
                }
                __syncwarp();
              }
            }
          }
          return true;
        });
        // copies still in flight must land before the CTA can leave
        const uint32_t n = zc < uint32_t(nz) ? zc : uint32_t(nz);
        for (uint32_t k = 1; k <= n; ++k) {
          const uint32_t idx = zc - k;
          drain_wait(bar(bars->z_full[idx % nz]), (idx / nz) & 1u);
        }
        if (kFp8 && pieces > 0) drain_wait(bar(bars->qpe_full), (pieces - 1) & 1u);
      }
    } else if (warp == 1) {
      // ---- QK^T issuer warp: per block 36 MMAs M128 N128 K16.  BF16 cache: 5
      // stages of 2 boxes (the last 1) x 4 MMAs, A = Q (TMEM), into S.  FP8 cache: the RoPE stage x 4 with
      // A = the query RoPE columns (shared memory) into S_rope, then the 4
      // e4m3 stages x (4 + 4) kind::f8f6f4 MMAs with A = the query's e4m3 hi
      // and lo parts (TMEM) into S_lat.
      // The warp waits and computes operands together; one lane issues.
      const bool leader = elect_one();
      const uint64_t zdesc0 = sdesc(sbase + L::z, 16, 1024);
      const uint64_t qdesc = sdesc(sbase + L::qpe, 16, 1024);
      uint32_t zc = 0, bc = 0, pieces = 0;
      each_piece(sv, [&](const Piece& pc) {
        // test hook (set only by the test library's stalled-decode entry
        // point): a wait on a barrier nothing arrives on runs out, and the
        // abort path (status bit, peer abort, drains, TMEM freed) runs
        if (p.test_stall && !ewait(ctl, bar(bars->never), 0)) return false;
        // FP8 cache: the ring is shorter than the query, so its stages are
        // released one by one.  This warp walks every stage of the ring in
        // order (a parity wait is only sound when the stage's previous use
        // has completed), and a stage is refilled after two releases: softmax
        // and issuer.  For the RoPE and e4m3 stages, which the softmax never
        // sees, the issuer releases twice.
        constexpr int nq = kFp8 ? 8 : 5;   // ring stages of the query
        if constexpr (kFp8) {
          for (int u = 0; u < nq; ++u, ++zc) {
            if (!ewait(ctl, bar(bars->z_full[zc % nz]), (zc / nz) & 1u)) return false;
            if (leader) mbar_arrive(bar(bars->z_empty[zc % nz]));
          }
        }
        if (!ewait(ctl, bar(bars->q_ready), pieces & 1u)) return false;
        if (kFp8 && !ewait(ctl, bar(bars->qpe_full), pieces & 1u)) return false;
        ++pieces;
        // the query rows are in TMEM: release their stages
        if constexpr (!kFp8) {
          if (leader)
            for (int u = 0; u < nq; ++u) mbar_arrive(bar(bars->z_empty[(zc + u) % nz]));
          zc += nq;
        }
        tc_fence_after();
        for (int j = pc.p0; j < pc.p1; j += 2, ++bc) {
          if (!ewait(ctl, bar(bars->s_empty), (bc & 1u) ^ 1u)) return false;
          tc_fence_after();
          if constexpr (kFp8) {
            {
              const uint32_t zs = zc % nz;
              if (!ewait(ctl, bar(bars->z_full[zs]), (zc / nz) & 1u)) return false;
              tc_fence_after();
              const uint64_t bd = zdesc0 + uint64_t(zs * (kZStage >> 4));
              const uint32_t d = tmem + kTmemS;
              if (leader) {
                mma_ss(d, qdesc, bd, kIdescQK, 0u);
                mma_ss(d, qdesc + 2u, bd + 2u, kIdescQK, 1u);
                mma_ss(d, qdesc + 4u, bd + 4u, kIdescQK, 1u);
                mma_ss(d, qdesc + 6u, bd + 6u, kIdescQK, 1u);
                mma_commit(bar(bars->z_empty[zs]));    // the issuer's release, when the MMAs are done
                mbar_arrive(bar(bars->z_empty[zs]));   // the softmax's
              }
              __syncwarp();
              ++zc;
            }
            // the four e4m3 stages, straight from the cache: S_lat =
            // Q_hi . K + Q_lo . K, 4 + 4 MMAs of K = 32 per stage
            for (int e = 0; e < 4; ++e, ++zc) {
              const uint32_t zs = zc % nz;
              if (!ewait(ctl, bar(bars->z_full[zs]), (zc / nz) & 1u)) return false;
              tc_fence_after();
              const uint64_t bd = zdesc0 + uint64_t(zs * (kZStage >> 4));
              const uint32_t d = tmem + kTmemSLat;
              if (leader) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  mma_ts_f8(d, tmem + 32u * e + 8u * k, bd + 2u * k, kIdescQK8, (e | k) != 0 ? 1u : 0u);
                  mma_ts_f8(d, tmem + kTmemQLo + 32u * e + 8u * k, bd + 2u * k, kIdescQK8, 1u);
                }
                mma_commit(bar(bars->z_empty[zs]));    // the issuer's release, when the MMAs are done
                mbar_arrive(bar(bars->z_empty[zs]));   // the softmax's
              }
              __syncwarp();
            }
          } else {
            for (int q = 0; q < 5; ++q, ++zc) {
              const uint32_t zs = zc % nz;
              if (!ewait(ctl, bar(bars->z_full[zs]), (zc / nz) & 1u)) return false;
              tc_fence_after();
              const uint32_t d = tmem + kTmemS;
              if (leader) {
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                  const int c = 2 * q + k;
                  if (c < 9) {
                    const uint64_t bd = zdesc0 + uint64_t((zs * L::zbytes + uint32_t(k) * kZStage) >> 4);
                    const uint32_t ad = tmem + 32u * uint32_t(c);
                    mma_ts(d, ad, bd, kIdescQK, c != 0);
                    mma_ts(d, ad + 8u, bd + 2u, kIdescQK, 1u);
                    mma_ts(d, ad + 16u, bd + 4u, kIdescQK, 1u);
                    mma_ts(d, ad + 24u, bd + 6u, kIdescQK, 1u);
                  }
                }
                mma_commit(bar(bars->z_empty[zs]));
              }
              __syncwarp();
            }
          }
          if (leader) {
            mma_commit(bar(bars->s_full));
          }
          __syncwarp();
        }
        if (kFp8 && leader) mma_commit(bar(bars->qpe_empty));   // the piece's RoPE MMAs are done with the buffer
        __syncwarp();
        return true;
      });
      if (leader) mma_commit(bar(bars->mma_done));
      __syncwarp();
      drain_wait(bar(bars->mma_done), 0);
    } else if (warp >= 4 && warp < 12) {
      // ---- softmax: two warpgroups; thread (h, i) owns row i of the tile
      // (TMEM lane i) for page h of each 2-page block
      const int g = tid - 128, h = g >> 7, i = g & 127, wq = warp & 3;
      const uint32_t lane_off = uint32_t(wq * 32) << 16;
      const uint32_t o_p = mapa(sbase + kOffP, 1);
      const uint32_t o_pfull = mapa(bar(bars->p_full[0]), 1);
      const uint32_t stg = sbase + L::stage;
      const uint32_t xmax = sbase + L::xchg, xsum = xmax + 2 * 128 * 4;
      const uint32_t scl = sbase + L::scales + uint32_t(h) * 256;   // FP8: this page's 64 scales
      uint32_t zc = 0, bc = 0, n1 = 0;   // n1: blocks with two pages so far (uses of slot 1)
      bool carry_ok = true;
      each_piece(sv, [&](const Piece& pc) {
        const int r = pc.T / sv.tiles_per_req, qt = pc.T % sv.tiles_per_req;
        const int rho = qt * MLA_TILE_ROWS + i;
        const bool valid = rho < rows_total;
        const int t = clamp_len(p.seqlens[r], sv);
        const int Lrow = valid ? visible_len(t, sv.s_q, rho / sv.heads, sv.causal) : 0;
        // query row i -> TMEM lane i.  Box c of the query (rows 0-63, then
        // 64-127 at +8 KB) is sub-stage c % qbs of stage zc + c / qbs.  BF16
        // cache: boxes 0-8, two per stage, as bf16 pairs in columns [0, 288),
        // group 0 moves boxes 0-4, group 1 boxes 5-8.  FP8 cache: the latent
        // boxes 0-7, one per stage, 0-3 / 4-7, as two e4m3 parts (the RoPE
        // box stays in shared memory): with a power-of-two scale 2^e per row
        // that takes the row's largest |value| to at most 448, hi = e4m3(q /
        // 2^e) keeps 4 of bf16's 8 significant bits and lo = e4m3(q / 2^e -
        // hi) the rest, exactly (values below 2^-11 of the row's largest
        // lose at most 2^-19 of it).  hi in columns [0, 128), lo in [128,
        // 256), four values per column.  Every QK MMA of the previous piece
        // has completed: its last S was read.
        float qscale = 1.f;   // FP8 cache: the row's 2^e
        {
          constexpr int nq = kFp8 ? 8 : 9, nq0 = kFp8 ? 4 : 5, qbs = kFp8 ? 1 : 2;
          const uint32_t roff = uint32_t(i >> 6) * kBox + uint32_t(i & 63) * 128;
          float qinv = 1.f;
          if constexpr (kFp8) {
            // the row's largest |value|: each of its two threads reads half
            // of the latent part from global memory
            float am = 0.f;
            if (valid) {
              const uint16_t* qrow = p.q + (size_t(r) * rows_total + rho) * MLA_D_QK + 256 * h;
#pragma unroll 4
              for (int k = 0; k < 32; ++k) {
                const uint4 w = ld_global_nc_v4(qrow + 8 * k);
                am = fmaxf(am, fmaxf(fmaxf(bf16_abs_max(w.x), bf16_abs_max(w.y)),
                                     fmaxf(bf16_abs_max(w.z), bf16_abs_max(w.w))));
              }
            }
            const uint32_t qam = sbase + L::qam;
            st_shared_u32(qam + 4u * uint32_t(128 * h + i), __float_as_uint(am));
            named_bar_sync(kSoftmaxBar, kSmThreads);
            am = fmaxf(am, ld_shared_f32(qam + 4u * uint32_t(128 * (h ^ 1) + i)));
            const int e = pow2_scale_exp(am);
            qscale = ldexpf(1.f, e);
            qinv = ldexpf(1.f, -e);
          }
#pragma unroll 1
          for (int c = 0; c < nq; ++c) {
            const uint32_t idx = zc + uint32_t(c / qbs);
            if (c % qbs == 0)
              if (!gwait(ctl, bar(bars->z_full[idx % nz]), (idx / nz) & 1u, g == 0, carry_ok)) return false;
            // FP8 cache: every thread has passed the barrier, so the previous
            // query stage has been read: the producer may refill it
            if (kFp8 && c > 0 && g == 0) mbar_arrive(bar(bars->z_empty[(idx - 1) % nz]));
            if ((c < nq0) == (h == 0)) {
              const uint32_t st = sbase + L::z + (idx % nz) * L::zbytes + uint32_t(c % qbs) * kZStage + roff;
              uint32_t v[32];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const uint4 x = ld_shared_v4(st + ((uint32_t(k) ^ uint32_t(i & 7)) << 4));
                v[4 * k + 0] = x.x;
                v[4 * k + 1] = x.y;
                v[4 * k + 2] = x.z;
                v[4 * k + 3] = x.w;
              }
              if constexpr (kFp8) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) split_e4m3x4(v[2 * k], v[2 * k + 1], qinv, &hi[k], &lo[k]);
                tmem_st16(tmem + lane_off + 16u * c, hi);
                tmem_st16(tmem + lane_off + kTmemQLo + 16u * c, lo);
              } else {
                tmem_st32(tmem + lane_off + 32u * c, v);
              }
            }
          }
          if constexpr (kFp8) {
            named_bar_sync(kSoftmaxBar, kSmThreads);
            if (g == 0) mbar_arrive(bar(bars->z_empty[(zc + nq - 1) % nz]));
          }
          zc += (kFp8 ? 8u : 5u) + 5u * uint32_t((pc.p1 - pc.p0 + 1) / 2);   // query stages, then 5 per block
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(bars->q_ready));
        }
        float m = -INFINITY, l = 0.f;
        for (int j = pc.p0; j < pc.p1; j += 2, ++bc) {
          const int jp = j + h;                      // this thread's page
          int nv = 0, page = -1;                     // its visible tokens here
          if (jp < pc.p1) {
            page = p.block_table[size_t(r) * sv.max_pages + jp];
            if (page >= 0 && page < p.num_pages) nv = Lrow - jp * MLA_PAGE_SIZE;
            else page = -1;
          }
          if constexpr (kFp8) {
            // the page's per-token scales, published by the barrier below
            if (i < 64) st_shared_u32(scl + 4u * uint32_t(i), __float_as_uint(page >= 0 ? p.kv_scale[size_t(page) * 64 + i] : 0.f));
          }
          if (!gwait(ctl, bar(bars->s_full), bc & 1u, g == 0, carry_ok)) return false;
          tc_fence_after();
          float x[64];
          {
            uint32_t sv0[32], sv1[32];
            if constexpr (kFp8) {
              // S = 2^e * scale_j * S_lat + S_rope: S_lat is the scaled
              // query against the unscaled e4m3 values
              tmem_ld32(tmem + lane_off + kTmemSLat + 64u * h, sv0);
              tmem_ld32(tmem + lane_off + kTmemSLat + 64u * h + 32u, sv1);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                const uint4 s0 = ld_shared_v4(scl + 4u * uint32_t(c)), s1 = ld_shared_v4(scl + 128u + 4u * uint32_t(c));
                x[c] = __uint_as_float(sv0[c]) * (qscale * __uint_as_float(s0.x));
                x[c + 1] = __uint_as_float(sv0[c + 1]) * (qscale * __uint_as_float(s0.y));
                x[c + 2] = __uint_as_float(sv0[c + 2]) * (qscale * __uint_as_float(s0.z));
                x[c + 3] = __uint_as_float(sv0[c + 3]) * (qscale * __uint_as_float(s0.w));
                x[c + 32] = __uint_as_float(sv1[c]) * (qscale * __uint_as_float(s1.x));
                x[c + 33] = __uint_as_float(sv1[c + 1]) * (qscale * __uint_as_float(s1.y));
                x[c + 34] = __uint_as_float(sv1[c + 2]) * (qscale * __uint_as_float(s1.z));
                x[c + 35] = __uint_as_float(sv1[c + 3]) * (qscale * __uint_as_float(s1.w));
              }
              tmem_ld32(tmem + lane_off + kTmemS + 64u * h, sv0);
              tmem_ld32(tmem + lane_off + kTmemS + 64u * h + 32u, sv1);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                x[c] += __uint_as_float(sv0[c]);
                x[c + 32] += __uint_as_float(sv1[c]);
              }
            } else {
              tmem_ld32(tmem + lane_off + kTmemS + 64u * h, sv0);
              tmem_ld32(tmem + lane_off + kTmemS + 64u * h + 32u, sv1);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                x[c] = __uint_as_float(sv0[c]);
                x[c + 32] = __uint_as_float(sv1[c]);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(bar(bars->s_empty));
          float mh = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = c < nv ? x[c] * p.scale_log2 : -INFINITY;
            x[c + 32] = c + 32 < nv ? x[c + 32] * p.scale_log2 : -INFINITY;
            mh = fmaxf(mh, fmaxf(x[c], x[c + 32]));
          }
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(xmax + 4u * uint32_t(g)), "f"(mh) : "memory");
          // staging is free once the previous block's copy has read it
          if (g == 0) bulk_wait_group_read<0>();
          named_bar_sync(kSoftmaxBar, kSmThreads);
          const float mb = fmaxf(mh, ld_shared_f32(xmax + 4u * uint32_t(g ^ 128)));
          float m_new = m, alpha = 1.f;
          bool need = false;
          if (mb > m + kLazyMax) {
            m_new = mb;
            alpha = ex2(m - m_new);            // 0 when m = -inf
            need = (j != pc.p0) && (m != -INFINITY);
          }
          const bool live = m_new != -INFINITY;
          float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            x[c] = live ? ex2(x[c] - m_new) : 0.f;
            x[c + 1] = live ? ex2(x[c + 1] - m_new) : 0.f;
            x[c + 2] = live ? ex2(x[c + 2] - m_new) : 0.f;
            x[c + 3] = live ? ex2(x[c + 3] - m_new) : 0.f;
            s0 += x[c];
            s1 += x[c + 1];
            s2 += x[c + 2];
            s3 += x[c + 3];
          }
          const float ph = (s0 + s1) + (s2 + s3);
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(xsum + 4u * uint32_t(g)), "f"(ph) : "memory");
          const uint32_t prow = stg + uint32_t(h) * kPSlot0 + (i >> 3) * 1024 + (i & 7) * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            st_shared_v4(prow + ((uint32_t(k) ^ uint32_t(i & 7)) << 4), pack_f16(x[8 * k], x[8 * k + 1]),
                         pack_f16(x[8 * k + 2], x[8 * k + 3]), pack_f16(x[8 * k + 4], x[8 * k + 5]),
                         pack_f16(x[8 * k + 6], x[8 * k + 7]));
          named_bar_sync(kSoftmaxBar, kSmThreads);
          l = l * alpha + ph + ld_shared_f32(xsum + 4u * uint32_t(g ^ 128));
          m = m_new;
          if (h == 0) {
            st_shared_u32(stg + kPPage + 4 * i, __float_as_uint(need ? alpha : 1.f));
            st_shared_u32(stg + kPPage + 512 + 4 * i, __float_as_uint(l));
          }
          fence_proxy_async_cta();
          // publishes every staging write to thread 0, which ships page 0
          // (with the meta) and page 1 to the output CTA's slots, each once
          // the PVs of the previous block's same page completed.  A failed
          // wait is reported at the group's next barrier.
          named_bar_sync(kSoftmaxBar, kSmThreads);
          const bool two = j + 1 < pc.p1;
          if (g == 0) {
            bool ok = bwait<true>(ctl, bar(bars->x_free[0]), (bc & 1u) ^ 1u);
            if (ok) bulk_copy_to_peer(o_p, stg, kPSlot0, o_pfull);
            if (ok && two) {
              ok = bwait<true>(ctl, bar(bars->x_free[1]), (n1 & 1u) ^ 1u);
              if (ok) bulk_copy_to_peer(o_p + kPSlot0, stg + kPSlot0, kPPage, o_pfull + 8u);
            }
            bulk_commit_group();
            carry_ok = ok;
          }
          n1 += two ? 1u : 0u;
        }
        if (valid && h == 0) {
          const float lse_v = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
          if (sv.tile_splits(pc.T) == 1) {
            p.lse[size_t(r) * rows_total + rho] = lse_v;
          } else {
            const int slot = sv.tile_slot_base(pc.T) + pc.split;
            if (slot < p.cap_slots) ws_partial_lse(p.ws, p.cap_slots, slot)[i] = lse_v;
            else flag_status(p.ws, kStatusWorkspace);
          }
        }
        return true;
      });
      // no copy may still be in flight when the CTAs leave
      if (g == 0) bulk_wait_group_all();
    }
  } else {
    // ======================= output CTA =======================
    if (warp == 1) {
      // ---- PV issuer warp: per block, per page 4 K-steps x 2 N halves.  One
      // lane issues; the warp reads the block's rescale factors and hands
      // them to the correction warpgroup only when one of them is not 1.
      const bool leader = elect_one();
      const uint64_t pdesc0 = sdesc(sbase + kOffP, 16, 1024);
      const uint64_t vdesc0 = sdesc(sbase + kOffV, kBox, 1024);
      const uint32_t meta = sbase + kOffP + kPPage + 16u * uint32_t(lane);   // alpha[4 lane..]; l at +512
      const uint32_t evv = smem_u32(&bars->ev_val[0]) + 16u * uint32_t(lane);
      uint32_t bc = 0, vc = 0, pieces = 0, n1 = 0, nr = 0;
      each_piece(sv, [&](const Piece& pc) {
        if (pieces > 0 && !ewait(ctl, bar(bars->o_free), (pieces - 1) & 1u)) return false;
        ++pieces;
        for (int j = pc.p0; j < pc.p1; j += 2, ++bc) {
          const bool two = j + 1 < pc.p1, last = j + 2 >= pc.p1;
          if (!ewait<true>(ctl, bar(bars->p_full[0]), bc & 1u)) return false;
          const float4 a4 = ld_shared_f4(meta);
          const float4 l4 = last ? ld_shared_f4(meta + 512u) : make_float4(0.f, 0.f, 0.f, 0.f);
          // re-arm slot 0: its next copy starts only after this block's
          // page-0 PVs complete
          if (leader) mbar_arrive_expect_tx(bar(bars->p_full[0]), kPSlot0);
          if (__any_sync(0xffffffffu, a4.x != 1.f || a4.y != 1.f || a4.z != 1.f || a4.w != 1.f)) {
            // the running max moved: O is rescaled (once every earlier PV
            // completed) before this block's PVs
            st_shared_f4(evv, a4);
            if (leader) {
              bars->ev_type = kEvRescale;
              bars->ev_blk = bc;
            }
            mbar_arrive(bar(bars->corr_go));
            if (!ewait(ctl, bar(bars->corr_done), nr & 1u)) return false;
            ++nr;
          }
          for (int u = 0; u < (two ? 2 : 1); ++u, ++vc) {
            if (u == 1) {
              if (!ewait<true>(ctl, bar(bars->p_full[1]), n1 & 1u)) return false;
              if (leader) mbar_arrive_expect_tx(bar(bars->p_full[1]), kPPage);
            }
            const uint32_t vs = vc % NV;
            if (!ewait(ctl, bar(bars->v_full[vs]), (vc / NV) & 1u)) return false;
            tc_fence_after();
            const uint64_t ad = pdesc0 + uint64_t((uint32_t(u) * kPSlot0) >> 4);
            const uint64_t bd = vdesc0 + uint64_t((vs * kVStage) >> 4);
            const uint32_t acc0 = (j > pc.p0 || u > 0) ? 1u : 0u;
            if (leader) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                mma_ss(tmem, ad + 2u * k, bd + (2048u >> 4) * k, kIdescPV, k > 0 ? 1u : acc0);
                mma_ss(tmem + 256u, ad + 2u * k, bd + ((4u * kBox + 2048u * k) >> 4), kIdescPV, k > 0 ? 1u : acc0);
              }
              mma_commit(bar(bars->pv_done[vs]));
              mma_commit_mc(bar(bars->x_free[u]), uint16_t(1u));   // the score CTA may refill slot u
            }
            __syncwarp();
          }
          n1 += two ? 1u : 0u;
          if (leader) {
            mma_commit(bar(bars->pv_blk[bc % NB]));
          }
          __syncwarp();
          if (last) {
            // the piece's row sums, for the epilogue (which waits for these PVs)
            st_shared_f4(evv, l4);
            if (leader) {
              bars->ev_type = kEvEnd;
              bars->ev_blk = bc;
            }
            mbar_arrive(bar(bars->corr_go));
          }
        }
        return true;
      });
      if (leader) mma_commit(bar(bars->mma_done));
      __syncwarp();
      drain_wait(bar(bars->mma_done), 0);
    } else if (warp >= 4 && warp < 8) {
      // ---- correction / epilogue warpgroup: thread i owns row i of O.  It
      // acts on the PV issuer's events: a block whose rescale factors are not
      // all 1 (rescale O once every earlier block's PVs completed) and the end
      // of a piece (normalise O by the row sums and store it).  An event's
      // data stays put until the issuer sees it handled (corr_done, o_free).
      const int i = tid - 128, wq = warp - 4;
      const uint32_t lane_off = uint32_t(wq * 32) << 16;
      const volatile Bars* vb = bars;
      uint32_t ne = 0;
      each_piece(sv, [&](const Piece& pc) {
        const int r = pc.T / sv.tiles_per_req, qt = pc.T % sv.tiles_per_req;
        const int rho = qt * MLA_TILE_ROWS + i;
        const bool valid = rho < rows_total;
        for (;;) {
          if (!wwait(ctl, bar(bars->corr_go), ne & 1u)) return false;
          ++ne;
          const uint32_t type = vb->ev_type, eb = vb->ev_blk;
          const float v = vb->ev_val[i];
          if (type == kEvRescale) {
            // O must hold every earlier block before it is rescaled (never
            // the piece's first block, so eb - 1 exists)
            const uint32_t pb = eb - 1;
            if (!wwait(ctl, bar(bars->pv_blk[pb % NB]), (pb / NB) & 1u)) return false;
            if (__any_sync(0xffffffffu, v != 1.f)) {
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < 16; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + 32u * c, o);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 32; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * v);
                tmem_st32(tmem + lane_off + 32u * c, o);
              }
              tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar(bars->corr_done));
            continue;
          }
          // end of the piece: wait for its last block of PVs, normalise, store
          const uint32_t pb = eb;
          if (!wwait(ctl, bar(bars->pv_blk[pb % NB]), (pb / NB) & 1u)) return false;
          tc_fence_after();
          const float lfin = v;
          const float inv = lfin > 0.f ? 1.f / lfin : 0.f;
          const bool whole = sv.tile_splits(pc.T) == 1;
          const int slot = whole ? 0 : sv.tile_slot_base(pc.T) + pc.split;
          const bool slot_ok = whole || slot < p.cap_slots;
          uint4* dst_b = reinterpret_cast<uint4*>(p.out + (size_t(r) * rows_total + (valid ? rho : 0)) * MLA_D_V);
          uint4* dst_f = slot_ok && !whole
                             ? reinterpret_cast<uint4*>(ws_partial_o(p.ws, p.cap_slots, slot) + size_t(i) * MLA_D_V)
                             : nullptr;
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + 32u * c, o);
            tmem_wait_ld();
            if (valid && slot_ok) {
              if (whole && p.out_lo == nullptr) {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  dst_b[c * 4 + u] = make_uint4(
                      pack_bf16(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv),
                      pack_bf16(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv),
                      pack_bf16(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv),
                      pack_bf16(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv));
              } else if (whole) {
                // two-term output: hi = bf16(x), lo = bf16(x - hi)
                uint4* dst_l =
                    reinterpret_cast<uint4*>(p.out_lo + (size_t(r) * rows_total + (valid ? rho : 0)) * MLA_D_V);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  uint32_t hi[4], lo[4];
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    split_bf16(__uint_as_float(o[8 * u + 2 * k]) * inv, __uint_as_float(o[8 * u + 2 * k + 1]) * inv,
                               &hi[k], &lo[k]);
                  dst_b[c * 4 + u] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                  dst_l[c * 4 + u] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
              } else {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  dst_f[c * 8 + u] = make_uint4(__float_as_uint(__uint_as_float(o[4 * u + 0]) * inv),
                                                __float_as_uint(__uint_as_float(o[4 * u + 1]) * inv),
                                                __float_as_uint(__uint_as_float(o[4 * u + 2]) * inv),
                                                __float_as_uint(__uint_as_float(o[4 * u + 3]) * inv));
              }
            }
          }
          tc_fence_before();
          mbar_arrive(bar(bars->o_free));
          return true;
        }
      });
    } else if (warp == 0) {
      // ---- V producer: the page's 512 latent columns per stage.  BF16 cache:
      // 8 boxes of 64 columns.  FP8 cache: 4 e4m3 boxes of 128 columns into
      // the upper half of the stage (the converters expand them in place).
      if (lane == 0) {
        uint32_t vc = 0;
        each_piece(sv, [&](const Piece& pc) {
          const int r = pc.T / sv.tiles_per_req;
          for (int j = pc.p0; j < pc.p1; ++j, ++vc) {
            const uint32_t vs = vc % NV, vph = (vc / NV) & 1u;
            if (!swait(ctl, bar(bars->pv_done[vs]), vph ^ 1u)) return false;
            int page = p.block_table[size_t(r) * sv.max_pages + j];
            if (page < 0 || page >= p.num_pages) page = 0;   // the converters zero it
            const uint32_t fb = bar(bars->v_loaded[vs]);
            const uint32_t dst = sbase + kOffV + vs * kVStage;
            if constexpr (kFp8) {
              mbar_arrive_expect_tx(fb, kVStage / 2);
#pragma unroll
              for (int c = 0; c < 4; ++c) tma_load_3d(dst + kVStage / 2 + c * kBox, &pool_map, 128 * c, 0, page, fb);
            } else {
              mbar_arrive_expect_tx(fb, kVStage);
#pragma unroll
              for (int c = 0; c < 8; ++c) tma_load_3d(dst + c * kBox, &pool_map, 64 * c, 0, page, fb);
            }
          }
          return true;
        });
        const uint32_t n = vc < NV ? vc : NV;
        for (uint32_t k = 1; k <= n; ++k) {
          const uint32_t idx = vc - k;
          drain_wait(bar(bars->v_loaded[idx % NV]), (idx / NV) & 1u);
        }
      }
    } else if (conv_rank(warp) >= 0) {
      // ---- V converters: each landed stage is rewritten in place from bf16
      // to fp16 (same size, same swizzled N-major layout).  Tokens at or
      // past the request's length become zero: their bytes may be anything
      // and 0 * NaN would poison O.  Thread -> 16 chunks of 16 bytes.  A
      // value that does not fit fp16 sets kStatusBadInput (the output of its
      // tile is then not valid).
      const int ct = conv_rank(warp) * 32 + lane;
      uint32_t vc = 0;
      __half2 vmax = __float2half2_rn(0.f);
      const bool done = each_piece(sv, [&](const Piece& pc) {
        const int r = pc.T / sv.tiles_per_req;
        const int t = clamp_len(p.seqlens[r], sv);
        for (int j = pc.p0; j < pc.p1; ++j, ++vc) {
          const uint32_t vs = vc % NV, vph = (vc / NV) & 1u;
          const int page = p.block_table[size_t(r) * sv.max_pages + j];
          const bool ok = page >= 0 && page < p.num_pages;
          const int nvalid = ok ? t - j * MLA_PAGE_SIZE : 0;
          const uint32_t st = sbase + kOffV + vs * kVStage;
          if constexpr (kFp8) {
            // FP8 cache: output chunk o = ct + 256u (8 fp16 of token rr, in
            // the N-major swizzled layout) comes from 8 e4m3 bytes of the
            // upper half, times the token's scale.  The input and output
            // regions overlap: every thread reads all its input before any
            // thread writes.  Thread ct's chunks belong to tokens ct/8 and
            // ct/8 + 32.
            const int ta = ct >> 3;
            const float sa = ok ? p.kv_scale[size_t(page) * 64 + ta] : 0.f;
            const float sb = ok ? p.kv_scale[size_t(page) * 64 + ta + 32] : 0.f;
            const bool vwait = ct == 0 ? bwait(ctl, bar(bars->v_loaded[vs]), vph) : true;
            if (!named_bar_and(kConvBar, kConvThreads, vwait)) return false;
            uint2 in[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const uint32_t o = uint32_t(ct + kConvThreads * u), b = o >> 9, rr = (o & 511u) >> 3;
              const uint32_t lc = (o & 7u) ^ (rr & 7u), k = 4u * (b & 1u) + (lc >> 1);
              in[u] = ld_shared_v2(st + kVStage / 2 + (b >> 1) * kBox + rr * 128u + ((k ^ (rr & 7u)) << 4) +
                                   (lc & 1u) * 8u);
            }
            named_bar_sync(kConvBar, kConvThreads);
            const __half2 ha = __float2half2_rn(sa), hb = __float2half2_rn(sb);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const uint32_t o = uint32_t(ct + kConvThreads * u), rr = (o & 511u) >> 3;
              if (int(rr) < nvalid) {
                const __half2 sc = (u & 1) ? hb : ha;
                const uint32_t a = e4m3x2_scaled(in[u].x & 0xFFFFu, sc), b = e4m3x2_scaled(in[u].x >> 16, sc);
                const uint32_t c = e4m3x2_scaled(in[u].y & 0xFFFFu, sc), d = e4m3x2_scaled(in[u].y >> 16, sc);
                track_absmax(vmax, a);
                track_absmax(vmax, b);
                track_absmax(vmax, c);
                track_absmax(vmax, d);
                st_shared_v4(st + o * 16u, a, b, c, d);
              } else {
                st_shared_v4(st + o * 16u, 0u, 0u, 0u, 0u);
              }
            }
          } else {
            if (!wwait(ctl, bar(bars->v_loaded[vs]), vph)) return false;
            // Loads go out in groups of kConvGroup ahead of the group's
            // stores (a thread's 16 chunks are its own, so the order is
            // free): the shared-memory load latency is paid once per group
            // instead of once per chunk.  Chunk u of this thread holds token
            // ct / 8 + 32 (u & 1).  A page whose 64 tokens all count (every
            // page but a request's last, and valid) takes the loop without
            // the per-token test; the CTA's converters all agree on it.  The
            // converters are issue-bound: dropping the test took the b=64,
            // h=128, t=4096 decode from 111.1 to 104.8 us.
            auto convert = [&](auto masked) {
              constexpr bool kMasked = decltype(masked)::value;
              const bool va = (ct >> 3) < nvalid, vb = (ct >> 3) + 32 < nvalid;
#pragma unroll
              for (int u0 = 0; u0 < 16; u0 += kConvGroup) {
                uint4 v[kConvGroup];
#pragma unroll
                for (int k = 0; k < kConvGroup; ++k)
                  v[k] = ld_shared_v4(st + uint32_t(ct + kConvThreads * (u0 + k)) * 16u);
#pragma unroll
                for (int k = 0; k < kConvGroup; ++k) {
                  const uint32_t off = uint32_t(ct + kConvThreads * (u0 + k)) * 16u;
                  if (!kMasked || (((u0 + k) & 1) ? vb : va)) {
                    const uint32_t a = bf16x2_to_f16x2(v[k].x), b = bf16x2_to_f16x2(v[k].y);
                    const uint32_t c = bf16x2_to_f16x2(v[k].z), d = bf16x2_to_f16x2(v[k].w);
                    track_absmax(vmax, a);
                    track_absmax(vmax, b);
                    track_absmax(vmax, c);
                    track_absmax(vmax, d);
                    st_shared_v4(st + off, a, b, c, d);
                  } else {
                    st_shared_v4(st + off, 0u, 0u, 0u, 0u);
                  }
                }
              }
            };
            if (nvalid >= MLA_PAGE_SIZE) convert(std::false_type{});
            else convert(std::true_type{});
          }
          fence_proxy_async_cta();
          mbar_arrive(bar(bars->v_full[vs]));
        }
        return true;
      });
      if (done && !absmax_finite(vmax)) flag_status(p.ws, kStatusBadInput);
    }
  }

  // ---- teardown: every MMA has completed (mma_done), every TMEM access has
  // been waited on; free TMEM and leave together with the peer CTA
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  cluster_sync();
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Tensor map over the bf16 page pool viewed as [pages][64 tokens][576]:
// boxes of 64 columns x 64 tokens x 1 page, 128-byte swizzle.
bool make_pool_map(CUtensorMap* map, const void* kv, int num_pages) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cuuint64_t(MLA_D_QK), cuuint64_t(MLA_PAGE_SIZE), cuuint64_t(num_pages)};
  cuuint64_t strides[2] = {cuuint64_t(MLA_D_QK) * 2, cuuint64_t(MLA_D_QK) * 2 * MLA_PAGE_SIZE};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// FP8 cache pages [pages][40960 B]: the e4m3 latent block viewed as
// [pages][64 tokens][512 bytes] with boxes of 128 bytes (columns) x 64
// tokens, and the bf16 RoPE block (at +32 KB in each page) viewed as
// [pages][64 tokens][64] with boxes of 64 columns x 64 tokens; both with the
// 128-byte swizzle.
bool make_fp8_maps(CUtensorMap* lat, CUtensorMap* rope, const void* kv, int num_pages) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dl[3] = {512, cuuint64_t(MLA_PAGE_SIZE), cuuint64_t(num_pages)};
  cuuint64_t sl[2] = {512, kFp8PageBytes};
  cuuint32_t bl[3] = {128, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(lat, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(kv), dl, sl, bl, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cuuint64_t dr[3] = {64, cuuint64_t(MLA_PAGE_SIZE), cuuint64_t(num_pages)};
  cuuint64_t sr[2] = {128, kFp8PageBytes};
  cuuint32_t br[3] = {64, 64, 1};
  r = fn(rope, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
         const_cast<uint8_t*>(static_cast<const uint8_t*>(kv)) + 64 * 512, dr, sr, br, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the query rows [batch * s_q * heads][576] bf16: boxes of
// 64 columns x 64 rows, 128-byte swizzle.  Rows past the end read as zero.
bool make_q_map(CUtensorMap* map, const void* q, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(MLA_D_QK), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(MLA_D_QK) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace


int prepare_decode_sm100(const mla_shape_t* shape, const void* q, const void* kv, DecodePrepared* pr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&pr->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || pr->sms <= 0)
    return MLA_ERR_CUDA;
  pr->fp8 = shape->cache_dtype == MLA_CACHE_FP8_E4M3;
  const int q_rows = shape->batch * shape->s_q * shape->num_heads;
  if (pr->fp8) {
    if (!make_fp8_maps(&pr->pool_map, &pr->rope_map, kv, shape->num_pages)) return MLA_ERR_CUDA;
  } else {
    if (!make_pool_map(&pr->pool_map, kv, shape->num_pages)) return MLA_ERR_CUDA;
    pr->rope_map = pr->pool_map;   // not read
  }
  if (!make_q_map(&pr->q_map, q, q_rows)) return MLA_ERR_CUDA;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(pr->fp8 ? &decode_sm100_kernel<true>
                                                               : &decode_sm100_kernel<false>),
                        int(kSmemBytes)))
    return MLA_ERR_CUDA;
  return MLA_OK;
}

int enqueue_decode_sm100(const DecodePrepared& pr, const mla_shape_t* shape, const void* q, const void* kv,
                         const float* kv_scale, const int32_t* block_table, const int32_t* seqlens, float scale,
                         const void* sched, void* ws, int cap_slots, void* out, float* lse, cudaStream_t stream,
                         void* out_lo, int test_stall) {
  Params prm;
  prm.q = static_cast<const uint16_t*>(q);
  prm.kv = static_cast<const uint8_t*>(kv);
  prm.kv_scale = kv_scale;
  prm.block_table = block_table;
  prm.seqlens = seqlens;
  prm.sched = sched;
  prm.ws = ws;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.out_lo = static_cast<__nv_bfloat16*>(out_lo);
  prm.lse = lse;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.num_pages = shape->num_pages;
  prm.cap_slots = cap_slots;
  prm.q_rows = shape->batch * shape->s_q * shape->num_heads;
  prm.test_stall = test_stall;
  const int clusters = pr.sms / 2 > 0 ? pr.sms / 2 : 1;
  // programmatic dependent launch: the prologue (barriers, TMEM, descriptor
  // prefetch) overlaps the scheduler kernel; the kernel waits for it before
  // reading the schedule
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      pr.fp8 ? cudaLaunchKernelEx(&cfg, decode_sm100_kernel<true>, pr.pool_map, pr.q_map, pr.rope_map, prm)
             : cudaLaunchKernelEx(&cfg, decode_sm100_kernel<false>, pr.pool_map, pr.q_map, pr.rope_map, prm);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int launch_decode_sm100(const mla_shape_t* shape, const void* q, const void* kv, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seqlens, float scale, const void* sched,
                        void* ws, int cap_slots, void* out, float* lse, cudaStream_t stream, void* out_lo) {
  DecodePrepared pr;
  const int rc = prepare_decode_sm100(shape, q, kv, &pr);
  if (rc != MLA_OK) return rc;
  return enqueue_decode_sm100(pr, shape, q, kv, kv_scale, block_table, seqlens, scale, sched, ws, cap_slots, out,
                              lse, stream, out_lo);
}

}  // namespace mla
