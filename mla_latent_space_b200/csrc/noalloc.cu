// mla_decode_fwd_noalloc: the whole decode step (schedule, decode, combine)
// with no caller-provided scratch and no allocation.  Its schedule and the
// device status word live in a file-scope __device__ array, sized for at
// most kNoAllocMaxTiles tiles; the schedule assigns whole tiles to workers
// (schedule_whole_tiles_kernel), so no fp32 partial slot is ever needed.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <mutex>

#include "decode_launch.cuh"

namespace mla {

size_t schedule_whole_tiles_smem(int num_tiles);
cudaError_t launch_schedule_whole_tiles(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched,
                                        int32_t* status, cudaStream_t stream);

namespace {

// [status word block, kStatusBytes][schedule].  One copy per device (the
// module is loaded per device); zero-initialised at module load.
constexpr size_t kNoAllocScratchBytes = 320 * 1024;
constexpr int kNoAllocMaxTiles = 16384;
constexpr int kMaxDevices = 64;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// NVTX range around the call's host work (as for the other entry points).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// Address of this device's scratch and its SM count, looked up once per
// device (the first call on a device, which therefore must not be made while
// the stream is being captured).  The cached address belongs to the device's
// primary context: after cudaDeviceReset it is stale, and this entry point is
// not supported in a process that resets a device it has used.
int scratch_for_device(uint8_t** base, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MLA_ERR_CUDA;
  static std::mutex mu;
  static uint8_t* addr[kMaxDevices] = {nullptr};
  static int nsm[kMaxDevices] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return MLA_ERR_CUDA;
    addr[dev] = static_cast<uint8_t*>(p);
    nsm[dev] = n;
  }
  *base = addr[dev];
  *sms = nsm[dev];
  return MLA_OK;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" int mla_decode_fwd_noalloc(const mla_shape_t* shape, const void* q, const void* kv_cache,
                                      const float* kv_scale, const int32_t* block_table, const int32_t* seqlens,
                                      float softmax_scale, void* out, float* lse, int32_t* device_status,
                                      void* stream) {
  CallRange range_("mla_decode_fwd_noalloc");
  if (!shape) return MLA_ERR_INVALID_ARG;
  if (shape->batch < 1 || shape->s_q < 1 || shape->num_heads < 1 || shape->max_pages_per_seq < 1 ||
      shape->num_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (shape->d_qk != MLA_D_QK || shape->d_v != MLA_D_V || shape->page_size != MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED;
  if (shape->cache_dtype != MLA_CACHE_BF16 && shape->cache_dtype != MLA_CACHE_FP8_E4M3) return MLA_ERR_UNSUPPORTED;
  if (shape->causal != 0 && shape->causal != 1) return MLA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(shape->s_q) * shape->num_heads;
  const int64_t tiles_per_req = (rows + MLA_TILE_ROWS - 1) / MLA_TILE_ROWS;
  const int64_t num_tiles = int64_t(shape->batch) * tiles_per_req;
  // the size limit of the static scratch, checked before touching the device
  if (num_tiles > kNoAllocMaxTiles) return MLA_ERR_WORKSPACE;
  if (int64_t(shape->max_pages_per_seq) * MLA_PAGE_SIZE >= (int64_t(1) << 30)) return MLA_ERR_UNSUPPORTED;
  if (num_tiles * (int64_t(shape->max_pages_per_seq) + kPieceOverhead) >= (int64_t(1) << 31))
    return MLA_ERR_UNSUPPORTED;
  if (!q || !kv_cache || !block_table || !seqlens || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (shape->cache_dtype == MLA_CACHE_FP8_E4M3 && !kv_scale) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_cache, 256) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(seqlens, 4) || (kv_scale && !aligned(kv_scale, 4)) ||
      (device_status && !aligned(device_status, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || softmax_scale - softmax_scale != 0.f) return MLA_ERR_INVALID_ARG;

  uint8_t* base = nullptr;
  int sms = 0;
  int rc = scratch_for_device(&base, &sms);
  if (rc != MLA_OK) return rc;
  ShapeInfo si;
  si.batch = shape->batch;
  si.s_q = shape->s_q;
  si.heads = shape->num_heads;
  si.causal = shape->causal;
  si.max_pages = shape->max_pages_per_seq;
  si.tiles_per_req = int(tiles_per_req);
  const int W = num_workers_for(sms);
  const size_t sched_bytes = 4 * (size_t(kHeaderInts) + size_t(W) * kWorkerInts + size_t(num_tiles) * kTileInts);
  if (kStatusBytes + sched_bytes > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE;
  void* ws = base;
  int32_t* sched = reinterpret_cast<int32_t*>(base + kStatusBytes);

  // every check that can fail on the host comes before the first enqueue, so
  // an error return leaves nothing of this call on the stream
  if (schedule_whole_tiles_smem(int(num_tiles)) == 0) return MLA_ERR_WORKSPACE;
  DecodePrepared prep;
  rc = prepare_decode_sm100(shape, q, kv_cache, &prep);
  if (rc != MLA_OK) return rc;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word must start at zero: the kernels only OR flags into it
  if (cudaMemsetAsync(ws, 0, kStatusBytes, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (launch_schedule_whole_tiles(seqlens, si, W, sched, static_cast<int32_t*>(ws), st) != cudaSuccess)
    return MLA_ERR_CUDA;
  rc = enqueue_decode_sm100(prep, shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, ws, 0,
                            out, lse, st);
  if (rc != MLA_OK) return rc;
  if (launch_combine(sched, ws, out, lse, int(num_tiles), 0, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (device_status && cudaMemcpyAsync(device_status, ws, 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}
