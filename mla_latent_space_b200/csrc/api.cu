// Host side of libmla_b200.so: argument validation, buffer sizing and the
// launches behind the C ABI declared in include/mla.h.  Every check runs
// before anything is enqueued; an error return means the stream is untouched.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "decode_launch.cuh"
#ifdef MLA_TEST_ENTRY_POINTS
#include "test_entry.h"
#endif

namespace mla {
void plan_schedule_host(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched);
cudaError_t launch_schedule(const int32_t* seqlens, const ShapeInfo& s, int W, int32_t* sched, cudaStream_t st);
#ifdef MLA_TEST_ENTRY_POINTS
cudaError_t launch_decode_simt(const void* q, const void* kv, const float* kv_scale, const int32_t* block_table,
                               const int32_t* seqlens, float scale, const void* sched, void* ws, void* out,
                               float* lse, int num_pages, int fp8, int cap_slots, int grid_ctas,
                               cudaStream_t stream);
#endif
cudaError_t launch_sparse_gather(const int32_t* indices, int topk, const int32_t* seqlens, int batch, int s_q,
                                 const int32_t* block_table, int max_pages, int num_pages, const void* pool,
                                 const float* kv_scale, void* scratch, float* vscale, int vpages, int32_t* vseqlens,
                                 int32_t* vbt, void* status_ws, bool fp8, cudaStream_t stream);
cudaError_t launch_var6_old_len(const int32_t* seqlens, int batch, int n_new, int max_pages, int32_t* old_len,
                                cudaStream_t stream);
cudaError_t launch_var6_new(const void* q, const void* k_new, const void* v_new, const void* pool, bool fp8,
                            const int32_t* block_table, const int32_t* seqlens, const void* o_old,
                            const void* o_old_lo, const float* lse_old, int batch, int s_q, int heads, int n_new,
                            int max_pages, int num_pages, int causal, float scale, void* out, float* lse,
                            void* status_ws, cudaStream_t stream);
int launch_absorb_q(int rows, int heads, const void* q, const void* w_k, void* qz, int32_t* status,
                    cudaStream_t stream);
int launch_decompress_o(int rows, int heads, const void* o_lat, const void* w_kvb2, void* out, int32_t* status,
                        cudaStream_t stream, const void* o_lat_lo = nullptr, void* out_lo = nullptr);
}  // namespace mla

using namespace mla;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// NVTX range around an entry point's host work (argument checks, tensor-map
// encoding, launches), so a profiler's timeline names each call.  Costs a
// few nanoseconds when no tool is attached.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// Shape checks shared by every entry point.
int check_shape(const mla_shape_t* s) {
  if (!s) return MLA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->s_q < 1 || s->num_heads < 1 || s->max_pages_per_seq < 1 || s->num_pages < 1)
    return MLA_ERR_INVALID_ARG;
  if (s->d_qk != MLA_D_QK || s->d_v != MLA_D_V || s->page_size != MLA_PAGE_SIZE) return MLA_ERR_UNSUPPORTED;
  if (s->cache_dtype != MLA_CACHE_BF16 && s->cache_dtype != MLA_CACHE_FP8_E4M3) return MLA_ERR_UNSUPPORTED;
  if (s->causal != 0 && s->causal != 1) return MLA_ERR_INVALID_ARG;
  const int64_t rows = int64_t(s->s_q) * s->num_heads;
  const int64_t tiles = int64_t(s->batch) * ((rows + MLA_TILE_ROWS - 1) / MLA_TILE_ROWS);
  if (rows * s->batch >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED;
  if (int64_t(s->max_pages_per_seq) * MLA_PAGE_SIZE >= (int64_t(1) << 30)) return MLA_ERR_UNSUPPORTED;
  if (tiles * (int64_t(s->max_pages_per_seq) + kPieceOverhead) >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

ShapeInfo shape_info(const mla_shape_t* s) {
  ShapeInfo si;
  si.batch = s->batch;
  si.s_q = s->s_q;
  si.heads = s->num_heads;
  si.causal = s->causal;
  si.max_pages = s->max_pages_per_seq;
  si.tiles_per_req = (s->s_q * s->num_heads + MLA_TILE_ROWS - 1) / MLA_TILE_ROWS;
  return si;
}

size_t sched_bytes_for(const mla_shape_t* s, int num_sms) {
  ShapeInfo si = shape_info(s);
  int W = num_workers_for(num_sms);
  return 4 * (size_t(kHeaderInts) + size_t(W) * kWorkerInts + size_t(si.batch) * si.tiles_per_req * kTileInts);
}

int cap_slots_for(size_t ws_bytes) {
  if (ws_bytes < kStatusBytes) return -1;
  size_t cap = (ws_bytes - kStatusBytes) / kSlotBytes;
  return cap > (1u << 30) ? (1 << 30) : int(cap);
}

int device_sms(int* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return MLA_ERR_CUDA;
    cache[dev] = n;
  }
  *out = cache[dev];
  return MLA_OK;
}

int check_decode_args(const mla_shape_t* shape, const void* q, const void* kv, const float* kv_scale,
                      const int32_t* block_table, const int32_t* seqlens, float scale, const void* sched,
                      void* ws, size_t ws_bytes, void* out, float* lse) {
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  if (!q || !kv || !block_table || !seqlens || !sched || !ws || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (shape->cache_dtype == MLA_CACHE_FP8_E4M3 && !kv_scale) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv, 256) || !aligned(out, 16) || !aligned(lse, 4) || !aligned(block_table, 4) ||
      !aligned(seqlens, 4) || !aligned(sched, 16) || !aligned(ws, 256) || (kv_scale && !aligned(kv_scale, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return MLA_ERR_INVALID_ARG;
  if (cap_slots_for(ws_bytes) < 0) return MLA_ERR_WORKSPACE;
  return MLA_OK;
}

// Workspace of the sparse decode (every region 256-byte aligned): the
// compacted lengths and identity block table of the b*s single-query
// "virtual" requests, their schedule, the decode workspace, the scratch
// pages the selected rows are gathered into (the cache's own page format)
// and, for the FP8 cache, their per-token scales.
struct SparseLayout {
  mla_shape_t vshape;
  int vpages;
  size_t vseq, vbt, sched, sched_bytes, ws, ws_bytes, scratch, vscale, total;
};

bool sparse_layout(const mla_shape_t* s, int topk, int num_sms, SparseLayout* L) {
  if (check_shape(s) != MLA_OK || topk < 1 || topk > (1 << 24) || num_sms < 1) return false;
  if (s->causal != 0) return false;
  const bool fp8 = s->cache_dtype == MLA_CACHE_FP8_E4M3;
  const int64_t V = int64_t(s->batch) * s->s_q;
  const int64_t vpages = (topk + MLA_PAGE_SIZE - 1) / MLA_PAGE_SIZE;
  if (V * vpages >= (int64_t(1) << 26)) return false;   // scratch rows stay below 2^32
  mla_shape_t vs = *s;
  vs.batch = int32_t(V);
  vs.s_q = 1;
  vs.max_pages_per_seq = int32_t(vpages);
  vs.num_pages = int32_t(V * vpages);
  vs.causal = 0;
  if (check_shape(&vs) != MLA_OK) return false;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  L->vshape = vs;
  L->vpages = int(vpages);
  size_t off = 0;
  L->vseq = off;
  off = up(off + 4 * size_t(V));
  L->vbt = off;
  off = up(off + 4 * size_t(V) * size_t(vpages));
  L->sched = off;
  L->sched_bytes = sched_bytes_for(&vs, num_sms);
  off = up(off + L->sched_bytes);
  L->ws = off;
  L->ws_bytes = kStatusBytes + size_t(max_slots_for(num_workers_for(num_sms))) * kSlotBytes;
  off = up(off + L->ws_bytes);
  L->scratch = off;
  const size_t page_bytes = fp8 ? size_t(MLA_PAGE_SIZE) * (MLA_D_V + 2 * MLA_D_ROPE)
                                : size_t(MLA_PAGE_SIZE) * (2 * MLA_D_QK);
  off = up(off + size_t(V) * size_t(vpages) * page_bytes);
  L->vscale = off;
  if (fp8) off = up(off + size_t(V) * size_t(vpages) * MLA_PAGE_SIZE * 4);
  L->total = off;
  return true;
}

// Workspace of the MLAvar6+ split decode (every region 256-byte aligned):
// the old lengths t - n, the schedule and decode workspace of the latent
// part (a non-causal decode over the old tokens), its latent output (two
// bf16 terms) and lse, and its decompressed output (two bf16 terms).
struct Var6Layout {
  mla_shape_t oshape;
  size_t oldlen, sched, sched_bytes, ws, ws_bytes, olat, olat_lo, lse_old, oold, oold_lo, total;
};

bool var6_layout(const mla_shape_t* s, int n_new, int num_sms, Var6Layout* L) {
  if (check_shape(s) != MLA_OK || num_sms < 1 || n_new < 0 || n_new > (1 << 20)) return false;
  if (s->s_q > 32 || s->num_heads > 65535) return false;
  if (s->causal && n_new < s->s_q) return false;   // every old token must be visible to every query row
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  L->oshape = *s;
  L->oshape.causal = 0;
  const size_t rows = size_t(s->batch) * s->s_q * s->num_heads;
  size_t off = 0;
  L->oldlen = off;
  off = up(off + 4 * size_t(s->batch));
  L->sched = off;
  L->sched_bytes = sched_bytes_for(&L->oshape, num_sms);
  off = up(off + L->sched_bytes);
  L->ws = off;
  L->ws_bytes = kStatusBytes + size_t(max_slots_for(num_workers_for(num_sms))) * kSlotBytes;
  off = up(off + L->ws_bytes);
  L->olat = off;
  off = up(off + rows * MLA_D_V * 2);
  L->olat_lo = off;
  off = up(off + rows * MLA_D_V * 2);
  L->lse_old = off;
  off = up(off + rows * 4);
  L->oold = off;
  off = up(off + rows * MLA_D_HEAD * 2);
  L->oold_lo = off;
  off = up(off + rows * MLA_D_HEAD * 2);
  L->total = off;
  return true;
}

}  // namespace

extern "C" {

size_t mla_schedule_bytes(const mla_shape_t* shape, int num_sms) {
  if (check_shape(shape) != MLA_OK || num_sms < 1) return 0;
  return sched_bytes_for(shape, num_sms);
}

size_t mla_workspace_bytes(const mla_shape_t* shape, int num_sms) {
  if (check_shape(shape) != MLA_OK || num_sms < 1) return 0;
  return kStatusBytes + size_t(max_slots_for(num_workers_for(num_sms))) * kSlotBytes;
}

int mla_get_schedule(const mla_shape_t* shape, const int32_t* seqlens, int num_sms, void* sched,
                     size_t sched_bytes, void* stream) {
  CallRange range_("mla_get_schedule");
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  if (!seqlens || !sched || num_sms < 1) return MLA_ERR_INVALID_ARG;
  if (!aligned(sched, 16) || !aligned(seqlens, 4)) return MLA_ERR_INVALID_ARG;
  if (sched_bytes < sched_bytes_for(shape, num_sms)) return MLA_ERR_WORKSPACE;
  cudaError_t e = launch_schedule(seqlens, shape_info(shape), num_workers_for(num_sms), static_cast<int32_t*>(sched),
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_plan_schedule_host(const mla_shape_t* shape, const int32_t* seqlens, int num_sms, void* sched,
                           size_t sched_bytes) {
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  if (!seqlens || !sched || num_sms < 1) return MLA_ERR_INVALID_ARG;
  if (sched_bytes < sched_bytes_for(shape, num_sms)) return MLA_ERR_WORKSPACE;
  plan_schedule_host(seqlens, shape_info(shape), num_workers_for(num_sms), static_cast<int32_t*>(sched));
  return MLA_OK;
}

int mla_decode_fwd(const mla_shape_t* shape, const void* q, const void* kv_cache, const float* kv_scale,
                   const int32_t* block_table, const int32_t* seqlens, float softmax_scale, const void* sched,
                   void* workspace, size_t workspace_bytes, void* out, float* lse, void* stream) {
  CallRange range_("mla_decode_fwd");
  int rc = check_decode_args(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                             workspace_bytes, out, lse);
  if (rc != MLA_OK) return rc;
  return launch_decode_sm100(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                             cap_slots_for(workspace_bytes), out, lse, static_cast<cudaStream_t>(stream));
}

#ifdef MLA_TEST_ENTRY_POINTS
// Test-only entry point (built into the test library alone): the SIMT
// decode kernel over the same schedule and workspace.
int mla_decode_fwd_simt(const mla_shape_t* shape, const void* q, const void* kv_cache, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seqlens, float softmax_scale,
                        const void* sched, void* workspace, size_t workspace_bytes, void* out, float* lse,
                        void* stream) {
  int rc = check_decode_args(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                             workspace_bytes, out, lse);
  if (rc != MLA_OK) return rc;
  int sms = 0;
  if ((rc = device_sms(&sms)) != MLA_OK) return rc;
  cudaError_t e = launch_decode_simt(q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                                     out, lse, shape->num_pages, shape->cache_dtype == MLA_CACHE_FP8_E4M3,
                                     cap_slots_for(workspace_bytes), sms, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
#endif

#ifdef MLA_TEST_ENTRY_POINTS
// Test-only entry point: mla_decode_fwd with the kernel's stall hook set, so
// that one bounded wait runs out (after about 2 s) and the abort path runs.
int mla_test_decode_stalled(const mla_shape_t* shape, const void* q, const void* kv_cache, const float* kv_scale,
                            const int32_t* block_table, const int32_t* seqlens, float softmax_scale,
                            const void* sched, void* workspace, size_t workspace_bytes, void* out, float* lse,
                            void* stream) {
  int rc = check_decode_args(shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched, workspace,
                             workspace_bytes, out, lse);
  if (rc != MLA_OK) return rc;
  DecodePrepared prep;
  if ((rc = prepare_decode_sm100(shape, q, kv_cache, &prep)) != MLA_OK) return rc;
  return enqueue_decode_sm100(prep, shape, q, kv_cache, kv_scale, block_table, seqlens, softmax_scale, sched,
                              workspace, cap_slots_for(workspace_bytes), out, lse, static_cast<cudaStream_t>(stream),
                              nullptr, 1);
}
#endif

int mla_combine(const mla_shape_t* shape, const void* sched, const void* workspace, size_t workspace_bytes,
                void* out, float* lse, void* stream) {
  CallRange range_("mla_combine");
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  if (!sched || !workspace || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (!aligned(sched, 16) || !aligned(workspace, 256) || !aligned(out, 16) || !aligned(lse, 4))
    return MLA_ERR_INVALID_ARG;
  const int cap = cap_slots_for(workspace_bytes);
  if (cap < 0) return MLA_ERR_WORKSPACE;
  ShapeInfo si = shape_info(shape);
  cudaError_t e = launch_combine(sched, workspace, out, lse, si.batch * si.tiles_per_req, cap,
                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_get_device_status(const void* sched, void* workspace, void* stream, int* status) {
  if (!sched || !workspace || !status) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t ws_word = 0, sched_word = 0;
  if (cudaMemcpyAsync(&ws_word, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyAsync(&sched_word, static_cast<const int32_t*>(sched) + H_STATUS, 4, cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, 4, st) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MLA_ERR_CUDA;
  const int32_t all = ws_word | sched_word;
  if (all & kStatusTimeout) *status = MLA_ERR_TIMEOUT;
  else if (all & kStatusWorkspace) *status = MLA_ERR_WORKSPACE;
  else if (all) *status = MLA_ERR_DEVICE_CHECK;
  else *status = MLA_OK;
  return MLA_OK;
}

size_t mla_sparse_workspace_bytes(const mla_shape_t* shape, int topk, int num_sms) {
  SparseLayout L;
  return sparse_layout(shape, topk, num_sms, &L) ? L.total : 0;
}

int mla_sparse_decode_fwd(const mla_shape_t* shape, int topk, const void* q, const void* kv_cache,
                          const float* kv_scale, const int32_t* block_table, const int32_t* seqlens,
                          const int32_t* indices, float softmax_scale, void* workspace, size_t workspace_bytes,
                          void* out, float* lse, void* stream) {
  CallRange range_("mla_sparse_decode_fwd");
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  const bool fp8 = shape->cache_dtype == MLA_CACHE_FP8_E4M3;
  if (shape->causal != 0 || topk < 1 || topk > (1 << 24)) return MLA_ERR_INVALID_ARG;
  if (!q || !kv_cache || !block_table || !seqlens || !indices || !workspace || !out || !lse)
    return MLA_ERR_INVALID_ARG;
  if (fp8 && (!kv_scale || !aligned(kv_scale, 4))) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_cache, 256) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(block_table, 4) || !aligned(seqlens, 4) || !aligned(indices, 4) || !aligned(workspace, 256))
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  int sms = 0;
  if ((rc = device_sms(&sms)) != MLA_OK) return rc;
  SparseLayout L;
  if (!sparse_layout(shape, topk, sms, &L)) return MLA_ERR_UNSUPPORTED;
  if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
  char* w = static_cast<char*>(workspace);
  int32_t* vseq = reinterpret_cast<int32_t*>(w + L.vseq);
  int32_t* vbt = reinterpret_cast<int32_t*>(w + L.vbt);
  void* sched = w + L.sched;
  void* ws = w + L.ws;
  void* scratch = w + L.scratch;
  float* vscale = fp8 ? reinterpret_cast<float*>(w + L.vscale) : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (launch_sparse_gather(indices, topk, seqlens, shape->batch, shape->s_q, block_table, shape->max_pages_per_seq,
                           shape->num_pages, kv_cache, kv_scale, scratch, vscale, L.vpages, vseq, vbt, ws, fp8,
                           st) != cudaSuccess)
    return MLA_ERR_CUDA;
  const ShapeInfo si = shape_info(&L.vshape);
  if (launch_schedule(vseq, si, num_workers_for(sms), static_cast<int32_t*>(sched), st) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int cap = cap_slots_for(L.ws_bytes);
  rc = launch_decode_sm100(&L.vshape, q, scratch, vscale, vbt, vseq, softmax_scale, sched, ws, cap, out, lse, st);
  if (rc != MLA_OK) return rc;
  return launch_combine(sched, ws, out, lse, si.batch * si.tiles_per_req, cap, st) == cudaSuccess ? MLA_OK
                                                                                                  : MLA_ERR_CUDA;
}

int mla_sparse_get_device_status(const mla_shape_t* shape, int topk, int num_sms, void* workspace, void* stream,
                                 int* status) {
  SparseLayout L;
  if (!workspace || !status || !sparse_layout(shape, topk, num_sms, &L)) return MLA_ERR_INVALID_ARG;
  char* w = static_cast<char*>(workspace);
  return mla_get_device_status(w + L.sched, w + L.ws, stream, status);
}

size_t mla_var6_workspace_bytes(const mla_shape_t* shape, int n_new, int num_sms) {
  Var6Layout L;
  return var6_layout(shape, n_new, num_sms, &L) ? L.total : 0;
}

int mla_var6_decode_fwd(const mla_shape_t* shape, int n_new, const void* qz, const void* q, const void* kv_cache,
                        const float* kv_scale, const int32_t* block_table, const int32_t* seqlens, const void* k_new,
                        const void* v_new, const void* w_kvb2, float softmax_scale, void* workspace,
                        size_t workspace_bytes, void* out, float* lse, void* stream) {
  CallRange range_("mla_var6_decode_fwd");
  int rc = check_shape(shape);
  if (rc != MLA_OK) return rc;
  const bool fp8 = shape->cache_dtype == MLA_CACHE_FP8_E4M3;
  if (n_new < 0 || n_new > (1 << 20) || (shape->causal && n_new < shape->s_q)) return MLA_ERR_INVALID_ARG;
  if (shape->s_q > 32 || shape->num_heads > 65535) return MLA_ERR_UNSUPPORTED;
  if (!qz || !q || !kv_cache || !block_table || !seqlens || !w_kvb2 || !workspace || !out || !lse)
    return MLA_ERR_INVALID_ARG;
  if (n_new > 0 && (!k_new || !v_new)) return MLA_ERR_INVALID_ARG;
  if (fp8 && !kv_scale) return MLA_ERR_INVALID_ARG;
  if (!aligned(qz, 16) || !aligned(q, 16) || !aligned(kv_cache, 256) || !aligned(block_table, 4) ||
      !aligned(seqlens, 4) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(w_kvb2, 16) ||
      !aligned(workspace, 256) || !aligned(out, 16) || !aligned(lse, 4) || (kv_scale && !aligned(kv_scale, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return MLA_ERR_INVALID_ARG;
  int sms = 0;
  if ((rc = device_sms(&sms)) != MLA_OK) return rc;
  Var6Layout L;
  if (!var6_layout(shape, n_new, sms, &L)) return MLA_ERR_UNSUPPORTED;
  if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE;
  char* w = static_cast<char*>(workspace);
  int32_t* oldlen = reinterpret_cast<int32_t*>(w + L.oldlen);
  void* sched = w + L.sched;
  void* ws = w + L.ws;
  void* olat = w + L.olat;
  void* olat_lo = w + L.olat_lo;
  float* lse_old = reinterpret_cast<float*>(w + L.lse_old);
  void* oold = w + L.oold;
  void* oold_lo = w + L.oold_lo;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int b = shape->batch, s = shape->s_q, h = shape->num_heads;
  if (launch_var6_old_len(seqlens, b, n_new, shape->max_pages_per_seq, oldlen, st) != cudaSuccess) return MLA_ERR_CUDA;
  const ShapeInfo si = shape_info(&L.oshape);
  if (launch_schedule(oldlen, si, num_workers_for(sms), static_cast<int32_t*>(sched), st) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int cap = cap_slots_for(L.ws_bytes);
  rc = launch_decode_sm100(&L.oshape, qz, kv_cache, kv_scale, block_table, oldlen, softmax_scale, sched, ws, cap, olat,
                           lse_old, st, olat_lo);
  if (rc != MLA_OK) return rc;
  if (launch_combine(sched, ws, olat, lse_old, si.batch * si.tiles_per_req, cap, st, olat_lo) != cudaSuccess)
    return MLA_ERR_CUDA;
  rc = launch_decompress_o(b * s, h, olat, w_kvb2, oold, static_cast<int32_t*>(ws), st, olat_lo, oold_lo);
  if (rc != MLA_OK) return rc;
  return launch_var6_new(q, k_new, v_new, kv_cache, fp8, block_table, seqlens, oold, oold_lo, lse_old, b, s, h, n_new,
                         shape->max_pages_per_seq, shape->num_pages, shape->causal, softmax_scale, out, lse, ws,
                         st) == cudaSuccess
             ? MLA_OK
             : MLA_ERR_CUDA;
}

int mla_var6_get_device_status(const mla_shape_t* shape, int n_new, int num_sms, void* workspace, void* stream,
                               int* status) {
  Var6Layout L;
  if (!workspace || !status || !var6_layout(shape, n_new, num_sms, &L)) return MLA_ERR_INVALID_ARG;
  char* w = static_cast<char*>(workspace);
  return mla_get_device_status(w + L.sched, w + L.ws, stream, status);
}

int mla_absorb_q(int32_t rows, int32_t num_heads, const void* q, const void* w_k, void* qz, int32_t* device_status,
                 void* stream) {
  CallRange range_("mla_absorb_q");
  if (rows < 0 || num_heads < 1 || num_heads > 65535) return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!q || !w_k || !qz) return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(w_k, 16) || !aligned(qz, 16) || !aligned(device_status, 4))
    return MLA_ERR_INVALID_ARG;
  return launch_absorb_q(rows, num_heads, q, w_k, qz, device_status, static_cast<cudaStream_t>(stream));
}

int mla_decompress_o(int32_t rows, int32_t num_heads, const void* o_lat, const void* w_kvb2, void* out,
                     int32_t* device_status, void* stream) {
  CallRange range_("mla_decompress_o");
  if (rows < 0 || num_heads < 1 || num_heads > 65535) return MLA_ERR_INVALID_ARG;
  if (rows == 0) return MLA_OK;
  if (!o_lat || !w_kvb2 || !out) return MLA_ERR_INVALID_ARG;
  if (!aligned(o_lat, 16) || !aligned(w_kvb2, 16) || !aligned(out, 16) || !aligned(device_status, 4))
    return MLA_ERR_INVALID_ARG;
  return launch_decompress_o(rows, num_heads, o_lat, w_kvb2, out, device_status, static_cast<cudaStream_t>(stream));
}

const char* mla_error_string(int code) {
  switch (code) {
    case MLA_OK: return "MLA_OK: success";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: null pointer, bad size or misaligned pointer";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: shape not implemented (d_qk 576, d_v 512, page 64)";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE: schedule or workspace buffer too small";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: a CUDA runtime call failed";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT: a bounded device wait gave up";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK: out-of-range seqlen or page id, or a value row outside fp16 range, seen on the device";
    default: return "MLA: unknown error code";
  }
}

const char* mla_version(void) { return "mla_b200 0.1 (sm_100a)"; }

}  // extern "C"
