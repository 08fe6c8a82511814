// Placeholder launcher: routes to the SIMT kernel until the tcgen05 kernel
// lands in this file.
#include "common.cuh"
#include <cuda_runtime.h>

namespace mla {
cudaError_t launch_decode_simt(const void* q, const void* kv, const float* kv_scale, const int32_t* block_table,
                               const int32_t* seqlens, float scale, const void* sched, void* ws, void* out,
                               float* lse, int num_pages, int fp8, int cap_slots, int grid_ctas,
                               cudaStream_t stream);

int launch_decode_sm100(const mla_shape_t* shape, const void* q, const void* kv, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seqlens, float scale, const void* sched,
                        void* ws, int cap_slots, void* out, float* lse, cudaStream_t stream) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MLA_ERR_CUDA;
  cudaError_t e = launch_decode_simt(q, kv, kv_scale, block_table, seqlens, scale, sched, ws, out, lse,
                                     shape->num_pages, shape->cache_dtype == MLA_CACHE_FP8_E4M3, cap_slots, sms,
                                     stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
}  // namespace mla
