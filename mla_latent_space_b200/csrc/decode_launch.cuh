// Host-side launch interface of the tcgen05 decode kernel, split in two so a
// caller can finish every check that can fail on the host (tensor-map
// encoding, the shared-memory attribute, the SM count) before it enqueues
// anything on the stream.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace mla {

// What prepare_decode_sm100 builds: the TMA descriptors over the page pool
// and the query rows, and the launch geometry.  Plain data, valid for the
// pointers and shape it was built from.
struct DecodePrepared {
  CUtensorMap pool_map, q_map, rope_map;
  int sms;
  bool fp8;
};

// Host work only: encodes the tensor maps and sets the kernel's dynamic
// shared-memory limit on the current device.  Returns MLA_OK or
// MLA_ERR_CUDA; enqueues nothing.
int prepare_decode_sm100(const mla_shape_t* shape, const void* q, const void* kv, DecodePrepared* pr);

// Enqueues the decode kernel built by prepare_decode_sm100 on `stream`.
// out_lo (optional, bf16 like out): whole tiles then write O as two terms,
// out = bf16(O) and out_lo = bf16(O - out); split tiles leave both to the
// combine (launch_combine with the same out_lo).
// test_stall: 0, except from the test library's stalled-decode entry point
// (a bounded wait in the kernel then runs out on purpose).
int enqueue_decode_sm100(const DecodePrepared& pr, const mla_shape_t* shape, const void* q, const void* kv,
                         const float* kv_scale, const int32_t* block_table, const int32_t* seqlens, float scale,
                         const void* sched, void* ws, int cap_slots, void* out, float* lse, cudaStream_t stream,
                         void* out_lo = nullptr, int test_stall = 0);

// prepare + enqueue.
int launch_decode_sm100(const mla_shape_t* shape, const void* q, const void* kv, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seqlens, float scale, const void* sched,
                        void* ws, int cap_slots, void* out, float* lse, cudaStream_t stream,
                        void* out_lo = nullptr);

// The log-sum-exp merge of split tiles (and O = 0, lse = -inf for tiles
// with no visible key); out_lo as for enqueue_decode_sm100.
cudaError_t launch_combine(const void* sched, const void* ws, void* out, float* lse, int num_tiles,
                           int cap_slots, cudaStream_t stream, void* out_lo = nullptr);

}  // namespace mla
