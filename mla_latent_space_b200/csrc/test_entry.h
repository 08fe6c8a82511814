/* Entry points of the TEST library only (libmla_b200_test.so, built from the
 * same sources with MLA_TEST_ENTRY_POINTS defined, plus the SIMT kernel).
 * The product library libmla_b200.so does not export them. */
#pragma once

#include "../../include/mla.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The decode of mla_decode_fwd computed by a plain SIMT kernel (fp32 FMA,
 * no tensor cores) over the same schedule and workspace: a second,
 * independently written device implementation for the parity tests.
 * Arguments, layouts and errors as for mla_decode_fwd. */
int mla_decode_fwd_simt(const mla_shape_t* shape, const void* q, const void* kv_cache,
                        const float* kv_scale, const int32_t* block_table,
                        const int32_t* seqlens, float softmax_scale, const void* sched,
                        void* workspace, size_t workspace_bytes, void* out, float* lse,
                        void* stream);

/* mla_decode_fwd with the decode kernel's test hook set: one of its bounded
 * waits waits on a barrier that nothing arrives on, runs out after about
 * 2 s, and the kernel's abort path runs (status bit, both CTAs stop, copies
 * and MMAs drained, tensor memory freed).  mla_get_device_status then
 * reports MLA_ERR_TIMEOUT; the outputs are not valid.  Faults nothing. */
int mla_test_decode_stalled(const mla_shape_t* shape, const void* q, const void* kv_cache,
                            const float* kv_scale, const int32_t* block_table,
                            const int32_t* seqlens, float softmax_scale, const void* sched,
                            void* workspace, size_t workspace_bytes, void* out, float* lse,
                            void* stream);

#ifdef __cplusplus
}
#endif
