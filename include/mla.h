/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA decode library, libmla_b200.so.
 *
 * Multi-head Latent Attention decode in absorbed latent space ("MLA Cost
 * Analysis & Regime Guide", section "Absorption Trick"): with the key and
 * value up-projections absorbed into the query and the output projection,
 * every head scores directly against the shared latent cache,
 *
 *     S = scale * Qz . C^T            C = cache rows [latent 512 | RoPE 64]
 *     O = softmax(S) . C[:, :512]     (decompressed by a separate GEMM)
 *
 * Shapes follow the page's "Tensor Shapes" table (h=128, k=512, p=64).  The
 * split-KV scheduler and the log-sum-exp merge of partial results follow the
 * FlashMLA-2 newsletter page ("Architectural Analysis": sequence partitions
 * balanced across SMs for jagged batches).
 *
 * Around the decode: the query absorption and the output decompression
 * (mla_absorb_q, mla_decompress_o), token-level sparse decode over listed
 * cache positions (mla_sparse_*), and the MLAvar6+ split decode with the
 * newest tokens held decompressed (mla_var6_*).
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library never allocates device memory, never frees caller memory and
 *    never synchronises the stream (except mla_get_device_status, which
 *    says so).
 *  - Every call takes the caller's cudaStream_t (passed as void*: NULL is
 *    the legacy default stream) and enqueues its work there.
 *  - Return value: MLA_OK (0) or a negative MLA_ERR_* code.  Arguments are
 *    validated on the host BEFORE anything is launched; an error return
 *    means nothing was enqueued.  mla_error_string() names each code.
 *  - Layouts are dense and row-major (innermost dimension last, contiguous).
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes --------------------------------------------------------- */
enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misaligned pointer      */
  MLA_ERR_UNSUPPORTED = -2,  /* shape the kernels do not implement             */
  MLA_ERR_WORKSPACE = -3,    /* workspace / schedule buffer too small          */
  MLA_ERR_CUDA = -4,         /* a CUDA runtime call failed (launch, attribute) */
  MLA_ERR_TIMEOUT = -5,      /* device status: a bounded wait gave up          */
  MLA_ERR_DEVICE_CHECK = -6  /* device status: seqlen / page id out of range,
                                or a value row outside fp16's range            */
};

/* ---- cache element types -------------------------------------------------- */
enum {
  MLA_CACHE_BF16 = 0,      /* page = 64 rows x 576 bf16 = 73,728 bytes           */
  MLA_CACHE_FP8_E4M3 = 1   /* page = 64x512 e4m3 bytes, then 64x64 bf16 RoPE
                              values (40,960 bytes); scales in kv_scale       */
};

/* Fixed geometry of this library (DeepSeek-V3 defaults of the page's
 * "Tensor Shapes" table; one 128-row tile = 128 (query token, head) rows). */
#define MLA_D_QK 576
#define MLA_D_V 512
#define MLA_PAGE_SIZE 64
#define MLA_TILE_ROWS 128
#define MLA_D_HEAD 128 /* d: per-head query/key/value dims before absorption */
#define MLA_D_ROPE 64  /* p: RoPE dims (the last 64 of the 576)              */

/* Problem description.  Every field is read on the host only. */
typedef struct {
  int32_t batch;             /* b: requests in the batch, >= 1                  */
  int32_t s_q;               /* query tokens per request (1 = decode, >1 = spec) */
  int32_t num_heads;         /* h: query heads; s_q*h rows are tiled by 128    */
  int32_t d_qk;              /* must be 576 (k + p)                             */
  int32_t d_v;               /* must be 512 (k)                                 */
  int32_t page_size;         /* must be 64                                      */
  int32_t max_pages_per_seq; /* row length of block_table, >= 1                 */
  int32_t num_pages;         /* pages in the cache pool, >= 1                   */
  int32_t cache_dtype;       /* MLA_CACHE_BF16 or MLA_CACHE_FP8_E4M3            */
  int32_t causal;            /* 1: query token i sees keys j <= t - s_q + i    */
} mla_shape_t;

/* Bytes of the device buffer mla_get_schedule fills.  num_sms is the SM
 * count of the device that will run the decode (one scheduler worker per
 * pair of SMs).  Returns 0 for an invalid shape. */
size_t mla_schedule_bytes(const mla_shape_t* shape, int num_sms);

/* Bytes of the device workspace mla_decode_fwd / mla_combine use: fp32
 * partial results of split tiles (at most 2 per worker, 128x512 O + 128
 * lse each) plus a 256-byte status area.  Returns 0 for an invalid shape. */
size_t mla_workspace_bytes(const mla_shape_t* shape, int num_sms);

/* a1 -- split-KV schedule (FlashMLA-2 newsletter, "Architectural Analysis").
 * Splits the work sum over tiles of (visible pages + a fixed per-piece
 * cost) into num_sms/2 contiguous, equally costed ranges of (tile, page)
 * units, and records for every tile how many pieces it was cut into and
 * where their partial results go.  Runs one small kernel on `stream`.
 *   seqlens : device int32 [batch], tokens in the cache per request
 *             INCLUDING the s_q new ones.  Values outside
 *             [0, max_pages_per_seq*64] are clamped and flagged
 *             (MLA_ERR_DEVICE_CHECK from mla_get_device_status).
 *   sched   : device buffer of mla_schedule_bytes(shape, num_sms) bytes,
 *             4-byte aligned; written entirely by this call.
 * The schedule depends only on seqlens, so one schedule serves every layer
 * of a decode step. */
int mla_get_schedule(const mla_shape_t* shape, const int32_t* seqlens, int num_sms,
                     void* sched, size_t sched_bytes, void* stream);

/* a2-a7 (+a9 FP8, a10 causal) -- the decode itself.
 *   q          : bf16 [batch, s_q, num_heads, 576], the absorbed query rows
 *                (q_nope . W_k ++ q_pe), 16-byte aligned.
 *   kv_cache   : page pool.  BF16: bf16 [num_pages, 64, 576].  FP8: uint8
 *                [num_pages, 40960] (64x512 e4m3 then 64x64 bf16 RoPE).
 *                256-byte aligned base.  Value rows are the first 512
 *                entries of each cache row.
 *   kv_scale   : FP8 only: fp32 [num_pages, 64], one dequantisation scale
 *                per cached token (value = e4m3 * scale).  NULL for BF16.
 *   block_table: int32 [batch, max_pages_per_seq]; entry [r][j] is the pool
 *                page holding tokens 64j..64j+63 of request r.  Entries past
 *                ceil(visible/64) are never read.  Out-of-range page ids are
 *                skipped and flagged (MLA_ERR_DEVICE_CHECK).
 *                The PV product runs in fp16: a value entry (or, FP8, an
 *                e4m3 value times its scale) of magnitude 65520 or more, or
 *                a NaN / infinity, is flagged (MLA_ERR_DEVICE_CHECK) and the
 *                output of the tiles that read it is not valid.
 *   seqlens    : the same int32 [batch] array given to mla_get_schedule.
 *   softmax_scale : multiplies the raw 576-d dot product before softmax.
 *   sched      : filled by mla_get_schedule for this shape and num_sms.
 *   workspace  : mla_workspace_bytes(shape, num_sms) bytes, 256-byte
 *                aligned; the caller must not touch it between this call and
 *                mla_combine.
 *   out        : bf16 [batch, s_q, num_heads, 512], the latent output rows.
 *                The tensor-core kernel (tcgen05, 2-SM clusters) rounds P to
 *                fp16 and converts V to fp16 on chip, so value rows must lie
 *                within fp16 range (|v| < 65504; FP8: |e4m3 * scale|).  FP8
 *                cache: the latent scores multiply the cache's e4m3 values
 *                directly with a two-part e4m3 copy of the query's latent
 *                part (per-row power-of-two scale), which holds every bf16
 *                query value exactly down to 2^-11 of its row's largest.
 *   lse        : fp32 [batch, s_q, num_heads], natural-log log-sum-exp of the
 *                scaled scores (-inf for a row that sees no key).
 * Tiles cut into several pieces are finished by mla_combine; tiles in one
 * piece are written directly.  Call mla_combine after every decode. */
int mla_decode_fwd(const mla_shape_t* shape, const void* q, const void* kv_cache,
                   const float* kv_scale, const int32_t* block_table, const int32_t* seqlens,
                   float softmax_scale, const void* sched, void* workspace, size_t workspace_bytes,
                   void* out, float* lse, void* stream);

/* a8 -- log-sum-exp merge of split pieces: for each split row,
 * L = ln sum_i e^{lse_i}, O = sum_i e^{lse_i - L} O_i; writes out/lse for
 * split tiles and for tiles that see no key at all (O = 0, lse = -inf).
 * Arguments as for mla_decode_fwd. */
int mla_combine(const mla_shape_t* shape, const void* sched, const void* workspace,
                size_t workspace_bytes, void* out, float* lse, void* stream);

/* Reads and clears the sticky device status words that the scheduler and
 * the decode kernels set instead of trapping (a bounded wait that gave up,
 * an out-of-range seqlen or page id, a value row outside fp16's range).
 * SYNCHRONISES `stream`.  *status
 * receives MLA_OK, MLA_ERR_TIMEOUT or MLA_ERR_DEVICE_CHECK. */
int mla_get_device_status(const void* sched, void* workspace, void* stream, int* status);

/* Host copy of the scheduler (same code as the device kernel), for tests
 * and tools: seqlens and sched are HOST pointers here. */
int mla_plan_schedule_host(const mla_shape_t* shape, const int32_t* seqlens, int num_sms,
                           void* sched, size_t sched_bytes);

/* The pages have no counterpart to this call: it is the whole decode step
 * (schedule, decode, combine) for callers that cannot allocate device
 * memory -- a host program linking only this C ABI with no device allocator
 * of its own, or a serving loop whose memory is entirely reserved up front --
 * and so cannot pass the sched and workspace buffers that mla_get_schedule /
 * mla_decode_fwd / mla_combine take.  It allocates nothing: its schedule and
 * its device status word live in a static device array of 320 KiB inside
 * the library (one per device), whose address is looked up with
 * cudaGetSymbolAddress on the first call on each device; that first call
 * must therefore not be made while `stream` is being captured.  To fit that
 * array, work is assigned to the SM pairs in whole 128-row tiles (no tile is
 * split, no fp32 partial result is kept), so a batch with one very long
 * request balances worse than with mla_get_schedule.
 *   Limit: batch * ceil(s_q * num_heads / 128) <= 16384 tiles; larger
 *   shapes return MLA_ERR_WORKSPACE before anything is enqueued.
 *   Arguments as for mla_decode_fwd; device_status: optional device int32
 *   (4-byte aligned) that receives, in stream order, this call's status
 *   word (0, or the bits behind MLA_ERR_TIMEOUT / MLA_ERR_DEVICE_CHECK);
 *   NULL to skip.  The call zeroes the status word before its kernels run.
 * Every check that can fail on the host (arguments, the tile limit, the
 * tensor-map encoding) is made before the first enqueue, so those errors
 * leave nothing on the stream; only a failing kernel launch itself
 * (MLA_ERR_CUDA) can leave this call's earlier kernels enqueued.
 * The static array's address is cached per device for the life of the
 * process; calling this after cudaDeviceReset on a device it was used on is
 * not supported.
 * Calls that overlap in time on one device (different streams, or threads
 * without ordering) share the static array and race: serialise them. */
int mla_decode_fwd_noalloc(const mla_shape_t* shape, const void* q, const void* kv_cache,
                           const float* kv_scale, const int32_t* block_table,
                           const int32_t* seqlens, float softmax_scale, void* out, float* lse,
                           int32_t* device_status, void* stream);

/* ---- token-level sparse decode --------------------------------------------
 * The FlashMLA product page lists token-level sparse attention for decoding.
 * Query token (r, i) attends, with all its heads, to exactly the cache rows
 * at the positions listed in indices[r][i][0..topk): S = scale * q . C_j^T
 * over those rows, O = softmax(S) . C[:, :512], lse as for mla_decode_fwd.
 * A position outside [0, seqlens[r]) (e.g. -1 padding) is skipped; a
 * position listed twice is two keys; a list with no valid position gives
 * O = 0 and lse = -inf.  Positions resolve through block_table as for the
 * dense decode.  Both cache types; causal must be 0 (the lists decide what
 * each query token sees).  The selected rows (FP8: with their scales) are
 * gathered into scratch pages of the workspace, in the cache's own page
 * format, then the tensor-core decode runs over them.
 *   shape, q, kv_cache, kv_scale, block_table, seqlens, out, lse: as for
 *             mla_decode_fwd (kv_scale NULL for a BF16 cache).
 *   topk    : list length per query token, 1 <= topk <= 2^24.
 *   indices : device int32 [batch, s_q, topk], 4-byte aligned.
 *   workspace: device buffer of mla_sparse_workspace_bytes(shape, topk,
 *             num_sms of this device) bytes, 256-byte aligned, zero-filled
 *             before its first use (it holds the status word); the caller
 *             must not touch it while the call's work runs.
 * Returns MLA_ERR_UNSUPPORTED for a shape whose b*s_q*ceil(topk/64) scratch
 * pages reach 2^26; MLA_ERR_WORKSPACE when workspace_bytes is too small. */
size_t mla_sparse_workspace_bytes(const mla_shape_t* shape, int topk, int num_sms);
int mla_sparse_decode_fwd(const mla_shape_t* shape, int topk, const void* q, const void* kv_cache,
                          const float* kv_scale, const int32_t* block_table, const int32_t* seqlens,
                          const int32_t* indices, float softmax_scale, void* workspace, size_t workspace_bytes,
                          void* out, float* lse, void* stream);
/* Device status of the sparse decode's kernels (bounded waits, out-of-range
 * lengths or page ids); as mla_get_device_status, SYNCHRONISES `stream`. */
int mla_sparse_get_device_status(const mla_shape_t* shape, int topk, int num_sms, void* workspace, void* stream,
                                 int* status);

/* ---- MLAvar6+ split attention for speculative steps -------------------------
 * "MLA Cost Analysis & Regime Guide", section "MLAvar6+ Design": each
 * request's o = t - n older tokens stay in latent form (the cache), its n
 * newest are given as decompressed per-head keys and values; one softmax
 * covers both.  Old token j scores scale * qz . C_j and contributes its
 * decompressed value C_j[:512] . w_kvb2[head]^T; new token m (position
 * t - n + m; absent when that is negative) scores scale * (q_nope . k_new[m]
 * + q_pe . C_{t-n+m}[512:]) and contributes v_new[m].  Query token i sees
 * positions below t - s_q + i + 1 (causal) or t.  Runs as the latent decode
 * over the old tokens, the output decompression of its result, and one
 * kernel that attends over the new tokens and merges by log-sum-exp.
 *   shape    : as for mla_decode_fwd; s_q <= 32; causal steps need n >= s_q
 *              (every old token then precedes every query position).
 *   n_new    : n, 0 <= n <= 2^20 (0: the latent path alone, decompressed).
 *   qz       : bf16 [batch, s_q, h, 576], the absorbed query (old tokens).
 *   q        : bf16 [batch, s_q, h, 192] = [q_nope | q_pe] (new tokens).
 *   kv_cache, kv_scale, block_table, seqlens: as for mla_decode_fwd.
 *   k_new    : bf16 [batch, n, h, 128] decompressed keys (RoPE part excluded).
 *   v_new    : bf16 [batch, n, h, 128] decompressed values.
 *   w_kvb2   : bf16 [h, 128, 512], as for mla_decompress_o.
 *   workspace: mla_var6_workspace_bytes(shape, n, num_sms of this device)
 *              bytes, 256-byte aligned, zero-filled before its first use.
 *   out      : bf16 [batch, s_q, h, 128];  lse: fp32 [batch, s_q, h]. */
size_t mla_var6_workspace_bytes(const mla_shape_t* shape, int n_new, int num_sms);
int mla_var6_decode_fwd(const mla_shape_t* shape, int n_new, const void* qz, const void* q, const void* kv_cache,
                        const float* kv_scale, const int32_t* block_table, const int32_t* seqlens, const void* k_new,
                        const void* v_new, const void* w_kvb2, float softmax_scale, void* workspace,
                        size_t workspace_bytes, void* out, float* lse, void* stream);
/* Device status of the split decode's kernels; as mla_get_device_status. */
int mla_var6_get_device_status(const mla_shape_t* shape, int n_new, int num_sms, void* workspace, void* stream,
                               int* status);

/* ---- the projections on either side of the decode -------------------------
 * "MLA Cost Analysis & Regime Guide", section "Absorption Trick": the key
 * up-projection Wk is folded into the query (Q . K^T = (Q . Wk^T) . Z^T),
 * and the latent output is decompressed by a separate GEMM after the
 * attention (O_latent . W_kvb2^T).  Both run on the tensor core (tcgen05,
 * bf16 operands, fp32 accumulation, bf16 result rounded to nearest even).
 * rows = batch * s_q query rows; every tensor is dense row-major and its
 * pointer 16-byte aligned; inputs and outputs must not overlap.  rows == 0
 * enqueues nothing and returns MLA_OK (pointers unchecked).  device_status: optional device int32 (4-byte aligned)
 * that a bounded wait which gave up ORs 1 into (NULL to skip; never cleared
 * by these calls).  Returns MLA_OK, MLA_ERR_INVALID_ARG (null or misaligned
 * pointer, rows < 0, num_heads outside [1, 65535]) or MLA_ERR_CUDA. */

/* f1a -- absorbed query rows, the q argument of mla_decode_fwd:
 *   qz[r, j, c]       = sum_n q[r, j, n] * w_k[j, c, n]   (c < 512, n < 128)
 *   qz[r, j, 512 + e] = q[r, j, 128 + e]                  (e < 64, copied)
 *   q   : bf16 [rows, num_heads, 192] = [q_nope 128 | q_pe 64] per head
 *   w_k : bf16 [num_heads, 512, 128]; head j's keys are K_j = Z . w_k[j]
 *   qz  : bf16 [rows, num_heads, 576] (written entirely) */
int mla_absorb_q(int32_t rows, int32_t num_heads, const void* q, const void* w_k, void* qz,
                 int32_t* device_status, void* stream);

/* f1b -- output decompression of the latent attention result:
 *   out[r, j, v] = sum_c o_lat[r, j, c] * w_kvb2[j, v, c]   (v < 128, c < 512)
 *   o_lat  : bf16 [rows, num_heads, 512] (the out of mla_decode_fwd)
 *   w_kvb2 : bf16 [num_heads, 128, 512]; head j's values are V_j = Z . w_kvb2[j]^T
 *   out    : bf16 [rows, num_heads, 128] (written entirely) */
int mla_decompress_o(int32_t rows, int32_t num_heads, const void* o_lat, const void* w_kvb2, void* out,
                     int32_t* device_status, void* stream);

/* Human-readable name of an MLA_* code (static storage). */
const char* mla_error_string(int code);

/* Library version string (static storage). */
const char* mla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
