/*
 * mla_b200.h — C ABI of the B200 (sm_100a) MLA paged-KV decode library.
 *
 * Operation (cnblogs "DeepSeek 开源记-第1天-FlashMLA", §2 核心功能 and §6.2
 * 基本使用): Multi-head Latent Attention decoding over a paged BF16 latent
 * KV cache.  Every cached token holds one row of d = 576 values per KV head
 * (512 latent + 64 rotary); the value vector is the first dv = 512 values of
 * the same row; pages hold 64 tokens (m.ygpos.cn "DeepSeek代碼開源第一彈Flash
 * MLA", release list) and are addressed through a block table; sequences have
 * variable lengths.  For every query row:
 *     x_j = scale * <q, K_j>,  lse = ln sum_j exp(x_j),
 *     O   = sum_j exp(x_j - lse) * V_j.
 *
 * Conventions for every call below
 *   - Pointers named *_d are device pointers; all are owned by the caller and
 *     must stay valid until the stream work completes.  The library allocates
 *     no device memory and never synchronises the stream.
 *   - All calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream), which must belong to the current device:
 *     kernels are launched on the current device.
 *   - Kernels are launched with programmatic stream serialization: each may
 *     start its set-up while the previous kernel of the stream is finishing,
 *     and waits for that kernel to complete before reading or writing any
 *     buffer, so stream order is kept.  The metadata and decode kernels, and
 *     the combine kernel (which the decode call launches last), let the next
 *     kernel start early in the same way: a kernel of the caller's launched
 *     after them with programmatic serialization must itself wait for its
 *     predecessor (griddepcontrol.wait / cudaGridDependencySynchronize) before
 *     reading `out`, `lse`, `tile_md` or `num_splits`; one launched normally
 *     needs nothing.
 *   - Return value: MLA_OK or a negative MLA_ERR_* code; on error nothing is
 *     launched.  Errors detected on the device (bad page ids, sequence longer
 *     than its block-table row, a bounded wait that ran out) are written to
 *     the optional `status_d` word (int32, 0 = OK) and the affected rows are
 *     zeroed; read it after synchronising.
 *   - Layouts are dense, row-major, contiguous (innermost index last).
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_OK                0
#define MLA_ERR_INVALID_ARG  -1   /* null pointer, bad alignment, bad sizes      */
#define MLA_ERR_UNSUPPORTED  -2   /* d != 576, dv != 512, device not sm_100       */
#define MLA_ERR_WORKSPACE    -3   /* workspace missing or too small              */
#define MLA_ERR_CUDA         -4   /* a CUDA runtime/driver call failed           */
#define MLA_ERR_TIMEOUT      -5   /* device-side bounded wait gave up (status_d) */
#define MLA_ERR_BAD_INPUT    -6   /* device-side input check failed (status_d)   */

/* Element type of q, k_cache and out (kind::f16 MMAs accumulate in fp32 for both). */
#define MLA_DTYPE_BF16  0
#define MLA_DTYPE_FP16  1

#define MLA_HEAD_DIM   576
#define MLA_VALUE_DIM  512
#define MLA_PAGE_SIZE  64
#define MLA_MD_WORDS   8      /* int32 words per tile-scheduler entry */

/* Human-readable name of a status code.  Never NULL. */
const char* mla_status_string(int status);

/* Number of SMs of the current device (cached per device), or a negative
 * MLA_ERR_* code. */
int mla_device_sm_count(void);

/* Rows per decode CTA for `rows_per_kv` query rows per KV head: 16, 32 or 64.
 * Host-only, pure. */
int mla_rows_per_block(int rows_per_kv);

/* Number G of scheduler parts ("tile_scheduler_metadata" entries) for the
 * given shape: max(1, num_sms / (h_kv * ceil(rows_per_kv / rows_per_block))).
 * Host-only, pure.  Returns a negative MLA_ERR_* code on bad arguments. */
int mla_num_parts(int rows_per_kv, int h_kv, int num_sms);

/*
 * Tile-scheduler metadata (jsxs2.com "什麼是FlashMLA", §3.1 分塊調度與並行
 * 計算: the work is cut into blocks and scheduled over the SMs; cnblogs §6.2:
 * get_mla_metadata(cache_seqlens, s_q*h_q//h_kv, h_kv) returns
 * tile_scheduler_metadata and num_splits).
 *
 *   cache_seqlens_d  int32[batch]            sequence lengths L_b >= 0
 *   rows_per_kv      s_q * h_q / h_kv
 *   h_kv             number of KV heads
 *   num_sms          SMs to schedule over (<= 0: this device's SM count)
 *   tile_md_d        int32[G * MLA_MD_WORDS]  out: per part
 *                    (begin_b, begin_page, end_b, end_page, first_piece,
 *                     n_pieces, 0, 0), end exclusive
 *   num_splits_d     int32[batch + 1]        out: prefix sum of pieces per
 *                    sequence
 *   num_parts_out    host int*, out: G (may be NULL)
 * One single-CTA kernel; integer arithmetic only (bit-exact, deterministic).
 * Limits: batch <= 8192 and G <= 4096 (MLA_ERR_INVALID_ARG otherwise).
 * The kernel reads cache_seqlens_d and computes the table before it waits for
 * the previous kernel of the stream (it waits only before writing its
 * outputs), so a kernel of the caller's that writes cache_seqlens_d right
 * before this call must not let its dependents launch early
 * (griddepcontrol.launch_dependents) before those writes.  Kernels launched
 * without programmatic launch and copies need nothing: the stream orders them.
 */
int mla_get_metadata(const int32_t* cache_seqlens_d, int batch, int rows_per_kv, int h_kv,
                     int num_sms, int32_t* tile_md_d, int32_t* num_splits_d,
                     int* num_parts_out, void* stream);

/* Bytes of device workspace mla_decode_paged needs for split partials:
 * (batch + num_parts) * h_kv * rows_per_kv * (dv + 1) * 4, rounded up to
 * 256.  Returns 0 on bad arguments. */
size_t mla_workspace_bytes(int batch, int rows_per_kv, int h_kv, int dv, int num_parts);

/*
 * Split-KV MLA decode (cnblogs §6.2: flash_mla_with_kvcache(q, blocked_k,
 * block_table, cache_seqlens, dv, tile_scheduler_metadata, num_splits,
 * causal) -> output, lse; compute flow cnblogs §4.1: load, blockwise scores,
 * softmax, merge of the outputs).
 *
 *   q_d             bf16 [batch, s_q, h_q, d]             (16-byte aligned)
 *   k_cache_d       bf16 [num_pages, 64, h_kv, d]          (16-byte aligned)
 *   block_table_d   int32 [batch, max_pages_per_seq]; entries for pages at
 *                   or beyond ceil(L_b/64) are never read
 *   cache_seqlens_d int32 [batch]; L_b <= 64 * max_pages_per_seq required;
 *                   batch <= 8192 (the limit of mla_get_metadata)
 *   d, dv           must be 576 and 512
 *   tile_md_d, num_splits_d, num_parts: exactly as produced by
 *                   mla_get_metadata for the same seqlens, rows_per_kv, h_kv
 *   causal          0/1; query token s sees keys j < L - (s_q - 1 - s)
 *   softmax_scale   multiplies <q, K_j>; pass 576^-0.5 for the usual scale
 *   workspace_d     >= mla_workspace_bytes(...) bytes, 256-byte aligned
 *   out_d           bf16 [batch, s_q, h_q, dv]             (16-byte aligned)
 *   lse_d           fp32 [batch, s_q, h_q]; natural log; -inf for rows that
 *                   see no key (their out row is 0)
 *   status_d        optional int32 device word (see conventions)
 * Launches the decode kernel and then the combine kernel, both on `stream`;
 * the combine merges the rows of split sequences and zero-fills empty ones
 * (its blocks for sequences the decode kernel finished return at once).
 */
int mla_decode_paged(const void* q_d, const void* k_cache_d, int num_pages,
                     const int32_t* block_table_d, int max_pages_per_seq,
                     const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                     int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d,
                     int num_parts, int causal, float softmax_scale,
                     void* workspace_d, size_t workspace_bytes,
                     void* out_d, float* lse_d, int32_t* status_d, void* stream);

/*
 * Debug/testing variant of mla_decode_paged with extra knobs; same contract
 * otherwise.
 *   debug_flags  bit 0: the softmax warps wait on a barrier that nothing
 *                signals, so the bounded wait must run out and report
 *                MLA_ERR_TIMEOUT through status_d (fault detection test).
 *                bit 1: launch only the decode kernel; the caller then calls
 *                mla_combine with the same workspace (used to time the two
 *                kernels separately).
 *                bit 2: for more than 64 rows per KV head, use one CTA per
 *                64-row block instead of CTA pairs (cross-check of the two
 *                decode kernels).
 *   timeout_ns   limit of every device-side wait (0 = default, 4 s).
 */
int mla_decode_paged_ex(const void* q_d, const void* k_cache_d, int num_pages,
                        const int32_t* block_table_d, int max_pages_per_seq,
                        const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                        int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d,
                        int num_parts, int causal, float softmax_scale,
                        void* workspace_d, size_t workspace_bytes,
                        void* out_d, float* lse_d, int32_t* status_d,
                        int debug_flags, unsigned long long timeout_ns, void* stream);

/*
 * Merge of split partials (cnblogs §4.1 计算流程, 输出结果合并): for every query
 * row of a sequence cut into n >= 2 pieces, lse = ln sum_i exp(lse_i) and
 * O = sum_i exp(lse_i - lse) * O_i; sequences with no piece get O = 0 and
 * lse = -inf; sequences with one piece are left untouched (the decode kernel
 * wrote them).  workspace_d holds the partials mla_decode_paged_ex left with
 * debug_flags bit 1; the other arguments are those of that call.
 */
int mla_combine(const int32_t* num_splits_d, const void* workspace_d, size_t workspace_bytes, int batch,
                int s_q, int h_q, int h_kv, int num_parts, void* out_d, float* lse_d, void* stream);

/*
 * mla_decode_paged_ex and mla_combine for either element type.  The pages list
 * FP16 next to BF16 among the kernel's data types (cnblogs §2 关键特性); the
 * release notes on every page name BF16, which the calls above use.
 *   dtype   MLA_DTYPE_BF16 or MLA_DTYPE_FP16: the type of q_d, k_cache_d and
 *           out_d (2 bytes per element either way; same layouts and alignment
 *           rules).  P is rounded to the same type before the value product.
 * Other arguments and results exactly as mla_decode_paged_ex / mla_combine;
 * MLA_ERR_INVALID_ARG for any other dtype.
 */
int mla_decode_paged_typed(int dtype, const void* q_d, const void* k_cache_d, int num_pages,
                           const int32_t* block_table_d, int max_pages_per_seq,
                           const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                           int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d,
                           int num_parts, int causal, float softmax_scale,
                           void* workspace_d, size_t workspace_bytes,
                           void* out_d, float* lse_d, int32_t* status_d,
                           int debug_flags, unsigned long long timeout_ns, void* stream);
int mla_combine_typed(int dtype, const int32_t* num_splits_d, const void* workspace_d, size_t workspace_bytes,
                      int batch, int s_q, int h_q, int h_kv, int num_parts, void* out_d, float* lse_d,
                      void* stream);

/*
 * Allocation-free variant of mla_decode_paged.  The pages describe no such
 * call; it has no counterpart there and exists for callers that cannot call
 * cudaMalloc: code that runs where the device allocator belongs to someone
 * else (a plugin or custom operator inside a host framework with its own
 * memory pool), where allocation after start-up is forbidden by a fixed
 * memory budget, or where the caller simply has no handle to allocate with.
 *
 * Same arguments and results as mla_decode_paged, minus the workspace: the
 * split partials go to a scratch array of MLA_NOALLOC_SCRATCH_BYTES that the
 * library holds in a file-scope __device__ variable, so every GPU that loads
 * the library keeps those bytes until the process exits.  Nothing is
 * allocated by this call (no cudaMalloc, cudaFree or allocating library
 * routine).
 *   - Returns MLA_ERR_WORKSPACE if the shape needs more than
 *     MLA_NOALLOC_SCRATCH_BYTES (mla_workspace_bytes(...) larger than it).
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it together
 *     with the unique id of the device's current context; a later call made
 *     in another context of that device (for example after cudaDeviceReset
 *     destroyed the old one) looks it up again.  Make the first call on a
 *     device, and the first call after such a reset, outside any stream
 *     capture.
 *   - `stream` must belong to the current device (as for every call of this
 *     library): the scratch array used is the current device's.
 *   - All calls share the one scratch array and it keeps the previous call's
 *     contents; nothing in it needs to start at zero (every partial is written
 *     before it is read).  Calls that overlap on the GPU (other streams, other
 *     host threads) race on it: serialise them.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

int mla_decode_paged_noalloc(const void* q_d, const void* k_cache_d, int num_pages,
                             const int32_t* block_table_d, int max_pages_per_seq,
                             const int32_t* cache_seqlens_d, int batch, int s_q, int h_q, int h_kv,
                             int d, int dv, const int32_t* tile_md_d, const int32_t* num_splits_d,
                             int num_parts, int causal, float softmax_scale,
                             void* out_d, float* lse_d, int32_t* status_d, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_H */
