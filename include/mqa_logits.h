/*
 * mqa_logits.h -- C ABI of the B200 (sm_100a) paged MQA-logits library.
 *
 * The operation (the page "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA
 * Logits 커널 도입", introduction: the DeepSeek MLA sparse-attention indexer's
 * "per-head weighted sum of rectified scores"):
 *
 *   for every batch row b, draft position n < next_n and token t < out_len:
 *     ctx_bn = clamp(context_lens[b] - next_n + 1 + n, 0, context_lens[b])
 *     out[b][n][t] = sum_h weights[b][n][h] * max(0, s_t * dot(q[b][n][h][:], k_t[:]))
 *                    when t < ctx_bn, and -inf otherwise,
 *   where k_t (and s_t) live in page block_table[b][t / page_size] at slot
 *   t % page_size of the paged K cache.
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is a DEVICE pointer, except `params`, which is a
 *     host pointer read during the call only. The caller allocates and owns
 *     every buffer (the page's third article, section 2, keeps TMA workspace
 *     and outputs caller-owned for the same reason: nothing is allocated per
 *     call, so every call can be captured in a CUDA graph).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and never synchronise the host.
 *   - Return value: MQA_OK, or a negative mqa_status. On error nothing is
 *     launched and mqa_logits_last_error() describes the failure.
 *   - The library needs a compute capability 10.0 device (B200); anything
 *     else returns MQA_ERR_ARCH (the page's fifth article, section on the
 *     target check, gates its SM100 kernels the same way).
 *   - Thread safety: calls from several host threads are safe; the error
 *     message is kept per thread.
 */
#ifndef MQA_LOGITS_H_
#define MQA_LOGITS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mqa_status {
    MQA_OK = 0,
    MQA_ERR_INVALID_ARG = -1,  /* a host-side argument check failed */
    MQA_ERR_ARCH = -2,         /* current device is not compute capability 10.0 */
    MQA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
    MQA_ERR_UNSUPPORTED = -4,  /* valid arguments outside the compiled kernel set */
    MQA_ERR_DEVICE_CHECK = -5  /* mqa_logits_check_status only: the device status word has
                                  bits set (a validate-mode check or an expired wait) */
} mqa_status;

/* Bits of a device status word. A logits kernel ORs them into the library's
 * own word for the device (always; read it with mqa_logits_get_status) and,
 * if given, into the caller's mqa_logits_params.status. The caller clears
 * them. No bit is ever raised by a trap. */
#define MQA_STATUS_TIMEOUT      0x1u  /* a pipeline wait exceeded timeout_ns; the CTA stopped and
                                         part of out may be unwritten */
#define MQA_STATUS_BAD_PAGE     0x2u  /* validate mode: a block_table entry outside [0, num_pages) */
#define MQA_STATUS_BAD_CONTEXT  0x4u  /* validate mode: context_lens[b] < 0 or > out_len or > max_pages_per_row*page_size */
#define MQA_STATUS_STALE_SCHEDULE 0x8u /* validate mode: the schedule does not match context_lens */
#define MQA_STATUS_Q_RANGE      0x10u /* fp4: a q row's largest |q| is outside [2^-86, 2^115), where
                                         its f16 image (see paged_mqa_logits_fp4) can lose
                                         precision or overflow */
#define MQA_STATUS_DEBUG_INVARIANT 0x20u /* raised only by a library compiled with -DMQA_DEBUG
                                         (libmqa_logits_debug.so, mqa_logits_version() ends in
                                         "-debug"): a pipeline invariant failed in some CTA -- a
                                         work-table entry outside its row, context or schedule
                                         range, roles that walked different numbers of units or
                                         tiles, or an mbarrier that ended in another phase than
                                         its use count predicts. The output is still written. */

/* mqa_logits_params.flags */
#define MQA_FLAG_VALIDATE 0x1u   /* device-side checks (also enabled by env MQA_LOGITS_VALIDATE=1) */
#define MQA_FLAG_NO_PDL   0x2u   /* launch without programmatic dependent launch */

/* The units of work of the split schedule are 256 tokens of one row. */
#define MQA_SCHEDULE_UNIT 256

typedef struct mqa_logits_params {
    int32_t batch;              /* B, number of rows (>= 0) */
    int32_t next_n;             /* draft positions per row, 1..4 */
    int32_t num_heads;          /* H: 4, 8, 16, 32, 64 or 128; H*next_n <= 256 */
    int32_t head_dim;           /* D: fp8 32, 64 or 128; fp4 64 or 128 */
    int32_t page_size;          /* tokens per page: a power of two, 8..256 (fp4: 16..256) */
    int32_t num_pages;          /* pages in kv_cache */
    int32_t max_pages_per_row;  /* row stride of block_table */
    int32_t out_len;            /* L: row length of out, multiple of 4, >= every context_lens[b] */
    int32_t num_ctas;           /* S: the value given to mqa_logits_schedule */
    uint32_t flags;             /* MQA_FLAG_* */
    int32_t* status;            /* optional device int32 for MQA_STATUS_* bits; may be NULL */
    uint64_t timeout_ns;        /* bound on every pipeline wait; 0 = 2 s */
} mqa_logits_params;

/*
 * Number of persistent CTAs the logits kernels are built for on `device`
 * (its SM count, 148 on B200). Writes it to *num_ctas.
 */
int mqa_logits_num_ctas(int device, int32_t* num_ctas);

/*
 * The split schedule (the page's section 2, "스케줄링 및 CUDA Graph 지원":
 * the persistent kernel's per-call work assignment is computed on the GPU, so
 * no host round trip is needed and the call can be captured in a CUDA graph;
 * section 1: partitions are found by binary search instead of a linear scan).
 *
 * context_lens: device int32 [B], tokens cached per row (negative = 0).
 * schedule:     device int32 [(num_ctas + 1) * 2], written. Entry i is the
 *               (row, unit offset) where CTA i starts; CTA i owns the units
 *               from entry i up to (not including) entry i + 1. With
 *               u_b = ceil(ctx_b / 256) and U = sum_b u_b, CTA i starts at
 *               global unit i*floor(U/S) + min(i, U mod S); rows with no
 *               units are never named; the end sentinel is (B, 0).
 * Limits: 0 <= B <= 32768, 1 <= num_ctas <= 4096, and U < 2^31.
 *
 * Reuse (the page's "general lessons" 1 and reviewer feedback): a schedule
 * stays valid while num_ctas and every ceil(context_lens[b] / 256) are
 * unchanged; recompute it when a row crosses a 256-token boundary.
 */
int mqa_logits_schedule(const int32_t* context_lens, int32_t batch, int32_t num_ctas,
                        int32_t* schedule, void* stream);

/*
 * FP8 logits (the page's introduction, fp8_paged_mqa_logits).
 *
 * q:            device e4m3 bytes [B][next_n][H][D], 16-byte aligned.
 * kv_cache:     device bytes [num_pages][page_size * (D + 4)], 16-byte aligned:
 *               each page holds page_size rows of D e4m3 K values followed by
 *               page_size fp32 per-token scales s_t.
 * block_table:  device int32 [B][max_pages_per_row]; entry j of row b is the
 *               page holding tokens [j*page_size, (j+1)*page_size). Entries
 *               past ceil(ctx_b / page_size) are never read.
 * context_lens: device int32 [B]; 0 <= ctx_b <= min(out_len, max_pages_per_row*page_size).
 * weights:      device fp32 [B][next_n][H], 16-byte aligned.
 * schedule:     device int32 [(num_ctas + 1) * 2] from mqa_logits_schedule
 *               for these context_lens (see its reuse rule).
 * out:          device fp32 [B][next_n][out_len], 16-byte aligned. Every
 *               element is written: the logit for t < ctx_bn, -inf otherwise
 *               (rows with ctx_b == 0 become all -inf and get no K traffic).
 * params:       host pointer, shapes and flags as documented above.
 */
int paged_mqa_logits_fp8(const void* q, const void* kv_cache, const int32_t* block_table,
                         const int32_t* context_lens, const float* weights,
                         const int32_t* schedule, float* out,
                         const mqa_logits_params* params, void* stream);

/*
 * FP4 logits (the page's introduction, fp4_paged_mqa_logits).
 *
 * q:        device bf16 [B][next_n][H][D], 16-byte aligned. The kernel
 *           multiplies in f16: each (b, n) row of q is scaled by a power of
 *           two that maps its largest |q| into [2^14, 2^15) (undone exactly
 *           in the epilogue), which is exact unless a nonzero |q| is below
 *           about 2^-31 of its row's largest; rows whose largest |q| is
 *           outside [2^-86, 2^115) raise MQA_STATUS_Q_RANGE.
 * kv_cache: device bytes [num_pages][page_size * (D/2 + D/16)]: each page
 *           holds page_size rows of D e2m1 codes packed two per byte (even
 *           element in the low nibble), then page_size rows of D/16 e4m3
 *           block scales (one per 16 consecutive elements). The K value is
 *           code * block scale; there is no per-token scale (s_t = 1).
 * Everything else as for paged_mqa_logits_fp8.
 */
int paged_mqa_logits_fp4(const void* q, const void* kv_cache, const int32_t* block_table,
                         const int32_t* context_lens, const float* weights,
                         const int32_t* schedule, float* out,
                         const mqa_logits_params* params, void* stream);

/*
 * Block-scaled FP4 logits: q and K both NVFP4, multiplied by the tensor
 * core's block-scaled FP4 MMA (the page's introduction, fp4_paged_mqa_logits;
 * "FP4 block-scaled" is this entry point's reading of it when q, too, is
 * supplied in FP4).
 *
 * q:        device bytes [B][next_n][H * (D/2 + D/16)], 16-byte aligned: per
 *           (b, n) row, H rows of D e2m1 codes packed two per byte (even
 *           element in the low nibble), then H rows of D/16 e4m3 block
 *           scales; q[b][n][h][d] = code * scale of block d / 16. Scales must
 *           be non-negative (the MMA reads them as unsigned e4m3).
 * kv_cache: the FP4 page format of paged_mqa_logits_fp4 (codes, then e4m3
 *           block scales; K scales non-negative as well); s_t = 1.
 * Everything else as for paged_mqa_logits_fp4 (D 64 or 128, H * next_n <= 128,
 * page_size 16..256).
 */
int paged_mqa_logits_nvfp4(const void* q, const void* kv_cache, const int32_t* block_table,
                           const int32_t* context_lens, const float* weights,
                           const int32_t* schedule, float* out,
                           const mqa_logits_params* params, void* stream);

/*
 * Top-k over the logits: the selection the DeepSeek sparse-attention indexer
 * makes from them (the page's introduction: the indexer scores every cached
 * token so that sparse attention reads only the best-scoring ones). No
 * counterpart call is named on the page; this is the step that consumes the
 * logits.
 *
 * logits:       device fp32 [B][next_n][out_len], 4-byte aligned (e.g. the
 *               output of paged_mqa_logits_fp8 / _fp4).
 * context_lens: device int32 [B]; with c = clamp(ctx_b, 0, out_len) the valid
 *               tokens of row (b, n) are t < ctx_bn = clamp(c - next_n + 1 + n, 0, c).
 * flags:        0, or MQA_TOPK_BY_TOKEN.
 * indices:      device int32 [B][next_n][k], written completely: per row the
 *               k valid tokens of largest logit, where among equal logits the
 *               lower tokens win (-0.0 equals +0.0); listed by logit descending
 *               and, for equal logits, by token ascending, or with
 *               MQA_TOPK_BY_TOKEN by token ascending (the order a sparse
 *               attention kernel reads pages in; no sort is needed). -1 after
 *               the last valid token when a row has fewer than k.
 * values:       NULL, or device fp32 [B][next_n][k], 4-byte aligned: the logit
 *               of each listed token (-0.0 reported as +0.0), -inf where the
 *               index is -1. These are what mqa_logits_topk_merge consumes.
 * Limits: 1 <= k <= MQA_TOPK_MAX, 1 <= next_n <= 4, B >= 0. Logits are expected
 * finite for valid tokens (NaN is outside the contract).
 * One CTA per row, or, when the rows are few (at most 148) and out_len is at
 * least 32768, every row split over a thread-block cluster of 2 CTAs that
 * combine their histograms and counts in distributed shared memory; the result
 * is the same either way. The environment variable MQA_TOPK_CLUSTER, read at
 * each call, forces the choice (1: one CTA per row; 2 or 4: that cluster size
 * for every row). Asynchronous on `stream`, allocates nothing. Invalid
 * arguments (range, NULL, alignment, unknown flag bits) return
 * MQA_ERR_INVALID_ARG before any launch.
 */
#define MQA_TOPK_MAX 4096
#define MQA_TOPK_BY_TOKEN 1
int mqa_logits_topk(const float* logits, const int32_t* context_lens, int32_t batch,
                    int32_t next_n, int32_t out_len, int32_t k, int32_t flags, int32_t* indices,
                    float* values, void* stream);

/*
 * Merge of per-shard top-k lists into the top-k of the whole row: the
 * exchange step when a row's tokens are split by range over several GPUs
 * (each GPU scores and selects within its own pages; the lists are gathered,
 * e.g. by an all-gather over NVLink, and merged here).
 *
 * cand_values:  device fp32 [shards][rows][k_in] (per-shard `values`).
 * cand_tokens:  device int32 [shards][rows][k_in]: each shard's LOCAL tokens
 *               listed by token ascending (MQA_TOPK_BY_TOKEN), -1 for empty
 *               slots (ignored).
 * token_offsets: HOST int32 [shards]: shard s's global token = local token +
 *               token_offsets[s].
 * token_counts: HOST int32 [shards]: the length of shard s's token range
 *               (its local tokens are 0 .. token_counts[s] - 1). The ranges
 *               must not overlap and must ascend with s:
 *               token_offsets[s] + token_counts[s] <= token_offsets[s + 1]
 *               (checked; MQA_ERR_INVALID_ARG otherwise). Ties between equal
 *               values are then broken by global token, as in one call over
 *               the whole row.
 * k, flags, indices, values: as for mqa_logits_topk, over the union of the
 *               shards' valid entries; indices are global tokens.
 * Limits: 1 <= shards <= MQA_TOPK_MERGE_MAX_SHARDS, k_in >= 1,
 * shards * k_in <= MQA_TOPK_MERGE_MAX, 1 <= k <= MQA_TOPK_MAX, rows >= 0.
 * One CTA per row; asynchronous on `stream`, allocates nothing; argument
 * errors return MQA_ERR_INVALID_ARG before any launch.
 */
#define MQA_TOPK_MERGE_MAX_SHARDS 8
#define MQA_TOPK_MERGE_MAX 16384
int mqa_logits_topk_merge(const float* cand_values, const int32_t* cand_tokens, int32_t shards,
                          int32_t rows, int32_t k_in, const int32_t* token_offsets,
                          const int32_t* token_counts, int32_t k, int32_t flags,
                          int32_t* indices, float* values, void* stream);

/*
 * The library's own status word on the current device (one 32-bit word per
 * device, allocated when the library is loaded there): every logits kernel
 * ORs its MQA_STATUS_* bits into it, whether or not params->status was given,
 * so a bounded wait that expired is never silent.
 *
 * mqa_logits_get_status waits for the work queued on `stream` so far, then
 * writes the word to *bits (a host pointer). mqa_logits_clear_status zeroes
 * it, asynchronously on `stream`. The first call of the library on a device
 * looks the word up (a runtime call that is not a stream operation), so make
 * one call on each device before capturing a CUDA graph there.
 */
int mqa_logits_get_status(uint32_t* bits, void* stream);
int mqa_logits_clear_status(void* stream);

/*
 * The same word as an error code: waits for the work queued on `stream` so
 * far and returns MQA_OK if no bit is set, else MQA_ERR_DEVICE_CHECK with
 * mqa_logits_last_error() naming the bits (e.g. "device status 0x3: TIMEOUT
 * BAD_PAGE"). The word is left as it is; clear it with
 * mqa_logits_clear_status. This is how a caller turns the kernels'
 * asynchronous device-side checks (validate mode, bounded waits) into a
 * return code at a point of its choosing, e.g. once per step.
 */
int mqa_logits_check_status(void* stream);

/* Message of the last failed call on this host thread ("" if none). */
const char* mqa_logits_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* mqa_logits_version(void);

/* ---- Test hooks: NOT part of the stable interface -------------------------
 * Declared only when MQA_LOGITS_TEST_HOOKS is defined before this header is
 * included. They let the test suite drive the failure paths without faulting
 * a GPU; production callers never set them. */
#ifdef MQA_LOGITS_TEST_HOOKS
/* mqa_logits_params.flags: the producers never fill the second unit of the
 * work, so a consumer's bounded wait must expire and raise MQA_STATUS_TIMEOUT. */
#define MQA_FLAG_TEST_DROP_ARRIVE 0x100u
#endif

#ifdef __cplusplus
}
#endif

#endif  /* MQA_LOGITS_H_ */
