/*
 * Diagnostics for the paged MQA logits library: calls that measure parts of
 * the logits path on their own. They are not steps of the indexer and the
 * pages describe no counterpart; the benchmark uses them to state what the
 * logits kernels could reach.
 */
#ifndef MQA_LOGITS_DIAG_H
#define MQA_LOGITS_DIAG_H

#include "mqa_logits.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The FP8 logits kernel's data movement alone: the same work table, builder,
 * producer, ring of shared-memory stages and tensor maps as
 * paged_mqa_logits_fp8 (every K row of every unit, and each row's q tile and
 * weights), with a consumer that releases each stage as soon as it lands and
 * no arithmetic. Timing it gives the copy-only time of a workload's page
 * gather. Arguments, their layout, checks and error codes are exactly those of
 * paged_mqa_logits_fp8 (head_dim 32, 64 or 128); `out` is not written.
 * Asynchronous on `stream`, allocates nothing; waits are bounded as in the
 * logits kernels (MQA_STATUS_TIMEOUT).
 */
int mqa_diag_fp8_gather(const void* q, const void* kv_cache, const int32_t* block_table,
                        const int32_t* context_lens, const float* weights,
                        const int32_t* schedule, float* out, const mqa_logits_params* params,
                        void* stream);

#ifdef __cplusplus
}
#endif

#endif  /* MQA_LOGITS_DIAG_H */
