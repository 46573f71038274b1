/*
 * pa_probe.h -- C ABI of the paged read-bandwidth probe.
 *
 * Source: "vLLM 定位与核心机制详解", 六.5 (decode is bound by memory
 * bandwidth) and "当大模型推理遇上内存瓶颈", 2.1 (the KV bytes a step reads).
 * The probe reads exactly the pages a decode call over the same block tables
 * reads -- every (block, KV head) page of K and of V under
 * ceil(context_len / block_size) table entries per sequence -- and nothing
 * else: no attention, no output besides a checksum.  Its time is the read
 * rate the paged layout allows on this device, the bound a decode call's
 * achieved bandwidth is compared with.
 *
 * pa_read_probe
 *   k_pool, v_pool     device pools, pa_pool_desc layout (see pa.h); a page is
 *                      block_size * head_dim bf16 values, contiguous.
 *   block_tables       device int32 [num_seqs][max_blocks_per_seq].
 *   context_lens       device int32 [num_seqs]; a length outside
 *                      [0, max_blocks_per_seq * block_size] is clamped and sets
 *                      PA_DEV_ERR_CONTEXT.
 *   partial_sums       device uint64 [num_ctas], written (not accumulated): CTA c
 *                      stores the sum, modulo 2^64, of the 32-bit words of the
 *                      pages it read.  Summed over all CTAs (modulo 2^64) this is
 *                      the sum of the words of every page read, whatever num_ctas.
 *   num_ctas           CTAs to launch, 1..65535; the SM count gives one per SM.
 * Pages are split into units of up to eight consecutive blocks of one KV head
 * of one sequence (K and V); CTA c takes units c, c + num_ctas, ...  A table
 * entry outside [0, num_blocks) is not read; it sets PA_DEV_ERR_BLOCK_ID.
 * Returns PA_ERR_ARG for NULL or misaligned pointers, num_seqs < 0 or
 * > PA_PROBE_MAX_SEQS, or num_ctas outside 1..65535; PA_ERR_UNSUPPORTED for a
 * pool shape pa.h does not support.  Asynchronous on `stream`.
 */
#ifndef PA_PROBE_H_
#define PA_PROBE_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

#define PA_PROBE_MAX_SEQS 4096

PA_API int pa_read_probe(const void* k_pool, const void* v_pool, pa_pool_desc pool,
                         const int32_t* block_tables, int32_t max_blocks_per_seq,
                         const int32_t* context_lens, int32_t num_seqs, uint64_t* partial_sums,
                         int32_t num_ctas, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_PROBE_H_ */
