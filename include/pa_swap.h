/*
 * pa_swap.h -- C ABI of block swapping between the device KV pools and host
 * pools in pinned memory.
 *
 * Source: "当大模型推理遇上内存瓶颈", 5.1 (a CPU swap space for offloading KV
 * blocks, --swap-space) and 7.3 (blocks whose reference count is 0 are written
 * to slower storage and read back when needed).  The host pools play that
 * storage; the block manager (pa_kv_manager.h) decides which blocks move and
 * returns the pairs this call takes.
 *
 * pa_swap_blocks copies whole blocks (all KV heads, all slots, K and V):
 *   direction PA_SWAP_OUT: device block src -> host block dst;
 *   direction PA_SWAP_IN:  host block src -> device block dst.
 * One kernel moves every pair: SMs read and write the host pools directly
 * through their unified addresses (no staging buffer, no per-block copy call).
 *
 *   k_pool, v_pool    device pools, pa_pool_desc layout (see pa.h).
 *   k_host, v_host    host pools, bf16 [num_host_blocks][num_kv_heads][block_size][head_dim],
 *                     in page-locked memory the device can address (cudaHostAlloc,
 *                     torch's pin_memory), 16-byte aligned.
 *   pairs_host        int64 [num_pairs][2] = (src, dst), HOST memory, read during
 *                     the call.  Checked: ids inside their pools, destinations
 *                     distinct (PA_ERR_ARG otherwise).
 * Asynchronous on `stream`: the host pools must stay allocated, and must not be
 * read (swap out) or written (swap in) by the host, until the stream reaches it.
 */
#ifndef PA_SWAP_H_
#define PA_SWAP_H_

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

#define PA_SWAP_OUT 0
#define PA_SWAP_IN 1

PA_API int pa_swap_blocks(void* k_pool, void* v_pool, pa_pool_desc pool, void* k_host,
                          void* v_host, int32_t num_host_blocks, const int64_t* pairs_host,
                          int32_t num_pairs, int32_t direction, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_SWAP_H_ */
