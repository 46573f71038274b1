/*
 * pa.h -- C ABI of a PagedAttention library for NVIDIA B200 (sm_100a).
 *
 * What it computes.  Attention for a batch of sequences whose keys and values
 * live in fixed-size physical blocks scattered through one KV pool, reached
 * through a per-sequence block table that maps logical block IDs to physical
 * block IDs ("vLLM 基本原理", section PagedAttention: logical blocks, physical
 * blocks, block table; "当大模型推理遇上内存瓶颈", section 3.1: the paged layout
 * [num_blocks, num_heads, block_size, head_dim] and the lookup
 * physical_block = block_tables[seq_idx][logic_block]).
 *
 * Conventions shared by every call:
 *   - Tensor arguments are DEVICE pointers into memory the caller owns, unless
 *     a parameter says "host".  The library allocates no device memory; the
 *     caller passes any scratch it needs (pa_decode's workspace).
 *   - bf16 tensors are passed as untyped pointers to 16-bit storage.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream).  Results are visible to later work on that stream.
 *   - The return value is PA_OK or a PA_ERR_* code.  Arguments are checked on
 *     the host before anything is launched; on an error nothing is launched.
 *   - Values that only the device sees (block-table entries, slots, context
 *     lengths) are range-checked by the kernels.  A bad value never causes an
 *     out-of-bounds access: the access is skipped (its token contributes
 *     nothing) and a bit is set in a sticky per-device error word that
 *     pa_get_device_error() returns and clears.
 *   - Every pointer argument must be 16-byte aligned; strides are in elements
 *     and must be multiples of 8 (16 bytes).
 *   - The library caches, per device and for the life of the process, the
 *     device address of its error word (and of the scratch array of
 *     pa_decode_noalloc).  Do not keep using it after cudaDeviceReset().
 *   - Each entry point opens an NVTX range named after itself (visible in
 *     Nsight Systems timelines); a build with -DPA_NO_NVTX has none.
 *
 * Pool layout (both pools):  bf16 [num_blocks][num_kv_heads][block_size][head_dim],
 * densely packed.  One (block, kv head) page is block_size*head_dim contiguous
 * elements (4 KiB at block_size 16, head_dim 128).
 *
 * Compiled sizes: block_size 16; head_dim 64 or 128; any num_q_heads that is a
 * multiple of num_kv_heads with group size num_q_heads/num_kv_heads <= 16.
 * Other sizes return PA_ERR_UNSUPPORTED.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_ABI_VERSION 1

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

/* Status codes. */
#define PA_OK 0
#define PA_ERR_ARG 1         /* NULL pointer, negative count, misaligned pointer or stride */
#define PA_ERR_SHAPE 2       /* inconsistent sizes, e.g. num_q_heads % num_kv_heads != 0 */
#define PA_ERR_UNSUPPORTED 3 /* a size this build has no kernel for */
#define PA_ERR_WORKSPACE 4   /* workspace NULL or smaller than pa_decode_workspace_size() */
#define PA_ERR_CUDA 5        /* a CUDA runtime call or a launch failed */

/* Bits of the sticky device error word (pa_get_device_error). */
#define PA_DEV_ERR_BLOCK_ID 0x1u    /* a block-table entry outside [0, num_blocks) was needed */
#define PA_DEV_ERR_SLOT 0x2u        /* a slot_mapping entry >= num_blocks * block_size */
#define PA_DEV_ERR_CONTEXT 0x4u     /* a context length < 0 or > max_blocks_per_seq * block_size,
                                       or a chunk longer than its context */
#define PA_DEV_ERR_TIMEOUT 0x8u     /* a pipeline wait gave up (bounded spin); results invalid */

/* The KV pool both pools share the shape of. */
typedef struct pa_pool_desc {
  int32_t num_blocks;   /* physical blocks in the pool */
  int32_t num_kv_heads; /* Hkv */
  int32_t block_size;   /* tokens per block (16) */
  int32_t head_dim;     /* D (64 or 128) */
} pa_pool_desc;

/*
 * pa_reshape_and_cache -- write this step's new tokens' K and V into their slots.
 *
 * Source: "vLLM 基本原理", PagedAttention / 按需分配 (tokens fill the current
 * block; only the last block of a sequence may be partly filled).  For every
 * token t with slot = slot_mapping[t] >= 0, and every KV head h:
 *     k_pool[slot / block_size][h][slot % block_size][:] = key[t][h][:]
 *     v_pool[...same...]                                = value[t][h][:]
 * A negative slot is padding and is skipped.
 *
 *   key, value     bf16 [num_tokens][num_kv_heads][head_dim], token stride
 *                  `token_stride` elements (>= num_kv_heads*head_dim), heads packed.
 *   k_pool, v_pool the pools, written in place.
 *   slot_mapping   int64 [num_tokens], device.
 *   Two tokens with the same slot race (which one lands is unspecified).
 *   A slot >= num_blocks*block_size is skipped and sets PA_DEV_ERR_SLOT.
 */
PA_API int pa_reshape_and_cache(const void* key, const void* value, int64_t token_stride,
                         void* k_pool, void* v_pool, pa_pool_desc pool,
                         const int64_t* slot_mapping, int32_t num_tokens, void* stream);

/*
 * pa_copy_blocks -- copy-on-write of shared blocks: whole blocks (all KV heads,
 * all slots, K and V) src -> dst.
 *
 * Source: "当大模型推理遇上内存瓶颈", section 3.3 (a sharer that must write gets
 * its own copy of the shared block; with reference counts only the first writer
 * copies) and section 2.2 (RefCounter for copy-on-write).
 *
 *   pairs_host     int64 [num_pairs][2] = (src, dst), in HOST memory; read
 *                  during the call (the pairs travel in the kernel parameters),
 *                  so the buffer may be reused as soon as the call returns.
 *   Rules checked on the host (PA_ERR_ARG): every id in [0, num_blocks);
 *   destinations distinct; no destination is also a source.  So the result
 *   does not depend on the order the copies run in.
 */
PA_API int pa_copy_blocks(void* k_pool, void* v_pool, pa_pool_desc pool, const int64_t* pairs_host,
                   int32_t num_pairs, void* stream);

/*
 * pa_decode -- one query token per sequence attends to its whole paged context.
 *
 * Source: "vLLM 基本原理", PagedAttention ("the CUDA kernel fetches data from
 * every corner of physical memory according to the block table") and
 * Transformer 和 Attention (softmax-weighted lookup); "当大模型推理遇上内存瓶颈",
 * section 3.1 (kernel arguments Q, K, V, block_tables).  For sequence s with
 * L = context_lens[s] (which includes the query token itself, whose K/V
 * pa_reshape_and_cache wrote first) and q head h reading KV head
 * g = h / (num_q_heads / num_kv_heads):
 *     x_t = scale * dot(q[s][h], K_s[g][t])   for t in [0, L)
 *     out[s][h] = sum_t softmax(x)_t * V_s[g][t]
 *     lse[s][h] = log(sum_t exp(x_t))          (natural log)
 * where K_s[g][t] = k_pool[block_tables[s][t / bs]][g][t % bs].  Long contexts
 * are split into partitions whose partial results are merged by their
 * log-sum-exp (inside the tensor-core decode kernel, by the CTA that finishes
 * a sequence's last partition; by a second kernel on the same stream on the
 * CUDA-core path).  L == 0 gives out = 0 and lse = -inf.
 *
 *   q              bf16 [num_seqs][num_q_heads][head_dim], token stride q_stride
 *                  elements (>= num_q_heads*head_dim); heads packed.
 *   block_tables   int32 [num_seqs][max_blocks_per_seq]; entries past
 *                  ceil(L/bs) are never read.
 *   context_lens   int32 [num_seqs]; 0 <= L <= max_blocks_per_seq*block_size.
 *                  A table able to describe more than 65535 partitions of
 *                  the shortest partition length (about 8.4M tokens at 128)
 *                  returns PA_ERR_UNSUPPORTED, as do more than 32767 KV heads.
 *   out            bf16 [num_seqs][num_q_heads][head_dim], packed.
 *   lse            float [num_seqs][num_q_heads], or NULL.
 *   workspace      device scratch of at least pa_decode_workspace_size() bytes
 *                  for the partial results of split contexts; its contents
 *                  need no initialisation and are garbage afterwards.  Calls
 *                  that overlap on the GPU must not share a workspace.
 * Accumulation is fp32; the output is rounded to bf16 (nearest even).
 * Stream order: the first kernel of the call (the work plan) is a programmatic
 * dependent of the kernel before it on `stream`.  If that kernel signals that
 * its dependents may start early (this library's cache write and prefill
 * kernels do), the plan reads block_tables and context_lens while it still
 * runs -- they must be final by then -- and no K/V is read before it has
 * finished.  Kernels that do not signal (any other) are waited for as usual.
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, pa_pool_desc pool,
                                int32_t max_blocks_per_seq);

PA_API int pa_decode(const void* q, int64_t q_stride, const void* k_pool, const void* v_pool,
              pa_pool_desc pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
              const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
              void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Kernel choices for pa_decode_ex (testing and measurement). */
#define PA_KERNEL_AUTO 0   /* tensor-core kernel for head_dim 128, else CUDA cores */
#define PA_KERNEL_SIMT 1   /* CUDA-core kernel (any supported group size) */
#define PA_KERNEL_TCGEN05 2 /* tcgen05 tensor-core kernel (head_dim 128, group size <= 16) */

/*
 * pa_decode_ex -- pa_decode with the partition length and the kernel chosen
 * by the caller.  partition_tokens: tokens per split-context partition, a
 * multiple of 128 (0 = the kernel's default; a value >= the longest context
 * means no split).  The workspace must be sized with
 * pa_decode_workspace_size_ex() for the same partition length.
 */
PA_API size_t pa_decode_workspace_size_ex(int32_t num_seqs, int32_t num_q_heads, pa_pool_desc pool,
                                   int32_t max_blocks_per_seq, int32_t partition_tokens);

PA_API int pa_decode_ex(const void* q, int64_t q_stride, const void* k_pool, const void* v_pool,
                 pa_pool_desc pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                 const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads, float scale,
                 void* out, float* lse, void* workspace, size_t workspace_bytes,
                 int32_t partition_tokens, int32_t kernel, void* stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call: it only changes where the
 * split-context scratch comes from.  A caller that gives all free HBM to its KV
 * pool at start-up, or that runs inside a host framework whose op interface
 * passes no workspace, cannot provide the workspace pa_decode needs.  This call
 * takes the same arguments minus the workspace and uses a scratch array of
 * PA_NOALLOC_SCRATCH_BYTES compiled into the library instead; it allocates
 * nothing.
 *
 *   - Every GPU that loads the library holds the array until the process exits.
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture on the device.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls whose kernels
 *     overlap on the GPU (e.g. on two streams) race on it: do not issue them.
 *   - The call needs the workspace of the kernel pa_decode would choose for
 *     the same sizes.  pa_decode_workspace_size() is an upper bound of that
 *     need (it sizes for either kernel): a batch whose
 *     pa_decode_workspace_size() is at most PA_NOALLOC_SCRATCH_BYTES always
 *     fits.  A larger batch still runs when the chosen kernel's own need fits
 *     (typically GQA batches on the tensor-core kernel, whose partitions are
 *     longer); otherwise the call returns PA_ERR_WORKSPACE and launches
 *     nothing.  Other errors as for pa_decode.
 *   - The array's device address is cached per device for the life of the
 *     process: do not use the library across a cudaDeviceReset() (the same
 *     holds for the device error word every call uses).
 */
#define PA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

PA_API int pa_decode_noalloc(const void* q, int64_t q_stride, const void* k_pool,
                             const void* v_pool, pa_pool_desc pool, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t num_seqs, int32_t num_q_heads, float scale, void* out,
                             float* lse, void* stream);

/*
 * pa_chunked_prefill -- each sequence's new chunk of tokens attends causally to
 * its cached context plus the chunk itself.
 *
 * Source: "vLLM 定位与核心机制详解", section 六.4 (a long prompt is prefilled a
 * chunk per round, mixed with decode requests in one batch step).  Sequence s
 * owns query rows cu_q_lens[s] .. cu_q_lens[s+1]-1, i.e. n = cu_q_lens[s+1] -
 * cu_q_lens[s] new tokens on top of c = context_lens[s] - n cached tokens (the
 * chunk's own K/V were written by pa_reshape_and_cache first).  Query i sits at
 * absolute position c + i and attends to keys 0 .. c + i:
 *     out[r][h] = sum_{t <= c+i} softmax(scale * q[r][h] . K_s[g][t]) V_s[g][t]
 *
 *   q            bf16 [total_q][num_q_heads][head_dim], token stride q_stride.
 *   cu_q_lens    int32 [num_seqs + 1], device; cu_q_lens[0] = 0,
 *                cu_q_lens[num_seqs] = total_q.
 *   max_q_len    host bound on any n (sizes the grid).
 *   context_lens int32 [num_seqs], device, including the chunk.
 *   out          bf16 [total_q][num_q_heads][head_dim], packed.
 *   lse          float [total_q][num_q_heads], or NULL.
 *
 * Precision (head_dim 128, tensor cores): scores and the P.V product
 * accumulate in fp32; the softmax weights p enter P.V as p with its mantissa
 * cut to bf16 plus, where needed, the same cut of the remainder (about 16
 * significant bits together).  A 64-key half of a 128-key tile goes without
 * the remainder when, in every row of the 128-row tile, its weights sum to at
 * most a quarter of that half row's sum up to and including the tile: such a
 * tile's weights are then at most a quarter of their final denominator, and
 * each is short of itself by less than 2^-7 of itself.  pa_chunked_prefill_ex with
 * PA_PREFILL_EXACT_WEIGHTS carries the remainder on every tile.
 */
PA_API int pa_chunked_prefill(const void* q, int64_t q_stride, const int32_t* cu_q_lens,
                       int32_t total_q, int32_t max_q_len, const void* k_pool,
                       const void* v_pool, pa_pool_desc pool, const int32_t* block_tables,
                       int32_t max_blocks_per_seq, const int32_t* context_lens,
                       int32_t num_seqs, int32_t num_q_heads, float scale, void* out, float* lse,
                       void* stream);

/*
 * pa_chunked_prefill_ex -- pa_chunked_prefill with `flags`: 0, or
 * PA_PREFILL_EXACT_WEIGHTS (every key tile's P.V takes the weights' bf16
 * remainder as well, so each weight reaches the product to within 2^-15 of
 * itself; slower).  Other bits: PA_ERR_ARG.
 */
#define PA_PREFILL_EXACT_WEIGHTS 0x1u
PA_API int pa_chunked_prefill_ex(const void* q, int64_t q_stride, const int32_t* cu_q_lens,
                          int32_t total_q, int32_t max_q_len, const void* k_pool,
                          const void* v_pool, pa_pool_desc pool, const int32_t* block_tables,
                          int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_q_heads, float scale, void* out,
                          float* lse, uint32_t flags, void* stream);

/*
 * pa_gather_kv -- copy every sequence's paged K and V into contiguous,
 * packed rows (checks the block-table indexing bit for bit).
 *
 *   cu_kv_lens   int32 [num_seqs + 1], device: sequence s owns output rows
 *                cu_kv_lens[s] .. cu_kv_lens[s+1]-1; cu_kv_lens[s+1] -
 *                cu_kv_lens[s] must equal context_lens[s].
 *   max_context  host bound on any context length (sizes the grid).
 *   k_out, v_out bf16 [cu_kv_lens[num_seqs]][num_kv_heads][head_dim].
 *   Row r = cu_kv_lens[s] + t receives token t of sequence s.
 */
PA_API int pa_gather_kv(const void* k_pool, const void* v_pool, pa_pool_desc pool,
                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                 const int32_t* context_lens, const int32_t* cu_kv_lens, int32_t num_seqs,
                 int32_t max_context, void* k_out, void* v_out, void* stream);

/*
 * pa_get_device_error -- wait for `stream`, then return (in *flags_host) and
 * clear the sticky device error word of the current device (PA_DEV_ERR_* bits;
 * 0 = no error since the last call).
 */
PA_API int pa_get_device_error(uint32_t* flags_host, void* stream);

/* Human-readable name of a status code (static storage). */
PA_API const char* pa_status_string(int status);

/* PA_ABI_VERSION of the built library. */
PA_API int pa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
