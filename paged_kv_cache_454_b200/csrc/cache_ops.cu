// Cache write (reshape_and_cache), copy-on-write block copies and the
// contiguous gather used to check block-table indexing.  All three move bits
// only: 16-byte vector loads and stores, coalesced along head_dim.
#include <algorithm>
#include <set>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace pa {
namespace {

// ---------------------------------------------------------------------------
// reshape_and_cache: one thread per 16-byte chunk of one (token, head) row.
// Consecutive threads walk head_dim, then heads, then tokens, so both the
// source rows and each destination page row are read/written contiguously.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, int64_t token_stride_chunks,
    uint4* __restrict__ k_pool, uint4* __restrict__ v_pool, int num_blocks, int hkv, int chunks,
    const int64_t* __restrict__ slot_mapping, int num_tokens, unsigned int* err) {
  // the decode plan launched after this kernel may start now: it reads only
  // the tables and lengths, and it waits for this grid before it completes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t per_token = static_cast<int64_t>(hkv) * chunks;
  const int64_t total = per_token * num_tokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / per_token;
    const int rem = static_cast<int>(i - t * per_token);
    const int h = rem / chunks;
    const int c = rem - h * chunks;
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0) continue;  // padding token
    const int64_t b = slot >> 4;  // block_size 16
    const int o = static_cast<int>(slot & 15);
    if (b >= num_blocks) {
      raise_error(err, PA_DEV_ERR_SLOT);
      continue;
    }
    const int64_t src = t * token_stride_chunks + static_cast<int64_t>(h) * chunks + c;
    const int64_t dst = ((b * hkv + h) * 16 + o) * chunks + c;
    k_pool[dst] = __ldg(key + src);
    v_pool[dst] = __ldg(value + src);
  }
}

// ---------------------------------------------------------------------------
// copy_blocks: the (src, dst) pairs travel in the kernel parameters.
// ---------------------------------------------------------------------------
constexpr int kPairsPerLaunch = 480;
struct PairBatch {
  int n;
  int src[kPairsPerLaunch];
  int dst[kPairsPerLaunch];
};

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_pool,
                                                          uint4* __restrict__ v_pool,
                                                          int64_t block_chunks,
                                                          const __grid_constant__ PairBatch pb) {
  // grid.y = pair, grid.z = pool (0: K, 1: V); x strides over the block.
  const int pair = blockIdx.y;
  uint4* pool = blockIdx.z == 0 ? k_pool : v_pool;
  const int64_t s = static_cast<int64_t>(pb.src[pair]) * block_chunks;
  const int64_t d = static_cast<int64_t>(pb.dst[pair]) * block_chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  // four independent 16-byte loads in flight per thread
  for (; i + 3 * stride < block_chunks; i += 4 * stride) {
    uint4 a0 = pool[s + i], a1 = pool[s + i + stride], a2 = pool[s + i + 2 * stride],
          a3 = pool[s + i + 3 * stride];
    pool[d + i] = a0;
    pool[d + i + stride] = a1;
    pool[d + i + 2 * stride] = a2;
    pool[d + i + 3 * stride] = a3;
  }
  for (; i < block_chunks; i += stride) pool[d + i] = pool[s + i];
}

// ---------------------------------------------------------------------------
// gather_kv: grid (sequence, logical block); one thread per 16-byte chunk.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_kv_kernel(
    const uint4* __restrict__ k_pool, const uint4* __restrict__ v_pool, int num_blocks, int hkv,
    int chunks, const int32_t* __restrict__ block_tables, int max_blocks,
    const int32_t* __restrict__ context_lens, const int32_t* __restrict__ cu_kv,
    uint4* __restrict__ k_out, uint4* __restrict__ v_out, unsigned int* err) {
  const int s = blockIdx.y;
  const int lb = blockIdx.x;
  int L = context_lens[s];
  if (L < 0 || L > max_blocks * 16) {
    if (threadIdx.x == 0 && lb == 0) raise_error(err, PA_DEV_ERR_CONTEXT);
    L = L < 0 ? 0 : max_blocks * 16;
  }
  if (lb * 16 >= L) return;
  const int pb = block_tables[static_cast<int64_t>(s) * max_blocks + lb];
  if (pb < 0 || pb >= num_blocks) {
    if (threadIdx.x == 0) raise_error(err, PA_DEV_ERR_BLOCK_ID);
    return;
  }
  int ntok = min(16, L - lb * 16);
  const int64_t row0 = cu_kv[s] + lb * 16;
  const int64_t row_end = cu_kv[s + 1];
  if (row0 + ntok > row_end) {  // cu_kv_lens disagrees with context_lens
    if (threadIdx.x == 0) raise_error(err, PA_DEV_ERR_CONTEXT);
    ntok = row_end > row0 ? static_cast<int>(row_end - row0) : 0;
  }
  const int per_tok = hkv * chunks;
  for (int i = threadIdx.x; i < ntok * per_tok; i += blockDim.x) {
    const int t = i / per_tok;
    const int rem = i - t * per_tok;
    const int h = rem / chunks;
    const int c = rem - h * chunks;
    const int64_t src = ((static_cast<int64_t>(pb) * hkv + h) * 16 + t) * chunks + c;
    const int64_t dst = (row0 + t) * per_tok + rem;
    k_out[dst] = k_pool[src];
    v_out[dst] = v_pool[src];
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

int pa_reshape_and_cache(const void* key, const void* value, int64_t token_stride, void* k_pool,
                         void* v_pool, pa_pool_desc pool, const int64_t* slot_mapping,
                         int32_t num_tokens, void* stream) {
  PA_NVTX_RANGE("pa_reshape_and_cache");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_tokens < 0) return PA_ERR_ARG;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_pool || !v_pool || !slot_mapping) return PA_ERR_ARG;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
    return PA_ERR_ARG;
  const int chunks = pool.head_dim / 8;
  if (token_stride < static_cast<int64_t>(pool.num_kv_heads) * pool.head_dim || token_stride % 8)
    return PA_ERR_ARG;
  unsigned int* err = device_error_word();
  if (!err) return PA_ERR_CUDA;
  const int64_t total = static_cast<int64_t>(num_tokens) * pool.num_kv_heads * chunks;
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int blocks = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(num_sms()) * 8));
  reshape_and_cache_kernel<<<blocks, threads, 0, as_stream(stream)>>>(
      static_cast<const uint4*>(key), static_cast<const uint4*>(value), token_stride / 8,
      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), pool.num_blocks,
      pool.num_kv_heads, chunks, slot_mapping, num_tokens, err);
  return launch_status();
}

int pa_copy_blocks(void* k_pool, void* v_pool, pa_pool_desc pool, const int64_t* pairs_host,
                   int32_t num_pairs, void* stream) {
  PA_NVTX_RANGE("pa_copy_blocks");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_pairs < 0) return PA_ERR_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_pool || !v_pool || !pairs_host) return PA_ERR_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_ARG;
  std::set<int64_t> srcs, dsts;
  for (int i = 0; i < num_pairs; ++i) {
    const int64_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || s >= pool.num_blocks || d < 0 || d >= pool.num_blocks) return PA_ERR_ARG;
    if (!dsts.insert(d).second) return PA_ERR_ARG;  // repeated destination
    srcs.insert(s);
  }
  for (int64_t d : dsts)
    if (srcs.count(d)) return PA_ERR_ARG;  // a destination is also a source
  const int64_t block_chunks =
      static_cast<int64_t>(pool.num_kv_heads) * pool.block_size * pool.head_dim / 8;
  const int threads = 256;
  const int gx = static_cast<int>(std::min<int64_t>(
      std::max<int64_t>(1, (block_chunks + threads * 4 - 1) / (threads * 4)), 64));
  for (int base = 0; base < num_pairs; base += kPairsPerLaunch) {
    PairBatch pb;
    pb.n = std::min(kPairsPerLaunch, num_pairs - base);
    for (int i = 0; i < pb.n; ++i) {
      pb.src[i] = static_cast<int>(pairs_host[2 * (base + i)]);
      pb.dst[i] = static_cast<int>(pairs_host[2 * (base + i) + 1]);
    }
    dim3 grid(gx, pb.n, 2);
    copy_blocks_kernel<<<grid, threads, 0, as_stream(stream)>>>(
        static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), block_chunks, pb);
    st = launch_status();
    if (st != PA_OK) return st;
  }
  return PA_OK;
}

int pa_gather_kv(const void* k_pool, const void* v_pool, pa_pool_desc pool,
                 const int32_t* block_tables, int32_t max_blocks_per_seq,
                 const int32_t* context_lens, const int32_t* cu_kv_lens, int32_t num_seqs,
                 int32_t max_context, void* k_out, void* v_out, void* stream) {
  PA_NVTX_RANGE("pa_gather_kv");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || max_context < 0 || max_blocks_per_seq <= 0) return PA_ERR_ARG;
  if (num_seqs == 0 || max_context == 0) return PA_OK;
  if (!k_pool || !v_pool || !block_tables || !context_lens || !cu_kv_lens || !k_out || !v_out)
    return PA_ERR_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_out) || !aligned16(v_out))
    return PA_ERR_ARG;
  if (num_seqs > 65535) return PA_ERR_UNSUPPORTED;
  unsigned int* err = device_error_word();
  if (!err) return PA_ERR_CUDA;
  const int pages = std::min((max_context + 15) / 16, max_blocks_per_seq);
  dim3 grid(pages, num_seqs);
  gather_kv_kernel<<<grid, 256, 0, as_stream(stream)>>>(
      static_cast<const uint4*>(k_pool), static_cast<const uint4*>(v_pool), pool.num_blocks,
      pool.num_kv_heads, pool.head_dim / 8, block_tables, max_blocks_per_seq, context_lens,
      cu_kv_lens, static_cast<uint4*>(k_out), static_cast<uint4*>(v_out), err);
  return launch_status();
}

}  // extern "C"
