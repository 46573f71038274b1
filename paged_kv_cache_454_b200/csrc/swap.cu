// Block swapping between the device pools and page-locked host pools
// (pa_swap_blocks).  One launch per 480 pairs: the pairs travel in the kernel
// parameters; grid.y is the pair, grid.z the pool (K, V); each thread keeps
// eight independent 16-byte transfers in flight, since reads of host memory
// cross the bus with microseconds of latency.
#include <algorithm>
#include <set>

#include "common.cuh"
#include "internal.h"
#include "../../include/pa_swap.h"

namespace pa {
namespace {

constexpr int kSwapPairs = 480;
constexpr int kInFlight = 8;

struct SwapBatch {
  int n;
  int src[kSwapPairs];
  int dst[kSwapPairs];
};

__global__ void __launch_bounds__(256) swap_kernel(const uint4* __restrict__ src_k,
                                                   const uint4* __restrict__ src_v,
                                                   uint4* __restrict__ dst_k,
                                                   uint4* __restrict__ dst_v,
                                                   int64_t block_chunks,
                                                   const __grid_constant__ SwapBatch sb) {
  const int pair = blockIdx.y;
  const uint4* src = blockIdx.z == 0 ? src_k : src_v;
  uint4* dst = blockIdx.z == 0 ? dst_k : dst_v;
  const int64_t s = static_cast<int64_t>(sb.src[pair]) * block_chunks;
  const int64_t d = static_cast<int64_t>(sb.dst[pair]) * block_chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  for (; i + (kInFlight - 1) * stride < block_chunks; i += kInFlight * stride) {
    uint4 a[kInFlight];
#pragma unroll
    for (int q = 0; q < kInFlight; ++q) a[q] = src[s + i + q * stride];
#pragma unroll
    for (int q = 0; q < kInFlight; ++q) dst[d + i + q * stride] = a[q];
  }
  for (; i < block_chunks; i += stride) dst[d + i] = src[s + i];
}

// The device-side address of page-locked host memory, or NULL if `p` is not
// page-locked host memory the current device can address.
void* host_device_ptr(void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
  return at.devicePointer;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_swap_blocks(void* k_pool, void* v_pool, pa_pool_desc pool, void* k_host,
                              void* v_host, int32_t num_host_blocks, const int64_t* pairs_host,
                              int32_t num_pairs, int32_t direction, void* stream) {
  PA_NVTX_RANGE("pa_swap_blocks");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_pairs < 0 || num_host_blocks < 0) return PA_ERR_ARG;
  if (direction != PA_SWAP_OUT && direction != PA_SWAP_IN) return PA_ERR_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!k_pool || !v_pool || !k_host || !v_host || !pairs_host) return PA_ERR_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_host) || !aligned16(v_host))
    return PA_ERR_ARG;
  void* kh = host_device_ptr(k_host);
  void* vh = host_device_ptr(v_host);
  if (!kh || !vh) return PA_ERR_ARG;
  const int64_t src_n = direction == PA_SWAP_OUT ? pool.num_blocks : num_host_blocks;
  const int64_t dst_n = direction == PA_SWAP_OUT ? num_host_blocks : pool.num_blocks;
  std::set<int64_t> dsts;
  for (int i = 0; i < num_pairs; ++i) {
    const int64_t s = pairs_host[2 * i], d = pairs_host[2 * i + 1];
    if (s < 0 || s >= src_n || d < 0 || d >= dst_n) return PA_ERR_ARG;
    if (!dsts.insert(d).second) return PA_ERR_ARG;  // repeated destination
  }
  const int64_t block_chunks =
      static_cast<int64_t>(pool.num_kv_heads) * pool.block_size * pool.head_dim / 8;
  const uint4* sk = static_cast<const uint4*>(direction == PA_SWAP_OUT ? k_pool : kh);
  const uint4* sv = static_cast<const uint4*>(direction == PA_SWAP_OUT ? v_pool : vh);
  uint4* dk = static_cast<uint4*>(direction == PA_SWAP_OUT ? kh : k_pool);
  uint4* dv = static_cast<uint4*>(direction == PA_SWAP_OUT ? vh : v_pool);
  const int threads = 256;
  const int gx = static_cast<int>(std::min<int64_t>(
      std::max<int64_t>(1, (block_chunks + threads * kInFlight - 1) / (threads * kInFlight)), 64));
  for (int base = 0; base < num_pairs; base += kSwapPairs) {
    SwapBatch sb;
    sb.n = std::min(kSwapPairs, num_pairs - base);
    for (int i = 0; i < sb.n; ++i) {
      sb.src[i] = static_cast<int>(pairs_host[2 * (base + i)]);
      sb.dst[i] = static_cast<int>(pairs_host[2 * (base + i) + 1]);
    }
    dim3 grid(gx, sb.n, 2);
    swap_kernel<<<grid, threads, 0, as_stream(stream)>>>(sk, sv, dk, dv, block_chunks, sb);
    st = launch_status();
    if (st != PA_OK) return st;
  }
  return PA_OK;
}
