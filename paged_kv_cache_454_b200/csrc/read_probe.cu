// The paged read-bandwidth probe (pa_read_probe): reads, once each, the K and
// V pages a decode call over the same tables reads, and nothing else.
//
// A unit is up to eight consecutive blocks of one KV head of one sequence; its
// K and V pages land in one shared-memory stage by bulk copies (one per page,
// issued by the lanes of warp 0 with an evict-first L2 hint, as the decode
// kernels use, completion counted in bytes on the stage's mbarrier); the table
// entries of the next unit are read while the current one is issued.  Four warps sum the stage's 32-bit words -- so the bytes are
// used and the result can be checked -- and release the stage.  Three stages
// of 64 KiB keep 192 KiB of reads in flight per SM, well above what the
// latency-bandwidth product of one SM's share of HBM needs.  Units go to CTAs
// round-robin; every CTA derives the unit layout (units per sequence and
// their prefix) from the context lengths itself, so there is no plan launch.
#include "common.cuh"
#include "internal.h"
#include "../../include/pa_probe.h"

namespace pa {
namespace {

constexpr int kProbeStages = 3;
constexpr int kUnitBlocks = 8;
constexpr int kMaxPageBytes = 16 * 128 * 2;              // block 16, head_dim 128, bf16
constexpr int kStageBytes = 2 * kUnitBlocks * kMaxPageBytes;
constexpr int kSumWarps = 4;
constexpr int kProbeThreads = 32 * (1 + kSumWarps);      // warp 0 issues copies
constexpr int kProbeSmem = kProbeStages * kStageBytes + 4 * (2 * PA_PROBE_MAX_SEQS + 1);

// Blocks of sequence s the probe reads: ceil(L / bs) of the clamped length.
__device__ __forceinline__ int probe_blocks(const int32_t* lens, int s, int max_blocks, int bs,
                                            unsigned int* err) {
  int L = lens[s];
  const int cap = max_blocks * bs;
  if (L < 0 || L > cap) {
    raise_error(err, PA_DEV_ERR_CONTEXT);
    L = L < 0 ? 0 : cap;
  }
  return (L + bs - 1) / bs;
}

__device__ __forceinline__ int units_of(int nblk, int hkv) {
  return (nblk + kUnitBlocks - 1) / kUnitBlocks * hkv;
}

// Where unit u lies: its sequence (the last s with prefix[s] <= u), KV head and
// first block, and how many blocks it holds.
struct ProbeUnit {
  int s, h, b0, nb;
};
__device__ __forceinline__ ProbeUnit locate(int u, const int* prefix, const int* nblk, int S) {
  int lo = 0, hi = S;  // prefix[lo] <= u < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= u) lo = mid; else hi = mid;
  }
  ProbeUnit p;
  p.s = lo;
  const int nb = nblk[lo];
  const int chunks = (nb + kUnitBlocks - 1) / kUnitBlocks;
  const int r = u - prefix[lo];
  p.h = r / chunks;
  p.b0 = (r - p.h * chunks) * kUnitBlocks;
  p.nb = min(kUnitBlocks, nb - p.b0);
  return p;
}

__global__ void __launch_bounds__(kProbeThreads, 1)
    read_probe_kernel(const uint8_t* __restrict__ k_pool, const uint8_t* __restrict__ v_pool,
                      int num_blocks, int hkv, int bs, int page_bytes,
                      const int32_t* __restrict__ tables, int max_blocks,
                      const int32_t* __restrict__ lens, int S,
                      unsigned long long* __restrict__ partial, unsigned int* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  int* prefix = reinterpret_cast<int*>(smem + kProbeStages * kStageBytes);  // [S + 1]
  int* nblk = prefix + PA_PROBE_MAX_SEQS + 1;                                // [S]
  __shared__ uint64_t full_bar[kProbeStages], empty_bar[kProbeStages];
  __shared__ int stage_len[kProbeStages];
  __shared__ int warp_tot[kProbeThreads / 32];
  __shared__ unsigned long long cta_sum;
  __shared__ int abort_flag;
  __shared__ int n_issued;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- blocks and units per sequence, and the units' exclusive prefix:
  // thread t owns a contiguous run of sequences ----
  const int per = (S + kProbeThreads - 1) / kProbeThreads;
  const int s0 = min(S, tid * per), s1 = min(S, s0 + per);
  int mine = 0;
  for (int s = s0; s < s1; ++s) {
    const int nb = probe_blocks(lens, s, max_blocks, bs, blockIdx.x == 0 ? err : nullptr);
    nblk[s] = nb;
    mine += units_of(nb, hkv);
  }
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  if (tid < kProbeStages) {
    mbar_init(&full_bar[tid], 1);
    mbar_init(&empty_bar[tid], kSumWarps);
    fence_barrier_init();
  }
  if (tid == 0) {
    cta_sum = 0;
    abort_flag = 0;
    n_issued = 0;
  }
  __syncthreads();
  int run = incl - mine;
  for (int w = 0; w < warp; ++w) run += warp_tot[w];
  for (int s = s0; s < s1; ++s) {
    prefix[s] = run;
    run += units_of(nblk[s], hkv);
  }
  if (tid == 0) {
    int total = 0;
    for (int w = 0; w < kProbeThreads / 32; ++w) total += warp_tot[w];
    prefix[S] = total;
  }
  __syncthreads();
  const int total = prefix[S];

  if (warp == 0) {
    // ---- copies.  The table entries of the next unit are loaded while the
    // current one is waited for and issued, so no copy waits on a table read.
    ProbeUnit cur{}, nxt{};
    int id_nxt = -1;
    const uint64_t pol = l2_policy_evict_first();  // read once: leave L2 to others
    if (static_cast<int>(blockIdx.x) < total) {
      nxt = locate(blockIdx.x, prefix, nblk, S);
      if (lane < nxt.nb) id_nxt = tables[static_cast<int64_t>(nxt.s) * max_blocks + nxt.b0 + lane];
    }
    int k = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++k) {
      cur = nxt;
      const int id = id_nxt;
      const int un = u + gridDim.x;
      if (un < total) {
        nxt = locate(un, prefix, nblk, S);
        id_nxt = lane < nxt.nb ? tables[static_cast<int64_t>(nxt.s) * max_blocks + nxt.b0 + lane]
                               : -1;
      }
      const int st = k % kProbeStages;
      if (k >= kProbeStages) {
        bool ok = true;
        if (lane == 0)
          ok = mbar_wait(&empty_bar[st], ((k / kProbeStages) - 1) & 1, &abort_flag, err);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
      }
      const bool valid = lane < cur.nb && id >= 0 && id < num_blocks;
      if (lane < cur.nb && !valid) raise_error(err, PA_DEV_ERR_BLOCK_ID);
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      const int nvalid = __popc(vmask);
      if (lane == 0) {
        stage_len[st] = 2 * nvalid * page_bytes;
        mbar_arrive_expect_tx(&full_bar[st], 2u * nvalid * page_bytes);
      }
      __syncwarp();
      if (valid) {
        const int slot = __popc(vmask & ((1u << lane) - 1u));
        uint8_t* dst = smem + st * kStageBytes;
        const int64_t off = (static_cast<int64_t>(id) * hkv + cur.h) * page_bytes;
        bulk_g2s_hint(dst + slot * page_bytes, k_pool + off, page_bytes, &full_bar[st], pol);
        bulk_g2s_hint(dst + (nvalid + slot) * page_bytes, v_pool + off, page_bytes, &full_bar[st],
                      pol);
      }
    }
    if (lane == 0) n_issued = k;
  } else {
    // ---- sums ----
    const int ctid = tid - 32;
    unsigned long long acc = 0;
    int k = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++k) {
      const int st = k % kProbeStages;
      if (!mbar_wait(&full_bar[st], (k / kProbeStages) & 1, &abort_flag, err)) break;
      const int bytes = stage_len[st];
      const uint32_t base = smem_u32(smem + st * kStageBytes);
      // four independent 16-byte loads per thread per round
      constexpr int kStride = 32 * kSumWarps * 16;
      for (int off = ctid * 16; off < bytes; off += 4 * kStride) {
        uint4 w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          w[j] = off + j * kStride < bytes ? lds128(base + off + j * kStride) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          acc += (static_cast<unsigned long long>(w[j].x) + w[j].y) +
                 (static_cast<unsigned long long>(w[j].z) + w[j].w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicAdd(&cta_sum, acc);
  }
  __syncthreads();
  if (tid == 0) {
    if (abort_flag) {
      // a wait gave up: let the copies already issued land before the CTA's
      // shared memory goes away (the last use of each stage; bounded waits)
      for (int k = n_issued - kProbeStages < 0 ? 0 : n_issued - kProbeStages; k < n_issued; ++k)
        mbar_wait(&full_bar[k % kProbeStages], (k / kProbeStages) & 1, nullptr, err);
    }
    partial[blockIdx.x] = cta_sum;
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_read_probe(const void* k_pool, const void* v_pool, pa_pool_desc pool,
                             const int32_t* block_tables, int32_t max_blocks_per_seq,
                             const int32_t* context_lens, int32_t num_seqs,
                             uint64_t* partial_sums, int32_t num_ctas, void* stream) {
  PA_NVTX_RANGE("pa_read_probe");
  int st = check_pool(pool);
  if (st != PA_OK) return st;
  if (num_seqs < 0 || num_seqs > PA_PROBE_MAX_SEQS || max_blocks_per_seq < 0) return PA_ERR_ARG;
  if (num_ctas < 1 || num_ctas > 65535) return PA_ERR_ARG;
  if (!k_pool || !v_pool || !partial_sums) return PA_ERR_ARG;
  if (num_seqs > 0 && (!block_tables || !context_lens)) return PA_ERR_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) ||
      (reinterpret_cast<uintptr_t>(partial_sums) & 7u) != 0)
    return PA_ERR_ARG;
  const int page_bytes = pool.block_size * pool.head_dim * 2;
  if (page_bytes > kMaxPageBytes) return PA_ERR_UNSUPPORTED;
  static KernelLaunchCache cache;
  if (cache.blocks_per_sm(reinterpret_cast<const void*>(read_probe_kernel), kProbeThreads,
                          kProbeSmem) < 1)
    return PA_ERR_CUDA;
  read_probe_kernel<<<num_ctas, kProbeThreads, kProbeSmem, as_stream(stream)>>>(
      static_cast<const uint8_t*>(k_pool), static_cast<const uint8_t*>(v_pool), pool.num_blocks,
      pool.num_kv_heads, pool.block_size, page_bytes, block_tables, max_blocks_per_seq,
      context_lens, num_seqs, reinterpret_cast<unsigned long long*>(partial_sums),
      device_error_word());
  return launch_status();
}
