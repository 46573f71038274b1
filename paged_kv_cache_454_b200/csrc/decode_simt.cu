// Paged decode on CUDA cores (any group size up to 16), the work plan
// shared by both decode kernels, and the log-sum-exp merge of split contexts.
//
// Design (B200):
//   * A persistent grid walks a flat work list of (sequence, KV head,
//     partition) items written by a one-CTA plan kernel.
//   * Each warp of a CTA streams its own share of the item's pages through a
//     private ring of shared-memory stages.  A page (16 tokens x head_dim of one
//     KV head) is one contiguous span of the pool, so it moves with one
//     cp.async.bulk per tensor, completed on the stage's mbarrier; the ring runs
//     ahead across item boundaries.
//   * q.k: 8 lanes per token, 16-byte conflict-free shared loads, xor-shuffle
//     reduction; online softmax in the log2 domain per warp; p.v: each lane owns
//     head_dim/32 output dimensions.
//   * The warps' (max, sum, output) triples are merged through shared memory;
//     a single-partition sequence writes its bf16 output directly, otherwise
//     the partition's normalised fp32 output and log-sum-exp go to the
//     workspace for the merge kernel.
#include <algorithm>
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"

namespace pa {

// ---------------------------------------------------------------------------
// Context lengths are clamped to the table width (the plan kernel flags it).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int clamp_context(int L, int max_blocks, unsigned int* err) {
  const int cap = max_blocks * 16;
  if (L < 0 || L > cap) {
    raise_error(err, PA_DEV_ERR_CONTEXT);
    return L < 0 ? 0 : cap;
  }
  return L;
}

// ---------------------------------------------------------------------------
// Item descriptors (decode: from the work list; prefill: one query row each)
// ---------------------------------------------------------------------------
struct SimtParams {
  const uint16_t* q;
  int64_t q_stride;
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  int num_blocks;
  int hkv;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  int num_seqs;
  int hq;
  float scale_log2;  // scale * log2(e)
  uint16_t* out;
  float* lse;
  // decode mode
  const int* header;
  const int* part_base;
  const int2* items;
  float* part_o;
  float* part_lse;
  int part_tokens;
  // prefill mode (one item per (query row, KV head), whole causal context)
  int prefill;
  const int32_t* cu_q;
  int total_q;
  unsigned int* err;
};

struct Item {
  int row;    // q / out row
  int seq;    // block-table row
  int g;      // KV head
  int part;   // partition index (decode)
  int tok0;   // first token of the partition
  int tok1;   // one past the last token
  int npart;  // partitions of the sequence (1: write the final output)
  int pbase;  // part_base[seq]
};

__device__ __forceinline__ Item load_item(const SimtParams& p, int item, int part_tokens) {
  Item it;
  if (!p.prefill) {
    const int2 d = p.items[item];
    it.seq = d.x;
    it.row = d.x;
    it.g = d.y >> 16;
    it.part = d.y & 0xffff;
    const int L = clamp_context(p.context_lens[it.seq], p.max_blocks, nullptr);
    it.tok0 = it.part * part_tokens;
    it.tok1 = min(L, it.tok0 + part_tokens);
    it.pbase = p.part_base[it.seq];
    it.npart = p.part_base[it.seq + 1] - it.pbase;
  } else {
    const int r = item / p.hkv;
    it.g = item - r * p.hkv;
    it.row = r;
    // sequence owning query row r: largest s with cu_q[s] <= r
    int lo = 0, hi = p.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.cu_q[mid] <= r) lo = mid; else hi = mid - 1;
    }
    it.seq = lo;
    const int q0 = p.cu_q[lo], q1 = p.cu_q[lo + 1];
    const int L = clamp_context(p.context_lens[lo], p.max_blocks, nullptr);
    const int c = L - (q1 - q0);
    int ctx = c + (r - q0) + 1;
    if (c < 0 || ctx > L) {  // a chunk longer than its context, or rows past cu_q[S]
      raise_error(p.err, PA_DEV_ERR_CONTEXT);
      ctx = c < 0 ? 0 : L;
    }
    it.part = 0;
    it.tok0 = 0;
    it.tok1 = ctx;
    it.npart = 1;
    it.pbase = 0;
  }
  return it;
}

// ---------------------------------------------------------------------------
// The CUDA-core decode kernel
// ---------------------------------------------------------------------------
template <int D, int G, int NW, int NST>
struct SimtCfg {
  static constexpr int kPageElems = 16 * D;
  static constexpr int kPageBytes = kPageElems * 2;
  static constexpr int kStageBytes = 2 * kPageBytes;            // K + V
  static constexpr int kRingBytes = NW * NST * kStageBytes;
  static constexpr int kBarBytes = NW * NST * 8;
  static constexpr int kRedFloats = NW * G * (D + 2);
  static constexpr int kSmemBytes = kRingBytes + kBarBytes + 16 * NW * NST + kRedFloats * 4 + 16;
  static constexpr int kNQ = D / 8;   // q values per lane per head (chunks j and j+8)
  static constexpr int kVD = D / 32;  // output dims per lane
};

template <int D, int G, int NW, int NST>
__global__ void __launch_bounds__(NW * 32) decode_simt_kernel(const SimtParams p) {
  using C = SimtCfg<D, G, NW, NST>;
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kRingBytes);
  int* stage_nvalid = reinterpret_cast<int*>(smem + C::kRingBytes + C::kBarBytes);
  float* red = reinterpret_cast<float*>(smem + C::kRingBytes + C::kBarBytes + 16 * NW * NST);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(red + C::kRedFloats);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid < NW * NST) mbar_init(&bars[tid], 1);
  if (tid == 0) *abort_flag = 0;
  fence_barrier_init();
  __syncthreads();

  const int total_items = p.prefill ? p.total_q * p.hkv : p.header[0];
  const int part_tokens = p.prefill ? (1 << 30) : p.header[3];
  const int64_t head_stride = 16LL * D;  // elements per (block, head) page

  // ---- producer cursor (all lanes track it; lane 0 issues) ----
  int l_item = blockIdx.x;
  int l_lp = warp;
  Item l_it;
  int l_npages = 0;
  auto enter_item = [&](int item) {
    l_it = load_item(p, item, part_tokens);
    l_npages = (l_it.tok1 - l_it.tok0 + 15) >> 4;
    if (l_it.tok1 <= l_it.tok0) l_npages = 0;
  };
  // find the first page of this warp at or after (l_item, l_lp)
  auto settle = [&]() {
    while (l_item < total_items && l_lp >= l_npages) {
      l_item += gridDim.x;
      l_lp = warp;
      if (l_item < total_items) enter_item(l_item);
    }
  };
  if (l_item < total_items) enter_item(l_item);
  settle();

  uint32_t n_issued = 0;
  auto issue = [&]() {
    // issue the producer cursor's page into stage n_issued % NST, then advance
    const int st = n_issued % NST;
    uint64_t* bar = &bars[warp * NST + st];
    unsigned char* kdst = ring + (warp * NST + st) * C::kStageBytes;
    if (lane == 0) {
      const int lb = (l_it.tok0 >> 4) + l_lp;
      const int pb = p.block_tables[static_cast<int64_t>(l_it.seq) * p.max_blocks + lb];
      const int ntok = min(16, l_it.tok1 - (lb << 4));
      if (pb < 0 || pb >= p.num_blocks) {
        raise_error(p.err, PA_DEV_ERR_BLOCK_ID);
        stage_nvalid[warp * NST + st] = 0;
        mbar_arrive(bar);
      } else {
        stage_nvalid[warp * NST + st] = ntok;
        const int64_t off = (static_cast<int64_t>(pb) * p.hkv + l_it.g) * head_stride;
        mbar_arrive_expect_tx(bar, 2 * C::kPageBytes);
        bulk_g2s(kdst, p.k_pool + off, C::kPageBytes, bar);
        bulk_g2s(kdst + C::kPageBytes, p.v_pool + off, C::kPageBytes, bar);
      }
    }
    ++n_issued;
    l_lp += NW;
    settle();
  };
  for (int i = 0; i < NST && l_item < total_items; ++i) issue();

  // ---- consumer ----
  const int tp = lane >> 3;  // token within a pass of 4
  const int j = lane & 7;    // 16-byte chunk (and chunk j + 8 when D == 128)
  uint32_t n_used = 0;
  const uint32_t ring_base = smem_u32(ring);

  for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
    const Item it = load_item(p, item, part_tokens);
    const int npages = it.tok1 > it.tok0 ? (it.tok1 - it.tok0 + 15) >> 4 : 0;

    // q fragments of this lane, pre-scaled into the log2 domain
    float qf[G][C::kNQ];
    {
      const uint16_t* qrow = p.q + static_cast<int64_t>(it.row) * p.q_stride +
                             static_cast<int64_t>(it.g) * G * D;
#pragma unroll
      for (int h = 0; h < G; ++h) {
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          const uint4 w = *reinterpret_cast<const uint4*>(qrow + h * D + (j + 8 * half) * 8);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            qf[h][half * 8 + 2 * e] = bf16lo(ws[e]) * p.scale_log2;
            qf[h][half * 8 + 2 * e + 1] = bf16hi(ws[e]) * p.scale_log2;
          }
        }
      }
    }
    float m[G], l[G], o[G][C::kVD];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -CUDART_INF_F;
      l[h] = 0.f;
#pragma unroll
      for (int i = 0; i < C::kVD; ++i) o[h][i] = 0.f;
    }

    for (int lp = warp; lp < npages; lp += NW) {
      const int st = n_used % NST;
      const uint32_t par = (n_used / NST) & 1;
      bool ok = mbar_wait(&bars[warp * NST + st], par, abort_flag, p.err);
      const int nvalid = ok ? stage_nvalid[warp * NST + st] : 0;
      const uint32_t kbase = ring_base + (warp * NST + st) * C::kStageBytes;
      const uint32_t vbase = kbase + C::kPageBytes;

      // ---- scores of this lane's 4 tokens ----
      float sc[4][G];
#pragma unroll
      for (int pass = 0; pass < 4; ++pass) {
        const int t = pass * 4 + tp;
        const uint32_t row = kbase + t * D * 2;
        float kf[C::kNQ];
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          const uint4 w = lds128(row + (j + 8 * half) * 16);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            kf[half * 8 + 2 * e] = bf16lo(ws[e]);
            kf[half * 8 + 2 * e + 1] = bf16hi(ws[e]);
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < C::kNQ; ++i) acc = fmaf(qf[h][i], kf[i], acc);
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          acc += __shfl_xor_sync(0xffffffffu, acc, 4);
          sc[pass][h] = (t < nvalid) ? acc : -CUDART_INF_F;
        }
      }
      // ---- online softmax (log2 domain) ----
      float pr[4][G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float mx = fmaxf(fmaxf(sc[0][h], sc[1][h]), fmaxf(sc[2][h], sc[3][h]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float mn = fmaxf(m[h], mx);
        const float alpha = (mn == -CUDART_INF_F) ? 1.f : exp2f(m[h] - mn);
        m[h] = mn;
        float sum = 0.f;
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          pr[pass][h] = (sc[pass][h] == -CUDART_INF_F) ? 0.f : exp2f(sc[pass][h] - mn);
          sum += pr[pass][h];
        }
        l[h] = l[h] * alpha + sum;
#pragma unroll
        for (int i = 0; i < C::kVD; ++i) o[h][i] *= alpha;
      }
      // ---- p . v ----
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        if (t < nvalid) {
          float pt[G];
#pragma unroll
          for (int h = 0; h < G; ++h) pt[h] = __shfl_sync(0xffffffffu, pr[t >> 2][h], (t & 3) * 8);
          const uint32_t vaddr = vbase + t * D * 2 + lane * C::kVD * 2;
          float vf[C::kVD];
          if constexpr (C::kVD == 4) {
            const uint2 w = lds64(vaddr);
            vf[0] = bf16lo(w.x);
            vf[1] = bf16hi(w.x);
            vf[2] = bf16lo(w.y);
            vf[3] = bf16hi(w.y);
          } else {
            const uint32_t w = lds32(vaddr);
            vf[0] = bf16lo(w);
            vf[1] = bf16hi(w);
          }
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < C::kVD; ++i) o[h][i] = fmaf(pt[h], vf[i], o[h][i]);
        }
      }
      __syncwarp();
      ++n_used;
      // refill the stage just consumed
      if (l_item < total_items && !*abort_flag) {
        fence_proxy_async_smem();
        issue();
      }
    }

    // ---- merge the warps' partial results ----
    float* red_m = red;
    float* red_l = red + NW * G;
    float* red_o = red + 2 * NW * G;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float lt = l[h];
      lt += __shfl_xor_sync(0xffffffffu, lt, 8);
      lt += __shfl_xor_sync(0xffffffffu, lt, 16);
      if (lane == 0) {
        red_m[warp * G + h] = m[h];
        red_l[warp * G + h] = lt;
      }
#pragma unroll
      for (int i = 0; i < C::kVD; ++i) red_o[(warp * G + h) * D + lane * C::kVD + i] = o[h][i];
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += NW * 32) {
      const int h = idx / D, d = idx - h * D;
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w * G + h]);
      float res = 0.f, lse2 = -CUDART_INF_F;
      if (M != -CUDART_INF_F) {
        float wsum = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float mw = red_m[w * G + h];
          if (mw != -CUDART_INF_F) {
            const float f = exp2f(mw - M);
            wsum += f * red_l[w * G + h];
            acc += f * red_o[(w * G + h) * D + d];
          }
        }
        res = acc / wsum;
        lse2 = M + log2f(wsum);
      }
      const int hq = it.g * G + h;
      if (it.npart == 1) {
        p.out[(static_cast<int64_t>(it.row) * p.hq + hq) * D + d] = f32_to_bf16_bits(res);
        if (d == 0 && p.lse) p.lse[static_cast<int64_t>(it.row) * p.hq + hq] = lse2 * kLn2;
      } else {
        const int64_t rec = static_cast<int64_t>(it.pbase + it.part) * p.hq + hq;
        p.part_o[rec * D + d] = res;
        if (d == 0) p.part_lse[rec] = lse2;
      }
    }
    __syncthreads();
  }
  // Wind down: wait (bounded) for this warp's copies still in flight.
  while (n_used < n_issued) {
    const int st = n_used % NST;
    if (!mbar_wait(&bars[warp * NST + st], (n_used / NST) & 1, nullptr, p.err)) break;
    ++n_used;
  }
}

// ---------------------------------------------------------------------------
// Merge of split-context partitions by their log-sum-exp.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const int* __restrict__ part_base,
                                                         const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse,
                                                         int hq, uint16_t* __restrict__ out,
                                                         float* __restrict__ lse) {
  const int s = blockIdx.x / hq;
  const int h = blockIdx.x - s * hq;
  const int b = part_base[s];
  const int np = part_base[s + 1] - b;
  if (np <= 1) return;  // written by the decode kernel
  const int d = threadIdx.x;
  float M = -CUDART_INF_F;
  for (int i = 0; i < np; ++i) M = fmaxf(M, part_lse[static_cast<int64_t>(b + i) * hq + h]);
  float res = 0.f, lse2 = -CUDART_INF_F;
  if (M != -CUDART_INF_F) {
    float wsum = 0.f, acc = 0.f;
    for (int i = 0; i < np; ++i) {
      const int64_t rec = static_cast<int64_t>(b + i) * hq + h;
      const float li = part_lse[rec];
      if (li == -CUDART_INF_F) continue;
      const float f = exp2f(li - M);
      wsum += f;
      acc += f * part_o[rec * D + d];
    }
    res = acc / wsum;
    lse2 = M + log2f(wsum);
  }
  out[(static_cast<int64_t>(s) * hq + h) * D + d] = f32_to_bf16_bits(res);
  if (d == 0 && lse) lse[static_cast<int64_t>(s) * hq + h] = lse2 * kLn2;
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
namespace {

template <int D, int G>
int launch_simt_impl(const SimtParams& prm, int64_t item_bound, cudaStream_t stream) {
  constexpr int NW = 4;
  constexpr int NST = (D == 64) ? 6 : 3;
  using C = SimtCfg<D, G, NW, NST>;
  auto kern = decode_simt_kernel<D, G, NW, NST>;
  static KernelLaunchCache cache;
  const int per_sm = cache.blocks_per_sm(reinterpret_cast<const void*>(kern), NW * 32,
                                         C::kSmemBytes);
  if (per_sm < 1) return PA_ERR_CUDA;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(cap, item_bound)));
  kern<<<grid, NW * 32, C::kSmemBytes, stream>>>(prm);
  return launch_status();
}

template <int D>
int launch_simt_d(const SimtParams& prm, int group, int64_t item_bound, cudaStream_t stream) {
  switch (group) {
    case 1: return launch_simt_impl<D, 1>(prm, item_bound, stream);
    case 2: return launch_simt_impl<D, 2>(prm, item_bound, stream);
    case 3: return launch_simt_impl<D, 3>(prm, item_bound, stream);
    case 4: return launch_simt_impl<D, 4>(prm, item_bound, stream);
    case 5: return launch_simt_impl<D, 5>(prm, item_bound, stream);
    case 6: return launch_simt_impl<D, 6>(prm, item_bound, stream);
    case 7: return launch_simt_impl<D, 7>(prm, item_bound, stream);
    case 8: return launch_simt_impl<D, 8>(prm, item_bound, stream);
    case 9: return launch_simt_impl<D, 9>(prm, item_bound, stream);
    case 10: return launch_simt_impl<D, 10>(prm, item_bound, stream);
    case 11: return launch_simt_impl<D, 11>(prm, item_bound, stream);
    case 12: return launch_simt_impl<D, 12>(prm, item_bound, stream);
    case 13: return launch_simt_impl<D, 13>(prm, item_bound, stream);
    case 14: return launch_simt_impl<D, 14>(prm, item_bound, stream);
    case 15: return launch_simt_impl<D, 15>(prm, item_bound, stream);
    case 16: return launch_simt_impl<D, 16>(prm, item_bound, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

int launch_simt(const SimtParams& prm, int head_dim, int group, int64_t item_bound,
                cudaStream_t stream) {
  if (head_dim == 128) return launch_simt_d<128>(prm, group, item_bound, stream);
  if (head_dim == 64) return launch_simt_d<64>(prm, group, item_bound, stream);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

int launch_decode_merge(const DecodeArgs& a) {
  const int64_t n = static_cast<int64_t>(a.num_seqs) * a.num_q_heads;
  if (n > 0x7fffffff) return PA_ERR_UNSUPPORTED;
  if (a.pool.head_dim == 128)
    decode_merge_kernel<128><<<static_cast<int>(n), 128, 0, a.stream>>>(
        a.ws.part_base, a.ws.part_o, a.ws.part_lse, a.num_q_heads, a.out, a.lse);
  else
    decode_merge_kernel<64><<<static_cast<int>(n), 64, 0, a.stream>>>(
        a.ws.part_base, a.ws.part_o, a.ws.part_lse, a.num_q_heads, a.out, a.lse);
  return launch_status();
}

int launch_decode_simt(const DecodeArgs& a) {
  SimtParams p{};
  p.q = a.q;
  p.q_stride = a.q_stride;
  p.k_pool = a.k_pool;
  p.v_pool = a.v_pool;
  p.num_blocks = a.pool.num_blocks;
  p.hkv = a.pool.num_kv_heads;
  p.block_tables = a.block_tables;
  p.max_blocks = a.max_blocks;
  p.context_lens = a.context_lens;
  p.num_seqs = a.num_seqs;
  p.hq = a.num_q_heads;
  p.scale_log2 = a.scale * kLog2e;
  p.out = a.out;
  p.lse = a.lse;
  p.header = a.ws.header;
  p.part_base = a.ws.part_base;
  p.items = a.ws.items;
  p.part_o = a.ws.part_o;
  p.part_lse = a.ws.part_lse;
  p.part_tokens = 0;  // read from the plan's header
  p.prefill = 0;
  p.err = a.err;
  const int64_t bound = static_cast<int64_t>(a.num_seqs) * a.max_parts * a.pool.num_kv_heads;
  return launch_simt(p, a.pool.head_dim, a.num_q_heads / a.pool.num_kv_heads, bound, a.stream);
}

int launch_prefill_simt(const PrefillArgs& a) {
  SimtParams p{};
  p.q = a.q;
  p.q_stride = a.q_stride;
  p.k_pool = a.k_pool;
  p.v_pool = a.v_pool;
  p.num_blocks = a.pool.num_blocks;
  p.hkv = a.pool.num_kv_heads;
  p.block_tables = a.block_tables;
  p.max_blocks = a.max_blocks;
  p.context_lens = a.context_lens;
  p.num_seqs = a.num_seqs;
  p.hq = a.num_q_heads;
  p.scale_log2 = a.scale * kLog2e;
  p.out = a.out;
  p.lse = a.lse;
  p.part_tokens = 1 << 30;
  p.prefill = 1;
  p.cu_q = a.cu_q;
  p.total_q = a.total_q;
  p.err = a.err;
  const int64_t bound = static_cast<int64_t>(a.total_q) * a.pool.num_kv_heads;
  return launch_simt(p, a.pool.head_dim, a.num_q_heads / a.pool.num_kv_heads, bound, a.stream);
}

}  // namespace pa
