// Chunked prefill on the 5th-generation tensor cores.
//
// A sequence adds a chunk of n new tokens on top of c cached ones; query i of
// the chunk (absolute position c + i) attends to keys 0 .. c + i.  For one KV
// head g, the G = Hq/Hkv query heads of the chunk form rows (token i, head h),
// ordered token-major, so one 128-row tile holds floor(128/G) tokens x G heads
// and shares every K/V tile among them.  Per 128-key tile of the paged context:
//     S [128 rows x 128 keys] = Q_tile [128 x D] . K_tile^T         (8 MMAs, K = 16)
//     O [128 rows x D]        = P [128 x 128 keys] . V_tile         (16 MMAs, K = 16)
// where P = P_hi + P_lo: the bf16 rounding of p and the bf16 rounding of what it
// left out, so the weights reach the product with about 16 significant bits
// (bf16 p alone misses the output tolerance on contexts of a few keys)
// with fp32 accumulators in tensor memory (S and O double-buffered: all 512
// columns) and operands in 128-byte-swizzled shared memory.
//
// Roles (one CTA per SM, persistent over (sequence, KV head, row tile) items,
// longest causal ranges first):
//   warp 0     producer: the row tile of q with one 3-D tensor copy (tokens x
//              heads x 64 dims, twice; one q slot), then each key tile's 8 pages, K and V
//              in separate two-slot rings so a K slot frees as soon as its
//              scores are computed.
//   warp 1     allocates tensor memory; one lane issues S of tile t, then O of
//              tile t-1.
//   warps 2-5  softmax: thread r owns row r.  Two passes over its S row
//              (maximum, then exponentials written as bf16 into the P operand),
//              online rescaling, and the tile's O folded into registers; the
//              row is normalised and written at the end of the item.
// Keys past a row's causal limit get p = 0; key rows past the context or in
// pages with a bad block id are zeroed in V before the second product.  Every
// wait is bounded; no unbounded barrier is used inside the role loops.
#include <math_constants.h>

#include "internal.h"
#include "tc_common.cuh"

namespace pa {
namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kRegion = 128 * 128;            // 128 rows x 128 bytes
constexpr int kTileBytes = 2 * kRegion;       // one 128 x 128 bf16 operand tile
constexpr int kOffQ = 0;                      // Q
constexpr int kOffK = kOffQ + kTileBytes;     // K[2]
constexpr int kOffV = kOffK + 2 * kTileBytes; // V[2]
constexpr int kOffP = kOffV + 2 * kTileBytes; // P high parts
constexpr int kOffPlo = kOffP + kTileBytes;   // P remainders
constexpr int kOffBar = kOffPlo + kTileBytes;
// q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, s_free (x2 each);
// p_full; o_full, o_free (x2); drain
constexpr int kNumBars = 8 * 2 + 1 + 4 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemUsed = kOffMisc + 64;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;  // S x2 (128 each), O x2 (128 each)
constexpr uint32_t kPageHalf = 16 * 128;  // one 64-dim half of one page: 2 KiB

constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, false, true);

struct __align__(64) PfParams {
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_q;
  const int32_t* cu_q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  uint16_t* out;
  float* lse;
  unsigned int* err;
  int max_blocks;
  int num_blocks;
  int hkv;
  int hq;
  int group;
  int tpt;      // tokens per row tile (floor(128 / group))
  int num_seqs;
  int mt_max;   // row tiles of the longest chunk
  int total;    // virtual items: mt_max * num_seqs * hkv
  float scale_log2;
};

struct PfItem {
  bool valid;
  int s, g, q0, i0, ntok, c, ctx, kv_end, ntiles;
};

// Virtual item v -> (row tile, sequence, KV head); later row tiles (longer
// causal ranges) first.
__device__ __forceinline__ PfItem pf_item(const PfParams& p, int v, bool flag_errors) {
  PfItem it;
  it.g = v % p.hkv;
  const int rest = v / p.hkv;
  it.s = rest % p.num_seqs;
  const int mt = p.mt_max - 1 - rest / p.num_seqs;
  it.q0 = p.cu_q[it.s];
  const int n = p.cu_q[it.s + 1] - it.q0;
  it.i0 = mt * p.tpt;
  it.valid = it.i0 < n;
  if (!it.valid) return it;
  it.ntok = min(p.tpt, n - it.i0);
  int L = p.context_lens[it.s];
  const int cap = p.max_blocks * 16;
  if (L < n || L > cap) {
    if (flag_errors) raise_error(p.err, PA_DEV_ERR_CONTEXT);
    L = L > cap ? cap : L;
    if (L < n) {  // a chunk longer than its context: nothing consistent to compute
      it.valid = false;
      return it;
    }
  }
  it.ctx = L;
  it.c = L - n;
  it.kv_end = min(L, it.c + it.i0 + it.ntok);
  it.ntiles = (it.kv_end + 127) / 128;
  return it;
}

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) |
         (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ PfParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sptr = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sptr + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* k_full = bars + 4;
  uint64_t* k_empty = bars + 6;
  uint64_t* v_full = bars + 8;
  uint64_t* v_empty = bars + 10;
  uint64_t* s_full = bars + 12;
  uint64_t* s_free = bars + 14;
  uint64_t* p_full = bars + 16;
  uint64_t* o_full = bars + 17;
  uint64_t* o_free = bars + 19;
  uint64_t* drain = bars + 21;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + kOffMisc + 4);
  uint32_t* kmask = reinterpret_cast<uint32_t*>(sptr + kOffMisc + 16);  // [4] valid pages per key tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_q);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  fence_barrier_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int rows_box = p.tpt * p.group;

  if (warp == 0) {
    // =========================== producer ===========================
    uint32_t t = 0, it = 0;
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, lane == 0);
      if (!I.valid) continue;
      const int qb = 0;
      mbar_wait(&q_empty[qb], (it & 1) ^ 1, abort_flag, p.err);
      if (!*abort_flag && lane == 0) {
        const uint32_t qd = sbase + kOffQ;
        mbar_arrive_expect_tx(&q_full[qb], 2 * rows_box * 128);
        tma_load_3d(qd, &p.tm_q, 0, I.g * p.group, I.q0 + I.i0, &q_full[qb]);
        tma_load_3d(qd + kRegion, &p.tm_q, 64, I.g * p.group, I.q0 + I.i0, &q_full[qb]);
      }
      ++it;
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int ptok = j * 128 + lane * 16;
        int pb = -1;
        if (lane < 8 && ptok < I.kv_end) {
          pb = p.block_tables[static_cast<int64_t>(I.s) * p.max_blocks + (ptok >> 4)];
          if (pb < 0 || pb >= p.num_blocks) {
            raise_error(p.err, PA_DEV_ERR_BLOCK_ID);
            pb = -1;
          }
        }
        const unsigned vm = __ballot_sync(0xffffffffu, pb >= 0) & 0xffu;
        const int st = t & 1;
        const uint32_t ph = (t >> 1) & 1;
        const int row = (pb * p.hkv + I.g) * 16;
        mbar_wait(&k_empty[st], ph ^ 1, abort_flag, p.err);
        if (!*abort_flag) {
          if (lane == 0) {
            kmask[t & 3] = vm;
            mbar_arrive_expect_tx(&k_full[st], __popc(vm) * 2 * kPageHalf);
          }
          __syncwarp();
          if (pb >= 0) {
            const uint32_t kd = sbase + kOffK + st * kTileBytes + lane * kPageHalf;
            tma_load_2d(kd, &p.tm_k, 0, row, &k_full[st]);
            tma_load_2d(kd + kRegion, &p.tm_k, 64, row, &k_full[st]);
          }
        }
        mbar_wait(&v_empty[st], ph ^ 1, abort_flag, p.err);
        if (!*abort_flag) {
          if (lane == 0) mbar_arrive_expect_tx(&v_full[st], __popc(vm) * 2 * kPageHalf);
          __syncwarp();
          if (pb >= 0) {
            const uint32_t vd = sbase + kOffV + st * kTileBytes + lane * kPageHalf;
            tma_load_2d(vd, &p.tm_v, 0, row, &v_full[st]);
            tma_load_2d(vd + kRegion, &p.tm_v, 64, row, &v_full[st]);
          }
        }
      }
    }
    if (*abort_flag && lane == 0) {
      // wait (bounded) for copies still in flight
      for (uint32_t u = t > 2 ? t - 2 : 0; u < t; ++u) {
        mbar_wait(&k_full[u & 1], (u >> 1) & 1, nullptr, p.err);
        mbar_wait(&v_full[u & 1], (u >> 1) & 1, nullptr, p.err);
      }
      if (it > 0) mbar_wait(&q_full[0], (it - 1) & 1, nullptr, p.err);
    }
  } else if (warp == 1) {
    // ============================= MMA ==============================
    if (lane == 0) {
      uint32_t t = 0, it = 0, prev = 0;
      bool have_prev = false;
      auto issue_pv = [&](uint32_t u) {
        const int st = u & 1;
        mbar_wait(&v_full[st], (u >> 1) & 1, abort_flag, p.err);
        mbar_wait(p_full, u & 1, abort_flag, p.err);
        mbar_wait(&o_free[st], ((u >> 1) & 1) ^ 1, abort_flag, p.err);
        if (*abort_flag) return;
        tc_fence_after();
        const uint32_t vb = sbase + kOffV + st * kTileBytes;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t pb = sbase + (part ? kOffPlo : kOffP);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t a = smem_desc_sw128(pb + (k >> 2) * kRegion + (k & 3) * 32, 16, 1024);
            const uint64_t b = smem_desc_sw128(vb + k * 2048, kRegion, 1024);
            umma_ss(tmem + 256 + st * 128, a, b, kIdescO, (part | k) ? 1u : 0u);
          }
        }
        umma_commit(&o_full[st]);
        umma_commit(&v_empty[st]);
      };
      for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
        const PfItem I = pf_item(p, v, false);
        if (!I.valid) continue;
        const int qb = 0;
        mbar_wait(&q_full[qb], it & 1, abort_flag, p.err);
        const uint32_t qa = sbase + kOffQ;
        for (int j = 0; j < I.ntiles; ++j, ++t) {
          const int st = t & 1;
          mbar_wait(&k_full[st], (t >> 1) & 1, abort_flag, p.err);
          mbar_wait(&s_free[st], ((t >> 1) & 1) ^ 1, abort_flag, p.err);
          if (!*abort_flag) {
            tc_fence_after();
            const uint32_t kb = sbase + kOffK + st * kTileBytes;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
              umma_ss(tmem + st * 128, smem_desc_sw128(qa + off, 16, 1024),
                      smem_desc_sw128(kb + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[st]);
            umma_commit(&k_empty[st]);
            if (j == I.ntiles - 1) umma_commit(&q_empty[qb]);
          }
          if (have_prev) issue_pv(prev);
          prev = t;
          have_prev = true;
        }
        ++it;
      }
      if (have_prev) issue_pv(prev);
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err);
    }
    __syncwarp();
  } else {
    // ============================ softmax ============================
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // row of the tile, TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    uint32_t t = 0;
    float acc[kD];
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, false);
      if (!I.valid) continue;
      const int ti = r / p.group;  // token of this row within the tile
      const bool row_ok = r < rows_box && ti < I.ntok;
      const int limit = row_ok ? I.c + I.i0 + ti + 1 : 0;  // keys 0 .. limit-1
      float m = -CUDART_INF_F, l = 0.f, alpha_prev = 1.f;
#pragma unroll
      for (int d = 0; d < kD; ++d) acc[d] = 0.f;
      auto fold = [&](uint32_t u) {
        const int b = u & 1;
        mbar_wait(&o_full[b], (u >> 1) & 1, abort_flag, p.err);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float ov[16];
          tmem_ld16(tmem + lane_addr + 256 + b * 128 + c * 16, ov);
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[c * 16 + k] = acc[c * 16 + k] * alpha_prev + ov[k];
        }
        tc_fence_before();
        mbar_arrive(&o_free[b]);
      };
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int b = t & 1;
        const int kv0 = j * 128;
        mbar_wait(&s_full[b], (t >> 1) & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t vm = kmask[t & 3];
        const uint32_t sa = tmem + lane_addr + b * 128;
        // keys kv0 + k are visible to this row when below its limit and in a loaded page
        auto visible = [&](int k) {
          return kv0 + k < limit && ((vm >> (k >> 4)) & 1u);
        };
        // pass 1: row maximum
        float mx = -CUDART_INF_F;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float sv[32];
          tmem_ld32(sa + c * 32, sv);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (visible(c * 32 + k)) mx = fmaxf(mx, sv[k] * p.scale_log2);
        }
        const float mn = fmaxf(m, mx);
        const float alpha = (mn == -CUDART_INF_F) ? 1.f : exp2f(m - mn);
        // O of the previous tile is done: P is free again, fold it in
        if (j > 0) fold(t - 1);
        // pass 2: exponentials into P (bf16, K-major 128B swizzle), row sum
        float rs = 0.f;
        const uint32_t prow = sbase + kOffP + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float sv[16];
          tmem_ld16(sa + c * 16, sv);
          uint32_t pk[8], pl[8];
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const float p0 = visible(c * 16 + k) ? exp2f(sv[k] * p.scale_log2 - mn) : 0.f;
            const float p1 = visible(c * 16 + k + 1) ? exp2f(sv[k + 1] * p.scale_log2 - mn) : 0.f;
            rs += p0 + p1;
            const uint32_t hi = pack_bf16x2(p0, p1);
            pk[k >> 1] = hi;
            pl[k >> 1] = pack_bf16x2(p0 - __uint_as_float(hi << 16),
                                     p1 - __uint_as_float(hi & 0xffff0000u));
          }
          // keys c*16 .. c*16+15: region (c*16)/64, 16-byte chunks 2*(c%4) and 2*(c%4)+1
          const uint32_t region = prow + (c >> 2) * kRegion;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int chunk = (c & 3) * 2 + q;
            const uint32_t off = region + ((chunk ^ (r & 7)) << 4);
            sts128(off, make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]));
            sts128(off + (kOffPlo - kOffP),
                   make_uint4(pl[4 * q], pl[4 * q + 1], pl[4 * q + 2], pl[4 * q + 3]));
          }
        }
        tc_fence_before();
        mbar_arrive(&s_free[b]);
        // key rows past the context or in an unloaded page: zero them in V
        if (kv0 + 128 > I.ctx || vm != 0xffu) {
          const int key = kv0 + r;
          if (key >= I.ctx || !((vm >> (r >> 4)) & 1u)) {
            mbar_wait(&v_full[b], (t >> 1) & 1, abort_flag, p.err);
            const uint32_t vrow = sbase + kOffV + b * kTileBytes + r * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              sts128_zero(vrow + k * 16);
              sts128_zero(vrow + kRegion + k * 16);
            }
          }
        }
        l = l * alpha + rs;
        m = mn;
        alpha_prev = alpha;
        fence_proxy_async_smem();
        mbar_arrive(p_full);
      }
      if (I.ntiles > 0) fold(t - 1);
      if (row_ok) {
        const int h = r - ti * p.group;
        const int64_t orow = static_cast<int64_t>(I.q0 + I.i0 + ti) * p.hq + I.g * p.group + h;
        const bool live = l > 0.f;
        const float inv = live ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kD);
#pragma unroll
        for (int q = 0; q < kD / 8; ++q) {
          uint4 w;
          w.x = pack_bf16x2(acc[8 * q] * inv, acc[8 * q + 1] * inv);
          w.y = pack_bf16x2(acc[8 * q + 2] * inv, acc[8 * q + 3] * inv);
          w.z = pack_bf16x2(acc[8 * q + 4] * inv, acc[8 * q + 5] * inv);
          w.w = pack_bf16x2(acc[8 * q + 6] * inv, acc[8 * q + 7] * inv);
          dst[q] = w;
        }
        if (p.lse) p.lse[orow] = live ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool prefill_tcgen05_supported(const PrefillArgs& a) {
  const int group = a.num_q_heads / a.pool.num_kv_heads;
  const int64_t rows = static_cast<int64_t>(a.pool.num_blocks) * a.pool.num_kv_heads * 16;
  return a.pool.head_dim == kD && group >= 1 && group <= 16 && rows < (1LL << 31) &&
         a.total_q < (1 << 30);
}

int launch_prefill_tcgen05(const PrefillArgs& a) {
  if (!prefill_tcgen05_supported(a)) return PA_ERR_UNSUPPORTED;
  const int group = a.num_q_heads / a.pool.num_kv_heads;
  PfParams p;
  const int64_t rows = static_cast<int64_t>(a.pool.num_blocks) * a.pool.num_kv_heads * 16;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(rows)};
    const uint64_t strides[1] = {kD * 2};
    const uint32_t box[2] = {64, 16};
    if (!encode_bf16_map(&p.tm_k, a.k_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
    if (!encode_bf16_map(&p.tm_v, a.v_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
  }
  p.tpt = 128 / group;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(a.num_q_heads),
                              static_cast<uint64_t>(a.total_q)};
    const uint64_t strides[2] = {kD * 2, static_cast<uint64_t>(a.q_stride) * 2};
    const uint32_t box[3] = {64, static_cast<uint32_t>(group), static_cast<uint32_t>(p.tpt)};
    if (!encode_bf16_map(&p.tm_q, a.q, 3, dims, strides, box)) return PA_ERR_CUDA;
  }
  p.cu_q = a.cu_q;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.pool.num_blocks;
  p.hkv = a.pool.num_kv_heads;
  p.hq = a.num_q_heads;
  p.group = group;
  p.num_seqs = a.num_seqs;
  p.mt_max = (a.max_q_len + p.tpt - 1) / p.tpt;
  const int64_t total = static_cast<int64_t>(p.mt_max) * a.num_seqs * p.hkv;
  if (total >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
  p.total = static_cast<int>(total);
  p.scale_log2 = a.scale * kLog2e;
  if (p.total == 0) return PA_OK;
  static KernelLaunchCache cache;
  const int per_sm = cache.blocks_per_sm(reinterpret_cast<const void*>(prefill_tc_kernel),
                                         kThreads, kSmemBytes);
  if (per_sm < 1) return PA_ERR_CUDA;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(p.total < cap ? p.total : cap);
  prefill_tc_kernel<<<grid, kThreads, kSmemBytes, a.stream>>>(p);
  return launch_status();
}

}  // namespace pa
