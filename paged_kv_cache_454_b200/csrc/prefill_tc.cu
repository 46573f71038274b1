// Chunked prefill on the 5th-generation tensor cores.
//
// A sequence adds a chunk of n new tokens on top of c cached ones; query i of
// the chunk (absolute position c + i) attends to keys 0 .. c + i.  For one KV
// head g, the G = Hq/Hkv query heads of the chunk form rows (token i, head h),
// ordered token-major, so one 128-row tile holds floor(128/G) tokens x G heads
// and shares every K/V tile among them.  Per 128-key tile of the paged context:
//     S [128 rows x 128 keys] = Q_tile [128 x D] . K_tile^T         (8 MMAs, K = 16)
//     O [128 rows x D]       += P [128 x 128 keys] . V_tile         (16 MMAs, K = 16)
// with fp32 accumulators in tensor memory.  P = P_hi + P_lo, the bf16 rounding
// of p and the bf16 rounding of what it left out, so the weights reach the
// product with about 16 significant bits (bf16 p alone misses the output
// tolerance on contexts of a few keys).  P is written back into the tensor
// memory its scores came from (for each 16-key group: 8 columns of P_hi, then 8
// of P_lo) and the second product reads it from there.
//
// Softmax with a lazily raised maximum: each row keeps the maximum m it last
// used; a tile whose maximum exceeds m by more than 8 (log2 units) raises m,
// and only then is the row of O in tensor memory (and the row sum) rescaled.
// Otherwise exp2(s - m) <= 256 is used as is; the final division by the row
// sum accumulated with the same m makes the result exact either way.
//
// Tensor memory (512 columns): S/P of three tiles (128 each) and O (128).
// Shared memory: q of one row tile, two K slots, three V slots (128B swizzle).
//
// Roles (one CTA per SM, persistent over (sequence, KV head, row tile) items,
// longest causal ranges first):
//   warp 0      producer of q and K: the row tile of q with one 3-D tensor copy
//               (tokens x heads x 64 dims, twice), then each key tile's 8 pages.
//   warp 10     producer of V: each key tile's 8 pages.
//   warp 1      allocates tensor memory; one lane issues S of tile t, then the
//               P.V of tile t-1.
//   warps 2-9   softmax, two warpgroups: thread (r, half) owns row r and key
//               columns (and output dims) 64*half .. +63; row maxima and sums
//               are exchanged with the partner warp through shared memory.
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
constexpr int kQSlots = 1, kKSlots = 2, kVSlots = 3, kSP = 3;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQSlots * kTileBytes;
constexpr int kOffV = kOffK + kKSlots * kTileBytes;
constexpr int kOffBar = kOffV + kVSlots * kTileBytes;
// q_full/empty, k_full/empty, v_full/empty (per slot); s_full, p_full, pv_done
// (per S/P buffer); o_free; drain; row-quadrant exchange (x4)
constexpr int kNumBars = 2 * (kQSlots + kKSlots + kVSlots) + 3 * kSP + 1 + 1 + 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem slot, abort flag, kmask[8]
constexpr int kOffX = kOffMisc + 64;                // exchange buffer [2][2][128] floats
constexpr int kSmemUsed = kOffX + 2 * 2 * 128 * 4;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kThreads = 352;   // q/K producer, MMA, 8 softmax warps, V producer
constexpr int kTmemCols = 512;  // S/P x3 (128 each), O (128)
constexpr int kOcol = kSP * 128;
constexpr uint32_t kPageHalf = 16 * 128;  // one 64-dim half of one page: 2 KiB
constexpr float kRescaleLog2 = 8.f;       // raise the row maximum only past 2^8

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

// The same in two steps for a thread that must not stall on the loads: the
// three loads of item v are issued early (volatile, so they stay where they
// are written) and the item is decoded when it is needed.
struct PfRaw {
  int v, q0, q1, L;
};

__device__ __forceinline__ int ld_early(const int32_t* ptr) {
  int x;
  asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(x) : "l"(ptr));
  return x;
}

__device__ __forceinline__ PfRaw pf_fetch(const PfParams& p, int v) {
  PfRaw r;
  r.v = v;
  const int s = (v / p.hkv) % p.num_seqs;
  r.q0 = ld_early(p.cu_q + s);
  r.q1 = ld_early(p.cu_q + s + 1);
  r.L = ld_early(p.context_lens + s);
  return r;
}

__device__ __forceinline__ PfItem pf_decode(const PfParams& p, const PfRaw& r) {
  PfItem it;
  it.g = r.v % p.hkv;
  const int rest = r.v / p.hkv;
  it.s = rest % p.num_seqs;
  const int mt = p.mt_max - 1 - rest / p.num_seqs;
  it.q0 = r.q0;
  const int n = r.q1 - r.q0;
  it.i0 = mt * p.tpt;
  it.valid = it.i0 < n;
  if (!it.valid) return it;
  it.ntok = min(p.tpt, n - it.i0);
  int L = r.L;
  const int cap = p.max_blocks * 16;
  if (L < n || L > cap) {
    L = L > cap ? cap : L;
    if (L < n) {
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return static_cast<uint32_t>(f32_to_bf16_bits(lo)) |
         (static_cast<uint32_t>(f32_to_bf16_bits(hi)) << 16);
}

// Block-table entries of one key tile (lanes 0-7), range-checked.
__device__ __forceinline__ int tile_page(const PfParams& p, const PfItem& I, int j, int lane,
                                         bool flag_errors) {
  const int ptok = j * 128 + lane * 16;
  int pb = -1;
  if (lane < 8 && ptok < I.kv_end) {
    pb = p.block_tables[static_cast<int64_t>(I.s) * p.max_blocks + (ptok >> 4)];
    if (pb < 0 || pb >= p.num_blocks) {
      if (flag_errors) raise_error(p.err, PA_DEV_ERR_BLOCK_ID);
      pb = -1;
    }
  }
  return pb;
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ PfParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sptr = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sptr + kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + kQSlots;
  uint64_t* k_full = q_empty + kQSlots;
  uint64_t* k_empty = k_full + kKSlots;
  uint64_t* v_full = k_empty + kKSlots;
  uint64_t* v_empty = v_full + kVSlots;
  uint64_t* s_full = v_empty + kVSlots;   // S of tile t in buffer t % 3
  uint64_t* p_full = s_full + kSP;        // P of tile t written back
  uint64_t* pv_done = p_full + kSP;       // P.V of tile t complete
  uint64_t* o_free = pv_done + kSP;       // O of an item read out
  uint64_t* drain = o_free + 1;
  uint64_t* xq = drain + 1;               // [4]: the two softmax warps sharing a row quadrant
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + kOffMisc + 4);
  // loaded pages of key tile t, in slot t % 8 (written by the K producer; the
  // slot is rewritten only after the scores of tile t + 6 are done)
  uint32_t* kmask = reinterpret_cast<uint32_t*>(sptr + kOffMisc + 16);
  float* xbuf = reinterpret_cast<float*>(sptr + kOffX);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(o_free, 256);
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xq[i], 2);
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
    // ========================= q and K producer =========================
    uint32_t t = 0, it = 0;
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, lane == 0);
      if (!I.valid) continue;
      const int qs = it % kQSlots;
      mbar_wait(&q_empty[qs], ((it / kQSlots) & 1) ^ 1, abort_flag, p.err);
      if (!*abort_flag && lane == 0) {
        const uint32_t qd = sbase + kOffQ + qs * kTileBytes;
        mbar_arrive_expect_tx(&q_full[qs], 2 * rows_box * 128);
        tma_load_3d(qd, &p.tm_q, 0, I.g * p.group, I.q0 + I.i0, &q_full[qs]);
        tma_load_3d(qd + kRegion, &p.tm_q, 64, I.g * p.group, I.q0 + I.i0, &q_full[qs]);
      }
      ++it;
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int pb = tile_page(p, I, j, lane, true);
        const unsigned vm = __ballot_sync(0xffffffffu, pb >= 0) & 0xffu;
        const int ks = t % kKSlots;
        mbar_wait(&k_empty[ks], ((t / kKSlots) & 1) ^ 1, abort_flag, p.err);
        if (*abort_flag) continue;
        if (lane == 0) {
          kmask[t & 7] = vm;
          mbar_arrive_expect_tx(&k_full[ks], __popc(vm) * 2 * kPageHalf);
        }
        __syncwarp();
        if (pb >= 0) {
          const int row = (pb * p.hkv + I.g) * 16;
          const uint32_t kd = sbase + kOffK + ks * kTileBytes + lane * kPageHalf;
          tma_load_2d(kd, &p.tm_k, 0, row, &k_full[ks]);
          tma_load_2d(kd + kRegion, &p.tm_k, 64, row, &k_full[ks]);
        }
      }
    }
    if (*abort_flag && lane == 0) {
      for (uint32_t u = t > kKSlots ? t - kKSlots : 0; u < t; ++u)
        mbar_wait(&k_full[u % kKSlots], (u / kKSlots) & 1, nullptr, p.err);
      for (uint32_t u = it > kQSlots ? it - kQSlots : 0; u < it; ++u)
        mbar_wait(&q_full[u % kQSlots], (u / kQSlots) & 1, nullptr, p.err);
    }
  } else if (warp == 10) {
    // =========================== V producer ===========================
    uint32_t t = 0;
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, false);
      if (!I.valid) continue;
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int pb = tile_page(p, I, j, lane, false);
        const unsigned vm = __ballot_sync(0xffffffffu, pb >= 0) & 0xffu;
        const int vs = t % kVSlots;
        mbar_wait(&v_empty[vs], ((t / kVSlots) & 1) ^ 1, abort_flag, p.err);
        if (*abort_flag) continue;
        if (lane == 0) mbar_arrive_expect_tx(&v_full[vs], __popc(vm) * 2 * kPageHalf);
        __syncwarp();
        if (pb >= 0) {
          const int row = (pb * p.hkv + I.g) * 16;
          const uint32_t vd = sbase + kOffV + vs * kTileBytes + lane * kPageHalf;
          tma_load_2d(vd, &p.tm_v, 0, row, &v_full[vs]);
          tma_load_2d(vd + kRegion, &p.tm_v, 64, row, &v_full[vs]);
        }
      }
    }
    if (*abort_flag && lane == 0)
      for (uint32_t u = t > kVSlots ? t - kVSlots : 0; u < t; ++u)
        mbar_wait(&v_full[u % kVSlots], (u / kVSlots) & 1, nullptr, p.err);
  } else if (warp == 1) {
    // ============================= MMA ==============================
    // One lane issues S of the next key tile and P.V of an earlier one, each as
    // soon as its inputs are ready (non-blocking polls, one shared limit on time
    // without progress).  Operand descriptors are computed once; an issue is
    // then a constant add.  The next item's indices are loaded while the
    // current one runs.
    if (lane == 0) {
      const uint64_t dq0 = smem_desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + kOffK, 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(sbase + kOffV, kRegion, 1024);
      uint32_t ts = 0, tpv = 0, it = 0, items_pv = 0;
      uint32_t first_bits = 0;  // bit t % 8: tile t is the first of its item
      PfItem I{};
      int j = 0;
      bool have = false, s_end = false;
      PfRaw nxt = pf_fetch(p, blockIdx.x < p.total ? blockIdx.x : 0);
      bool nxt_ok = blockIdx.x < p.total;
      long long last = clock64();
      while (!*abort_flag) {
        bool prog = false;
        if (tpv < ts) {
          const int sb = tpv % kSP, vs = tpv % kVSlots;
          const bool first = (first_bits >> (tpv & 7)) & 1u;
          if (mbar_test_wait(&v_full[vs], (tpv / kVSlots) & 1) &&
              mbar_test_wait(&p_full[sb], (tpv / kSP) & 1) &&
              (!first || mbar_test_wait(o_free, (items_pv & 1) ^ 1))) {
            if (first) ++items_pv;  // O of the previous item has been read out
            tc_fence_after();
            const uint64_t vb = desc_add(dv0, vs * kTileBytes);
            const uint32_t sp = tmem + sb * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t bd = desc_add(vb, k * 2048);
              umma_ts(tmem + kOcol, sp + 16 * k, bd, kIdescO, (first && k == 0) ? 0u : 1u);
              umma_ts(tmem + kOcol, sp + 16 * k + 8, bd, kIdescO, 1u);
            }
            umma_commit(&pv_done[sb]);
            umma_commit(&v_empty[vs]);
            ++tpv;
            prog = true;
          }
        }
        if (!have && !s_end) {
          // the next valid item: the prefetched one, else load in place
          while (nxt_ok) {
            I = pf_decode(p, nxt);
            const int vn = nxt.v + gridDim.x;
            nxt_ok = vn < p.total;
            if (I.valid) {
              if (nxt_ok) nxt = pf_fetch(p, vn);
              break;
            }
            if (nxt_ok) nxt = pf_fetch(p, vn);
          }
          if (I.valid) {
            have = true;
            j = 0;
          } else {
            s_end = true;
          }
          I.valid = false;  // consumed
          prog = true;
        }
        if (have) {
          const int sb = ts % kSP, ks = ts % kKSlots, qs = it % kQSlots;
          // S/P buffer sb is free once the P.V of tile ts - 3 is done
          if ((j > 0 || mbar_test_wait(&q_full[qs], (it / kQSlots) & 1)) &&
              mbar_test_wait(&k_full[ks], (ts / kKSlots) & 1) &&
              mbar_test_wait(&pv_done[sb], ((ts / kSP) & 1) ^ 1)) {
            tc_fence_after();
            const uint64_t qa = desc_add(dq0, qs * kTileBytes);
            const uint64_t kb = desc_add(dk0, ks * kTileBytes);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
              umma_ss(tmem + sb * 128, desc_add(qa, off), desc_add(kb, off), kIdescS,
                      k > 0 ? 1u : 0u);
            }
            umma_commit(&s_full[sb]);
            umma_commit(&k_empty[ks]);
            if (j == 0) first_bits |= 1u << (ts & 7);
            else first_bits &= ~(1u << (ts & 7));
            ++ts;
            if (++j == I.ntiles) {
              umma_commit(&q_empty[qs]);
              ++it;
              have = false;
            }
            prog = true;
          }
        }
        if (s_end && tpv == ts) break;
        if (prog) {
          last = clock64();
        } else if (clock64() - last > kWaitLimitCycles) {
          *abort_flag = 1;
          raise_error(p.err, PA_DEV_ERR_TIMEOUT);
        }
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err);
    }
    __syncwarp();
  } else {
    // ============================ softmax ============================
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;        // row of the tile, TMEM lane
    const int half = (warp - 2) >> 2;    // key columns / output dims 64*half .. +63
    const int cofs = half * 64;
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t ocol = tmem + lane_addr + kOcol + cofs;
    uint32_t t = 0, xk = 0;
    // the two warps that share this row quadrant have both passed this point
    auto exchange = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&xq[q4]);
      mbar_wait(&xq[q4], xk & 1, abort_flag, p.err);
      ++xk;
    };
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, false);
      if (!I.valid) continue;
      const int ti = r / p.group;  // token of this row within the tile
      const bool row_ok = r < rows_box && ti < I.ntok;
      const int limit = row_ok ? I.c + I.i0 + ti + 1 : 0;  // keys 0 .. limit-1
      float m = -CUDART_INF_F, l = 0.f;
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int sb = t % kSP;
        const int kv0 = j * 128;
        mbar_wait(&s_full[sb], (t / kSP) & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t vm = kmask[t & 7];
        float sv[64];
        tmem_ld64(tmem + lane_addr + sb * 128 + cofs, sv);
        // visibility of this half row's 64 keys as two 32-bit masks: keys below
        // the row's causal limit, in pages that were loaded
        uint32_t vis[2];
        {
          const int nvis = min(max(limit - kv0 - cofs, 0), 64);  // leading visible keys
          const uint32_t pages = (vm >> (cofs >> 4)) & 0xfu;     // this half's 4 pages
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int nw = min(max(nvis - 32 * w, 0), 32);
            const uint32_t lead = nw >= 32 ? 0xffffffffu : ((1u << nw) - 1u);
            const uint32_t pg = (((pages >> (2 * w)) & 1u) ? 0x0000ffffu : 0u) |
                                (((pages >> (2 * w + 1)) & 1u) ? 0xffff0000u : 0u);
            vis[w] = lead & pg;
          }
        }
        // Row maximum of the scaled scores.  Scaling is folded into the
        // exponent's FMA below, so the maximum is taken on the raw scores (the
        // largest for a positive scale, the smallest for a negative one).  A
        // warp whose rows see all 64 keys skips the per-key visibility test.
        const bool all_vis = __all_sync(0xffffffffu, (vis[0] & vis[1]) == 0xffffffffu);
        const float sc = p.scale_log2;
        float mx;
        if (sc >= 0.f) {
          float mx4[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
          if (all_vis) {
#pragma unroll
            for (int k = 0; k < 64; ++k) mx4[k & 3] = fmaxf(mx4[k & 3], sv[k]);
          } else {
#pragma unroll
            for (int k = 0; k < 64; ++k) {
              const bool on = (vis[k >> 5] >> (k & 31)) & 1u;
              mx4[k & 3] = fmaxf(mx4[k & 3], on ? sv[k] : -CUDART_INF_F);
            }
          }
          mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        } else {  // a negative scale turns the smallest raw score into the largest
          float mn4[4] = {CUDART_INF_F, CUDART_INF_F, CUDART_INF_F, CUDART_INF_F};
#pragma unroll
          for (int k = 0; k < 64; ++k) {
            const bool on = (vis[k >> 5] >> (k & 31)) & 1u;
            mn4[k & 3] = fminf(mn4[k & 3], on ? sv[k] : CUDART_INF_F);
          }
          mx = fminf(fminf(mn4[0], mn4[1]), fminf(mn4[2], mn4[3]));
          mx = mx == CUDART_INF_F ? -CUDART_INF_F : mx;
        }
        mx = mx == -CUDART_INF_F ? mx : mx * sc;  // scaled maximum
        float* px = xbuf + (xk & 1) * 256;
        px[half * 128 + r] = mx;
        exchange();
        mx = fmaxf(mx, px[(half ^ 1) * 128 + r]);
        // raise the row maximum only when it grows past 2^8; then rescale O and l
        const bool raise = mx > m + kRescaleLog2;
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
          const float f = raise ? exp2f(m - mx) : 1.f;
          mbar_wait(&pv_done[(t - 1) % kSP], ((t - 1) / kSP) & 1, abort_flag, p.err);
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float ov[16];
            tmem_ld16(ocol + c * 16, ov);
            uint32_t ow[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) ow[k] = __float_as_uint(ov[k] * f);
            tmem_st16_nowait(ocol + c * 16, ow);
          }
          tmem_wait_st();
          l *= f;
        }
        if (raise) m = mx;
        // Exponentials written back over the scores as P_hi / P_lo.  P_hi is
        // p with its mantissa cut to bf16, P_lo the same cut of the remainder
        // (p = P_hi + P_lo to within 2^-15 of p); both are formed with integer
        // masks and byte permutes, leaving the multi-function unit to ex2.
        const float negm = m == -CUDART_INF_F ? 0.f : -m;
        // pairs of keys go through the packed fp32x2 FMA/add instructions
        const float2 sc2 = make_float2(sc, sc), nm2 = make_float2(negm, negm);
        const float2 neg1 = make_float2(-1.f, -1.f);
        float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pw[16];
#pragma unroll
          for (int k = 0; k < 16; k += 2) {
            const int kk = c * 16 + k;
            const float2 x = __ffma2_rn(make_float2(sv[kk], sv[kk + 1]), sc2, nm2);
            float p0 = exp2f(x.x);
            float p1 = exp2f(x.y);
            if (!all_vis) {
              p0 = ((vis[kk >> 5] >> (kk & 31)) & 1u) ? p0 : 0.f;
              p1 = ((vis[kk >> 5] >> ((kk + 1) & 31)) & 1u) ? p1 : 0.f;
            }
            const float2 pp = make_float2(p0, p1);
            rs2[(k >> 1) & 1] = __fadd2_rn(rs2[(k >> 1) & 1], pp);
            const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
            const float2 hi =
                make_float2(__uint_as_float(b0 & 0xffff0000u), __uint_as_float(b1 & 0xffff0000u));
            const float2 lo = __ffma2_rn(hi, neg1, pp);  // p - P_hi, exact
            pw[k >> 1] = __byte_perm(b0, b1, 0x7632);
            pw[8 + (k >> 1)] = __byte_perm(__float_as_uint(lo.x), __float_as_uint(lo.y), 0x7632);
          }
          tmem_st16_nowait(tmem + lane_addr + sb * 128 + cofs + c * 16, pw);
        }
        const float rs = (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        tmem_wait_st();
        l += rs;
        // key rows past the context or in an unloaded page: zero this half of them in V
        if (kv0 + 128 > I.ctx || vm != 0xffu) {
          const int key = kv0 + r;
          if (key >= I.ctx || !((vm >> (r >> 4)) & 1u)) {
            const int vs = t % kVSlots;
            mbar_wait(&v_full[vs], (t / kVSlots) & 1, abort_flag, p.err);
            const uint32_t vrow = sbase + kOffV + vs * kTileBytes + half * kRegion + r * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) sts128_zero(vrow + k * 16);
            fence_proxy_async_smem();
          }
        }
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
      }
      // end of the item: O is final once the last P.V is done
      float ov[64];
      if (I.ntiles > 0) {
        mbar_wait(&pv_done[(t - 1) % kSP], ((t - 1) / kSP) & 1, abort_flag, p.err);
        tc_fence_after();
        tmem_ld64(ocol, ov);
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) ov[k] = 0.f;
      }
      tc_fence_before();
      mbar_arrive(o_free);
      // row sum over both halves
      float* px = xbuf + (xk & 1) * 256;
      px[half * 128 + r] = l;
      exchange();
      l += px[(half ^ 1) * 128 + r];
      if (row_ok) {
        const int h = r - ti * p.group;
        const int64_t orow = static_cast<int64_t>(I.q0 + I.i0 + ti) * p.hq + I.g * p.group + h;
        const bool live = l > 0.f;
        const float inv = live ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kD + cofs);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 w;
          w.x = pack_bf16x2(ov[8 * q] * inv, ov[8 * q + 1] * inv);
          w.y = pack_bf16x2(ov[8 * q + 2] * inv, ov[8 * q + 3] * inv);
          w.z = pack_bf16x2(ov[8 * q + 4] * inv, ov[8 * q + 5] * inv);
          w.w = pack_bf16x2(ov[8 * q + 6] * inv, ov[8 * q + 7] * inv);
          dst[q] = w;
        }
        if (half == 0 && p.lse) p.lse[orow] = live ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
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
