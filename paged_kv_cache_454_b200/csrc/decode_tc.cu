// Paged decode for grouped-query attention on the 5th-generation tensor cores.
//
// All G = Hq/Hkv query heads of one KV head read the same K/V pages, so for a
// tile of 128 context tokens the work is two small dense products:
//     S^T [128 tokens x 16] = K_tile [128 x D] . Q^T [D x 16]       (q heads padded to 16)
//     O^T [D x 16]          = V_tile^T [D x 128] . P [128 x 16]
// (for group sizes up to 8, columns 8-15 of P carry the bf16 remainder of p, so
// the weights reach the product with about 16 significant bits)
// each issued as 8 tcgen05.mma (M = 128, N = 16, K = 16) with fp32 accumulators
// in tensor memory.  Every K/V byte is read from HBM once for all G heads.
//
// Roles (one CTA per SM, persistent; items handed out dynamically in the
// plan's longest-first order):
//   warp 6      scheduler: takes the next work item with an atomic counter,
//               reads its block-table entries (4 tiles per fetch) and publishes
//               one descriptor per 128-token tile (sequence, KV head, token
//               range, physical block of each page) into an 8-slot ring.
//   warp 0      producer: for each tile descriptor, moves the 8 pages (16 tokens
//               x 64 dims per copy, 128-byte swizzle) with tiled tensor copies
//               into a 3-stage ring; q of the group rides along.
//   warp 1      allocates 64 TMEM columns; one lane issues the MMAs and commits
//               them to mbarriers (S of tile t before O of tile t-1, so the
//               tensor core computes scores while the softmax warps work).
//   warps 2-5   softmax: thread r owns token r of S^T and output dimension r of
//               O^T.  Online softmax in the log2 domain with one max exchange
//               per tile; p goes to shared memory as bf16 in the operand layout
//               of the second product; the tile's O^T is folded into registers
//               (acc = acc * alpha + O).  At the end of an item they hand the
//               normalised result and its log-sum-exp to the epilogue through a
//               shared-memory buffer and move on.
//   warps 7-10  epilogue: write the output, or the partition's partial result;
//               the last partition of a (sequence, KV head) to finish merges all
//               of them by log-sum-exp (one pass over the partitions).
// Tokens past the context (and pages with a bad block id) get p = 0 and their
// V rows are zeroed before the second product, so NaN padding is never read
// into a result.  Every wait is bounded and the softmax warps exchange data
// through mbarriers, never unbounded barriers: after a timeout the CTA stops
// issuing work, the scheduler ends the descriptor stream, every loop runs out
// without waiting, and the CTA drains its own copies and MMAs and frees its
// tensor memory.
#include <mutex>

#include <math_constants.h>

#include "internal.h"
#include "tc_common.cuh"

namespace pa {
namespace {

using namespace tc;

constexpr int kD = 128;       // head dim
constexpr int kN = 16;        // MMA N: q heads of one group, padded
constexpr int kTile = 128;    // tokens per tile (8 pages)
constexpr int kStages = 3;
constexpr int kDescSlots = 8;
constexpr int kRegion = kTile * 128;             // 128 rows x 128 B (one 64-dim half)
constexpr int kKBytes = 2 * kRegion;              // K tile, 32 KiB
constexpr int kQRegion = kN * 128;                // 16 rows x 128 B
constexpr int kStageBytes = 2 * kKBytes + 2 * kQRegion;  // K, V, Q: 69632
constexpr int kPBytes = 2 * kN * 128;             // P: 2 token halves x 16 rows x 128 B
constexpr int kOffP = kStages * kStageBytes;
constexpr int kOffDesc = kOffP + 2 * kPBytes;
constexpr int kOffRes = kOffDesc + kDescSlots * 64;  // item result handed to the epilogue
constexpr int kResBytes = kN * 128 * 4 + kN * 4 + 32;  // res[16][128], lse2[16], meta
constexpr int kOffBar = kOffRes + kResBytes;
// full, empty (x stages); s_full, s_free, p_full, o_full, o_free (x2);
// desc_full, desc_empty (x slots); drain; softmax exchange; res_full, res_empty;
// epilogue exchange
constexpr int kNumBars = 2 * kStages + 10 + 2 * kDescSlots + 2 + 3;
constexpr int kOffRed = kOffBar + kNumBars * 8;
constexpr int kRedFloats = 2 * 4 * kN + 2 * 4 * kN;  // tile max (x2), l sums (x2)
constexpr int kOffMisc = kOffRed + kRedFloats * 4;
constexpr int kSmemUsed = kOffMisc + 64;
constexpr int kSmemBytes = kSmemUsed + 1024;  // slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kTmemCols = 64;                 // S x2, O x2
constexpr int kThreads = 352;                 // 11 warps
constexpr uint32_t kQBytes = 2 * kQRegion;
constexpr uint32_t kPageBytes = 4 * 16 * 128;  // K and V halves of one page: 8 KiB

constexpr uint32_t kIdescS = idesc_bf16_f32(128, kN, false, false);
constexpr uint32_t kIdescO = idesc_bf16_f32(128, kN, true, false);

// Tile descriptor flags.
constexpr int kFirst = 1, kLast = 2, kEmpty = 4, kEnd = 8;

struct TileDesc {
  int s, g, part, npart;
  int pbase, tok0, tok1, flags;  // tok0: first token of the tile; tok1: end of the item
  int pb[8];                     // physical block of each page, -1 = skip
};
static_assert(sizeof(TileDesc) == 64, "descriptor slot size");

struct __align__(64) TcParams {
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int* header;
  const int* part_base;
  int* merge_cnt;
  const int2* items;
  float* part_o;
  float* part_lse;
  uint16_t* out;
  float* lse;
  unsigned int* err;
  int max_blocks;
  int num_blocks;
  int hkv;
  int hq;
  int group;
  float scale_log2;
};

// Swizzled byte offset of (row, 16-byte chunk) inside a 128-byte-row region.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int NH>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sptr = smem_raw + (sbase - raw);

  uint64_t* bars = reinterpret_cast<uint64_t*>(sptr + kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_free = o_full + 2;
  uint64_t* desc_full = o_free + 2;
  uint64_t* desc_empty = desc_full + kDescSlots;
  uint64_t* drain = desc_empty + kDescSlots;
  uint64_t* xbar = drain + 1;       // softmax warps' exchange barrier
  uint64_t* res_full = xbar + 1;    // softmax -> epilogue: an item result is ready
  uint64_t* res_empty = res_full + 1;
  uint64_t* ebar = res_empty + 1;   // epilogue warps' exchange barrier
  float* resbuf = reinterpret_cast<float*>(sptr + kOffRes);          // [kN][128]
  float* reslse = resbuf + kN * 128;                                  // [kN]
  int* resmeta = reinterpret_cast<int*>(reslse + kN);                 // s, g, part, npart, pbase
  TileDesc* descs = reinterpret_cast<TileDesc*>(sptr + kOffDesc);
  float* red = reinterpret_cast<float*>(sptr + kOffRed);
  float* red_max = red;               // [2][4][kN]
  float* red_l = red + 2 * 4 * kN;    // [2][4][kN]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + kOffMisc + 4);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(sptr + kOffMisc + 8);  // [2]
  (void)merge_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 128);
    }
    for (int i = 0; i < kDescSlots; ++i) {
      mbar_init(&desc_full[i], 1);
      mbar_init(&desc_empty[i], 6);  // producer, MMA, four softmax warps
    }
    mbar_init(drain, 1);
    mbar_init(xbar, 4);
    mbar_init(res_full, 4);
    mbar_init(res_empty, 4);
    mbar_init(ebar, 4);
    *abort_flag = 0;
    prefetch_tmap(&p.tm_k);
    prefetch_tmap(&p.tm_v);
    prefetch_tmap(&p.tm_q);
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp >= 2 && warp <= 5) {
    // P rows >= group stay zero for the whole kernel
    for (int i = tid - 64; i < 2 * kPBytes / 16; i += 128) sts128_zero(sbase + kOffP + i * 16);
    fence_proxy_async_smem();
  }
  fence_barrier_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 6) {
    // =========================== scheduler ===========================
    const int total = p.header[0];
    const int part = p.header[3];
    uint32_t d = 0;
    auto publish = [&](const TileDesc& td, int pbk) {
      const int slot = d % kDescSlots;
      mbar_wait(&desc_empty[slot], ((d / kDescSlots) & 1) ^ 1, abort_flag, p.err);
      TileDesc* o = descs + slot;
      if (lane < 8) o->pb[lane] = pbk;
      if (lane == 0) {
        o->s = td.s;
        o->g = td.g;
        o->part = td.part;
        o->npart = td.npart;
        o->pbase = td.pbase;
        o->tok0 = td.tok0;
        o->tok1 = td.tok1;
        o->flags = td.flags;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_full[slot]);
      ++d;
    };
    while (!*abort_flag) {
      int item = 0;
      if (lane == 0) item = atomicAdd(p.header + 2, 1);
      item = __shfl_sync(0xffffffffu, item, 0);
      if (item >= total) break;
      const int2 dd = p.items[item];
      TileDesc td;
      td.s = dd.x;
      td.g = dd.y >> 16;
      td.part = dd.y & 0xffff;
      int L = p.context_lens[td.s];
      const int cap = p.max_blocks * 16;
      L = L < 0 ? 0 : (L > cap ? cap : L);
      const int tok0 = td.part * part;
      td.tok1 = min(L, tok0 + part);
      td.pbase = p.part_base[td.s];
      td.npart = p.part_base[td.s + 1] - td.pbase;
      const int ntiles = td.tok1 > tok0 ? (td.tok1 - tok0 + kTile - 1) / kTile : 0;
      if (ntiles == 0) {
        td.tok0 = tok0;
        td.flags = kFirst | kLast | kEmpty;
        publish(td, -1);
        continue;
      }
      for (int j0 = 0; j0 < ntiles; j0 += 4) {
        // lane l reads page l % 8 of tile j0 + l / 8
        const int jt = j0 + (lane >> 3);
        const int ptok = tok0 + jt * kTile + (lane & 7) * 16;
        int pb = -1;
        if (jt < ntiles && ptok < td.tok1) {
          pb = p.block_tables[static_cast<int64_t>(td.s) * p.max_blocks + (ptok >> 4)];
          if (pb < 0 || pb >= p.num_blocks) {
            raise_error(p.err, PA_DEV_ERR_BLOCK_ID);
            pb = -1;
          }
        }
        for (int k = 0; k < 4 && j0 + k < ntiles; ++k) {
          const int pbk = __shfl_sync(0xffffffffu, pb, k * 8 + (lane & 7));
          td.tok0 = tok0 + (j0 + k) * kTile;
          td.flags = (j0 + k == 0 ? kFirst : 0) | (j0 + k == ntiles - 1 ? kLast : 0);
          publish(td, pbk);
        }
      }
    }
    // end of the stream (after a timeout: in every slot, without waiting)
    if (!*abort_flag) {
      TileDesc td{};
      td.flags = kEnd;
      publish(td, -1);
    } else if (lane == 0) {
      for (int i = 0; i < kDescSlots; ++i) descs[i].flags = kEnd;
    }
  } else if (warp == 0) {
    // =========================== producer ===========================
    uint32_t d = 0, t = 0;
    const uint64_t pol = l2_policy_evict_first();
    while (true) {
      const int slot = d % kDescSlots;
      mbar_wait(&desc_full[slot], (d / kDescSlots) & 1, abort_flag, p.err);
      const TileDesc* td = descs + slot;
      const int flags = td->flags;
      if (flags & kEnd) break;
      if (!(flags & kEmpty)) {
        const int pb = lane < 8 ? td->pb[lane] : -1;
        const int s = td->s, g = td->g;
        const unsigned vmask = __ballot_sync(0xffffffffu, pb >= 0);
        const int st = t % kStages;
        mbar_wait(&empty[st], ((t / kStages) & 1) ^ 1, abort_flag, p.err);
        if (!*abort_flag) {
          const uint32_t stage = sbase + st * kStageBytes;
          if (lane == 0) mbar_arrive_expect_tx(&full[st], kQBytes + __popc(vmask) * kPageBytes);
          __syncwarp();
          if (lane == 0) {
            const uint32_t q0 = stage + 2 * kKBytes;
            tma_load_3d(q0, &p.tm_q, 0, g * p.group, s, &full[st]);
            tma_load_3d(q0 + kQRegion, &p.tm_q, 64, g * p.group, s, &full[st]);
          }
          if (pb >= 0) {
            const int row = (pb * p.hkv + g) * 16;
            const uint32_t kdst = stage + lane * 2048;
            const uint32_t vdst = stage + kKBytes + lane * 2048;
            tma_load_2d_hint(kdst, &p.tm_k, 0, row, &full[st], pol);
            tma_load_2d_hint(kdst + kRegion, &p.tm_k, 64, row, &full[st], pol);
            tma_load_2d_hint(vdst, &p.tm_v, 0, row, &full[st], pol);
            tma_load_2d_hint(vdst + kRegion, &p.tm_v, 64, row, &full[st], pol);
          }
        }
        ++t;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_empty[slot]);
      ++d;
    }
    if (*abort_flag && lane == 0) {
      // wait (bounded) for this CTA's copies still in flight
      const uint32_t first = t > kStages ? t - kStages : 0;
      for (uint32_t u = first; u < t; ++u)
        mbar_wait(&full[u % kStages], (u / kStages) & 1, nullptr, p.err);
    }
  } else if (warp == 1) {
    // ============================= MMA ==============================
    if (lane == 0) {
      uint32_t d = 0, t = 0, prev = 0;
      bool have_prev = false;
      auto issue_pv = [&](uint32_t u) {
        const int st = u % kStages;
        const int b = u & 1;
        const uint32_t bph = (u >> 1) & 1;
        mbar_wait(&p_full[b], bph, abort_flag, p.err);
        mbar_wait(&o_free[b], bph ^ 1, abort_flag, p.err);
        if (*abort_flag) return;
        tc_fence_after();
        const uint32_t vbase = sbase + st * kStageBytes + kKBytes;
        const uint32_t pbase = sbase + kOffP + b * kPBytes;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          // A = V^T (MN-major): 16 tokens = 2 groups of 8 rows; D halves kRegion apart
          const uint64_t a = smem_desc_sw128(vbase + k * 2048, kRegion, 1024);
          // B = P (K-major, rows = heads): token half k/4, 32 bytes per 16 tokens
          const uint64_t bd =
              smem_desc_sw128(pbase + (k >> 2) * (kN * 128) + (k & 3) * 32, 16, 1024);
          umma_ss(tmem + 2 * kN + b * kN, a, bd, kIdescO, k > 0 ? 1u : 0u);
        }
        umma_commit(&o_full[b]);
        umma_commit(&empty[st]);
      };
      while (true) {
        const int slot = d % kDescSlots;
        mbar_wait(&desc_full[slot], (d / kDescSlots) & 1, abort_flag, p.err);
        const int flags = descs[slot].flags;
        if (flags & kEnd) break;
        mbar_arrive(&desc_empty[slot]);
        ++d;
        if (flags & kEmpty) continue;
        const int st = t % kStages;
        const int b = t & 1;
        mbar_wait(&full[st], (t / kStages) & 1, abort_flag, p.err);
        mbar_wait(&s_free[b], ((t >> 1) & 1) ^ 1, abort_flag, p.err);
        if (!*abort_flag) {
          tc_fence_after();
          const uint32_t kbase = sbase + st * kStageBytes;
          const uint32_t qbase = kbase + 2 * kKBytes;
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) {
            const uint32_t off = (k >> 2) * kRegion + (k & 3) * 32;
            const uint64_t a = smem_desc_sw128(kbase + off, 16, 1024);
            const uint64_t bq =
                smem_desc_sw128(qbase + (k >> 2) * kQRegion + (k & 3) * 32, 16, 1024);
            umma_ss(tmem + b * kN, a, bq, kIdescS, k > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[b]);
        }
        if (have_prev) issue_pv(prev);
        prev = t;
        have_prev = true;
        ++t;
      }
      if (have_prev) issue_pv(prev);
      // drain: every MMA issued above has completed before TMEM is freed
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.err);
    }
    __syncwarp();
  } else if (warp >= 7) {
    // =========================== epilogue ============================
    const int e = tid - 224;  // output dimension
    uint32_t k = 0, ek = 0;
    auto eexchange = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(ebar);
      mbar_wait(ebar, ek & 1, abort_flag, p.err);
      ++ek;
    };
    while (!*abort_flag) {
      mbar_wait(res_full, k & 1, abort_flag, p.err);
      const int npart = resmeta[3];
      if (npart < 0 || *abort_flag) break;
      const int s = resmeta[0], g = resmeta[1], part = resmeta[2], pbase = resmeta[4];
      float res[NH], l2[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        res[h] = h < p.group ? resbuf[h * 128 + e] : 0.f;
        l2[h] = reslse[h];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(res_empty);
      ++k;
      if (npart == 1) {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < p.group) {
            const int64_t o = static_cast<int64_t>(s) * p.hq + g * p.group + h;
            p.out[o * kD + e] = f32_to_bf16_bits(res[h]);
            if (e == 0 && p.lse) p.lse[o] = l2[h] * kLn2;
          }
        }
        continue;
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (h < p.group) {
          const int64_t rec = static_cast<int64_t>(pbase + part) * p.hq + g * p.group + h;
          __stcg(p.part_o + rec * kD + e, res[h]);
          if (e == 0) __stcg(p.part_lse + rec, l2[h]);
        }
      }
      // the last partition of (s, g) to finish merges all of them
      eexchange();
      if (e == 0) {
        __threadfence();
        const int old = atomicAdd(p.merge_cnt + s * p.hkv + g, 1);
        merge_flag[k & 1] = (old == npart - 1);
      }
      eexchange();
      if (!merge_flag[k & 1]) continue;
      __threadfence();
      float M[NH], W[NH], A[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        M[h] = -CUDART_INF_F;
        W[h] = 0.f;
        A[h] = 0.f;
      }
      const int64_t rec0 = static_cast<int64_t>(pbase) * p.hq + g * p.group;
      for (int q = 0; q < npart; ++q) {
        float li[NH], oi[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < p.group) {
            const int64_t rec = rec0 + static_cast<int64_t>(q) * p.hq + h;
            li[h] = __ldcg(p.part_lse + rec);
            oi[h] = __ldcg(p.part_o + rec * kD + e);
          }
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < p.group && li[h] != -CUDART_INF_F) {
            // one-pass log-sum-exp merge: rescale when a larger partition max appears
            if (li[h] > M[h]) {
              const float sc = exp2f(M[h] - li[h]);
              W[h] = W[h] * sc + 1.f;
              A[h] = A[h] * sc + oi[h];
              M[h] = li[h];
            } else {
              const float f = exp2f(li[h] - M[h]);
              W[h] += f;
              A[h] += f * oi[h];
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (h < p.group) {
          const bool live = W[h] > 0.f;
          const int64_t o = static_cast<int64_t>(s) * p.hq + g * p.group + h;
          p.out[o * kD + e] = f32_to_bf16_bits(live ? A[h] / W[h] : 0.f);
          if (e == 0 && p.lse) p.lse[o] = live ? (M[h] + log2f(W[h])) * kLn2 : -CUDART_INF_F;
        }
      }
    }
  } else {
    // ============================ softmax =============================
    const int q4 = warp & 3;          // TMEM lane quadrant of this warp
    const int r = q4 * 32 + lane;     // token row of S^T, output dim of O^T
    const int wi = warp - 2;          // index among the softmax warps
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    uint32_t d = 0, t = 0, xk = 0, nfin = 0;
    // all four softmax warps have passed this point (bounded, unlike bar.sync)
    auto exchange = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(xbar);
      mbar_wait(xbar, xk & 1, abort_flag, p.err);
      ++xk;
    };
    float m_run[NH], l_part[NH], acc[NH], alpha_prev[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      m_run[h] = -CUDART_INF_F;
      l_part[h] = 0.f;
      acc[h] = 0.f;
      alpha_prev[h] = 1.f;
    }
    auto fold = [&](uint32_t u) {
      const int b = u & 1;
      mbar_wait(&o_full[b], (u >> 1) & 1, abort_flag, p.err);
      tc_fence_after();
      float ov[16];
      tmem_ld16(tmem + lane_addr + 2 * kN + b * kN, ov);
      tc_fence_before();
      mbar_arrive(&o_free[b]);
#pragma unroll
      for (int h = 0; h < NH; ++h)
        acc[h] = acc[h] * alpha_prev[h] + ov[h] + (NH <= 8 ? ov[(h + 8) & 15] : 0.f);
    };
    while (true) {
      const int slot = d % kDescSlots;
      mbar_wait(&desc_full[slot], (d / kDescSlots) & 1, abort_flag, p.err);
      const TileDesc* td = descs + slot;
      const int flags = td->flags;
      if ((flags & kEnd) || *abort_flag) {
        // no more items: tell the epilogue warps
        mbar_wait(res_empty, (nfin & 1) ^ 1, abort_flag, p.err);
        if (r == 0) resmeta[3] = -1;
        __syncwarp();
        if (lane == 0) mbar_arrive(res_full);
        break;
      }
      const int s = td->s, g = td->g, part = td->part, npart = td->npart, pbase = td->pbase;
      const int tok0 = td->tok0, tok1 = td->tok1;
      const int mypb = td->pb[r >> 4];
      __syncwarp();
      if (lane == 0) mbar_arrive(&desc_empty[slot]);
      ++d;
      if (flags & kFirst) {
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          m_run[h] = -CUDART_INF_F;
          l_part[h] = 0.f;
          acc[h] = 0.f;
          alpha_prev[h] = 1.f;
        }
      }
      if (!(flags & kEmpty)) {
        const int st = t % kStages;
        const int b = t & 1;
        mbar_wait(&s_full[b], (t >> 1) & 1, abort_flag, p.err);
        tc_fence_after();
        float sv[16];
        tmem_ld16(tmem + lane_addr + b * kN, sv);
        tc_fence_before();
        mbar_arrive(&s_free[b]);
        const bool valid = tok0 + r < tok1 && mypb >= 0;
        float x[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) x[h] = valid ? sv[h] * p.scale_log2 : -CUDART_INF_F;
        // tile max per head: warp shuffle, then across the four softmax warps
        float* rm = red_max + (t & 1) * 4 * kN;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          float v = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rm[wi * kN + h] = v;
        }
        exchange();
        float pr[NH], alpha[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float tmax =
              fmaxf(fmaxf(rm[h], rm[kN + h]), fmaxf(rm[2 * kN + h], rm[3 * kN + h]));
          const float mn = fmaxf(m_run[h], tmax);
          alpha[h] = (mn == -CUDART_INF_F) ? 1.f : exp2f(m_run[h] - mn);
          pr[h] = (x[h] == -CUDART_INF_F) ? 0.f : exp2f(x[h] - mn);
          l_part[h] = l_part[h] * alpha[h] + pr[h];
          m_run[h] = mn;
        }
        // p into P[b]: row h (head), column r (token), K-major 128B swizzle.  For
        // group sizes up to 8, p is split into a bf16 high part (row h) and the
        // bf16 rounding of its remainder (row 8 + h), so the product carries p to
        // about 16 significant bits; larger groups use the high part only.
        const uint32_t pbuf = sbase + kOffP + b * kPBytes + (r >> 6) * (kN * 128);
        const int c = r & 63;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if (h < p.group) {
            const uint16_t hi = f32_to_bf16_bits(pr[h]);
            sts16(pbuf + swz(h, c >> 3) + (c & 7) * 2, hi);
            if (NH <= 8) {
              const float rem = pr[h] - __uint_as_float(static_cast<uint32_t>(hi) << 16);
              sts16(pbuf + swz(h + 8, c >> 3) + (c & 7) * 2, f32_to_bf16_bits(rem));
            }
          }
        }
        if (!valid) {
          // zero this token's V row (both 64-dim halves) so padding never reaches O
          const uint32_t vrow = sbase + st * kStageBytes + kKBytes + r * 128;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            sts128_zero(vrow + k * 16);
            sts128_zero(vrow + kRegion + k * 16);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&p_full[b]);
        if (!(flags & kFirst)) fold(t - 1);
#pragma unroll
        for (int h = 0; h < NH; ++h) alpha_prev[h] = alpha[h];
        ++t;
      }
      if (!(flags & kLast)) continue;
      if (!(flags & kEmpty)) fold(t - 1);

      // ---- finalize the item: l over the 128 token rows, then output dim r ----
      float* rl = red_l + (nfin & 1) * 4 * kN;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = l_part[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rl[wi * kN + h] = v;
      }
      exchange();
      float res[NH], lse2[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float l = rl[h] + rl[kN + h] + rl[2 * kN + h] + rl[3 * kN + h];
        const bool live = m_run[h] != -CUDART_INF_F && l > 0.f;
        res[h] = live ? acc[h] / l : 0.f;
        lse2[h] = live ? m_run[h] + log2f(l) : -CUDART_INF_F;
      }
      // hand the item's result to the epilogue warps
      mbar_wait(res_empty, (nfin & 1) ^ 1, abort_flag, p.err);
#pragma unroll
      for (int h = 0; h < NH; ++h)
        if (h < p.group) resbuf[h * 128 + r] = res[h];
      if (r == 0) {
#pragma unroll
        for (int h = 0; h < NH; ++h) reslse[h] = lse2[h];
        resmeta[0] = s;
        resmeta[1] = g;
        resmeta[2] = part;
        resmeta[3] = npart;
        resmeta[4] = pbase;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(res_full);
      ++nfin;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int NH>
int launch_nh(const TcParams& prm, int64_t item_bound, cudaStream_t stream) {
  auto kern = decode_tc_kernel<NH>;
  static KernelLaunchCache cache;
  const int per_sm = cache.blocks_per_sm(reinterpret_cast<const void*>(kern), kThreads, kSmemBytes);
  if (per_sm < 1) return PA_ERR_CUDA;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(item_bound < cap ? (item_bound < 1 ? 1 : item_bound) : cap);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(prm);
  return launch_status();
}

}  // namespace

bool decode_tcgen05_supported(int head_dim, int group) {
  return head_dim == kD && group >= 1 && group <= kN;
}

int launch_decode_tcgen05(const DecodeArgs& a) {
  const int group = a.num_q_heads / a.pool.num_kv_heads;
  if (!decode_tcgen05_supported(a.pool.head_dim, group)) return PA_ERR_UNSUPPORTED;
  const int64_t rows = static_cast<int64_t>(a.pool.num_blocks) * a.pool.num_kv_heads * 16;
  if (rows >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
  TcParams p;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(rows)};
    const uint64_t strides[1] = {kD * 2};
    const uint32_t box[2] = {64, 16};
    if (!encode_bf16_map(&p.tm_k, a.k_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
    if (!encode_bf16_map(&p.tm_v, a.v_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(a.num_q_heads),
                              static_cast<uint64_t>(a.num_seqs)};
    const uint64_t strides[2] = {kD * 2, static_cast<uint64_t>(a.q_stride) * 2};
    const uint32_t box[3] = {64, 16, 1};
    if (!encode_bf16_map(&p.tm_q, a.q, 3, dims, strides, box)) return PA_ERR_CUDA;
  }
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.header = a.ws.header;
  p.part_base = a.ws.part_base;
  p.merge_cnt = a.ws.merge_cnt;
  p.items = a.ws.items;
  p.part_o = a.ws.part_o;
  p.part_lse = a.ws.part_lse;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  p.max_blocks = a.max_blocks;
  p.num_blocks = a.pool.num_blocks;
  p.hkv = a.pool.num_kv_heads;
  p.hq = a.num_q_heads;
  p.group = group;
  p.scale_log2 = a.scale * kLog2e;
  const int64_t bound = static_cast<int64_t>(a.num_seqs) * a.max_parts * a.pool.num_kv_heads;
  if (group <= 4) return launch_nh<4>(p, bound, a.stream);
  if (group <= 8) return launch_nh<8>(p, bound, a.stream);
  return launch_nh<16>(p, bound, a.stream);
}

}  // namespace pa
