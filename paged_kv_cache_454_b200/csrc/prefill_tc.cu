// Chunked prefill on the 5th-generation tensor cores.
//
// A sequence adds a chunk of n new tokens on top of c cached ones; query i of
// the chunk (absolute position c + i) attends to keys 0 .. c + i.  For one KV
// head g, the G = Hq/Hkv query heads of the chunk form rows (token i, head h),
// ordered token-major, so one 128-row tile holds floor(128/G) tokens x G heads
// and shares every K/V tile among them.  Per 128-key tile of the paged context:
//     S [128 rows x 128 keys] = Q_tile [128 x D] . K_tile^T         (8 MMAs, K = 16)
//     O [128 rows x D]       += P [128 x 128 keys] . V_tile         (16 MMAs, K = 16)
// with fp32 accumulators in tensor memory.  P = P_hi + P_lo, p with its
// mantissa cut to bf16 and the same cut of what that left out, so the weights
// reach the product with about 16 significant bits where they need them: a
// key half of a tile whose weights are at most a quarter of the half row's
// sum so far (in every row of the tile) goes to the product as P_hi alone,
// since its share of the output bounds what the cut can change; the first
// tiles of a row, and every tile of a row of a few keys, take P_lo as well
// (bf16 p alone misses the output tolerance on contexts of a few keys).  P is
// written back into the tensor memory its scores came from (per 64-key half:
// 32 columns of P_hi, then 32 of P_lo) and the second product reads it there.
//
// Softmax: two warpgroups; warpgroup h owns key columns 64h .. 64h+63 of
// every key tile and thread r of it row r of those, so no warp exchanges
// anything with another inside an item.  Each half row keeps its own maximum
// m, row sum l and accumulator O_h (P.V of keys 0-63 goes to O_0, of keys
// 64-127 to O_1); at the end of an item the halves meet once in shared memory
// and the result is O = (2^(m_0 - M) O_0 + 2^(m_1 - M) O_1) / L with
// M = max(m_0, m_1) and L the matching sum of l_0, l_1.  The maximum is kept
// lazily: a half row with none yet takes its first visible tile's maximum;
// after that the weights exp2(s - m) are formed with the maximum in use, and
// only when they sum past 2^32 (or not to a finite number) is the tile's
// maximum computed and, if it exceeds m by more than 32 (log2 units), m is
// raised to it and the row of O_h, l and the tile's weights are rescaled.
// Weights up to 2^32 cannot overflow fp32 sums, and the final division by l,
// accumulated with the same m as O_h, makes the result exact either way.
//
// Tensor memory (512 columns): S/P of two key tiles (128 each) and O_0, O_1
// (128 each), so the scores of the next tile are computed while the softmax
// works on this one and the P.V of the previous one runs.
// Shared memory: q of one row tile, two K slots, three V slots (128-byte
// swizzle).  K is laid out half by half (each 64-dim half of the 128 key rows
// evenly spaced, as the first product needs), moved as two 2 KiB copies per
// page; V page by page, one 4 KiB copy per page (the second product takes a
// page per 16-key step).
//
// Roles (one CTA per SM, persistent over (sequence, KV head, row tile) items):
//   warp 0      producer of q and K: each item's row tile of q (one 3-D tensor
//               copy per 64-dim half: tokens x heads x dims), then each key
//               tile's 8 pages.
//   warp 1      allocates tensor memory; one lane issues S of the next key
//               tile and P.V of an earlier one, each as soon as its inputs are
//               ready.
//   warp 2      producer of V: each key tile's 8 pages.
//   warps 4-11  softmax: two warpgroups, one per 64-key half of a tile.
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
constexpr int kQSlots = 1, kKSlots = 2, kVSlots = 3, kSP = 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQSlots * kTileBytes;
constexpr int kOffV = kOffK + kKSlots * kTileBytes;
constexpr int kOffBar = kOffV + kVSlots * kTileBytes;
// q_full/empty, k_full/empty, v_full/empty (per slot); s_full, p_full, pv_done
// (per S/P buffer); o_free; drain; the halves' exchange at the end of an item
constexpr int kNumBars = 2 * (kQSlots + kKSlots + kVSlots) + 3 * kSP + 1 + 1 + 1;
constexpr int kMaskRing = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem slot, abort flag, kmask ring, lo flags
constexpr int kOffLo = kOffMisc + 16 + 4 * kMaskRing;  // [S/P buffer][key half] tile number
constexpr int kOffX = kOffLo + 8 * kSP;  // [2 items][2 halves][128 rows] (m, l)
constexpr int kSmemUsed = kOffX + 2 * 2 * 128 * 8;
constexpr int kSmemBytes = kSmemUsed + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kThreads = 384;   // q/K producer, MMA, V producer, (idle), 2 softmax warpgroups
constexpr int kTmemCols = 512;  // S/P x2 (128 each), O of each key half (128 each)
constexpr int kOcol = kSP * 128;  // O_0 at kOcol, O_1 at kOcol + 128
constexpr uint32_t kPageHalf = 16 * 128;  // one 64-dim half of one page: 2 KiB
constexpr float kRescaleLog2 = 32.f;      // raise the row maximum only past 2^32
constexpr float kRaiseSum = 4294967296.f;  // 2^32: weights summing to less need no raise
// A half row's weights of a key tile go to the second product as P_hi alone
// when they sum to at most a quarter of the half row's sum so far (their sum
// is then at most 1/3 of the sum before the tile).
constexpr float kLoSkipRatio = 3.f;

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
  int lo_always;  // every key tile's P.V takes P_lo as well
  float scale_log2;
};

struct PfItem {
  bool valid;
  int s, g, q0, i0, ntok, c, ctx, kv_end, ntiles;
};

// AND of `pred` over the 128 threads of a warpgroup (named barrier `id`).
__device__ __forceinline__ bool warpgroup_all(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q, a;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred a, %2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, a;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint2 lds_volatile_u32x2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.volatile.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ int ld_early(const int32_t* ptr) {
  int x;
  asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(x) : "l"(ptr));
  return x;
}

// Virtual item v -> (sequence, KV head, row tile), row tile fastest: the row
// tiles of one (sequence, KV head) are consecutive items, so the persistent
// CTAs work on them at the same time and stream the same K/V pages -- read
// from HBM once, from L2 for the rest (in another order each row tile's pass
// over the pages comes long after the previous one, and a batch's pages
// outgrow L2).  Row tiles are counted from the end of the sequence's chunk
// (k = 0: its last row tile, the longest causal range).  The three loads are
// issued early (pf_fetch) and decoded later (pf_decode), so a thread that must
// not stall can overlap them with other work.
struct PfRaw {
  int v, q0, q1, L;
};

__device__ __forceinline__ PfRaw pf_fetch(const PfParams& p, int v) {
  PfRaw r;
  r.v = v;
  const int s = v / (p.mt_max * p.hkv);
  r.q0 = ld_early(p.cu_q + s);
  r.q1 = ld_early(p.cu_q + s + 1);
  r.L = ld_early(p.context_lens + s);
  return r;
}

__device__ __forceinline__ PfItem pf_decode(const PfParams& p, const PfRaw& r, bool flag_errors) {
  PfItem it;
  const int k = r.v % p.mt_max;
  const int q = r.v / p.mt_max;
  it.g = q % p.hkv;
  it.s = q / p.hkv;
  it.q0 = r.q0;
  const int n = r.q1 - r.q0;
  const int mt = (n + p.tpt - 1) / p.tpt;  // row tiles of this chunk
  const int ti = mt - 1 - k;
  it.valid = n > 0 && ti >= 0;
  it.ntiles = 0;
  if (!it.valid) return it;
  int L = r.L;
  const int cap = p.max_blocks * 16;
  if (L < n || L > cap) {
    if (flag_errors) raise_error(p.err, PA_DEV_ERR_CONTEXT);
    L = L > cap ? cap : L;
    if (L < n) {  // a chunk longer than its context: nothing consistent to compute
      it.valid = false;
      return it;
    }
  }
  it.i0 = ti * p.tpt;
  it.ntok = min(p.tpt, n - it.i0);
  it.ctx = L;
  it.c = L - n;
  it.kv_end = min(L, it.c + it.i0 + it.ntok);
  it.ntiles = (it.kv_end + 127) / 128;
  return it;
}

__device__ __forceinline__ PfItem pf_item(const PfParams& p, int v, bool flag_errors) {
  return pf_decode(p, pf_fetch(p, v), flag_errors);
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
  uint64_t* xchg = drain + 1;             // both key halves' (m, l) of an item written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + kOffMisc + 4);
  // loaded pages of key tile t, in slot t % kMaskRing (written by the K
  // producer before the tile's copies; the softmax reads it after the tile's
  // scores, long before the producer can come round to the slot again)
  uint32_t* kmask = reinterpret_cast<uint32_t*>(sptr + kOffMisc + 16);
  // lo_seq[2 b + h] = t + 1 when key half h of key tile t (in S/P buffer
  // b = t % kSP) has P_lo written; then the MMA issues that half's P_lo
  // products.  The first warp of each softmax warpgroup writes it, before its
  // arrival on p_full; the MMA reads both halves' words in one load.
  static_assert(kOffLo % 8 == 0, "lo_seq pairs are read as 8 bytes");
  volatile uint32_t* lo_seq = reinterpret_cast<volatile uint32_t*>(sptr + kOffLo);
  float2* xbuf = reinterpret_cast<float2*>(sptr + kOffX);

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
      mbar_init(&p_full[i], 8);  // one arrival per softmax warp
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(o_free, 8);
    mbar_init(drain, 1);
    mbar_init(xchg, 8);
    *abort_flag = 0;
    for (int i = 0; i < kSP * 2; ++i) lo_seq[i] = 0;
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
          kmask[t % kMaskRing] = vm;
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
    // this CTA has issued its last item: a programmatic dependent launched
    // after this kernel (the decode plan) may start on the SMs that free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (*abort_flag && lane == 0) {
      for (uint32_t u = t > kKSlots ? t - kKSlots : 0; u < t; ++u)
        mbar_wait(&k_full[u % kKSlots], (u / kKSlots) & 1, nullptr, p.err);
      for (uint32_t u = it > kQSlots ? it - kQSlots : 0; u < it; ++u)
        mbar_wait(&q_full[u % kQSlots], (u / kQSlots) & 1, nullptr, p.err);
    }
  } else if (warp == 2) {
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
          // one 3-D copy of the page: both 64-dim halves, next to each other
          const uint32_t vd = sbase + kOffV + vs * kTileBytes + lane * (2 * kPageHalf);
          tma_load_3d(vd, &p.tm_v, 0, row, 0, &v_full[vs]);
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
    // without progress).  S of tile t may run ahead of the softmax by a tile
    // (two S/P buffers).  Operand descriptors are computed once; an
    // issue is then a constant add.  The next item's indices are loaded while
    // the current one runs.
    if (lane == 0) {
      const uint64_t dq0 = smem_desc_sw128(sbase + kOffQ, 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(sbase + kOffK, 16, 1024);
      // V page by page: [page][64-dim half][16 rows][128 B]; the second
      // product's 16-key step is one page, its two halves 2 KiB apart
      const uint64_t dv0 = smem_desc_sw128(sbase + kOffV, 2 * 1024, 1024);
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
            // the halves' P_lo flags, read while the P_hi products issue
            const uint2 lf = lds_volatile_u32x2(sbase + kOffLo + sb * 8);
            // keys 0-63 of the tile into O_0, keys 64-127 into O_1; a half's
            // 64 columns of P are 32 of P_hi, then 32 of P_lo
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t oc = tmem + kOcol + (k >> 2) * 128;
              umma_ts(oc, sp + 64 * (k >> 2) + 8 * (k & 3), desc_add(vb, k * 4096), kIdescO,
                      (first && (k & 3) == 0) ? 0u : 1u);
            }
            const bool lo0 = lf.x == tpv + 1, lo1 = lf.y == tpv + 1;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if ((k >> 2) ? lo1 : lo0)
                umma_ts(tmem + kOcol + (k >> 2) * 128, sp + 64 * (k >> 2) + 32 + 8 * (k & 3),
                        desc_add(vb, k * 4096), kIdescO, 1u);
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
            I = pf_decode(p, nxt, false);
            const int vn = nxt.v + gridDim.x;
            nxt_ok = vn < p.total;
            if (nxt_ok) nxt = pf_fetch(p, vn);
            if (I.valid) break;
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
          // S/P buffer sb is free once the P.V of tile ts - 2 is done
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
  } else if (warp >= 4) {
    // ============================ softmax ============================
    // Warpgroup h (0: warps 4-7, 1: warps 8-11) owns key columns 64h .. 64h+63
    // of every tile; thread r of it owns row r of those.  Each half keeps its
    // own maximum, row sum and accumulator O_h, so the halves never wait for
    // each other inside an item; at its end they merge by log-sum-exp.
    const int hf = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // row of the tile, TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t ocol = tmem + lane_addr + kOcol + hf * 128;  // this half's O_h row
    const float sc = p.scale_log2;
    const float2 sc2 = make_float2(sc, sc);
    const float2 neg1 = make_float2(-1.f, -1.f);
    uint32_t t = 0, nit = 0;
    for (int v = blockIdx.x; v < p.total; v += gridDim.x) {
      const PfItem I = pf_item(p, v, false);
      if (!I.valid) continue;
      const int ti = r / p.group;  // token of this row within the tile
      const bool row_ok = r < rows_box && ti < I.ntok;
      const int limit = row_ok ? I.c + I.i0 + ti + 1 : 0;  // keys 0 .. limit-1
      float m = -CUDART_INF_F, l = 0.f;
      for (int j = 0; j < I.ntiles; ++j, ++t) {
        const int sb = t % kSP;
        const int kv0 = j * 128 + 64 * hf;  // first key of this half
        const uint32_t scol = tmem + lane_addr + sb * 128 + 64 * hf;
        mbar_wait(&s_full[sb], (t / kSP) & 1, abort_flag, p.err);
        tc_fence_after();
        const uint32_t vm = (kmask[t % kMaskRing] >> (4 * hf)) & 0xfu;  // this half's pages
        // Visibility of the half row's keys: below the row's causal limit, in
        // pages that were loaded.  A row outside the tile's tokens sees
        // everything: its weights are never read out, and treating it as fully
        // visible keeps its warp on the unmasked path.
        const int nvis = min(max(limit - kv0, 0), 64);  // leading visible keys
        const bool all_vis = __all_sync(0xffffffffu, !row_ok || (nvis == 64 && vm == 0xfu));
        // The half row of scores in registers (one wait), scaled with the
        // maximum in use; keys that are not visible become -inf (p = 0),
        // whatever their score.
        float xv[64];
        auto load_x = [&]() {
          uint32_t sa[32], sb2[32];
          tmem_ld32_nowait(scol, sa);
          tmem_ld32_nowait(scol + 32, sb2);
          tmem_wait_ld_regs(sa);
          tmem_wait_ld_regs(sb2);
          const float negm = m == -CUDART_INF_F ? 0.f : -m;
          const float2 nm2 = make_float2(negm, negm);
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 xa = __ffma2_rn(
                make_float2(__uint_as_float(sa[k]), __uint_as_float(sa[k + 1])), sc2, nm2);
            const float2 xb = __ffma2_rn(
                make_float2(__uint_as_float(sb2[k]), __uint_as_float(sb2[k + 1])), sc2, nm2);
            xv[k] = xa.x;
            xv[k + 1] = xa.y;
            xv[32 + k] = xb.x;
            xv[32 + k + 1] = xb.y;
          }
          if (!all_vis) {
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const int nw = min(max(nvis - 32 * w, 0), 32);
              const uint32_t lead = nw >= 32 ? 0xffffffffu : ((1u << nw) - 1u);
              const uint32_t pg = (((vm >> (2 * w)) & 1u) ? 0x0000ffffu : 0u) |
                                  (((vm >> (2 * w + 1)) & 1u) ? 0xffff0000u : 0u);
              const uint32_t vw = row_ok ? (lead & pg) : 0xffffffffu;
#pragma unroll
              for (int k = 0; k < 32; ++k)
                xv[32 * w + k] = ((vw >> k) & 1u) ? xv[32 * w + k] : -CUDART_INF_F;
            }
          }
        };
        load_x();
        // Weights of the half row with the maximum in use, in place of the
        // scores, and P_hi (p with its mantissa cut to bf16, two keys a
        // column) in hw, formed with byte permutes between the multi-function
        // unit's ex2; returns the sum of the weights.
        uint32_t hw[32];
        auto exp_pass = [&]() -> float {
          float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int k = 0; k < 64; k += 2) {
            const float p0 = exp2f(xv[k]);
            const float p1 = exp2f(xv[k + 1]);
            xv[k] = p0;
            xv[k + 1] = p1;
            rs2[(k >> 1) & 1] = __fadd2_rn(rs2[(k >> 1) & 1], make_float2(p0, p1));
            hw[k >> 1] = __byte_perm(__float_as_uint(p0), __float_as_uint(p1), 0x7632);
          }
          return (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        };
        // P_lo, the same cut of p - P_hi (so P_hi + P_lo is p to within 2^-15
        // of p), in the next 32 columns, formed with integer masks and byte
        // permutes.
        auto store_lo = [&]() {
          uint32_t lw[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const float2 pp = make_float2(xv[2 * k], xv[2 * k + 1]);
            const float2 hi = make_float2(__uint_as_float(__float_as_uint(pp.x) & 0xffff0000u),
                                          __uint_as_float(__float_as_uint(pp.y) & 0xffff0000u));
            const float2 lo = __ffma2_rn(hi, neg1, pp);  // p - P_hi, exact
            lw[k] = __byte_perm(__float_as_uint(lo.x), __float_as_uint(lo.y), 0x7632);
          }
          tmem_st32_nowait(scol + 32, lw);
        };
        // Raise the maximum in use to the tile's maximum xm (scaled, relative
        // to the old one); then this half's row of O_h (earlier key tiles of
        // this item) and l are rescaled.  The P.V of the previous tile may
        // still be running, so that waits for it first.
        auto raise_to = [&](bool raise, float xm) {
          float f = 1.f;
          if (raise) {
            f = m == -CUDART_INF_F ? 0.f : exp2f(-xm);
            m = m == -CUDART_INF_F ? xm : m + xm;
            const float2 d2 = make_float2(-xm, -xm);
#pragma unroll
            for (int k = 0; k < 64; k += 2) {
              const float2 xx = __fadd2_rn(make_float2(xv[k], xv[k + 1]), d2);
              xv[k] = xx.x;
              xv[k + 1] = xx.y;
            }
          }
          l *= f;
          if (j > 0) {
            mbar_wait(&pv_done[(t - 1) % kSP], ((t - 1) / kSP) & 1, abort_flag, p.err);
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
              float ov[16];
              tmem_ld16(ocol + cc * 16, ov);
              uint32_t ow[16];
#pragma unroll
              for (int k = 0; k < 16; ++k) ow[k] = __float_as_uint(ov[k] * f);
              tmem_st16(ocol + cc * 16, ow);
            }
          }
        };
        auto row_max = [&]() -> float {
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = xv[k];
#pragma unroll
          for (int k = 8; k < 64; ++k) m8[k & 7] = fmaxf(m8[k & 7], xv[k]);
          return fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        };
        // A half row without a maximum yet (its first visible keys) takes the
        // tile's maximum first.  Every other one goes straight to the weights:
        // a sum of at most 2^32 means no weight exceeds 2^32, so the maximum
        // in use stands (no maximum is computed in the common case); a larger
        // (or non-finite) sum raises it to the tile's maximum and the weights
        // are computed again.
        if (__any_sync(0xffffffffu, m == -CUDART_INF_F)) {
          const float xm = row_max();
          const bool raise = m == -CUDART_INF_F ? xm != -CUDART_INF_F : xm > kRescaleLog2;
          if (__any_sync(0xffffffffu, raise)) raise_to(raise, xm);
        }
        float rs = exp_pass();
        {
          const bool check = row_ok && !(rs <= kRaiseSum);
          if (__any_sync(0xffffffffu, check)) {
            // the weights took the scores' registers: reload the scores
            // (still in tensor memory) for the tile's maximum
            load_x();
            const float xm = row_max();
            const bool raise = check && xm > kRescaleLog2;
            if (__any_sync(0xffffffffu, raise)) raise_to(raise, xm);
            rs = exp_pass();
          }
        }
        // P_lo is left out for this key half of the tile when, in every row
        // of the warpgroup, the tile's weights are at most a quarter of the
        // half row's sum with them: each such weight is then at most 1/4 of
        // its final value's denominator, and the cut's relative error (below
        // 2^-7) reaches the output scaled by that share.
        tmem_st32_nowait(scol, hw);  // P_hi over the scores' first 32 columns
        const bool with_lo =
            !warpgroup_all(1 + hf, !p.lo_always && (!row_ok || kLoSkipRatio * rs <= l));
        if (with_lo) store_lo();
        tmem_wait_st();
        l += rs;
        if (with_lo && q4 == 0 && lane == 0) lo_seq[sb * 2 + hf] = t + 1;
        // key rows of this half past the context or in an unloaded page: zero
        // them in V (threads 0-63 of the warpgroup, one key row each)
        if (j * 128 + 128 > I.ctx || vm != 0xfu) {
          const int key = kv0 + r;
          if (r < 64 && (key >= I.ctx || !((vm >> (r >> 4)) & 1u))) {
            const int vs = t % kVSlots;
            mbar_wait(&v_full[vs], (t / kVSlots) & 1, abort_flag, p.err);
            const int kr = 64 * hf + r;  // key row of the tile: page kr / 16, row kr % 16
            const uint32_t vrow =
                sbase + kOffV + vs * kTileBytes + (kr >> 4) * 4096 + (kr & 15) * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              sts128_zero(vrow + k * 16);
              sts128_zero(vrow + 2048 + k * 16);
            }
            fence_proxy_async_smem();
          }
        }
        // every lane's stores are done (waited and fenced) before its warp's arrival
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      // End of the item: the halves' (m, l) meet in shared memory; O = s_0 O_0 +
      // s_1 O_1 with s_h = 2^(m_h - M) / L, M = max(m_0, m_1) and
      // L = l_0 2^(m_0 - M) + l_1 2^(m_1 - M).  Half h writes output dims
      // 64h .. 64h+63 from both accumulators, once the last P.V is done.
      float2* xb = xbuf + (nit & 1) * 256;
      xb[hf * 128 + r] = make_float2(m, l);
      __syncwarp();
      if (lane == 0) mbar_arrive(xchg);
      mbar_wait(xchg, nit & 1, abort_flag, p.err);
      const float2 other = xb[(hf ^ 1) * 128 + r];
      ++nit;
      const float m0 = hf == 0 ? m : other.x, l0 = hf == 0 ? l : other.y;
      const float m1 = hf == 0 ? other.x : m, l1 = hf == 0 ? other.y : l;
      const float M = fmaxf(m0, m1);
      const float e0 = M == -CUDART_INF_F ? 0.f : exp2f(m0 - M);
      const float e1 = M == -CUDART_INF_F ? 0.f : exp2f(m1 - M);
      const float L = l0 * e0 + l1 * e1;
      const bool live = L > 0.f;
      const float inv = live ? 1.f / L : 0.f;
      const float s0 = e0 * inv, s1 = e1 * inv;
      if (I.ntiles > 0) {
        mbar_wait(&pv_done[(t - 1) % kSP], ((t - 1) / kSP) & 1, abort_flag, p.err);
        tc_fence_after();
      }
      const int h = r - ti * p.group;
      const int64_t orow = static_cast<int64_t>(I.q0 + I.i0 + ti) * p.hq + I.g * p.group + h;
      uint4* dst = reinterpret_cast<uint4*>(p.out + orow * kD + 64 * hf);
      const uint32_t o0 = tmem + lane_addr + kOcol + 64 * hf;  // dims 64h.. of O_0
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float a0[32], a1[32];
        tmem_ld32(o0 + 32 * c, a0);
        tmem_ld32(o0 + 128 + 32 * c, a1);
        if (c == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] = a0[8 * q + k] * s0 + a1[8 * q + k] * s1;
            uint4 w;
            w.x = pack_bf16x2(o[0], o[1]);
            w.y = pack_bf16x2(o[2], o[3]);
            w.z = pack_bf16x2(o[4], o[5]);
            w.w = pack_bf16x2(o[6], o[7]);
            dst[4 * c + q] = w;
          }
        }
      }
      if (hf == 0 && row_ok && p.lse) p.lse[orow] = live ? (M + log2f(L)) * kLn2 : -CUDART_INF_F;
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
  }
  {
    // V: (dim within a 64-dim half, pool row, half) -- one copy moves a page's
    // 16 rows for both halves, half 0 first
    const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), 2};
    const uint64_t strides[2] = {kD * 2, 128};
    const uint32_t box[3] = {64, 16, 2};
    if (!encode_bf16_map(&p.tm_v, a.v_pool, 3, dims, strides, box)) return PA_ERR_CUDA;
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
  p.lo_always = a.exact_weights ? 1 : 0;
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
