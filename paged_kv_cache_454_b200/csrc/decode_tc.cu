// Paged decode on the 5th-generation tensor cores.
//
// All G = Hq/Hkv query heads of one KV head read the same K/V pages.  A tile
// is 128 rows of the pool: HT KV heads x 16 tokens of each of 8/HT pages (the
// HT heads of one page are adjacent in the pool, so a page of K moves as one
// HT*2 KiB tensor copy per 64-dim half).  HT = 1 for large groups; for small
// groups (MHA above all) several KV heads share a tile, which keeps the copies
// large -- the copy engine moves 2 KiB boxes at well under the HBM rate -- and
// fills the product's N dimension with useful columns.  A page of V (HT < 8)
// moves as one 3-D copy of both halves, which land next to each other: the
// second product takes its K = 16 slices page by page, so per-page halves
// suit it, while the first product's M = 128 rows span all pages of the tile
// and need each half's rows evenly spaced, so K keeps one copy per half.
// With NH q columns per tile (the group's q heads of the tile's KV heads,
// padded) the work is two small dense products:
//     S^T [128 rows x 16] = K_tile [128 x D] . Q^T [D x 16]
//     O^T [D x 2NH]       = V_tile^T [D x 128] . P [128 x 2NH]
// where row r of the tile only scores against its own KV head's q columns
// (the others get p = 0), and columns NH.. of P carry the bf16 remainder of p,
// so the weights reach the product with about 16 significant bits.  Each is
// issued as 8 tcgen05.mma (M = 128, K = 16) with fp32 accumulators in tensor
// memory.  Every K/V byte is read from HBM once for all of its q heads.
//
// Roles (one CTA per SM, persistent; items handed out dynamically in the
// plan's order):
//   warp 6      scheduler: takes the next work item (sequence, KV-head group,
//               partition) with an atomic counter, reads its block-table entries
//               (32 pages per fetch) and publishes one descriptor per tile
//               (sequence, head group, token range, physical block of each
//               page) into an 8-slot ring.
//   warp 0      producer: q of an item into one of two q slots, then for each
//               tile descriptor the K and V pages (128-byte swizzle) with tiled
//               tensor copies into a 3-stage ring.
//   warp 1      allocates the tensor memory; one lane issues the MMAs and
//               commits them to mbarriers (S of tile t before O of tile t-1, so
//               the tensor core computes scores while the softmax warps work).
//   warps 2-5   softmax: thread r owns row r of S^T and output dimension r of
//               O^T.  Online softmax in the log2 domain with one max exchange
//               per tile; p goes to shared memory as bf16 in the operand layout
//               of the second product; the tile's O^T is folded into registers
//               (acc = acc * alpha + O).  At the end of an item they hand the
//               normalised result and its log-sum-exp to the epilogue through a
//               shared-memory buffer and move on.
//   warps 7-10  epilogue: write the output, or the partition's partial result;
//               the last partition of a (sequence, KV head) to finish merges
//               all of them by log-sum-exp (one pass over the partitions).
// Shared prefixes (cascade; groups up to 4): sequences whose tables start
// with the same blocks (parallel samples of one prompt, "vLLM 基本原理",
// PagedAttention / 内存共享) are grouped by the plan into sub-runs of up to M
// sharers, and the span their tables have in common becomes shared-prefix
// items, which the scheduler hands out before the sequences' own items (those
// then cover only each sequence's tokens after its span).  A shared-prefix
// tile is read once and scored against the q heads of every sharer: the q
// columns are ordered (KV head of the item, sharer, q head of the group), so a
// row's columns -- those of its KV head -- are M * G contiguous ones, exactly
// as for a group of M * G q heads, and the same softmax serves both kinds.
// The two kinds pack different numbers of KV heads per tile (the plan picks
// the shared-prefix one), so each role keeps both tile geometries and takes
// the one a tile's descriptor names.  Each sharer gets its own partial result
// for a shared-prefix partition; all partitions of a (sequence, KV head) are
// merged by whichever finishes last.
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
constexpr int kN = 16;        // N of the score product: q rows of one tile, padded
constexpr int kRows = 128;    // pool rows per tile
constexpr int kStages = 3;
constexpr int kDescSlots = 8;
constexpr int kRegion = kRows * 128;              // 128 rows x 128 B (one 64-dim half)
constexpr int kKBytes = 2 * kRegion;              // K tile, 32 KiB
constexpr int kStageBytes = 2 * kKBytes;          // K, V: 65536
constexpr int kQRegion = kN * 128;                // 16 rows x 128 B
constexpr uint32_t kQBytes = 2 * kQRegion;        // one q slot
constexpr int kQSlots = 2;

// Shared-memory plan for NH q columns per tile.
template <int NH>
struct Smem {
  static constexpr int kNpv = 2 * NH;                       // N of the second product
  static constexpr int kPBytes = 2 * kNpv * 128;            // 2 token halves x kNpv rows x 128 B
  static constexpr int kOffQ = kStages * kStageBytes;
  static constexpr int kOffP = kOffQ + kQSlots * kQBytes;
  static constexpr int kOffDesc = kOffP + 2 * kPBytes;
  static constexpr int kOffRes = kOffDesc + kDescSlots * 64;
  static constexpr int kResBytes = NH * 128 * 4 + NH * 4 + 32;  // res[NH][128], lse2[NH], meta
  static constexpr int kOffBar = kOffRes + kResBytes;
  // full, empty (x stages); s_full, s_free, p_full, o_full, o_free, q_full,
  // q_empty (x2); desc_full, desc_empty (x slots); drain; softmax exchange;
  // res_full, res_empty; epilogue exchange
  static constexpr int kNumBars = 2 * kStages + 14 + 2 * kDescSlots + 2 + 3;
  static constexpr int kOffRed = kOffBar + kNumBars * 8;
  // tile max (x2), l sums (x2)
  static constexpr int kRedFloats = 2 * 4 * NH + 2 * 4 * NH;
  static constexpr int kOffMisc = kOffRed + kRedFloats * 4;
  static constexpr int kUsed = kOffMisc + 64;
  static constexpr int kBytes = kUsed + 1024;  // slack to align the base to 1024
  static constexpr int kTmemCols = NH <= 8 ? 64 : 128;  // S x2 (16 columns each), O x2
  static_assert(kBytes <= 232448, "shared memory per CTA");
  static_assert(2 * kN + 2 * kNpv <= kTmemCols, "tensor memory columns");
};
constexpr int kThreads = 352;  // 11 warps

constexpr uint32_t kIdescS = idesc_bf16_f32(128, kN, false, false);

// Tile descriptor flags (kPre: a tile of a shared-prefix item).
constexpr int kFirst = 1, kLast = 2, kEmpty = 4, kEnd = 8, kPre = 16;

struct TileDesc {
  int s, g, part, npart;         // g: KV-head group of the item
  int pbase, tok0, tok1, flags;  // tok0: first token of the tile; tok1: end of the item
  int pb[8];                     // physical block of each page of the tile, -1 = skip
};
static_assert(sizeof(TileDesc) == 64, "descriptor slot size");

struct __align__(64) TcParams {
  CUtensorMap tm_k;
  CUtensorMap tm_v;   // V as rows of 64 dims (two copies per page, one per half)
  CUtensorMap tm_v3;  // V as (64 dims, row, half): one copy per page
  CUtensorMap tm_q;
  CUtensorMap tm_kc[4];  // shared-prefix launch: K and V maps for 1, 2, 4, 8 KV heads per tile
  CUtensorMap tm_vc[4];
  const uint16_t* q;     // shared-prefix launch: q rows are gathered with plain loads
  int64_t q_stride;      // elements between sequences' q rows
  const int32_t* block_tables;
  const int32_t* context_lens;
  int* header;
  const int* part_base;
  int* merge_cnt;
  const int2* items;
  const int2* pitems;    // shared-prefix items
  const int* runs;       // sub-runs: span, members, member sequences
  const int* seq_span;   // per sequence: tokens of its shared span
  const int* seq_pp;     // per sequence: partitions of that span
  float* part_o;
  float* part_lse;
  uint16_t* out;
  float* lse;
  unsigned int* err;
  int max_blocks;
  int num_blocks;
  int hkv;
  int hq;
  int group;     // q heads per KV head
  int ht_shift;  // log2 of the KV heads per tile (and per item)
  int ngroups;   // KV-head groups: hkv >> ht_shift
  int nq;        // q columns of a tile: group << ht_shift
  float scale_log2;
};

// Swizzled byte offset of (row, 16-byte chunk) inside a 128-byte-row region.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int NH>
__device__ __forceinline__ void tmem_ld_o(uint32_t taddr, float (&v)[2 * NH]);
template <>
__device__ __forceinline__ void tmem_ld_o<8>(uint32_t taddr, float (&v)[16]) {
  tmem_ld16(taddr, v);
}
template <>
__device__ __forceinline__ void tmem_ld_o<16>(uint32_t taddr, float (&v)[32]) {
  tmem_ld32(taddr, v);
}

// NH: q columns per tile (every row computes all of them, masked to its own
// KV head's).  kCasc: the launch also runs the plan's shared-prefix items,
// before the sequences' own items.
template <int NH, bool kCasc>
__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ TcParams p) {
  static_assert(!kCasc || NH == 8, "shared-prefix items use 8 q columns");
  using L = Smem<NH>;
  constexpr int kNpv = L::kNpv;
  constexpr uint32_t kIdescO = idesc_bf16_f32(128, kNpv, true, false);
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  unsigned char* sptr = smem_raw + (sbase - raw);

  uint64_t* bars = reinterpret_cast<uint64_t*>(sptr + L::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* s_full = bars + 2 * kStages;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* o_free = o_full + 2;
  uint64_t* q_full = o_free + 2;
  uint64_t* q_empty = q_full + 2;
  uint64_t* desc_full = q_empty + 2;
  uint64_t* desc_empty = desc_full + kDescSlots;
  uint64_t* drain = desc_empty + kDescSlots;
  uint64_t* xbar = drain + 1;       // softmax warps' exchange barrier
  uint64_t* res_full = xbar + 1;    // softmax -> epilogue: an item result is ready
  uint64_t* res_empty = res_full + 1;
  uint64_t* ebar = res_empty + 1;   // epilogue warps' exchange barrier
  float* resbuf = reinterpret_cast<float*>(sptr + L::kOffRes);        // [NH][128]
  float* reslse = resbuf + NH * 128;                                  // [NH]
  int* resmeta = reinterpret_cast<int*>(reslse + NH);                 // s, g, part, npart, pbase, kind
  TileDesc* descs = reinterpret_cast<TileDesc*>(sptr + L::kOffDesc);
  float* red = reinterpret_cast<float*>(sptr + L::kOffRed);
  float* red_max = red;                // [2][4][NH]
  float* red_l = red + 2 * 4 * NH;     // [2][4][NH]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sptr + L::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sptr + L::kOffMisc + 4);
  volatile int* merge_flag = reinterpret_cast<volatile int*>(sptr + L::kOffMisc + 8);  // [2]

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
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
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
    prefetch_tmap(&p.tm_v3);
    prefetch_tmap(&p.tm_q);
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::kTmemCols);
  fence_barrier_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The kernel may be launched while the plan kernel before it still runs (a
  // programmatic dependent launch): the set-up above overlaps it, and nothing
  // below reads the plan's results before the plan grid has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Tile geometry of the two item kinds.  A sequence's own items pack 2^hts_o
  // KV heads per tile (fixed by the host); shared-prefix items pack 2^hts_p
  // KV heads and msh_p sharers (chosen by the plan: log2 HT | M << 8).  A tile
  // holds 8 / HT pages; an item's q columns are cph = M G per KV head.
  const int hts_o = p.ht_shift;
  int hts_p = hts_o, msh_p = 1;
  if (kCasc) {
    const int hw = p.header[6];
    hts_p = hw & 0xff;
    msh_p = hw >> 8 > 0 ? hw >> 8 : 1;
  }
  const int cph_p = msh_p * p.group;

  if (warp == 6) {
    // =========================== scheduler ===========================
    // shared-prefix items first (their own list and counter), then the
    // sequences' own items
    const int ptotal = kCasc ? p.header[4] : 0;
    const int ppart = kCasc ? p.header[7] : 0;
    const int total = p.header[0];
    const int part = p.header[3];
    bool pre = ptotal > 0;
    uint32_t d = 0;
    int pages = 8 >> hts_o;
    auto publish = [&](const TileDesc& td, int pbk) {
      const int slot = d % kDescSlots;
      mbar_wait(&desc_empty[slot], ((d / kDescSlots) & 1) ^ 1, abort_flag, p.err);
      TileDesc* o = descs + slot;
      if (lane < 8) o->pb[lane] = lane < pages ? pbk : -1;
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
      if (lane == 0) item = atomicAdd(p.header + (pre ? 5 : 2), 1);
      item = __shfl_sync(0xffffffffu, item, 0);
      if (pre && item >= ptotal) {
        pre = false;
        continue;
      }
      if (!pre && item >= total) break;
      const int2 dd = pre ? p.pitems[item] : p.items[item];
      TileDesc td;
      td.s = dd.x;
      td.g = dd.y >> 16;
      const int q = dd.y & 0xffff;
      int tok0, srow;
      pages = 8 >> (pre ? hts_p : hts_o);
      const int kind = pre ? kPre : 0;
      if (pre) {
        // a sub-run (s = its index; npart = its members) over its shared span,
        // read through its first member's table
        const int* rr = p.runs + static_cast<int64_t>(td.s) * kRunInts;
        const int span = rr[0];
        td.npart = rr[1];
        srow = rr[2];
        td.part = q;
        td.pbase = 0;
        tok0 = q * ppart;
        td.tok1 = min(span, tok0 + ppart);
      } else {
        // a sequence's own tokens, after its shared span (if any)
        int Lc = p.context_lens[td.s];
        const int cap = p.max_blocks * 16;
        Lc = Lc < 0 ? 0 : (Lc > cap ? cap : Lc);
        srow = td.s;
        td.part = p.seq_pp[td.s] + q;
        tok0 = p.seq_span[td.s] + q * part;
        td.tok1 = min(Lc, tok0 + part);
        td.pbase = p.part_base[td.s];
        td.npart = p.part_base[td.s + 1] - td.pbase;
      }
      const int npages = td.tok1 > tok0 ? (td.tok1 - tok0 + 15) / 16 : 0;
      if (npages == 0) {
        td.tok0 = tok0;
        td.flags = kFirst | kLast | kEmpty | kind;
        publish(td, -1);
        continue;
      }
      const int32_t* row = p.block_tables + static_cast<int64_t>(srow) * p.max_blocks + (tok0 >> 4);
      for (int p0 = 0; p0 < npages; p0 += 32) {
        // lane l reads page p0 + l of the item
        int pb = -1;
        if (p0 + lane < npages) {
          pb = row[p0 + lane];
          if (pb < 0 || pb >= p.num_blocks) {
            raise_error(p.err, PA_DEV_ERR_BLOCK_ID);
            pb = -1;
          }
        }
        for (int k = 0; k < 32 && p0 + k < npages; k += pages) {
          const int pbk = __shfl_sync(0xffffffffu, pb, (k + (lane & (pages - 1))) & 31);
          td.tok0 = tok0 + (p0 + k) * 16;
          td.flags = (p0 + k == 0 ? kFirst : 0) | (p0 + k + pages >= npages ? kLast : 0) | kind;
          publish(td, p0 + k + (lane & (pages - 1)) < npages ? pbk : -1);
        }
      }
    }
    // the launch after this one may start as this CTA's last items drain
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
    uint32_t d = 0, t = 0, nq = 0;
    const uint64_t pol = l2_policy_evict_first();
    const CUtensorMap* tmk_p = &p.tm_kc[hts_p];
    const CUtensorMap* tmv_p = &p.tm_vc[hts_p];
    while (true) {
      const int slot = d % kDescSlots;
      mbar_wait(&desc_full[slot], (d / kDescSlots) & 1, abort_flag, p.err);
      const TileDesc* td = descs + slot;
      const int flags = td->flags;
      if (flags & kEnd) break;
      if (!(flags & kEmpty)) {
        const bool pre = kCasc && (flags & kPre);
        const int hts = pre ? hts_p : hts_o;
        const int ht = 1 << hts, pages = 8 >> hts;
        const uint32_t page_bytes = 4u * 2048u * static_cast<uint32_t>(ht);  // K and V, both halves
        const int pb = lane < pages ? td->pb[lane] : -1;
        const int s = td->s, g = td->g;
        if (flags & kFirst) {
          // q of the item's KV-head group into the next q slot
          const int qs = nq & 1;
          mbar_wait(&q_empty[qs], ((nq >> 1) & 1) ^ 1, abort_flag, p.err);
          const uint32_t q0 = sbase + L::kOffQ + qs * kQBytes;
          if (pre) {
            // the sharers' q heads of the item's KV heads, column by column
            // (row h of the slot: KV head hh = h / cph of the item, sharer
            // m = h % cph / G, q head j = h % G of the group; rows of absent
            // sharers and past HT * cph zero), with plain loads in the
            // swizzled layout
            if (!*abort_flag) {
              const int nsh = td->npart;
              const int my_s = lane < nsh ? p.runs[static_cast<int64_t>(s) * kRunInts + 2 + lane] : 0;
#pragma unroll
              for (int j = 0; j < 16 * NH / 32; ++j) {
                const int i = j * 32 + lane;
                const int h = i >> 4, c = i & 15;  // q column, 16-byte chunk of the 256-byte row
                const int hh = h / cph_p, w = h - hh * cph_p, m = w / p.group;
                const int sm = __shfl_sync(0xffffffffu, my_s, m & 31);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (hh < ht && m < nsh)
                  v = __ldg(reinterpret_cast<const uint4*>(
                      p.q + static_cast<int64_t>(sm) * p.q_stride +
                      static_cast<int64_t>((g * ht + hh) * p.group + w - m * p.group) * kD + c * 8));
                sts128(q0 + (c >> 3) * kQRegion + swz(h, c & 7), v);
              }
              // rows NH..15 of the q region (a 16-row operand) stay as they are:
              // no product column reads them
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) mbar_arrive(&q_full[qs]);
            }
          } else if (!*abort_flag && lane == 0) {
            mbar_arrive_expect_tx(&q_full[qs], kQBytes);
            tma_load_3d(q0, &p.tm_q, 0, g * p.nq, s, &q_full[qs]);
            tma_load_3d(q0 + kQRegion, &p.tm_q, 64, g * p.nq, s, &q_full[qs]);
          }
          ++nq;
        }
        const unsigned vmask = __ballot_sync(0xffffffffu, pb >= 0);
        const int st = t % kStages;
        mbar_wait(&empty[st], ((t / kStages) & 1) ^ 1, abort_flag, p.err);
        if (!*abort_flag) {
          const uint32_t stage = sbase + st * kStageBytes;
          if (lane == 0) mbar_arrive_expect_tx(&full[st], __popc(vmask) * page_bytes);
          __syncwarp();
          if (pb >= 0) {
            const int prow = (pb * p.hkv + (g << hts)) * 16;
            const uint32_t kdst = stage + lane * (ht * 2048);
            const uint32_t vdst = stage + kKBytes + lane * (ht * 4096);
            const CUtensorMap* tmk = pre ? tmk_p : &p.tm_k;
            tma_load_2d_hint(kdst, tmk, 0, prow, &full[st], pol);
            tma_load_2d_hint(kdst + kRegion, tmk, 64, prow, &full[st], pol);
            if (ht < 8 || pre) {
              tma_load_3d_hint(vdst, pre ? tmv_p : &p.tm_v3, 0, prow, 0, &full[st], pol);  // both halves
            } else {
              // a 128-row page: two 16 KiB copies ran faster than one of 32 KiB
              tma_load_2d_hint(vdst, &p.tm_v, 0, prow, &full[st], pol);
              tma_load_2d_hint(vdst + kRegion, &p.tm_v, 64, prow, &full[st], pol);
            }
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
      const uint32_t qfirst = nq > kQSlots ? nq - kQSlots : 0;
      for (uint32_t u = qfirst; u < nq; ++u) mbar_wait(&q_full[u & 1], (u >> 1) & 1, nullptr, p.err);
    }
  } else if (warp == 1) {
    // ============================= MMA ==============================
    // One lane issues both products as soon as each is ready: S of the next
    // tile once its pages have landed, O of an earlier tile once its p is in
    // shared memory.  Neither waits for the other, so a stage is released as
    // soon as its O product is done even while the next tile's pages are still
    // in flight.  All waits are non-blocking polls with one shared limit on
    // time without progress.
    if (lane == 0) {
      // Operand descriptors of every stage and buffer, computed once: issuing
      // a product then costs only constant adds (the single issuing thread is
      // otherwise bound by its own address arithmetic).
      const uint64_t desc_k0 = smem_desc_sw128(sbase, 16, 1024);
      // V of a tile of HT heads: its two 64-dim halves HT * 2 KiB apart; rows
      // 16k.. are page k >> log2 HT, its (k & (HT - 1))-th 16 rows (own items
      // and shared-prefix items each have their HT)
      const uint64_t desc_v0_o = smem_desc_sw128(sbase + kKBytes, (1 << hts_o) * 2048, 1024);
      const uint64_t desc_v0_p = smem_desc_sw128(sbase + kKBytes, (1 << hts_p) * 2048, 1024);
      uint32_t voff_o[kRows / 16], voff_p[kRows / 16];
#pragma unroll
      for (int k = 0; k < kRows / 16; ++k) {
        voff_o[k] = 2048u * (k + ((k >> hts_o) << hts_o));
        voff_p[k] = 2048u * (k + ((k >> hts_p) << hts_p));
      }
      uint32_t pre_tiles = 0;  // bit t % 32: tile t is a shared-prefix tile
      const uint64_t desc_q0 = smem_desc_sw128(sbase + L::kOffQ, 16, 1024);
      const uint64_t desc_p0 = smem_desc_sw128(sbase + L::kOffP, 16, 1024);
      uint32_t d = 0, ts = 0, tpv = 0, mq = 0;  // ts: next S tile; tpv: next O tile
      bool have_desc = false, s_end = false;
      int flags = 0;
      long long last = clock64();
      while (!*abort_flag) {
        bool progressed = false;
        if (tpv < ts) {
          const int b = tpv & 1;
          const uint32_t bph = (tpv >> 1) & 1;
          if (mbar_test_wait(&p_full[b], bph) && mbar_test_wait(&o_free[b], bph ^ 1)) {
            tc_fence_after();
            const int st = tpv % kStages;
            const bool pt = kCasc && ((pre_tiles >> (tpv & 31)) & 1u);
            const uint64_t a0 = desc_add(pt ? desc_v0_p : desc_v0_o, st * kStageBytes);
            const uint64_t b0 = desc_add(desc_p0, b * L::kPBytes);
            const uint32_t dt = tmem + 2 * kN + b * kNpv;
            // A = V^T (MN-major): 16 rows = 2 groups of 8; D halves HT*2 KiB apart
            // B = P (K-major, kNpv rows = q columns): row half k/4, 32 bytes per 16 rows
            if (!kCasc && hts_o == 3) {  // one page: slices 2 KiB apart (constant offsets)
#pragma unroll
              for (int k = 0; k < kRows / 16; ++k)
                umma_ss(dt, desc_add(a0, k * 2048),
                        desc_add(b0, (k >> 2) * (kNpv * 128) + (k & 3) * 32), kIdescO,
                        k > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int k = 0; k < kRows / 16; ++k)
                umma_ss(dt, desc_add(a0, pt ? voff_p[k] : voff_o[k]),
                        desc_add(b0, (k >> 2) * (kNpv * 128) + (k & 3) * 32), kIdescO,
                        k > 0 ? 1u : 0u);
            }
            umma_commit(&o_full[b]);
            umma_commit(&empty[st]);
            ++tpv;
            progressed = true;
          }
        }
        if (!s_end && !have_desc) {
          const int slot = d % kDescSlots;
          if (mbar_test_wait(&desc_full[slot], (d / kDescSlots) & 1)) {
            flags = descs[slot].flags;
            if (flags & kEnd) {
              s_end = true;
            } else {
              mbar_arrive(&desc_empty[slot]);
              ++d;
              have_desc = !(flags & kEmpty);
            }
            progressed = true;
          }
        }
        if (have_desc) {
          const int st = ts % kStages;
          const int b = ts & 1;
          const int qs = mq & 1;
          if ((!(flags & kFirst) || mbar_test_wait(&q_full[qs], (mq >> 1) & 1)) &&
              mbar_test_wait(&full[st], (ts / kStages) & 1) &&
              mbar_test_wait(&s_free[b], ((ts >> 1) & 1) ^ 1)) {
            tc_fence_after();
            const uint64_t a0 = desc_add(desc_k0, st * kStageBytes);
            const uint64_t b0 = desc_add(desc_q0, qs * kQBytes);
            const uint32_t dt = tmem + b * kN;
#pragma unroll
            for (int k = 0; k < kD / 16; ++k)
              umma_ss(dt, desc_add(a0, (k >> 2) * kRegion + (k & 3) * 32),
                      desc_add(b0, (k >> 2) * kQRegion + (k & 3) * 32), kIdescS, k > 0 ? 1u : 0u);
            umma_commit(&s_full[b]);
            if (kCasc) pre_tiles = (flags & kPre) ? (pre_tiles | (1u << (ts & 31))) : (pre_tiles & ~(1u << (ts & 31)));
            if (flags & kLast) {
              umma_commit(&q_empty[qs]);
              ++mq;
            }
            ++ts;
            have_desc = false;
            progressed = true;
          }
        }
        if (s_end && tpv == ts) break;
        if (progressed) {
          last = clock64();
        } else if (clock64() - last > kWaitLimitCycles) {
          *abort_flag = 1;
          raise_error(p.err, PA_DEV_ERR_TIMEOUT);
        }
      }
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
    // Column h of an item: KV head h / cph of the item, sharer (h % cph) / G,
    // q head (h / cph) * G + h % G among the item's q heads of that sequence
    // (an own item: one sequence, cph = G, so q head h).
    while (!*abort_flag) {
      mbar_wait(res_full, k & 1, abort_flag, p.err);
      const int npart = resmeta[3];  // shared-prefix items: the sharers
      if (npart < 0 || *abort_flag) break;
      const int s = resmeta[0], g = resmeta[1], part = resmeta[2], pbase = resmeta[4];
      const bool pre = kCasc && resmeta[5];
      const int hts = pre ? hts_p : hts_o, ht = 1 << hts;
      const int msh = pre ? msh_p : 1, cph = pre ? cph_p : p.group;
      auto sharer_cols = [&](int m) {  // the columns of sharer m
        uint32_t mm = 0;
        for (int hh = 0; hh < ht; ++hh) mm |= ((1u << p.group) - 1u) << (hh * cph + m * p.group);
        return mm & ((1u << NH) - 1u);
      };
      auto col_qhead = [&](int h) { return pre ? (h / cph) * p.group + h % p.group : h; };
      const int nsh = pre ? npart : 1;  // sequences of the item
      float res[NH], l2[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        res[h] = resbuf[h * 128 + e];
        l2[h] = reslse[h];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(res_empty);
      ++k;
      // lane m of every epilogue warp holds sequence m of the item: its index,
      // first partition record and partition count
      int my_s = s, my_pb = pbase, my_np = npart;
      if (pre) {
        my_s = lane < nsh ? p.runs[static_cast<int64_t>(s) * kRunInts + 2 + lane] : 0;
        my_pb = lane < nsh ? p.part_base[my_s] : 0;
        my_np = lane < nsh ? p.part_base[my_s + 1] - my_pb : 1;
      }
      const int qh0 = g * ht * p.group;  // first q head of the item in each sequence
      bool any_multi = false;
      for (int m = 0; m < nsh; ++m) {
        const int sm = __shfl_sync(0xffffffffu, my_s, m);
        const int pbm = __shfl_sync(0xffffffffu, my_pb, m);
        const int npm = __shfl_sync(0xffffffffu, my_np, m);
        const uint32_t mm = pre ? sharer_cols(m) : (1u << (ht * p.group)) - 1u;
        any_multi |= npm > 1;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if ((mm >> h) & 1u) {
            const int qh = qh0 + col_qhead(h);
            if (npm == 1) {
              const int64_t o = static_cast<int64_t>(sm) * p.hq + qh;
              p.out[o * kD + e] = f32_to_bf16_bits(res[h]);
              if (e == 0 && p.lse) p.lse[o] = l2[h] * kLn2;
            } else {
              const int64_t rec = static_cast<int64_t>(pbm + part) * p.hq + qh;
              __stcg(p.part_o + rec * kD + e, res[h]);
              if (e == 0) __stcg(p.part_lse + rec, l2[h]);
            }
          }
        }
      }
      if (!any_multi) continue;
      // The last partition of a (sequence, KV head) to finish merges all of
      // them.  Thread e < ht * M counts (KV head g ht + e / M, sharer e % M),
      // whose G columns are [e G, (e + 1) G).
      __threadfence();
      eexchange();
      if (warp == 7) {
        bool last = false;
        const int hh = e / msh, m = e - hh * msh;
        const int sm = __shfl_sync(0xffffffffu, my_s, m & 31);
        const int npm = __shfl_sync(0xffffffffu, my_np, m & 31);
        if (e < ht * msh && m < nsh && npm > 1) {
          const int old =
              atomicAdd(p.merge_cnt + static_cast<int64_t>(sm) * p.hkv + g * ht + hh, 1);
          last = old == npm - 1;
        }
        const unsigned done = __ballot_sync(0xffffffffu, last);
        if (lane == 0) merge_flag[k & 1] = static_cast<int>(done);
      }
      eexchange();
      const unsigned done = static_cast<unsigned>(merge_flag[k & 1]);
      if (!done) continue;
      __threadfence();
      // bit b of `done`: q columns [b G, (b + 1) G)
      uint32_t colsel = 0;
      for (unsigned bits = done; bits; bits &= bits - 1)
        colsel |= ((1u << p.group) - 1u) << ((__ffs(bits) - 1) * p.group);
      for (int m = 0; m < nsh; ++m) {
        const int sm = __shfl_sync(0xffffffffu, my_s, m);
        const int pbm = __shfl_sync(0xffffffffu, my_pb, m);
        const int npm = __shfl_sync(0xffffffffu, my_np, m);
        const uint32_t mc = pre ? colsel & sharer_cols(m) : colsel;
        if (!mc) continue;
        float M[NH], W[NH], A[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          M[h] = -CUDART_INF_F;
          W[h] = 0.f;
          A[h] = 0.f;
        }
        const int64_t rec0 = static_cast<int64_t>(pbm) * p.hq + qh0;
        for (int q = 0; q < npm; ++q) {
          float li[NH], oi[NH];
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            li[h] = -CUDART_INF_F;
            oi[h] = 0.f;
            if ((mc >> h) & 1u) {
              const int64_t rec = rec0 + static_cast<int64_t>(q) * p.hq + col_qhead(h);
              li[h] = __ldcg(p.part_lse + rec);
              oi[h] = __ldcg(p.part_o + rec * kD + e);
            }
          }
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            if (li[h] != -CUDART_INF_F) {
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
          if ((mc >> h) & 1u) {
            const bool live = W[h] > 0.f;
            const int64_t o = static_cast<int64_t>(sm) * p.hq + qh0 + col_qhead(h);
            p.out[o * kD + e] = f32_to_bf16_bits(live ? A[h] / W[h] : 0.f);
            if (e == 0 && p.lse) p.lse[o] = live ? (M[h] + log2f(W[h])) * kLn2 : -CUDART_INF_F;
          }
        }
      }
    }
  } else {
    // ============================ softmax =============================
    const int q4 = warp & 3;          // TMEM lane quadrant of this warp
    const int r = q4 * 32 + lane;     // tile row of S^T, output dim of O^T
    const int wi = warp - 2;          // index among the softmax warps
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    // Tile row r, for either item kind (own: _o, shared prefix: _p): page pj,
    // KV head (r >> 4) & (HT - 1) of the tile, token pj * 16 + r % 16.  Row r
    // of the V tile: page pj holds its rows for dims 0-63, then 64-127.  The
    // row's q columns start at its KV head's block of cph columns (an item
    // with k sharers uses the first k G of them).
    const int pj_o = r >> (4 + hts_o), pj_p = r >> (4 + hts_p);
    const uint32_t vro_o = pj_o * ((1 << hts_o) * 4096) + (r & ((16 << hts_o) - 1)) * 128;
    const uint32_t vro_p = pj_p * ((1 << hts_p) * 4096) + (r & ((16 << hts_p) - 1)) * 128;
    const int crow_o = ((r >> 4) & ((1 << hts_o) - 1)) * p.group;
    const int crow_p = ((r >> 4) & ((1 << hts_p) - 1)) * cph_p;
    const int rtok_o = (pj_o << 4) | (r & 15), rtok_p = (pj_p << 4) | (r & 15);
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
      float ov[2 * NH];
      tmem_ld_o<NH>(tmem + lane_addr + 2 * kN + b * kNpv, ov);
      tc_fence_before();
      mbar_arrive(&o_free[b]);
#pragma unroll
      for (int h = 0; h < NH; ++h) acc[h] = acc[h] * alpha_prev[h] + ov[h] + ov[NH + h];
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
      const bool pre = kCasc && (flags & kPre);
      const int pj = pre ? pj_p : pj_o;
      const int mypb = td->pb[pj];
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
        const bool valid = tok0 + (pre ? rtok_p : rtok_o) < tok1 && mypb >= 0;
        // the row's columns: its KV head's G q heads for each of the item's sharers
        const uint32_t cm = ((1u << ((pre ? npart : 1) * p.group)) - 1u) << (pre ? crow_p : crow_o);
        float x[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h)
          x[h] = (valid && ((cm >> h) & 1u)) ? sv[h] * p.scale_log2 : -CUDART_INF_F;
        // tile max per q column: warp shuffle, then across the four softmax warps
        float* rm = red_max + (t & 1) * 4 * NH;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          float v = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rm[wi * NH + h] = v;
        }
        exchange();
        float pr[NH], alpha[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float tmax =
              fmaxf(fmaxf(rm[h], rm[NH + h]), fmaxf(rm[2 * NH + h], rm[3 * NH + h]));
          const float mn = fmaxf(m_run[h], tmax);
          alpha[h] = (mn == -CUDART_INF_F) ? 1.f : exp2f(m_run[h] - mn);
          pr[h] = (x[h] == -CUDART_INF_F) ? 0.f : exp2f(x[h] - mn);
          l_part[h] = l_part[h] * alpha[h] + pr[h];
          m_run[h] = mn;
        }
        // p into P[b]: row h (q column) and row NH + h (the bf16 remainder),
        // column r (tile row), K-major 128B swizzle
        const uint32_t pbuf = sbase + L::kOffP + b * L::kPBytes + (r >> 6) * (kNpv * 128);
        const int c = r & 63;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const uint16_t hi = f32_to_bf16_bits(pr[h]);
          const float rem = pr[h] - __uint_as_float(static_cast<uint32_t>(hi) << 16);
          sts16(pbuf + swz(h, c >> 3) + (c & 7) * 2, hi);
          sts16(pbuf + swz(NH + h, c >> 3) + (c & 7) * 2, f32_to_bf16_bits(rem));
        }
        if (!valid) {
          // zero this row of V (both 64-dim halves) so padding never reaches O
          const uint32_t vrow = sbase + st * kStageBytes + kKBytes + (pre ? vro_p : vro_o);
          const uint32_t vhalf = (1u << (pre ? hts_p : hts_o)) * 2048u;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            sts128_zero(vrow + k * 16);
            sts128_zero(vrow + vhalf + k * 16);
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

      // ---- finalize the item: l over the 128 tile rows, then output dim r ----
      float* rl = red_l + (nfin & 1) * 4 * NH;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = l_part[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rl[wi * NH + h] = v;
      }
      exchange();
      float res[NH], lse2[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float l = rl[h] + rl[NH + h] + rl[2 * NH + h] + rl[3 * NH + h];
        const bool live = m_run[h] != -CUDART_INF_F && l > 0.f;
        res[h] = live ? acc[h] / l : 0.f;
        lse2[h] = live ? m_run[h] + log2f(l) : -CUDART_INF_F;
      }
      // hand the item's result to the epilogue warps
      mbar_wait(res_empty, (nfin & 1) ^ 1, abort_flag, p.err);
#pragma unroll
      for (int h = 0; h < NH; ++h) resbuf[h * 128 + r] = res[h];
      if (r == 0) {
#pragma unroll
        for (int h = 0; h < NH; ++h) reslse[h] = lse2[h];
        resmeta[0] = s;
        resmeta[1] = g;
        resmeta[2] = part;
        resmeta[3] = npart;
        resmeta[4] = pbase;
        resmeta[5] = pre ? 1 : 0;
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
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int NH, bool kCasc = false>
int launch_nh(const TcParams& prm, int64_t item_bound, cudaStream_t stream) {
  auto kern = decode_tc_kernel<NH, kCasc>;
  static KernelLaunchCache cache;
  const int per_sm =
      cache.blocks_per_sm(reinterpret_cast<const void*>(kern), kThreads, Smem<NH>::kBytes);
  if (per_sm < 1) return PA_ERR_CUDA;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int grid = static_cast<int>(item_bound < cap ? (item_bound < 1 ? 1 : item_bound) : cap);
  // programmatic dependent launch: the CTAs start and set up while the plan
  // kernel (launched just before on the same stream) finishes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Smem<NH>::kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return launch_status();
}

// q columns per tile (8 or 16) and KV heads per tile for a group size.
struct TcShape {
  int nh;
  int ht_shift;
};

TcShape tc_shape(int group, int hkv) {
  TcShape sh{group <= 8 ? 8 : 16, 0};
  // pack KV heads while their q heads fit the tile's columns and the heads
  // divide evenly into groups
  while ((1 << (sh.ht_shift + 1)) <= 8 && (group << (sh.ht_shift + 1)) <= sh.nh &&
         hkv % (1 << (sh.ht_shift + 1)) == 0)
    ++sh.ht_shift;
  return sh;
}

}  // namespace

bool decode_tcgen05_supported(int head_dim, int group) {
  return head_dim == kD && group >= 1 && group <= kN;
}

int decode_tcgen05_heads_per_item(int group, int hkv) {
  return 1 << tc_shape(group, hkv).ht_shift;
}

int launch_decode_tcgen05(const DecodeArgs& a) {
  const int group = a.num_q_heads / a.pool.num_kv_heads;
  if (!decode_tcgen05_supported(a.pool.head_dim, group)) return PA_ERR_UNSUPPORTED;
  const TcShape sh = tc_shape(group, a.pool.num_kv_heads);
  if ((1 << sh.ht_shift) != a.item_heads) return PA_ERR_ARG;  // the plan's items differ
  const int64_t rows = static_cast<int64_t>(a.pool.num_blocks) * a.pool.num_kv_heads * 16;
  if (rows >= (1LL << 31)) return PA_ERR_UNSUPPORTED;
  TcParams p{};
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(rows)};
    const uint64_t strides[1] = {kD * 2};
    const uint32_t box[2] = {64, static_cast<uint32_t>(16 << sh.ht_shift)};
    if (!encode_bf16_map(&p.tm_k, a.k_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
    if (!encode_bf16_map(&p.tm_v, a.v_pool, 2, dims, strides, box)) return PA_ERR_CUDA;
  }
  {
    // V: (dim within a 64-dim half, pool row, half) -- one copy moves a page's
    // rows for both halves, half 0 first, as the second product reads them
    const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), 2};
    const uint64_t strides[2] = {kD * 2, 128};
    const uint32_t box[3] = {64, static_cast<uint32_t>(16 << sh.ht_shift), 2};
    if (!encode_bf16_map(&p.tm_v3, a.v_pool, 3, dims, strides, box)) return PA_ERR_CUDA;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(a.num_q_heads),
                              static_cast<uint64_t>(a.num_seqs)};
    const uint64_t strides[2] = {kD * 2, static_cast<uint64_t>(a.q_stride) * 2};
    const uint32_t box[3] = {64, 16, 1};
    if (!encode_bf16_map(&p.tm_q, a.q, 3, dims, strides, box)) return PA_ERR_CUDA;
  }
  const bool casc = a.casc_cols == 8;
  if (casc) {
    // shared-prefix launch: the plan picks 1, 2, 4 or 8 KV heads per tile
    for (int h = 0; h < 4; ++h) {
      if (a.pool.num_kv_heads % (1 << h)) continue;  // never chosen
      const uint64_t dk[2] = {static_cast<uint64_t>(kD), static_cast<uint64_t>(rows)};
      const uint64_t sk[1] = {kD * 2};
      const uint32_t bk[2] = {64, static_cast<uint32_t>(16 << h)};
      if (!encode_bf16_map(&p.tm_kc[h], a.k_pool, 2, dk, sk, bk)) return PA_ERR_CUDA;
      const uint64_t dv[3] = {64, static_cast<uint64_t>(rows), 2};
      const uint64_t sv[2] = {kD * 2, 128};
      const uint32_t bv[3] = {64, static_cast<uint32_t>(16 << h), 2};
      if (!encode_bf16_map(&p.tm_vc[h], a.v_pool, 3, dv, sv, bv)) return PA_ERR_CUDA;
    }
  }
  p.q = a.q;
  p.q_stride = a.q_stride;
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.header = a.ws.header;
  p.part_base = a.ws.part_base;
  p.merge_cnt = a.ws.merge_cnt;
  p.items = a.ws.items;
  p.pitems = a.ws.pitems;
  p.runs = a.ws.runs;
  p.seq_span = a.ws.seq_span;
  p.seq_pp = a.ws.seq_pp;
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
  p.ht_shift = sh.ht_shift;
  p.ngroups = a.pool.num_kv_heads >> sh.ht_shift;
  p.nq = group << sh.ht_shift;
  p.scale_log2 = a.scale * kLog2e;
  const int64_t bound = static_cast<int64_t>(a.num_seqs) * (a.max_parts + 1) * p.ngroups +
                        (casc ? static_cast<int64_t>(a.num_seqs / 2 + 1) * a.max_parts * a.pool.num_kv_heads : 0);
  // one launch: the shared-prefix items (none unless the plan found shared
  // prefixes) and then the sequences' own items
  if (casc) return launch_nh<8, true>(p, bound, a.stream);
  if (sh.nh == 8) return launch_nh<8>(p, bound, a.stream);
  return launch_nh<16>(p, bound, a.stream);
}

}  // namespace pa
