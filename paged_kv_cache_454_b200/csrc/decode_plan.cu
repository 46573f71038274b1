// The decode work plan: one CTA turns context lengths into the list of
// (sequence, KV-head group, partition) work items both decode kernels consume
// (a group is one KV head for the CUDA-core kernel, one to eight for the
// tensor-core kernel).
//
//  * Partition length: `min_part` tokens, or -- when the caller leaves the
//    choice to the library -- a power-of-two multiple of it up to `max_part`:
//    the longest that still leaves at least `target_items` items (every item
//    has a fixed cost, and longest-first order keeps the tail short), or, for
//    shared prefixes, the longest whose items stay small next to one SM's
//    share of the work (see below).
//  * Order: longest items first (all full partitions, then the tails by
//    decreasing length, then empty contexts), so a kernel that hands items out
//    dynamically schedules them longest-processing-time first.
//  * Shared prefixes: when sequences share their first physical block (parallel
//    samples of one prompt, "vLLM 基本原理" / 内存共享) and every item is small
//    next to one SM's share of the work, the list is instead ordered by that
//    block, then KV head, then sequence: the samples of a group read the shared
//    pages of one KV head at the same time, so DRAM serves them once and L2
//    the rest.  (Up to kSortMax sequences.)  A hash set of first blocks finds
//    whether any repeats; the sort runs only then, and only if some candidate
//    length keeps every item at most 1/kLocalityShare of one SM's share.
//  * Shared-prefix cascade (tensor-core kernel, when the caller enables it
//    with `casc_cols`, the q columns of one shared-prefix item):
//    sequences sorted by first block form runs.  The longest run fixes the
//    sharers per item M (at most casc_cols / G) and the KV heads per item HT
//    (the most, up to 8, with G * HT * M <= casc_cols that divide the KV
//    heads); runs are
//    cut into sub-runs of at most M sequences, and a sub-run's shared span is
//    the longest stretch of leading table entries all its members have in
//    common (whole blocks inside every member's context).  A span of at least
//    kMinCascSpan tokens becomes shared-prefix items (sub-run, KV-head group,
//    partition) in a list of their own, read once for all members, with a
//    partition length of their own (several items per SM, so they end
//    together); each member's own items then cover
//    only its tokens after the span, and its partitions count the span's
//    first.  header[4..7]: prefix items, their counter, log2 HT | M << 8,
//    their partition length.
//  * It also clears the dynamic item counters and the per-(sequence, KV head)
//    counters the tensor-core kernel uses to find the last partition to finish.
#include "common.cuh"
#include "internal.h"

namespace pa {
namespace {

__device__ __forceinline__ int clamp_len(int L, int max_blocks, unsigned int* err) {
  const int cap = max_blocks * 16;
  if (L < 0 || L > cap) {
    raise_error(err, PA_DEV_ERR_CONTEXT);
    return L < 0 ? 0 : cap;
  }
  return L;
}

// Items are bucketed by their length n in units (a page or a few): bucket 0
// holds n >= 64, bucket 64 - n holds 1 <= n < 64, bucket 64 the empty items.
constexpr int kMaxBuckets = 65;
__device__ __forceinline__ int bucket_of(int nunits) {
  return nunits == 0 ? 64 : (nunits >= 64 ? 0 : 64 - nunits);
}

constexpr int kSortMax = 1024;  // sequences the locality order sorts (one per thread)
constexpr int kLensCache = 2048;  // sequences whose lengths the plan keeps in shared memory
constexpr int kFirstSet = 2 * kSortMax;  // slots of the set that detects shared first blocks
// In prefix order the longest item is at most 1/kLocalityShare of one SM's
// share of the work (measured: 13B-shaped sampling batches are fastest with
// 256-token items at this bound; longer items leave a long tail).
constexpr int kLocalityShare = 16;
static_assert(kFirstSet == 2048, "the set's hash keeps 11 bits");
// A shared prefix shorter than this is left to each sequence's own items.
constexpr int kMinCascSpan = 128;
// sharers per sub-run at most (the span search compares this many tables per
// entry; the columns of a tile, 8, already bound it)
constexpr int kCascMaxMembers = 8;
// Shared-prefix items per SM the prefix partition length aims for.
constexpr int kCascItemsPerSm = 8;

// Inclusive block-wide scan (sum or max) of one value per thread, 1024 threads.
template <bool kMax>
__device__ __forceinline__ int block_scan(int x, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x = kMax ? max(x, y) : x + y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w = kMax ? max(w, y) : w + y;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  const int r = warp > 0 ? (kMax ? max(x, warp_tot[warp - 1]) : x + warp_tot[warp - 1]) : x;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) decode_plan_kernel(const int32_t* __restrict__ context_lens,
                                                           const int32_t* __restrict__ block_tables,
                                                           int S, int max_blocks, int hkv,
                                                           int kv_heads, int min_part, int max_part,
                                                           int target_items, int num_sms,
                                                           int group, int casc_cols,
                                                           int* header, int* part_base,
                                                           int2* items, int* merge_cnt,
                                                           int* seq_span, int* seq_pp, int* runs,
                                                           int2* pitems, unsigned int* err) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  __shared__ int cand[4];      // items per KV-head group at each candidate length
  __shared__ int cand_mx[4];   // longest item at each candidate length, in 128-token units
  __shared__ int tiles_tot;    // context of all items in 128-token units (any length)
  __shared__ int bucket[kMaxBuckets];
  __shared__ int cursor[kMaxBuckets];
  __shared__ unsigned long long skey[kSortMax];  // (first block << 32 | sequence), sorted
  __shared__ int run_tab[2 * kSortMax];           // per run start: partition prefix, run total
  __shared__ int sflag[4];                        // [0] some first block repeats
  __shared__ int slens[kLensCache];               // context lengths as given (S <= kLensCache)
  __shared__ unsigned first_set[kFirstSet];       // open-addressing set of first blocks
  __shared__ int sspan[kSortMax];                 // shared-prefix span per sequence (cascade)
  __shared__ int nruns;                           // sub-runs (cascade)
  __shared__ int rspan[kSortMax / 2];             // each sub-run's shared span (cascade)
  __shared__ int roff[kSortMax / 2];              // each sub-run's first prefix item (cascade)
  __shared__ int rmax;                            // longest run of shared first blocks
  __shared__ int cand_pp[4];                      // prefix items at each candidate length
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // The decode kernel that follows may start its prologue now; it waits for
  // this grid's results before reading them.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // Thread i's sequence's first table entry, loaded now so its latency overlaps
  // the passes below (used only when S fits the locality sort).
  const bool sortable = S > 1 && S <= kSortMax && max_blocks > 0;
  unsigned my_first = 0xffffffffu;
  if (sortable && tid < S) my_first = static_cast<unsigned>(block_tables[static_cast<int64_t>(tid) * max_blocks]);
  for (int i = tid; i < kFirstSet; i += 1024) first_set[i] = 0xffffffffu;

  // Context lengths are read once into shared memory when they fit; every pass
  // below reads them through `lens`.
  const int32_t* lens = context_lens;
  if (S <= kLensCache) {
    for (int s = tid; s < S; s += 1024) slens[s] = context_lens[s];
    __syncthreads();
    lens = slens;
  }

  // ---- shared prefixes: does any first physical block repeat?  (a set in
  // shared memory; the sort below runs only if one does and the items end up
  // small enough) ----
  if (tid < 4) sflag[tid] = 0;
  __syncthreads();  // the set's initialisation and sflag
  if (sortable && tid < S && clamp_len(lens[tid], max_blocks, nullptr) > 0) {
    unsigned h = (my_first * 2654435761u) >> 21;  // 11 bits: kFirstSet slots
    for (int probe = 0; probe < kFirstSet; ++probe, h = (h + 1) & (kFirstSet - 1)) {
      const unsigned old = atomicCAS(&first_set[h], 0xffffffffu, my_first);
      if (old == 0xffffffffu) break;
      if (old == my_first) {
        atomicOr(&sflag[0], 1);
        break;
      }
    }
  }

  // ---- partition length ----
  // Without shared prefixes items run longest first, so the tail is short
  // whatever their lengths, and every item costs a fixed start and finish:
  // the longest candidate that still gives `target_items` items wins (the
  // shortest when none does -- a small batch needs the parallelism).  With
  // shared prefixes items run in prefix order instead, so the longest item
  // must stay small next to one SM's share of the work: the longest candidate
  // whose longest item is at most 1/kLocalityShare of that share, in which
  // case the list takes the locality order.
  int ncand = 1;
  while (ncand < 4 && (min_part << ncand) <= max_part) ++ncand;
  if (tid < 4) {
    cand[tid] = 0;
    cand_mx[tid] = 0;
  }
  if (tid == 0) tiles_tot = 0;
  __syncthreads();
  {
    int cnt[4] = {0, 0, 0, 0}, mx[4] = {0, 0, 0, 0}, tt = 0;
    for (int s = tid; s < S; s += 1024) {
      const int L = clamp_len(lens[s], max_blocks, nullptr);
      tt += (L + 127) / 128;
      for (int k = 0; k < ncand; ++k) {
        const int pk = min_part << k;
        const int n = (L + pk - 1) / pk;
        cnt[k] += n < 1 ? 1 : n;
        mx[k] = max(mx[k], (min(L, pk) + 127) / 128);
      }
    }
    for (int o = 16; o > 0; o >>= 1) tt += __shfl_xor_sync(0xffffffffu, tt, o);
    if (lane == 0) atomicAdd(&tiles_tot, tt);
    for (int k = 0; k < ncand; ++k) {
      int v = cnt[k], m = mx[k];
      for (int o = 16; o > 0; o >>= 1) {
        v += __shfl_xor_sync(0xffffffffu, v, o);
        m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      }
      if (lane == 0) {
        atomicAdd(&cand[k], v);
        atomicMax(&cand_mx[k], m);
      }
    }
  }
  __syncthreads();
  int part = -1;
  bool locality = false;
  bool casc = casc_cols >= 2 * group && sortable && sflag[0] != 0;
  if (sortable && sflag[0] && !casc) {
    const long long share = static_cast<long long>(tiles_tot) * hkv;
    for (int k = ncand - 1; k >= 0; --k)
      if (static_cast<long long>(cand_mx[k]) * kLocalityShare * num_sms <= share) {
        part = min_part << k;
        locality = true;
        break;
      }
  }
  if (part < 0) {
    part = min_part;
    for (int k = ncand - 1; k > 0; --k)
      if (static_cast<long long>(cand[k]) * hkv >= target_items) {
        part = min_part << k;
        break;
      }
  }
  // items are bucketed by length in units of `unit` tokens: a page for short
  // partitions, coarser for long ones, so a partition is at most 64 units
  const int unit = part / 64 > 16 ? part / 64 : 16;
  const int full_bucket = bucket_of(part / unit);

  // ---- sort sequences by their first physical block ----
  // Keys (first block << 32 | sequence) are distinct, so each sequence's
  // sorted position is the number of keys below its own: one pass over the S
  // keys per thread (shared-memory broadcasts) and two barriers.
  if (locality || casc) {
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(run_tab);  // unsorted
    unsigned long long k = 0;
    if (tid < S) {
      const int L = clamp_len(lens[tid], max_blocks, nullptr);
      const unsigned first = L > 0 ? my_first : 0xffffffffu;
      k = (static_cast<unsigned long long>(first) << 32) | static_cast<unsigned>(tid);
      keys[tid] = k;
    }
    __syncthreads();
    if (tid < S) {
      int r = 0, j = 0;
      for (; j + 8 <= S; j += 8) {
#pragma unroll
        for (int q = 0; q < 8; ++q) r += keys[j + q] < k;
      }
      for (; j < S; ++j) r += keys[j] < k;
      skey[r] = k;
    }
    __syncthreads();
  }
  // ---- shared-prefix cascade: runs of sequences with a common first block,
  // cut into sub-runs, and the span each sub-run's tables have in common ----
  if (tid < kSortMax) sspan[tid] = 0;
  if (tid < 4) cand_pp[tid] = 0;
  if (tid == 0) {
    nruns = 0;
    rmax = 0;
  }
  __syncthreads();
  int members = 0, hts = 0, pp_len = part;
  if (casc) {
    // thread i: sorted position i.  A run's length is stored at its start.
    int* run_len = run_tab;           // by a run's first sorted position
    int* sub_pos = run_tab + kSortMax;  // per sub-run: first sorted position | members << 16
    const int i = tid;
    unsigned long long f = 0xffffffffull;
    bool head = false, last = false;
    if (i < S) {
      f = skey[i] >> 32;
      head = i == 0 || f != (skey[i - 1] >> 32);
      last = i == S - 1 || f != (skey[i + 1] >> 32);
    }
    const int start = block_scan<true>(head ? i : 0, warp_tot);
    if (i < S && last && f != 0xffffffffull) {
      run_len[start] = i - start + 1;
      atomicMax(&rmax, i - start + 1);
    }
    __syncthreads();
    // sharers per item and KV heads per item
    members = min(min(rmax, casc_cols / group), kCascMaxMembers);
    hts = 0;
    while (hts < 3 && group * (2 << hts) * members <= casc_cols && kv_heads % (2 << hts) == 0) ++hts;
    casc = members >= 2;
    if (casc) {
      // sub-runs: every members-th sequence of a run starts one, if at least
      // one more follows it
      bool sub = false;
      int k = 0;
      if (i < S && f != 0xffffffffull) {
        const int w = i - start, n = run_len[start];
        sub = w % members == 0 && n - w >= 2;
        k = min(members, n - w);
      }
      const int idx = block_scan<false>(sub ? 1 : 0, warp_tot);
      if (sub) sub_pos[idx - 1] = i | (k << 16);
      if (tid == 1023) nruns = idx;
      __syncthreads();
      // a half-warp per sub-run (two per warp, so 64 sub-runs take one round
      // of table loads): its members and the span of table entries they
      // share.  Lane l of a half covers entries b0 + l and b0 + 16 + l of
      // each 32-entry window.
      const int nr = nruns;
      const int hl = lane & 15, hw = lane >> 4;
      for (int r0 = 2 * warp; r0 < nr; r0 += 64) {
        const int r = r0 + hw;
        const bool live = r < nr;
        int i0 = 0, k = 0;
        int full = 0;  // whole blocks inside every member's context
        if (live) {
          i0 = sub_pos[r] & 0xffff;
          k = sub_pos[r] >> 16;
          full = max_blocks;
          for (int q = 0; q < k; ++q) {
            const int sq = static_cast<int>(skey[i0 + q] & 0xffffffffull);
            full = min(full, clamp_len(lens[sq], max_blocks, nullptr) >> 4);
          }
        }
        int lcp = full;
        bool open = live;  // this half has not found its first differing entry
        for (int b0 = 0; __any_sync(0xffffffffu, open && b0 < full); b0 += 32) {
          bool same0 = true, same1 = true;
          if (open && b0 < full) {
            // every member's entries are loaded before any is compared, so
            // the loads are in flight together
            int32_t v0[kCascMaxMembers], v1[kCascMaxMembers];
            const int bj0 = b0 + hl, bj1 = b0 + 16 + hl;
#pragma unroll
            for (int q = 0; q < kCascMaxMembers; ++q) {
              const int64_t rowq =
                  q < k ? static_cast<int64_t>(skey[i0 + q] & 0xffffffffull) * max_blocks : 0;
              v0[q] = q < k && bj0 < full ? block_tables[rowq + bj0] : 0;
              v1[q] = q < k && bj1 < full ? block_tables[rowq + bj1] : 0;
            }
#pragma unroll
            for (int q = 1; q < kCascMaxMembers; ++q) {
              same0 = same0 && (q >= k || v0[q] == v0[0]);
              same1 = same1 && (q >= k || v1[q] == v1[0]);
            }
          }
          const unsigned d0 = (__ballot_sync(0xffffffffu, !same0) >> (16 * hw)) & 0xffffu;
          const unsigned d1 = (__ballot_sync(0xffffffffu, !same1) >> (16 * hw)) & 0xffffu;
          const unsigned diff = d0 | (d1 << 16);  // bit i: entry b0 + i differs
          if (open && b0 < full && diff) {
            lcp = b0 + __ffs(diff) - 1;
            open = false;
          }
        }
        if (live) {
          const int span = lcp * 16 >= kMinCascSpan ? lcp * 16 : 0;
          int* rr = runs + static_cast<int64_t>(r) * kRunInts;
          if (hl == 0) {
            rr[0] = span;
            rr[1] = k;
            rspan[r] = span;
          }
          if (hl < k) {
            const int sq = static_cast<int>(skey[i0 + hl] & 0xffffffffull);
            rr[2 + hl] = sq;
            sspan[sq] = span;
          }
        }
      }
      __syncthreads();
      // prefix partition length: the longest candidate that still gives
      // kCascItemsPerSm items per SM (the shortest when none does)
      {
        const int cg = kv_heads >> hts;
        int cnt[4] = {0, 0, 0, 0};
        for (int r = tid; r < nr; r += 1024) {
          const int span = rspan[r];
          for (int k = 0; k < ncand; ++k) cnt[k] += cg * ((span + (min_part << k) - 1) / (min_part << k));
        }
        for (int k = 0; k < ncand; ++k) {
          int v = cnt[k];
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0 && v) atomicAdd(&cand_pp[k], v);
        }
      }
      __syncthreads();
      pp_len = min_part;
      for (int k = ncand - 1; k > 0; --k)
        if (static_cast<long long>(cand_pp[k]) >= static_cast<long long>(kCascItemsPerSm) * num_sms) {
          pp_len = min_part << k;
          break;
        }
    }
  }

  // ---- partitions per sequence and their exclusive prefix ----
  if (tid == 0) carry = 0;
  if (tid < kMaxBuckets) bucket[tid] = 0;
  __syncthreads();
  for (int base = 0; base < S; base += 1024) {
    const int s = base + tid;
    int np = 0;
    if (s < S) {
      const int L = clamp_len(lens[s], max_blocks, err);
      // a shared span (cascade) first, then the sequence's own tokens
      const int span = casc ? sspan[s] : 0;
      const int pp = (span + pp_len - 1) / pp_len;
      const int Ls = L - span;
      np = pp + (Ls + part - 1) / part;
      if (np < 1) np = 1;
      seq_span[s] = span;
      seq_pp[s] = pp;
      // bucket counts of the sequence's own items: full partitions, the tail,
      // or an empty context
      const int full = Ls / part, rem = Ls - full * part;
      if (full) atomicAdd(&bucket[full_bucket], full * hkv);
      if (rem) atomicAdd(&bucket[bucket_of((rem + unit - 1) / unit)], hkv);
      if (L == 0) atomicAdd(&bucket[bucket_of(0)], hkv);
    }
    int x = np;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int incl = x + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (s < S) part_base[s] = carry + incl - np;
    __syncthreads();
    if (tid == 1023) carry += incl;
    __syncthreads();
  }
  if (warp == 0) {
    // bucket start offsets: lane l owns buckets 3l .. 3l + 2
    int c[3], sum = 0;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int b = 3 * lane + j;
      c[j] = b < kMaxBuckets ? bucket[b] : 0;
      sum += c[j];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int acc = incl - sum;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int b = 3 * lane + j;
      if (b < kMaxBuckets) cursor[b] = acc;
      acc += c[j];
    }
    if (lane == 0) {
      int own = 0;  // the sequences' own items: every bucket
      for (int b = 0; b < kMaxBuckets; ++b) own += bucket[b];
      part_base[S] = carry;
      header[0] = own;          // items (the sequences' own)
      header[1] = carry;        // partitions
      header[2] = 0;            // dynamic item counter
      header[3] = part;         // partition length
      header[5] = 0;            // dynamic counter of the shared-prefix items
      header[6] = hts | (members << 8);  // log2 KV heads, sharers per shared-prefix item
      header[7] = pp_len;       // partition length of the shared prefixes
    }
  }
  __syncthreads();

  if (locality && !casc) {
    // thread i handles sorted position i (S <= 1024).  A run of equal first
    // blocks is laid out KV head by KV head, the run's sequences in each head.
    const int i = tid;
    int s = 0, np = 0, start = 0;
    bool last = false;
    if (i < S) {
      s = static_cast<int>(skey[i] & 0xffffffffull);
      const int L = clamp_len(lens[s], max_blocks, nullptr);
      np = max(1, (L + part - 1) / part);
      const unsigned long long f = skey[i] >> 32;
      const bool st = i == 0 || f == 0xffffffffull || f != (skey[i - 1] >> 32);
      start = st ? i : 0;
      last = i == S - 1 || (skey[i + 1] >> 32) == 0xffffffffull || (skey[i + 1] >> 32) != f;
    }
    const int pincl = block_scan<false>(np, warp_tot);
    const int gs = block_scan<true>(start, warp_tot);  // first sorted position of this run
    int* runP = run_tab;              // indexed by a run's first sorted position
    int* runT = run_tab + kSortMax;
    if (i < S && start == i) runP[i] = pincl - np;
    __syncthreads();
    if (i < S && last) runT[gs] = pincl - runP[gs];
    __syncthreads();
    if (i < S) {
      const int p0 = runP[gs], tot = runT[gs];
      const int within = (pincl - np) - p0;
      for (int g = 0; g < hkv; ++g)
        for (int q = 0; q < np; ++q)
          items[static_cast<int64_t>(p0) * hkv + static_cast<int64_t>(g) * tot + within + q] =
              make_int2(s, (g << 16) | q);
    }
  }

  // ---- the work list, longest items first ----
  for (int s = tid; s < S && (!locality || casc); s += 1024) {
    const int L = clamp_len(lens[s], max_blocks, nullptr);
    const int Ls = L - (casc ? sspan[s] : 0);
    const int full = Ls / part, rem = Ls - full * part;
    if (full) {
      int at = atomicAdd(&cursor[full_bucket], full * hkv);
      for (int g = 0; g < hkv; ++g)
        for (int q = 0; q < full; ++q) items[at++] = make_int2(s, (g << 16) | q);
    }
    if (rem) {
      const int at = atomicAdd(&cursor[bucket_of((rem + unit - 1) / unit)], hkv);
      for (int g = 0; g < hkv; ++g) items[at + g] = make_int2(s, (g << 16) | full);
    }
    if (L == 0) {
      const int at = atomicAdd(&cursor[bucket_of(0)], hkv);
      for (int g = 0; g < hkv; ++g) items[at + g] = make_int2(s, g << 16);
    }
  }
  // ---- the shared-prefix items: (sub-run, KV-head group, partition) ----
  {
    const int nr = casc ? nruns : 0;
    int cnt = 0;
    const int cg = kv_heads >> hts;
    if (tid < nr) cnt = cg * ((rspan[tid] + pp_len - 1) / pp_len);
    const int incl = block_scan<false>(cnt, warp_tot);  // (nr <= 512 < 1024)
    if (tid < nr) roff[tid] = incl - cnt;
    __shared__ int ptotal;
    if (tid == 1023) {
      header[4] = incl;  // shared-prefix items
      ptotal = incl;
    }
    __syncthreads();
    // item i: the sub-run whose first item is the last one <= i (binary
    // search), then KV-head group and partition within it; consecutive
    // threads write consecutive items
    for (int i = tid; i < ptotal; i += 1024) {
      int lo = 0, hi = nr - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (roff[mid] <= i) lo = mid; else hi = mid - 1;
      }
      const int np = (rspan[lo] + pp_len - 1) / pp_len;
      const int o = i - roff[lo];
      pitems[i] = make_int2(lo, ((o / np) << 16) | (o % np));
    }
  }
  for (int i = tid; i < S * kv_heads; i += 1024) merge_cnt[i] = 0;
  // The plan is a programmatic dependent of the kernel before it (the cache
  // write that puts this step's tokens in the pool, or a prefill): it reads
  // only the tables and lengths, so it runs while that kernel finishes, and
  // it completes only after that kernel has -- the decode kernel, which waits
  // for this grid, then sees the pool as written.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace

int launch_decode_plan(const DecodeArgs& a) {
  // a programmatic dependent of the previous kernel on the stream (see the end
  // of the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(1024);
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, decode_plan_kernel, a.context_lens, a.block_tables, a.num_seqs,
                         a.max_blocks, a.pool.num_kv_heads / a.item_heads, a.pool.num_kv_heads,
                         a.min_part, a.max_part, a.target_items, num_sms(),
                         a.num_q_heads / a.pool.num_kv_heads, a.casc_cols, a.ws.header,
                         a.ws.part_base, a.ws.items, a.ws.merge_cnt, a.ws.seq_span, a.ws.seq_pp,
                         a.ws.runs, a.ws.pitems, a.err) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace pa
