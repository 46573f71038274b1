// Fused next-token sampling: temperature, Top-K, Top-P and the draw in one
// kernel, one CTA per row, without sorting the vocabulary ("vLLM 基本原理",
// FlashInfer 采样器: the fused kernel avoids sorting the logits and is
// statistically equivalent to the sort-based sampler).
//
// Each logit is mapped to a 32-bit key that orders like the float.  The K-th
// largest key is found by a radix select (four passes over the row, 8 bits at
// a time, a 256-bin count histogram each); the Top-P cut is a second radix
// select over the same keys whose histograms hold probability mass instead of
// counts.  Masses are exp((x - max) / T) in 32.32 fixed point, summed as
// 64-bit integers, so every sum and comparison is exact and the result does not
// depend on the order the threads add in: the same inputs always draw the
// same token.  The draw is inverse-CDF in vocabulary order: the first kept
// token whose running mass exceeds floor(u * total).
//
// Semantics (the readings of the page's sampler):
//   T <= 0: greedy, the largest logit, lowest index among equals.
//   0 < K < V: keep the tokens whose logit is at least the K-th largest.
//   P < 1: over those, keep the tokens in decreasing logit order until their
//   mass reaches P of the kept mass, with every token tied with the last one.
//   NaN logits are never drawn (their key is the smallest).
#include <cstdint>

#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "../../include/pa_sampler.h"

namespace pa {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCand = 4096;   // candidates the small-K path keeps in shared memory
constexpr int kFastK = 1024;  // Top-K values the small-K path takes

__device__ __forceinline__ uint32_t key_of(float x) {
  if (x != x) return 0u;  // NaN: below everything
  uint32_t b = __float_as_uint(x);
  if ((b << 1) == 0u) b = 0u;  // -0 is the same logit as +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float float_of(uint32_t k) {
  const uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(b);
}

// Calls f(value, index) for every element of row x[0, V), each thread keeping
// kInflight loads in flight: 16-byte vectors when the row is 16-byte aligned
// (128 KiB in flight per CTA: one CTA per row streams a row at about its SM's
// share of HBM), single floats otherwise.  Each thread sees its elements in
// increasing index order.
constexpr int kInflight = 8;
template <typename F>
__device__ __forceinline__ void for_each_logit(const float* __restrict__ x, int V, F f) {
  const int tid = threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    int i = tid;
    for (; i + (kInflight - 1) * kThreads < V4; i += kInflight * kThreads) {
      float4 a[kInflight];
#pragma unroll
      for (int q = 0; q < kInflight; ++q) a[q] = __ldg(x4 + i + q * kThreads);
#pragma unroll
      for (int q = 0; q < kInflight; ++q) {
        const int b = 4 * (i + q * kThreads);
        f(a[q].x, b);
        f(a[q].y, b + 1);
        f(a[q].z, b + 2);
        f(a[q].w, b + 3);
      }
    }
    for (; i < V4; i += kThreads) {
      const float4 a = __ldg(x4 + i);
      f(a.x, 4 * i);
      f(a.y, 4 * i + 1);
      f(a.z, 4 * i + 2);
      f(a.w, 4 * i + 3);
    }
    for (int j = 4 * V4 + tid; j < V; j += kThreads) f(x[j], j);
    return;
  }
  int i = tid;
  for (; i + (kInflight - 1) * kThreads < V; i += kInflight * kThreads) {
    float a[kInflight];
#pragma unroll
    for (int q = 0; q < kInflight; ++q) a[q] = x[i + q * kThreads];
#pragma unroll
    for (int q = 0; q < kInflight; ++q) f(a[q], i + q * kThreads);
  }
  for (; i < V; i += kThreads) f(x[i], i);
}

// As for_each_logit, but hands 16-byte vectors to f4(vector, index of its
// first element) and single elements to f1(value, index).
template <typename F4, typename F1>
__device__ __forceinline__ void for_each_logit4(const float* __restrict__ x, int V, F4 f4, F1 f1) {
  const int tid = threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) == 0) {
    const float4* x4 = reinterpret_cast<const float4*>(x);
    const int V4 = V >> 2;
    int i = tid;
    for (; i + (kInflight - 1) * kThreads < V4; i += kInflight * kThreads) {
      float4 a[kInflight];
#pragma unroll
      for (int q = 0; q < kInflight; ++q) a[q] = __ldg(x4 + i + q * kThreads);
#pragma unroll
      for (int q = 0; q < kInflight; ++q) f4(a[q], 4 * (i + q * kThreads));
    }
    for (; i < V4; i += kThreads) f4(__ldg(x4 + i), 4 * i);
    for (int j = 4 * V4 + tid; j < V; j += kThreads) f1(x[j], j);
    return;
  }
  for_each_logit(x, V, f1);
}

// Mass of logit x in 32.32 fixed point: exp2((x - xmax) * scale) * 2^32.
__device__ __forceinline__ uint64_t mass_of(float x, float xmax, float scale) {
  if (x != x) return 0ull;
  const float e = exp2f((x - xmax) * scale);  // in [0, 1]
  return static_cast<uint64_t>(__float2ull_rn(e * 4294967296.0f));
}

// Warp 0 scans a 256-bin histogram from the highest bin down and returns the
// first nonempty bin at which the running total reaches `need`, and the total
// of the bins above it.  The caller has made sure the total reaches `need`.
template <typename T>
__device__ void pick_bin(const T* hist, T need, int* bin_out, T* above_out) {
  const int lane = threadIdx.x & 31;
  T part = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) part += hist[255 - 8 * lane - j];
  T incl = part;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const unsigned hit = __ballot_sync(0xffffffffu, incl >= need && part > 0);
  const int L = hit ? __ffs(hit) - 1 : 31;
  if (lane == L) {
    T c = incl - part;
    int b = 255 - 8 * lane - 7;
    T above = c;
    for (int j = 0; j < 8; ++j) {
      const int bb = 255 - 8 * lane - j;
      const T h = hist[bb];
      if (h > 0 && c + h >= need) {
        b = bb;
        above = c;
        break;
      }
      c += h;
    }
    *bin_out = b;
    *above_out = above;
  }
}

// Bitonic sort of v[0, n2) (n2 a power of two <= kCand) by all threads of the CTA;
// descending if `desc`.  Ends with a barrier.
__device__ void block_sort(uint64_t* v, int n2, bool desc) {
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += kThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = v[i], b = v[ixj];
          const bool up = ((i & k) == 0) != desc;  // this pair's order: ascending if up
          if (up ? (a > b) : (a < b)) {
            v[i] = b;
            v[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Sort of the n <= kThreads distinct entries v[0, n) by rank: thread t counts
// the entries ahead of v[t] and writes it to that position of tmp (which must
// not overlap v[0, n)), then v takes tmp.  Descending if `desc`.  Two barriers
// in all, against the bitonic network's one per stage.  Ends with a barrier.
__device__ void rank_sort(uint64_t* v, int n, uint64_t* tmp, bool desc) {
  const int t = threadIdx.x;
  if (t < n) {
    const uint64_t x = v[t];
    int r = 0;
    int j = 0;
    for (; j + 8 <= n; j += 8) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint64_t y = v[j + q];
        r += desc ? (y > x) : (y < x);
      }
    }
    for (; j < n; ++j) {
      const uint64_t y = v[j];
      r += desc ? (y > x) : (y < x);
    }
    tmp[r] = x;
  }
  __syncthreads();
  if (t < n) v[t] = tmp[t];
  __syncthreads();
}

// Inclusive scan of one uint64 per thread over the CTA; `tot` gets the total.
__device__ uint64_t block_scan64(uint64_t x, uint64_t* wbuf, uint64_t* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wbuf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint64_t w = wbuf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wbuf[lane] = w;
  }
  __syncthreads();
  const uint64_t r = x + (warp > 0 ? wbuf[warp - 1] : 0ull);
  *tot = wbuf[kWarps - 1];
  __syncthreads();
  return r;
}

// The cuts and the draw of the small-K path by one warp, for n <= kWarpTail
// candidates sorted by (key, -index) descending in cand[0, n): Top-K keeps the
// first K and every tie with the K-th; Top-P keeps the shortest prefix whose
// mass reaches P of the kept mass, and its ties; the draw is inverse-CDF in
// vocabulary order, each kept entry's index-order prefix mass counted over
// the kept entries.  `mass` is scratch for n masses.  Lane l holds entries
// 8l .. 8l + 7 (so sorted order is lane-major).
constexpr int kWarpTail = 256;
__device__ void warp_tail(const uint64_t* cand, int n, int K, float P, float u, float xmax,
                          float scale, uint64_t* mass, int32_t* token) {
  const int lane = threadIdx.x & 31;
  const uint32_t tk = static_cast<uint32_t>(cand[K - 1] >> 32);
  uint32_t key[8];
  int first_below = n;  // the first entry past the K-th that is below it
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = 8 * lane + j;
    key[j] = e < n ? static_cast<uint32_t>(cand[e] >> 32) : 0u;
    if (e >= K && e < n && key[j] < tk) first_below = min(first_below, e);
  }
  const int m = __reduce_min_sync(0xffffffffu, first_below);
  uint64_t ms[8], lsum = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ms[j] = 8 * lane + j < m ? mass_of(float_of(key[j]), xmax, scale) : 0ull;
    lsum += ms[j];
  }
  uint64_t incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint64_t mk = __shfl_sync(0xffffffffu, incl, 31);
  int m2 = m;
  if (P < 1.f) {
    const double want = static_cast<double>(P > 0.f ? P : 0.f) * static_cast<double>(mk);
    uint64_t need = static_cast<uint64_t>(ceil(want));
    if (need < 1) need = 1;
    // the first entry at which the running mass reaches `need` (the last one
    // if rounding keeps the run short of it), then its ties
    uint64_t run = incl - lsum;
    int cut_l = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = 8 * lane + j;
      if (e < m && run < need && run + ms[j] >= need) cut_l = min(cut_l, e);
      run += ms[j];
    }
    int cut = __reduce_min_sync(0xffffffffu, cut_l);
    if (cut > m - 1) cut = m - 1;
    const uint32_t cutkey = static_cast<uint32_t>(cand[cut] >> 32);
    int tie_l = m;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = 8 * lane + j;
      if (e > cut && e < m && key[j] < cutkey) tie_l = min(tie_l, e);
    }
    m2 = __reduce_min_sync(0xffffffffu, tie_l);
  }
  // the draw: kept entries e < m2, in vocabulary order
  uint64_t total = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = 8 * lane + j;
    if (e >= m2) ms[j] = 0ull;
    if (e < n) mass[e] = ms[j];
    total += ms[j];
  }
  for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  __syncwarp();
  const uint64_t tg = static_cast<uint64_t>(static_cast<double>(u) * static_cast<double>(total));
  const uint64_t tgt = tg < total ? tg : total - 1;
  // each kept entry's mass before it in vocabulary order, a lane per entry
  // (entries e0 + lane of each 32): the entry whose span holds tgt is drawn
  for (int e0 = 0; e0 < m2; e0 += 32) {
    const int e = e0 + lane;
    const bool live = e < m2;
    const uint32_t ie = live ? 0xffffffffu - static_cast<uint32_t>(cand[e]) : 0xffffffffu;
    const uint64_t me = live ? mass[e] : 0ull;
    uint64_t pre = 0;
#pragma unroll 4
    for (int f = 0; f < m2; ++f)
      pre += (0xffffffffu - static_cast<uint32_t>(cand[f])) < ie ? mass[f] : 0ull;
    if (live && me > 0 && pre <= tgt && pre + me > tgt) *token = static_cast<int32_t>(ie);
  }
}

struct Smem {
  uint32_t hcnt[256];
  uint64_t hmass[256];
  uint64_t wsum[kWarps];
  uint64_t cand[kCand];       // small-K path: candidates, packed for sorting
  uint32_t tmax[kThreads];    // each thread's largest key (K > 256)
  unsigned long long red64;
  int count;
  int overflow;
  int cut;
  int cutk, cutp, cutt;  // first entry below the K-th / the Top-P cut / its ties
  int bin;
  uint32_t above_cnt;
  uint64_t above_mass;
};

__global__ void __launch_bounds__(kThreads, 1) sample_kernel(const float* __restrict__ logits,
                                                          int64_t row_stride, int V,
                                                          const float* __restrict__ temperature,
                                                          const int32_t* __restrict__ top_k,
                                                          const float* __restrict__ top_p,
                                                          const float* __restrict__ uniform,
                                                          int32_t* __restrict__ tokens) {
  __shared__ Smem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const float* x = logits + static_cast<int64_t>(row) * row_stride;
  const float T = temperature[row];
  const int K = top_k[row];
  const float P = top_p[row];
  float u = uniform[row];
  u = (u >= 0.f && u < 1.f) ? u : 0.f;

  // ---- pass 1: each thread's four largest groups -- a group is a 16-byte
  // vector of four logits, or a single logit where the row is not 16-byte
  // aligned and in its tail -- by their largest value, the first group among
  // equal ones.  The common case (a vector below the fourth kept one) costs
  // three maxima and a compare. ----
  constexpr int kNone = 0x7fffffff;  // group index of an empty slot
  const int V4 = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 ? (V >> 2) : 0;  // vector elements: [0, 4 V4)
  float g0 = -CUDART_INF_F, g1 = -CUDART_INF_F, g2 = -CUDART_INF_F, g3 = -CUDART_INF_F;
  int b0 = kNone, b1 = kNone, b2 = kNone, b3 = kNone;
  // groups arrive in increasing index order, so `>` keeps the first of equals;
  // NaN and -inf maxima never enter
  auto add_group = [&](float m, int b) {
    if (m > g3) {
      if (m > g2) {
        g3 = g2;
        b3 = b2;
        if (m > g1) {
          g2 = g1;
          b2 = b1;
          if (m > g0) {
            g1 = g0;
            b1 = b0;
            g0 = m;
            b0 = b;
          } else {
            g1 = m;
            b1 = b;
          }
        } else {
          g2 = m;
          b2 = b;
        }
      } else {
        g3 = m;
        b3 = b;
      }
    }
  };
  for_each_logit4(
      x, V, [&](float4 a, int b) { add_group(fmaxf(fmaxf(a.x, a.y), fmaxf(a.z, a.w)), b); },
      [&](float v, int i) { add_group(v, i); });
  // the elements of group b (4 or 1) into v; returns how many
  auto load_group = [&](int b, float (&v)[4]) {
    if (b < 4 * V4) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(x) + (b >> 2));
      v[0] = a.x;
      v[1] = a.y;
      v[2] = a.z;
      v[3] = a.w;
      return 4;
    }
    v[0] = x[b];
    return 1;
  };
  // The values of the two largest kept groups, loaded now so the loads are in
  // flight while the row maximum and the Top-K bound are found (the others
  // are loaded when needed: rarely does a thread keep more than two groups at
  // or above the bound).
  float pv0[4], pv1[4];
  int pw0 = 0, pw1 = 0;
  if (b0 != kNone) pw0 = load_group(b0, pv0);
  if (b1 != kNone) pw1 = load_group(b1, pv1);
  // this thread's largest key; its index (bi) is known here only when every
  // element of the thread is -inf or NaN (or it has none)
  uint32_t bk = 0;
  int bi = kNone;
  if (b0 != kNone) {
    bk = key_of(g0);
  } else {
    for_each_logit(x, V, [&](float v, int i) {
      const uint32_t k = key_of(v);
      if (k > bk || (k == bk && i < bi)) {
        bk = k;
        bi = i;
      }
    });
  }
  const uint32_t kown = bk;  // this thread's largest key (the reduction below overwrites bk)
  bk = __reduce_max_sync(0xffffffffu, bk);
  __shared__ uint32_t best;
  __shared__ int best_i;
  if (tid == 0) {
    best = 0u;
    best_i = 0x7fffffff;
  }
  __syncthreads();
  if (lane == 0) atomicMax(&best, bk);
  __syncthreads();
  const uint32_t kmax = best;
  // The row's argmax, the first index of the largest key: every thread whose
  // own largest key it is finds its first such element (in its first group of
  // that maximum: groups come in index order) and the least index wins.  Only
  // the paths that use it call this (every thread, at one point).
  auto block_argmax = [&]() -> int {
    int ci = 0x7fffffff;
    if (kown == kmax) {
      if (b0 != kNone) {
#pragma unroll
        for (int j = 3; j >= 0; --j)
          if (j < pw0 && pv0[j] == g0) ci = b0 + j;
      } else {
        ci = bi;
      }
    }
    ci = __reduce_min_sync(0xffffffffu, ci);
    if (lane == 0 && ci != 0x7fffffff) atomicMin(&best_i, ci);
    __syncthreads();
    return best_i;
  };
  if (!(T > 0.f) || kmax == 0u) {
    const int argmax = block_argmax();
    if (tid == 0) tokens[row] = argmax;
    return;
  }
  const float xmax = float_of(kmax);
  const float scale = kLog2e / T;

  // ---- small K: candidates in shared memory ----
  // t0 below is a lower bound of the K-th largest key, so every Top-K survivor
  // has key >= t0.  When those elements fit in shared memory, everything else
  // is done there: sort them, cut at the K-th, cut at Top-P, draw.
  if (K > 0 && K <= kFastK && K < V) {
    // t0.  K <= 256: each warp sorts its 32 threads' maxima (descending,
    // across the lanes) and puts its kw = min(32, 2 ceil(K / 32)) largest into
    // a pool of 32 kw >= K keys; t0 is the K-th largest key of the pool, by
    // rank (a subset's K-th largest is at most the whole set's, and the pool
    // misses a top maximum only when a warp holds more than kw of them).
    // Larger K: the K-th largest of all 1024 maxima by radix select.  Either
    // way K distinct elements are at or above t0.
    uint32_t t0 = 0;
    if (tid == 0) {
      sm.count = 0;
      sm.overflow = 0;
      sm.cutk = sm.cutp = sm.cutt = 0x7fffffff;
    }
    if (K <= 256) {
      uint32_t v = kown;
#pragma unroll
      for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
          const uint32_t o = __shfl_xor_sync(0xffffffffu, v, j);
          // blocks of k lanes alternate descending / ascending; the last is descending
          v = (((lane & j) == 0) == ((lane & k) == 0)) ? max(v, o) : min(v, o);
        }
      }
      const int kw = min(32, 2 * ((K + 31) / 32));
      // the pool: free space of the candidate array until the candidates come
      uint32_t* pool = reinterpret_cast<uint32_t*>(sm.cand + kCand / 2);
      if (lane < kw) pool[warp * kw + lane] = v;
      __syncthreads();
      const int np = kWarps * kw;
      if (tid < np) {
        const uint32_t x = pool[tid];
        int r = 0;
        for (int u = 0; u < np; ++u) {
          const uint32_t y = pool[u];
          r += (y > x) || (y == x && u < tid);
        }
        if (r == K - 1) sm.bin = static_cast<int>(x);
      }
      __syncthreads();
      t0 = static_cast<uint32_t>(sm.bin);
    } else {
      sm.tmax[tid] = kown;
      uint32_t prefix = 0, pmask = 0, need = static_cast<uint32_t>(K);
      for (int dgt = 3; dgt >= 0; --dgt) {
        if (tid < 256) sm.hcnt[tid] = 0;
        __syncthreads();
        const int sh = 8 * dgt;
        const uint32_t k = sm.tmax[tid];
        if ((k & pmask) == prefix) atomicAdd(&sm.hcnt[(k >> sh) & 255u], 1u);
        __syncthreads();
        if (warp == 0) pick_bin<uint32_t>(sm.hcnt, need, &sm.bin, &sm.above_cnt);
        __syncthreads();
        prefix |= static_cast<uint32_t>(sm.bin) << sh;
        pmask |= 255u << sh;
        need -= sm.above_cnt;
        __syncthreads();
      }
      t0 = prefix;
    }
    // (key, -index): descending order is by logit, then by index
    auto pack = [](uint32_t k, int i) {
      return (static_cast<uint64_t>(k) << 32) | (0xffffffffu - static_cast<uint32_t>(i));
    };
    // Every element at or above t0 lies in a group whose maximum is, so in one
    // of its thread's four kept groups -- unless the fourth is at or above t0
    // too (a fifth may be) or t0 admits -inf or NaN logits, which no group
    // maximum tracks: then the row is read again.
    if ((b3 != kNone && key_of(g3) >= t0) || t0 <= key_of(-CUDART_INF_F)) sm.overflow = 1;
    auto gather = [&](float gm, int gb, const float* pv, int pw) {
      if (gb == kNone || key_of(gm) < t0) return;
      float v[4];
      int w = pw;
      if (pv) {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = pv[j];
      } else {
        w = load_group(gb, v);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t k = j < w ? key_of(v[j]) : 0u;
        if (j < w && k >= t0) {
          const int pos = atomicAdd(&sm.count, 1);
          if (pos < kCand) sm.cand[pos] = pack(k, gb + j);
        }
      }
    };
    gather(g0, b0, pv0, pw0);
    gather(g1, b1, pv1, pw1);
    gather(g2, b2, nullptr, 0);
    gather(g3, b3, nullptr, 0);
    __syncthreads();
    if (sm.overflow) {
      __syncthreads();
      if (tid == 0) sm.count = 0;
      __syncthreads();
      auto collect = [&](float v, int i) {
        const uint32_t k = key_of(v);
        if (k >= t0) {
          const int pos = atomicAdd(&sm.count, 1);
          if (pos < kCand) sm.cand[pos] = pack(k, i);
        }
      };
      for_each_logit(x, V, collect);
      __syncthreads();
    }
    const int n = sm.count;
    if (n <= kCand) {
      int n2 = 1;
      while (n2 < n) n2 <<= 1;
      if (n <= kThreads) {
        rank_sort(sm.cand, n, sm.cand + kThreads, true);
      } else {
        for (int i = n + tid; i < n2; i += kThreads) sm.cand[i] = 0ull;  // below every real entry
        __syncthreads();
        block_sort(sm.cand, n2, true);
      }
      if (n <= kWarpTail) {
        // Up to kWarpTail candidates (the usual case): one warp takes the
        // cuts and the draw with shuffles and warp reductions, no barriers.
        if (warp == 0) warp_tail(sm.cand, n, K, P, u, xmax, scale, sm.cand + kCand / 2, tokens + row);
        return;
      }
      const uint32_t tk = static_cast<uint32_t>(sm.cand[K - 1] >> 32);
      // survivors of Top-K: the leading K entries and every tie with the K-th,
      // i.e. up to the first entry below it
      for (int c = K + tid; c < n; c += kThreads)
        if (static_cast<uint32_t>(sm.cand[c] >> 32) < tk) atomicMin(&sm.cutk, c);
      __syncthreads();
      const int m = min(sm.cutk, n);
      // thread t owns sorted entries [4t, 4t + 4)
      const int j0 = 4 * tid;
      uint64_t ms[4];
      uint64_t mine = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = j0 + q;
        ms[q] = j < m ? mass_of(float_of(static_cast<uint32_t>(sm.cand[j] >> 32)), xmax, scale) : 0ull;
        mine += ms[q];
      }
      uint64_t mk = 0;
      const uint64_t incl = block_scan64(mine, sm.wsum, &mk);
      int m2 = m;
      if (P < 1.f) {
        const double want = static_cast<double>(P > 0.f ? P : 0.f) * static_cast<double>(mk);
        uint64_t need = static_cast<uint64_t>(ceil(want));
        if (need < 1) need = 1;
        // the first sorted entry at which the running mass reaches `need`
        // (the last one if rounding keeps the run short of it)
        uint64_t run = incl - mine;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = j0 + q;
          if (j < m && run < need && run + ms[q] >= need) atomicMin(&sm.cutp, j);
          run += ms[q];
        }
        __syncthreads();
        const int cut = min(sm.cutp, m - 1);
        // and every tie with it: up to the first entry below it
        const uint32_t cutkey = static_cast<uint32_t>(sm.cand[cut] >> 32);
        for (int c = cut + 1 + tid; c < m; c += kThreads)
          if (static_cast<uint32_t>(sm.cand[c] >> 32) < cutkey) atomicMin(&sm.cutt, c);
        __syncthreads();
        m2 = min(sm.cutt, m);
      }
      // the draw: kept entries re-packed as (index, key) and sorted by index
      for (int i = tid; i < n2; i += kThreads) {
        const uint64_t e = sm.cand[i];
        sm.cand[i] = i < m2 ? ((static_cast<uint64_t>(0xffffffffu - static_cast<uint32_t>(e)) << 32) |
                               (e >> 32))
                            : ~0ull;
      }
      __syncthreads();
      if (m2 <= kThreads)
        rank_sort(sm.cand, m2, sm.cand + kThreads, false);
      else
        block_sort(sm.cand, n2, false);
      uint64_t mine2 = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = j0 + q;
        ms[q] = j < m2 ? mass_of(float_of(static_cast<uint32_t>(sm.cand[j])), xmax, scale) : 0ull;
        mine2 += ms[q];
      }
      uint64_t total = 0;
      const uint64_t incl2 = block_scan64(mine2, sm.wsum, &total);
      const uint64_t tg = static_cast<uint64_t>(static_cast<double>(u) * static_cast<double>(total));
      const uint64_t tgt = tg < total ? tg : total - 1;
      uint64_t run = incl2 - mine2;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = j0 + q;
        if (j < m2 && ms[q] > 0 && run <= tgt && run + ms[q] > tgt)
          tokens[row] = static_cast<int32_t>(sm.cand[j] >> 32);
        run += ms[q];
      }
      return;
    }
    __syncthreads();
  }

  // ---- Top-K: the K-th largest key by radix select ----
  uint32_t tk = 0;
  if (K > 0 && K < V) {
    uint32_t prefix = 0, pmask = 0, need = static_cast<uint32_t>(K);
    for (int d = 3; d >= 0; --d) {
      for (int b = tid; b < 256; b += kThreads) sm.hcnt[b] = 0;
      __syncthreads();
      const int sh = 8 * d;
      for (int i = tid; i < V; i += kThreads) {
        const uint32_t k = key_of(x[i]);
        if ((k & pmask) == prefix) atomicAdd(&sm.hcnt[(k >> sh) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) pick_bin<uint32_t>(sm.hcnt, need, &sm.bin, &sm.above_cnt);
      __syncthreads();
      prefix |= static_cast<uint32_t>(sm.bin) << sh;
      pmask |= 255u << sh;
      need -= sm.above_cnt;
      __syncthreads();
    }
    tk = prefix;
  }

  // ---- Top-P: the cut key by a radix select over mass ----
  uint32_t tcut = tk;
  if (P < 1.f) {
    // mass of the Top-K survivors
    uint64_t s = 0;
    for (int i = tid; i < V; i += kThreads) {
      const float xi = x[i];
      if (key_of(xi) >= tk) s += mass_of(xi, xmax, scale);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) sm.wsum[warp] = s;
    __syncthreads();
    if (tid == 0) {
      uint64_t t = 0;
      for (int w = 0; w < kWarps; ++w) t += sm.wsum[w];
      sm.red64 = t;
    }
    __syncthreads();
    const uint64_t mk = sm.red64;
    const double want = static_cast<double>(P > 0.f ? P : 0.f) * static_cast<double>(mk);
    uint64_t need = static_cast<uint64_t>(ceil(want));
    if (need < 1) need = 1;
    uint32_t prefix = 0, pmask = 0;
    for (int d = 3; d >= 0; --d) {
      for (int b = tid; b < 256; b += kThreads) sm.hmass[b] = 0;
      __syncthreads();
      const int sh = 8 * d;
      for (int i = tid; i < V; i += kThreads) {
        const float xi = x[i];
        const uint32_t k = key_of(xi);
        if (k >= tk && (k & pmask) == prefix) {
          const uint64_t m = mass_of(xi, xmax, scale);
          if (m) atomicAdd(reinterpret_cast<unsigned long long*>(&sm.hmass[(k >> sh) & 255u]),
                           static_cast<unsigned long long>(m));
        }
      }
      __syncthreads();
      if (warp == 0) pick_bin<uint64_t>(sm.hmass, need, &sm.bin, &sm.above_mass);
      __syncthreads();
      prefix |= static_cast<uint32_t>(sm.bin) << sh;
      pmask |= 255u << sh;
      need -= sm.above_mass;
      __syncthreads();
    }
    tcut = prefix > tk ? prefix : tk;
  }

  // ---- the draw: inverse CDF in vocabulary order over keys >= tcut ----
  // (the argmax is the answer if rounding leaves no entry to draw)
  const int argmax = block_argmax();
  // warp w owns the contiguous segment [w * seg, (w + 1) * seg)
  const int seg = (V + kWarps - 1) / kWarps;
  const int lo = min(V, warp * seg), hi = min(V, lo + seg);
  uint64_t s = 0;
  for (int i = lo + lane; i < hi; i += 32) {
    const float xi = x[i];
    if (key_of(xi) >= tcut) s += mass_of(xi, xmax, scale);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) sm.wsum[warp] = s;
  __syncthreads();
  if (warp == 0) {
    const uint64_t mine = sm.wsum[lane];
    uint64_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint64_t total = __shfl_sync(0xffffffffu, incl, 31);
    const uint64_t target =
        static_cast<uint64_t>(static_cast<double>(u) * static_cast<double>(total));
    const uint64_t tgt = target < total ? target : (total ? total - 1 : 0);
    const unsigned hit = __ballot_sync(0xffffffffu, incl > tgt && mine > 0);
    const int W = hit ? __ffs(hit) - 1 : 0;
    const uint64_t excl_w = __shfl_sync(0xffffffffu, incl - mine, W);
    if (lane == 0) {
      sm.bin = W;           // the warp whose segment holds the draw
      sm.above_mass = excl_w;
      sm.red64 = tgt;
    }
  }
  __syncthreads();
  if (warp == sm.bin) {
    const uint64_t tgt = sm.red64;
    uint64_t run = sm.above_mass;
    int found = -1;
    for (int base = lo; base < hi && found < 0; base += 32) {
      const int i = base + lane;
      uint64_t m = 0;
      if (i < hi) {
        const float xi = x[i];
        if (key_of(xi) >= tcut) m = mass_of(xi, xmax, scale);
      }
      uint64_t incl = m;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, m > 0 && run + incl > tgt);
      if (hit) found = base + __ffs(hit) - 1;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) tokens[row] = found >= 0 ? found : argmax;
  }
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_sample(const float* logits, int64_t row_stride, int32_t num_rows, int32_t vocab,
                         const float* temperature, const int32_t* top_k, const float* top_p,
                         const float* uniform, int32_t* tokens, void* stream) {
  PA_NVTX_RANGE("pa_sample");
  if (num_rows < 0 || vocab <= 0 || row_stride < vocab) return PA_ERR_ARG;
  if (num_rows == 0) return PA_OK;
  if (!logits || !temperature || !top_k || !top_p || !uniform || !tokens) return PA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(logits) % alignof(float)) return PA_ERR_ARG;
  sample_kernel<<<num_rows, kThreads, 0, as_stream(stream)>>>(logits, row_stride, vocab,
                                                             temperature, top_k, top_p, uniform,
                                                             tokens);
  return launch_status();
}
