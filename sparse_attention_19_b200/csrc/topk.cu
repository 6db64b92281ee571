// topk.cu -- per-query top-k over the indexer scores.
//
// Row (b, i) sits at position t = q_offset + i and selects, among the n =
// min(t+1, Lk) scores I[t, 0..n), the m = min(k, n) largest, ties to the smaller
// position ("Отбор и основное внимание": the k KV entries with the largest
// I_{t,s}).  The result is written in ascending position order, -1 padded.
//
// Method (one CTA per row).  fp32 scores become order-preserving 32-bit keys
// (-0.0 is first canonicalised to +0.0).  The exact key of the m-th largest
// element (the threshold) is found by histogram refinement:
//   1. a strided sample of the row (1024 scores) gives a key range [lo, hi];
//   2. one pass over the row builds a 2048-bin histogram over that range (bin =
//      (key - lo) >> shift, so the bins follow the data rather than the float
//      exponent; keys outside the range are clamped into the end bins) and
//      yields the bin b that holds the m-th largest key and the count above it;
//   3. a second pass records every element of a bin above b in a bitmap (warp
//      ballots, no atomics) and collects the elements of bin b as candidates;
//      the threshold is then refined on the candidates in shared memory, with
//      2048-bin histograms over the candidates' own key range, down to an exact key.
// The output takes every element above the threshold and the first
// (m - #above) elements equal to it in position order: two bitmaps (above,
// equal) are scanned word by word with warp prefix sums, so positions come out
// sorted and ties resolve to smaller positions.  When bin b holds more elements
// than the candidate buffer (many equal scores), the refinement runs over the
// row instead and a final pass rebuilds both bitmaps.
// Rows up to cache_cap elements are kept in shared memory after the first pass;
// longer rows are re-read (from L2) by each pass.
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_internal.h"
#include "ptx.cuh"
#include "warp_select.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBinBits = 11;
constexpr int kBins = 1 << kBinBits;
constexpr int kUnroll = 8;           // 4-byte loads in flight per thread in the row passes
constexpr int kUnroll4 = 4;          // 16-byte loads in flight per thread in the histogram pass
constexpr int kSample = 1024;        // strided sample that sets the first histogram's range
constexpr int kSmallSelect = 64;     // a boundary bin this small is ranked directly by one warp
constexpr int kPassUnroll = 8;       // 16-byte loads in flight per thread in the single passes

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;                       // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is `key` (inverse of score_key; +0.0 for the key of zero).
// For non-NaN f, score_key(f) >= key exactly when f >= key_score(key): the key
// order is the float order with -0.0 equal to +0.0, as in float comparison.
__device__ __forceinline__ float key_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// The score at a selected position as the selection saw it: -0.0 reads as +0.0.
__device__ __forceinline__ float selected_score(const float* src, int s) {
  const float v = __ldg(src + s);
  return v == 0.f ? 0.f : v;
}

// Block-wide scratch for scans and reductions.
struct ScanScratch {
  uint32_t warp_tot[kWarps];
  uint32_t warp_a[kWarps], warp_b[kWarps];
  uint32_t bin, above, ncand;
  uint32_t bcount;             // keys in bin (find_bin)
};

// The keys of a small boundary bin, ranked by one warp (small_select).
struct SmallSel {
  uint32_t key[kSmallSelect];
  uint32_t n, thr, need;
};

// 16-byte multiple, so the arrays that follow it in dynamic shared memory stay aligned.
struct alignas(16) TopkShared {
  uint32_t hist[kBins];
  ScanScratch x;
  SmallSel small;
};

// Block-wide inclusive scan of one value per thread (thread order).
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_tot, uint32_t& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    uint32_t t = lane < kWarps ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < kWarps) warp_tot[lane] = t;   // inclusive warp prefix
  }
  __syncthreads();
  const uint32_t before = (w > 0) ? warp_tot[w - 1] : 0u;
  total = warp_tot[kWarps - 1];
  __syncthreads();
  return x + before;
}

// Find the bin b (searching from the top) where the running count from above first
// reaches `need`; records b and the count strictly above it in x.bin / x.above.
__device__ void find_bin(const uint32_t* hist, ScanScratch& x, uint32_t need) {
  constexpr int per = kBins / kThreads;            // bins per thread
  const int lo = threadIdx.x * per;
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < per; ++i) mine += hist[lo + i];
  uint32_t total;
  const uint32_t incl = block_inclusive_scan(mine, x.warp_tot, total);
  uint32_t acc = total - incl;                      // count in bins above this thread's range
#pragma unroll
  for (int i = per - 1; i >= 0; --i) {
    const uint32_t c = hist[lo + i];
    if (acc < need && acc + c >= need) {
      x.bin = (uint32_t)(lo + i);
      x.above = acc;
      x.bcount = c;
    }
    acc += c;
  }
  __syncthreads();
}

// The exact threshold inside a boundary bin [wlo, whi] that holds at most
// kSmallSelect keys (of key_of(0 .. count)): warp 0 ranks them directly and the
// block receives the need-th largest key (thr) and how many keys equal to it are
// still to be taken (need).  Replaces the remaining histogram levels.  Every
// thread of the block calls it.
template <typename KeyOf>
__device__ __forceinline__ void small_select(SmallSel& ss, int count, KeyOf key_of, uint32_t wlo, uint32_t whi,
                                             uint32_t& thr, uint32_t& need) {
  if (threadIdx.x == 0) ss.n = 0u;
  __syncthreads();
  for (int x = threadIdx.x; x < count; x += kThreads) {
    const uint32_t key = key_of(x);
    if (key >= wlo && key <= whi) {
      const uint32_t a = atomicAdd(&ss.n, 1u);
      if (a < (uint32_t)kSmallSelect) ss.key[a] = key;
    }
  }
  __syncthreads();
  const int m = (int)min(ss.n, (uint32_t)kSmallSelect);
  if (threadIdx.x < 32) {
    for (int a = (int)threadIdx.x; a < m; a += 32) {
      const uint32_t key = ss.key[a];
      uint32_t gt = 0, eq = 0;
      for (int b = 0; b < m; ++b) {
        const uint32_t v = ss.key[b];
        gt += v > key ? 1u : 0u;
        eq += v == key ? 1u : 0u;
      }
      if (gt < need && need <= gt + eq) {           // equal keys write the same values
        ss.thr = key;
        ss.need = need - gt;
      }
    }
  }
  __syncthreads();
  thr = ss.thr;
  need = ss.need;
}

// Right shift that maps a key range of width range+1 onto at most kBins bins.
__device__ __forceinline__ int bin_shift(uint32_t range) {
  return range == 0u ? 0 : max(0, 32 - __clz(range) - kBinBits);
}

// Block-wide min and max (every thread receives both).
__device__ __forceinline__ void block_min_max(ScanScratch& x, uint32_t& mn, uint32_t& mx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __syncthreads();                                  // earlier readers of warp_a / warp_b are done
  if (lane == 0) { x.warp_a[warp] = mn; x.warp_b[warp] = mx; }
  __syncthreads();
  mn = x.warp_a[0];
  mx = x.warp_b[0];
  for (int w = 1; w < kWarps; ++w) { mn = min(mn, x.warp_a[w]); mx = max(mx, x.warp_b[w]); }
}

__device__ __forceinline__ void clear_hist(uint32_t* hist) {
  for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0u;
  __syncthreads();
}

// Visits every position s < n of the row in warp-aligned groups of 32 (lane =
// s % 32, so one warp's ballot covers one bitmap word), with kUnroll groups per
// thread in flight: f(s, valid, key), key = 0 when !valid.  Every lane of a warp
// calls f for the same groups.
template <typename KeyAt, typename F>
__device__ __forceinline__ void row_pass(int n, KeyAt key_at, F f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = warp * 32; base < n; base += kThreads * kUnroll) {
    uint32_t key[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + u * kThreads + lane;
      key[u] = (s < n) ? key_at(s) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int g = base + u * kThreads;           // warp-uniform
      if (g < n) f(g + lane, g + lane < n, key[u]);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 2) topk_kernel(const TopkParams p) {
  griddep_launch_dependents();
  griddep_wait();                                   // the scores are complete
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* cache = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));
  uint32_t* gt_bits = cache + p.cache_cap;          // cache_cap and bit_words are multiples of 4
  uint32_t* eq_bits = gt_bits + p.bit_words;
  uint2* cand = reinterpret_cast<uint2*>(eq_bits + p.bit_words);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x;                       // b * Lq + i
  const int i = row % p.Lq;
  const long long t = (long long)p.q_offset + i;
  const int n = (int)((t + 1 < p.Lk) ? t + 1 : p.Lk);
  const int k = p.k;
  int32_t* out = p.indices + (size_t)row * k;
  float* sel_out = p.sel_scores ? p.sel_scores + (size_t)row * k : nullptr;
  const float* src = p.scores + (size_t)row * p.Lk;

  if (n <= k) {                                     // everything up to t is selected
    for (int x = threadIdx.x; x < k; x += kThreads) {
      out[x] = (x < n) ? x : -1;
      if (sel_out) sel_out[x] = (x < n) ? selected_score(src, x) : -INFINITY;
    }
    return;
  }
  const bool cached = n <= p.cache_cap;
  auto key_at = [&](int s) -> uint32_t { return cached ? cache[s] : score_key(__ldg(src + s)); };
  auto load_key = [&](int s) -> uint32_t { return score_key(__ldg(src + s)); };

  // ---- 1. key range of a strided sample (kept in the candidate buffer for step 1b)
  const int ns = n < kSample ? n : kSample;
  const bool try_single = p.sampled && !cached && p.cand_cap >= kSample;
  uint32_t smin = 0xffffffffu, smax = 0u;
  for (int j = threadIdx.x; j < ns; j += kThreads) {
    const uint32_t key = load_key((int)(((long long)j * n) / ns));
    if (try_single) cand[j].x = key;
    smin = min(smin, key);
    smax = max(smax, key);
  }
  block_min_max(sh.x, smin, smax);
  const uint32_t lo = smin;
  const int shift = bin_shift(smax - smin);
  auto bin_of = [lo, shift](uint32_t key) -> uint32_t {
    return key < lo ? 0u : min((uint32_t)(kBins - 1), (key - lo) >> shift);
  };

  // ---- 1b. long rows, one pass: a threshold theta at the sample's j-th largest key
  // (its bin's lower edge), j six standard deviations above the count the sample
  // is expected to hold above the k-th largest key of the row.  Every key >= theta
  // is kept with its position; if at least k and at most cand_cap of them are
  // found, the row's top-k is among them (each key below theta has k keys above
  // it), and the threshold is resolved on the candidates alone.  Otherwise the
  // row takes the two-pass route below (a rare event by construction, or rows of
  // many equal keys).
  bool single = false;
  uint32_t nsingle = 0;
  if (try_single) {
    const float mu = (float)ns * (float)k / (float)n;
    const float sig = sqrtf(mu * (1.f - (float)k / (float)n));
    const uint32_t j = (uint32_t)ceilf(mu + 6.f * sig + 2.f);
    if (j < (uint32_t)ns) {
      clear_hist(sh.hist);
      for (int x = threadIdx.x; x < ns; x += kThreads) atomicAdd(&sh.hist[bin_of(cand[x].x)], 1u);
      __syncthreads();
      find_bin(sh.hist, sh.x, j);
      // The first histogram's bins are coarse when the sample spans both signs (its
      // key range then covers half the key space), and the lower edge of the bin
      // alone can let through more keys than the buffer holds; a second histogram
      // of the sample keys inside that bin places theta just below the sample's
      // j-th largest key.  (Any theta is safe: the count check below decides.)
      uint32_t theta;
      {
        const uint32_t tb = sh.x.bin, need2 = j - sh.x.above;
        const uint32_t wlo = lo + (tb << shift);
        const unsigned long long top = (unsigned long long)wlo + (1ull << shift) - 1ull;
        const uint32_t whi = (tb == (uint32_t)(kBins - 1) || top > smax) ? smax : (uint32_t)top;
        const int sh2 = bin_shift(whi - wlo);
        clear_hist(sh.hist);
        for (int x = threadIdx.x; x < ns; x += kThreads) {
          const uint32_t key = cand[x].x;
          if (key >= wlo && key <= whi) atomicAdd(&sh.hist[(key - wlo) >> sh2], 1u);
        }
        __syncthreads();
        find_bin(sh.hist, sh.x, need2);
        theta = wlo + (sh.x.bin << sh2);
      }
      const int W = (n + 31) >> 5;
      for (int x = threadIdx.x; x < W; x += kThreads) { gt_bits[x] = 0u; eq_bits[x] = 0u; }
      if (threadIdx.x == 0) sh.x.ncand = 0u;
      __syncthreads();
      auto keep = [&](int s, uint32_t key) {
        if (key >= theta) {
          const uint32_t at = atomicAdd(&sh.x.ncand, 1u);
          if (at < (uint32_t)p.cand_cap) cand[at] = make_uint2(key, (uint32_t)s);
        }
      };
      if (p.vec4) {
        // Float compares against theta's float value (no key conversion per score)
        // and one shared atomic per warp and step for the kept keys' slots.
        const float4* src4 = reinterpret_cast<const float4*>(src);
        const int nq = n >> 2;
        const float theta_f = key_score(theta);
        for (int q00 = warp * 32; q00 < nq; q00 += kThreads * kPassUnroll) {   // warp-uniform bound
          const int q0 = q00 + lane;
          float4 f[kPassUnroll];
#pragma unroll
          for (int u = 0; u < kPassUnroll; ++u) {
            const int q = q0 + u * kThreads;
            f[u] = (q < nq) ? __ldg(src4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          uint32_t mine = 0;
#pragma unroll
          for (int u = 0; u < kPassUnroll; ++u) {
            if (q0 + u * kThreads < nq) {
              mine += f[u].x >= theta_f ? 1u : 0u;
              mine += f[u].y >= theta_f ? 1u : 0u;
              mine += f[u].z >= theta_f ? 1u : 0u;
              mine += f[u].w >= theta_f ? 1u : 0u;
            }
          }
          uint32_t incl = mine;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const uint32_t wtot = __shfl_sync(0xffffffffu, incl, 31);
          if (wtot == 0u) continue;
          uint32_t at = 0;
          if (lane == 31) at = atomicAdd(&sh.x.ncand, wtot);
          at = __shfl_sync(0xffffffffu, at, 31) + incl - mine;
          if (mine != 0u) {
#pragma unroll
            for (int u = 0; u < kPassUnroll; ++u) {
              const int q = q0 + u * kThreads;
              if (q < nq) {
                const float fx[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  if (fx[c] >= theta_f) {                // the predicate the count used
                    if (at < (uint32_t)p.cand_cap) cand[at] = make_uint2(score_key(fx[c]), (uint32_t)(4 * q + c));
                    ++at;
                  }
                }
              }
            }
          }
        }
        for (int s = (nq << 2) + (int)threadIdx.x; s < n; s += kThreads) keep(s, load_key(s));
      } else {
        row_pass(n, load_key, [&](int s, bool valid, uint32_t key) {
          if (valid) keep(s, key);
        });
      }
      __syncthreads();
      nsingle = sh.x.ncand;
      single = nsingle >= (uint32_t)k && nsingle <= (uint32_t)p.cand_cap;
      __syncthreads();
    }
  }

  uint32_t need = (uint32_t)k;                       // n > k, so m = k
  uint32_t b = 0, cnt_b = nsingle;
  bool fits = true;
  if (!single) {
  // ---- 2. histogram over the sampled range (outliers clamped into the end bins)
  clear_hist(sh.hist);
  if (p.vec4) {
    // 16-byte loads (rows start 16-byte aligned): four scores per thread per step.
    const float4* src4 = reinterpret_cast<const float4*>(src);
    const int nq = n >> 2;
    for (int q0 = threadIdx.x; q0 < nq; q0 += kThreads * kUnroll4) {
      float4 f[kUnroll4];
#pragma unroll
      for (int u = 0; u < kUnroll4; ++u) {
        const int q = q0 + u * kThreads;
        f[u] = (q < nq) ? __ldg(src4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kUnroll4; ++u) {
        const int q = q0 + u * kThreads;
        if (q >= nq) break;
        const uint4 key = make_uint4(score_key(f[u].x), score_key(f[u].y), score_key(f[u].z), score_key(f[u].w));
        if (cached) reinterpret_cast<uint4*>(cache)[q] = key;
        atomicAdd(&sh.hist[bin_of(key.x)], 1u);
        atomicAdd(&sh.hist[bin_of(key.y)], 1u);
        atomicAdd(&sh.hist[bin_of(key.z)], 1u);
        atomicAdd(&sh.hist[bin_of(key.w)], 1u);
      }
    }
    for (int s = (nq << 2) + (int)threadIdx.x; s < n; s += kThreads) {
      const uint32_t key = load_key(s);
      if (cached) cache[s] = key;
      atomicAdd(&sh.hist[bin_of(key)], 1u);
    }
  } else {
    row_pass(n, load_key, [&](int s, bool valid, uint32_t key) {
      if (!valid) return;
      if (cached) cache[s] = key;
      atomicAdd(&sh.hist[bin_of(key)], 1u);
    });
  }
  __syncthreads();
  find_bin(sh.hist, sh.x, need);
  b = sh.x.bin;
  need -= sh.x.above;
  cnt_b = sh.hist[b];

  // ---- 3. bins above b are selected; bin b becomes the candidate list
  if (threadIdx.x == 0) sh.x.ncand = 0u;
  __syncthreads();
  row_pass(n, key_at, [&](int s, bool valid, uint32_t key) {
    const uint32_t d = bin_of(key);
    const uint32_t gbal = __ballot_sync(0xffffffffu, valid && d > b);
    if (lane == 0) { gt_bits[s >> 5] = gbal; eq_bits[s >> 5] = 0u; }
    if (valid && d == b) {
      const uint32_t pos = atomicAdd(&sh.x.ncand, 1u);
      if (pos < (uint32_t)p.cand_cap) cand[pos] = make_uint2(key, (uint32_t)s);
    }
  });
  __syncthreads();
  fits = cnt_b <= (uint32_t)p.cand_cap;
  }   // two-pass route

  // Exact threshold: the need-th largest key among the elements of bin b (or of
  // the single-pass candidates), found
  // by 2048-bin histograms over a shrinking key window [wlo, whi] (inclusive).
  uint32_t wlo, whi;
  if (fits) {
    uint32_t cmin = 0xffffffffu, cmax = 0u;
    for (int x = threadIdx.x; x < (int)cnt_b; x += kThreads) {
      cmin = min(cmin, cand[x].x);
      cmax = max(cmax, cand[x].x);
    }
    block_min_max(sh.x, cmin, cmax);
    wlo = cmin;
    whi = cmax;
  } else {
    wlo = (b == 0) ? 0u : lo + (b << shift);
    whi = (b == (uint32_t)(kBins - 1)) ? 0xffffffffu : lo + (((b + 1) << shift) - 1u);
  }
  uint32_t thr;
  for (;;) {
    const int wsh = bin_shift(whi - wlo);
    const uint32_t l0 = wlo, h0 = whi;
    clear_hist(sh.hist);
    if (fits) {
      for (int x = threadIdx.x; x < (int)cnt_b; x += kThreads) {
        const uint32_t key = cand[x].x;
        if (key >= l0 && key <= h0) atomicAdd(&sh.hist[(key - l0) >> wsh], 1u);
      }
    } else {
      row_pass(n, key_at, [&](int, bool valid, uint32_t key) {
        if (valid && key >= l0 && key <= h0) atomicAdd(&sh.hist[(key - l0) >> wsh], 1u);
      });
    }
    __syncthreads();
    find_bin(sh.hist, sh.x, need);
    const uint32_t bw = sh.x.bin;
    need -= sh.x.above;
    if (wsh == 0) { thr = wlo + bw; break; }
    wlo = l0 + (bw << wsh);
    const unsigned long long top = (unsigned long long)wlo + (1ull << wsh) - 1ull;
    whi = top < (unsigned long long)h0 ? (uint32_t)top : h0;
    if (fits && sh.x.bcount <= (uint32_t)kSmallSelect) {
      small_select(sh.small, (int)cnt_b, [&](int x) { return cand[x].x; }, wlo, whi, thr, need);
      break;
    }
  }
  if (fits) {
    for (int x = threadIdx.x; x < (int)cnt_b; x += kThreads) {
      const uint2 c = cand[x];
      if (c.x > thr) atomicOr(&gt_bits[c.y >> 5], 1u << (c.y & 31u));
      else if (c.x == thr) atomicOr(&eq_bits[c.y >> 5], 1u << (c.y & 31u));
    }
  } else {
    // Bitmaps rebuilt from one pass over the row: above = key > thr, equal = key == thr.
    row_pass(n, key_at, [&](int s, bool valid, uint32_t key) {
      const uint32_t gbal = __ballot_sync(0xffffffffu, valid && key > thr);
      const uint32_t ebal = __ballot_sync(0xffffffffu, valid && key == thr);
      if (lane == 0) { gt_bits[s >> 5] = gbal; eq_bits[s >> 5] = ebal; }
    });
  }
  __syncthreads();

  // ---- 4. ordered output: every "above" position and the first eq_take "equal" ones
  const uint32_t eq_take = need;
  const int W = (n + 31) >> 5;
  const int wpw = (W + kWarps - 1) / kWarps;         // bitmap words per warp
  const int w_begin = warp * wpw, w_end = min(W, w_begin + wpw);
  uint32_t cg = 0, ce = 0;
  for (int w = w_begin + lane; w < w_end; w += 32) { cg += __popc(gt_bits[w]); ce += __popc(eq_bits[w]); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cg += __shfl_xor_sync(0xffffffffu, cg, o);
    ce += __shfl_xor_sync(0xffffffffu, ce, o);
  }
  if (lane == 0) { sh.x.warp_a[warp] = cg; sh.x.warp_b[warp] = ce; }
  __syncthreads();
  uint32_t g = 0, e = 0;
  for (int w = 0; w < warp; ++w) { g += sh.x.warp_a[w]; e += sh.x.warp_b[w]; }
  for (int w0 = w_begin; w0 < w_end; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t gw = (w < w_end) ? gt_bits[w] : 0u;
    const uint32_t ew = (w < w_end) ? eq_bits[w] : 0u;
    // inclusive prefix of the per-word counts over the lanes (word order)
    const uint32_t tg = __popc(gw), te = __popc(ew);
    uint32_t pg = tg, pe = te;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yg = __shfl_up_sync(0xffffffffu, pg, o);
      const uint32_t ye = __shfl_up_sync(0xffffffffu, pe, o);
      if (lane >= o) { pg += yg; pe += ye; }
    }
    const uint32_t sum_g = __shfl_sync(0xffffffffu, pg, 31), sum_e = __shfl_sync(0xffffffffu, pe, 31);
    uint32_t gg = g + pg - tg, ee = e + pe - te;
    uint32_t sel = gw | ew;
    while (sel) {
      const int bit = __ffs(sel) - 1;
      sel &= sel - 1u;
      const int s = w * 32 + bit;
      if ((gw >> bit) & 1u) {
        const uint32_t pos = gg + min(ee, eq_take);
        if (pos < (uint32_t)k) {
          out[pos] = s;
          if (sel_out) sel_out[pos] = selected_score(src, s);
        }
        ++gg;
      } else {
        if (ee < eq_take && gg + ee < (uint32_t)k) {
          out[gg + ee] = s;
          if (sel_out) sel_out[gg + ee] = selected_score(src, s);
        }
        ++ee;
      }
    }
    g += sum_g;
    e += sum_e;
  }
}

// ------------------------------------------------------------------ few long rows
// The same selection with each row spread over a cluster of kClusterCtas CTAs
// (used when there are too few rows to fill the GPU, as in decode).  CTA r owns the
// 32-aligned segment [s0, s1) of the row.  Every CTA draws the same sample, so all
// agree on the first histogram's range; histograms are summed over the cluster
// through distributed shared memory, so every CTA finds the same bins and the same
// threshold; each CTA marks its own segment's bitmaps and candidates, and writes
// its selected positions after those of the lower-ranked CTAs.
constexpr int kClusterCtas = kTopkClusterCtas;
constexpr int kClusterGatherCap = 8192;   // kept keys a CTA copies from the whole cluster (gathered route)

struct alignas(16) TopkClusterShared {
  uint32_t hist[kBins];        // this CTA's histogram
  uint32_t tot[kBins];         // the cluster's
  ScanScratch x;
  uint32_t pub_a, pub_b;       // values this CTA publishes to the cluster
  uint32_t pub_c, pub_d;
  uint32_t lower_gt, lower_eq;  // gathered route: keys above / equal to the threshold in lower-ranked CTAs
  SmallSel small;               // gathered route: a small boundary bin's keys
};

// tot = sum over the cluster's CTAs of hist.
__device__ void cluster_sum_hist(TopkClusterShared& sh) {
  cluster_sync();                                   // every CTA's hist is complete
  const uint32_t base = smem_u32(sh.hist);
  for (int i = threadIdx.x; i < kBins; i += kThreads) {
    uint32_t t = 0;
#pragma unroll
    for (int c = 0; c < kClusterCtas; ++c) t += ld_shared_cluster_u32(mapa_shared(base + 4u * i, c));
    sh.tot[i] = t;
  }
  cluster_sync();                                   // no CTA rewrites hist while others read it
}

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kThreads, 2)
topk_cluster_kernel(const TopkParams p) {
  griddep_launch_dependents();
  griddep_wait();                                   // the scores are complete
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkClusterShared& sh = *reinterpret_cast<TopkClusterShared*>(smem_raw);
  uint32_t* gt_bits = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkClusterShared));   // segment words
  uint32_t* eq_bits = gt_bits + p.bit_words;
  uint2* cand = reinterpret_cast<uint2*>(eq_bits + p.bit_words);
  uint32_t* allk = reinterpret_cast<uint32_t*>(cand + p.cand_cap);   // kClusterGatherCap keys

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t r = cluster_ctarank();
  const int row = blockIdx.x / kClusterCtas;        // b * Lq + i
  const int i = row % p.Lq;
  const long long t = (long long)p.q_offset + i;
  const int n = (int)((t + 1 < p.Lk) ? t + 1 : p.Lk);
  const int k = p.k;
  int32_t* out = p.indices + (size_t)row * k;
  float* sel_out = p.sel_scores ? p.sel_scores + (size_t)row * k : nullptr;
  const float* src = p.scores + (size_t)row * p.Lk;

  if (n <= k) {                                     // the whole cluster leaves together
    if (r == 0)
      for (int x = threadIdx.x; x < k; x += kThreads) {
        out[x] = (x < n) ? x : -1;
        if (sel_out) sel_out[x] = (x < n) ? selected_score(src, x) : -INFINITY;
      }
    return;
  }
  const int seg = ((n + kClusterCtas - 1) / kClusterCtas + 31) / 32 * 32;
  const int s0 = min(n, (int)r * seg), s1 = min(n, s0 + seg);
  auto load_key = [&](int s) -> uint32_t { return score_key(__ldg(src + s)); };
  // row passes over this CTA's segment: positions s0 + (0 .. s1 - s0)
  auto seg_key = [&](int s) -> uint32_t { return load_key(s0 + s); };

  // ---- 1. sampled key range (the same in every CTA; kept in the candidate buffer
  // for step 1b): positions j * (n / ns), every load of a thread in flight at once
  const int ns = n < kSample ? n : kSample;
  const int stride = n / ns;
  const bool try_single = p.sampled && p.cand_cap >= kSample;
  uint32_t smin = 0xffffffffu, smax = 0u;
  {
    constexpr int kPer = (kSample + kThreads - 1) / kThreads;
    uint32_t sk[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int j = (int)threadIdx.x + u * kThreads;
      sk[u] = j < ns ? load_key(j * stride) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int j = (int)threadIdx.x + u * kThreads;
      if (j < ns) {
        if (try_single) cand[j].x = sk[u];
        smin = min(smin, sk[u]);
        smax = max(smax, sk[u]);
      }
    }
  }
  block_min_max(sh.x, smin, smax);
  const uint32_t lo = smin;
  const int shift = bin_shift(smax - smin);
  auto bin_of = [lo, shift](uint32_t key) -> uint32_t {
    return key < lo ? 0u : min((uint32_t)(kBins - 1), (key - lo) >> shift);
  };

  // ---- 1b. one pass, as in the one-CTA kernel: every key of the segment at or
  // above theta (just below the sample's j-th largest key, the same in every CTA)
  // is kept with its position.  The cluster takes this route when at least k keys
  // pass over the whole row and every segment's share fits its buffer; the
  // decision is taken from cluster-wide counts, so every CTA reaches the same
  // barriers.  Otherwise the two passes below.
  bool single = false;
  uint32_t single_lo = 0xffffffffu, single_hi = 0u;   // the cluster's kept-key range
  uint32_t total = 0;                                  // keys kept over the cluster
  uint32_t cnt_c[kClusterCtas] = {};                   // ... by each CTA
  if (try_single) {
    const float mu = (float)ns * (float)k / (float)n;
    const float sig = sqrtf(mu * (1.f - (float)k / (float)n));
    const uint32_t j = (uint32_t)ceilf(mu + 6.f * sig + 2.f);
    if (j < (uint32_t)ns) {
      clear_hist(sh.hist);
      for (int x = threadIdx.x; x < ns; x += kThreads) atomicAdd(&sh.hist[bin_of(cand[x].x)], 1u);
      __syncthreads();
      find_bin(sh.hist, sh.x, j);
      uint32_t theta;
      {
        const uint32_t tb = sh.x.bin, need2 = j - sh.x.above;
        const uint32_t wlo = lo + (tb << shift);
        const unsigned long long top = (unsigned long long)wlo + (1ull << shift) - 1ull;
        const uint32_t whi = (tb == (uint32_t)(kBins - 1) || top > smax) ? smax : (uint32_t)top;
        const int sh2 = bin_shift(whi - wlo);
        clear_hist(sh.hist);
        for (int x = threadIdx.x; x < ns; x += kThreads) {
          const uint32_t key = cand[x].x;
          if (key >= wlo && key <= whi) atomicAdd(&sh.hist[(key - wlo) >> sh2], 1u);
        }
        __syncthreads();
        find_bin(sh.hist, sh.x, need2);
        theta = wlo + (sh.x.bin << sh2);
      }
      const int W = (s1 - s0 + 31) >> 5;
      for (int x = threadIdx.x; x < W; x += kThreads) { gt_bits[x] = 0u; eq_bits[x] = 0u; }
      if (threadIdx.x == 0) sh.x.ncand = 0u;
      __syncthreads();
      auto keep = [&](int s, uint32_t key) {        // s relative to s0
        if (key >= theta) {
          const uint32_t at = atomicAdd(&sh.x.ncand, 1u);
          if (at < (uint32_t)p.cand_cap) cand[at] = make_uint2(key, (uint32_t)s);
        }
      };
      if (p.vec4) {
        // s0 is a multiple of 32 scores, so the segment starts 16-byte aligned
        // whenever the rows do: 16-byte loads, four in flight per thread (twice the
        // bytes in flight of the 4-byte row pass, which matters with one row per
        // four CTAs and nothing else on the GPU).  A warp appends its kept keys of
        // a step with one shared atomic (per-key atomics on the one counter
        // serialised the pass).
        const float4* src4 = reinterpret_cast<const float4*>(src + s0);
        const int nq = (s1 - s0) >> 2;
        const float theta_f = key_score(theta);
        for (int q00 = warp * 32; q00 < nq; q00 += kThreads * kPassUnroll) {   // warp-uniform bound
          const int q0 = q00 + lane;
          float4 f[kPassUnroll];
#pragma unroll
          for (int u = 0; u < kPassUnroll; ++u) {
            const int q = q0 + u * kThreads;
            f[u] = (q < nq) ? __ldg(src4 + q) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          uint32_t mine = 0;                          // kept keys of this lane in this step
#pragma unroll
          for (int u = 0; u < kPassUnroll; ++u) {
            const int q = q0 + u * kThreads;
            if (q < nq) {                              // float compares: no key conversion per score
              mine += f[u].x >= theta_f ? 1u : 0u;
              mine += f[u].y >= theta_f ? 1u : 0u;
              mine += f[u].z >= theta_f ? 1u : 0u;
              mine += f[u].w >= theta_f ? 1u : 0u;
            }
          }
          uint32_t incl = mine;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const uint32_t wtot = __shfl_sync(0xffffffffu, incl, 31);
          if (wtot == 0u) continue;
          uint32_t at = 0;
          if (lane == 31) at = atomicAdd(&sh.x.ncand, wtot);
          at = __shfl_sync(0xffffffffu, at, 31) + incl - mine;
          if (mine != 0u) {
#pragma unroll
            for (int u = 0; u < kPassUnroll; ++u) {
              const int q = q0 + u * kThreads;
              if (q < nq) {
                const float fx[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  if (fx[c] >= theta_f) {                // the predicate the count used
                    if (at < (uint32_t)p.cand_cap) cand[at] = make_uint2(score_key(fx[c]), (uint32_t)(4 * q + c));
                    ++at;
                  }
                }
              }
            }
          }
        }
        for (int s = (nq << 2) + (int)threadIdx.x; s < s1 - s0; s += kThreads) keep(s, seg_key(s));
      } else {
        row_pass(s1 - s0, seg_key, [&](int s, bool valid, uint32_t key) {
          if (valid) keep(s, key);
        });
      }
      __syncthreads();
      // The kept keys' range goes out with the counts, so the single route needs no
      // second exchange to open its refinement window.
      const uint32_t kept = min(sh.x.ncand, (uint32_t)p.cand_cap);
      uint32_t cmin = 0xffffffffu, cmax = 0u;
      for (int x = threadIdx.x; x < (int)kept; x += kThreads) {
        cmin = min(cmin, cand[x].x);
        cmax = max(cmax, cand[x].x);
      }
      block_min_max(sh.x, cmin, cmax);
      if (threadIdx.x == 0) {
        sh.pub_a = sh.x.ncand;
        sh.pub_b = sh.x.ncand > (uint32_t)p.cand_cap ? 1u : 0u;
        sh.pub_c = cmin;
        sh.pub_d = cmax;
      }
      cluster_sync();
      uint32_t over = 0;
#pragma unroll
      for (int c = 0; c < kClusterCtas; ++c) {
        cnt_c[c] = ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_a), c));
        total += cnt_c[c];
        over |= ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_b), c));
        single_lo = min(single_lo, ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_c), c)));
        single_hi = max(single_hi, ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_d), c)));
      }
      cluster_sync();                               // the pub_* words are not rewritten before all have read them
      single = over == 0u && total >= (uint32_t)k;
    }
  }

  uint32_t need = (uint32_t)k;
  uint32_t b = 0, cnt_b = 0;
  if (!single) {
  // ---- 2. segment histogram, summed over the cluster
  clear_hist(sh.hist);
  row_pass(s1 - s0, seg_key, [&](int, bool valid, uint32_t key) {
    if (valid) atomicAdd(&sh.hist[bin_of(key)], 1u);
  });
  __syncthreads();
  cluster_sum_hist(sh);
  find_bin(sh.tot, sh.x, need);
  b = sh.x.bin;
  need -= sh.x.above;
  cnt_b = sh.tot[b];

  // ---- 3. this segment's bins above b into the bitmap; its bin-b elements as candidates
  if (threadIdx.x == 0) sh.x.ncand = 0u;
  __syncthreads();
  row_pass(s1 - s0, seg_key, [&](int s, bool valid, uint32_t key) {
    const uint32_t d = bin_of(key);
    const uint32_t gbal = __ballot_sync(0xffffffffu, valid && d > b);
    if (lane == 0) { gt_bits[s >> 5] = gbal; eq_bits[s >> 5] = 0u; }
    if (valid && d == b) {
      const uint32_t pos = atomicAdd(&sh.x.ncand, 1u);
      if (pos < (uint32_t)p.cand_cap) cand[pos] = make_uint2(key, (uint32_t)s);
    }
  });
  __syncthreads();
  }   // two-pass route
  // After one pass every CTA's share fits its buffer; after two, the bin's whole
  // count must fit (then every CTA's share fits as well).
  const bool fits = single || cnt_b <= (uint32_t)p.cand_cap;
  const int own = (int)sh.x.ncand;

  // Single route with few kept keys (decode rows keep ~5 K): every CTA gets a copy
  // of the cluster's kept keys, in CTA order (each CTA stores its own keys into
  // every CTA's copy), and refines the threshold on it alone, with no cluster
  // barrier per level; the keys that lower-ranked CTAs hold above and at the
  // threshold then give this CTA's output offsets.
  const bool gathered = single && total <= (uint32_t)kClusterGatherCap;
  uint32_t lower = 0;                               // keys kept by lower-ranked CTAs
  if (gathered) {
#pragma unroll
    for (int c = 0; c < kClusterCtas; ++c) {
      if ((uint32_t)c < r) lower += cnt_c[c];
    }
    // each CTA stores its own keys into every CTA's copy, at its offset
    const uint32_t base = smem_u32(allk + lower);
    for (int x = threadIdx.x; x < own; x += kThreads) {
      const uint32_t key = cand[x].x;
#pragma unroll
      for (int c = 0; c < kClusterCtas; ++c) st_shared_cluster_u32(mapa_shared(base + 4u * (uint32_t)x, (uint32_t)c), key);
    }
    if (threadIdx.x == 0) { sh.lower_gt = 0u; sh.lower_eq = 0u; }
    cluster_sync();                                 // every copy is complete; no shared memory of a peer is touched after this
  }

  // Exact threshold, refined over the window [wlo, whi] with cluster-summed histograms
  // of the candidates (or of the segments when the candidates do not fit).
  uint32_t wlo, whi;
  if (single) {
    wlo = single_lo;
    whi = single_hi;
  } else if (fits) {
    uint32_t cmin = 0xffffffffu, cmax = 0u;
    for (int x = threadIdx.x; x < own; x += kThreads) {
      cmin = min(cmin, cand[x].x);
      cmax = max(cmax, cand[x].x);
    }
    block_min_max(sh.x, cmin, cmax);
    if (threadIdx.x == 0) { sh.pub_a = cmin; sh.pub_b = cmax; }
    cluster_sync();
    wlo = 0xffffffffu;
    whi = 0u;
#pragma unroll
    for (int c = 0; c < kClusterCtas; ++c) {
      wlo = min(wlo, ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_a), c)));
      whi = max(whi, ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_b), c)));
    }
    cluster_sync();
  } else {
    wlo = (b == 0) ? 0u : lo + (b << shift);
    whi = (b == (uint32_t)(kBins - 1)) ? 0xffffffffu : lo + (((b + 1) << shift) - 1u);
  }
  uint32_t thr;
  for (;;) {
    const int wsh = bin_shift(whi - wlo);
    const uint32_t l0 = wlo, h0 = whi;
    clear_hist(sh.hist);
    if (gathered) {
      for (int x = threadIdx.x; x < (int)total; x += kThreads) {
        const uint32_t key = allk[x];
        if (key >= l0 && key <= h0) atomicAdd(&sh.hist[(key - l0) >> wsh], 1u);
      }
    } else if (fits) {
      for (int x = threadIdx.x; x < own; x += kThreads) {
        const uint32_t key = cand[x].x;
        if (key >= l0 && key <= h0) atomicAdd(&sh.hist[(key - l0) >> wsh], 1u);
      }
    } else {
      row_pass(s1 - s0, seg_key, [&](int, bool valid, uint32_t key) {
        if (valid && key >= l0 && key <= h0) atomicAdd(&sh.hist[(key - l0) >> wsh], 1u);
      });
    }
    __syncthreads();
    if (!gathered) cluster_sum_hist(sh);
    find_bin(gathered ? sh.hist : sh.tot, sh.x, need);
    const uint32_t bw = sh.x.bin;
    need -= sh.x.above;
    if (wsh == 0) { thr = wlo + bw; break; }
    wlo = l0 + (bw << wsh);
    const unsigned long long top = (unsigned long long)wlo + (1ull << wsh) - 1ull;
    whi = top < (unsigned long long)h0 ? (uint32_t)top : h0;
    // Gathered route: once the boundary bin [wlo, whi] holds few keys, one warp
    // ranks them directly instead of further histogram levels.
    if (gathered && sh.x.bcount <= (uint32_t)kSmallSelect) {
      small_select(sh.small, (int)total, [&](int x) { return allk[x]; }, wlo, whi, thr, need);
      break;
    }
  }
  if (fits) {
    for (int x = threadIdx.x; x < own; x += kThreads) {
      const uint2 c = cand[x];
      if (c.x > thr) atomicOr(&gt_bits[c.y >> 5], 1u << (c.y & 31u));
      else if (c.x == thr) atomicOr(&eq_bits[c.y >> 5], 1u << (c.y & 31u));
    }
    if (gathered) {                                 // the lower-ranked CTAs' keys come first in allk
      uint32_t lg = 0, le = 0;
      for (int x = threadIdx.x; x < (int)lower; x += kThreads) {
        const uint32_t key = allk[x];
        lg += key > thr ? 1u : 0u;
        le += key == thr ? 1u : 0u;
      }
      lg = __reduce_add_sync(0xffffffffu, lg);
      le = __reduce_add_sync(0xffffffffu, le);
      if (lane == 0 && (lg | le) != 0u) {
        atomicAdd(&sh.lower_gt, lg);
        atomicAdd(&sh.lower_eq, le);
      }
    }
  } else {
    row_pass(s1 - s0, seg_key, [&](int s, bool valid, uint32_t key) {
      const uint32_t gbal = __ballot_sync(0xffffffffu, valid && key > thr);
      const uint32_t ebal = __ballot_sync(0xffffffffu, valid && key == thr);
      if (lane == 0) { gt_bits[s >> 5] = gbal; eq_bits[s >> 5] = ebal; }
    });
  }
  __syncthreads();

  // ---- 4. ordered output: offsets from the lower-ranked CTAs, then this segment
  const uint32_t eq_take = need;
  const int W = (s1 - s0 + 31) >> 5;
  const int wpw = (W + kWarps - 1) / kWarps;         // bitmap words per warp
  const int w_begin = warp * wpw, w_end = min(W, w_begin + wpw);
  uint32_t cg = 0, ce = 0;
  for (int w = w_begin + lane; w < w_end; w += 32) { cg += __popc(gt_bits[w]); ce += __popc(eq_bits[w]); }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cg += __shfl_xor_sync(0xffffffffu, cg, o);
    ce += __shfl_xor_sync(0xffffffffu, ce, o);
  }
  if (lane == 0) { sh.x.warp_a[warp] = cg; sh.x.warp_b[warp] = ce; }
  __syncthreads();
  uint32_t g = 0, e = 0, seg_g = 0, seg_e = 0;
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) { g += sh.x.warp_a[w]; e += sh.x.warp_b[w]; }
    seg_g += sh.x.warp_a[w];
    seg_e += sh.x.warp_b[w];
  }
  if (gathered) {
    g += sh.lower_gt;
    e += sh.lower_eq;
  } else {
    if (threadIdx.x == 0) { sh.pub_a = seg_g; sh.pub_b = seg_e; }
    cluster_sync();
    for (uint32_t c = 0; c < r; ++c) {
      g += ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_a), c));
      e += ld_shared_cluster_u32(mapa_shared(smem_u32(&sh.pub_b), c));
    }
    cluster_sync();                                 // peers' shared memory is no longer read
  }
  for (int w0 = w_begin; w0 < w_end; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t gw = (w < w_end) ? gt_bits[w] : 0u;
    const uint32_t ew = (w < w_end) ? eq_bits[w] : 0u;
    const uint32_t tg = __popc(gw), te = __popc(ew);
    uint32_t pg = tg, pe = te;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yg = __shfl_up_sync(0xffffffffu, pg, o);
      const uint32_t ye = __shfl_up_sync(0xffffffffu, pe, o);
      if (lane >= o) { pg += yg; pe += ye; }
    }
    const uint32_t sum_g = __shfl_sync(0xffffffffu, pg, 31), sum_e = __shfl_sync(0xffffffffu, pe, 31);
    uint32_t gg = g + pg - tg, ee = e + pe - te;
    uint32_t sel = gw | ew;
    while (sel) {
      const int bit = __ffs(sel) - 1;
      sel &= sel - 1u;
      const int s = s0 + w * 32 + bit;
      if ((gw >> bit) & 1u) {
        const uint32_t pos = gg + min(ee, eq_take);
        if (pos < (uint32_t)k) {
          out[pos] = s;
          if (sel_out) sel_out[pos] = selected_score(src, s);
        }
        ++gg;
      } else {
        if (ee < eq_take && gg + ee < (uint32_t)k) {
          out[gg + ee] = s;
          if (sel_out) sel_out[gg + ee] = selected_score(src, s);
        }
        ++ee;
      }
    }
    g += sum_g;
    e += sum_e;
  }
}

// ------------------------------------------------------------------ many rows
// One warp per row, eight rows per CTA: no block-wide barrier anywhere, so each
// warp streams its row (from L2 / HBM) at its own pace and an SM keeps many rows
// in flight.  The same selection as above:
//   1. a strided sample of 256 scores sets the key range [lo, hi] of a 1024-bin
//      histogram (keys outside it are counted in the end bins);
//   2. one pass over the row builds that histogram and gives the bin b holding the
//      m-th largest key and the count above it;
//   3. the exact threshold inside bin b's key window: histogram levels over the
//      window's keys until the boundary bin's keys fit the warp's candidate buffer,
//      then levels over the candidates (warp_find_threshold);
//   4. one ordered pass writes every position above the threshold and the first
//      positions equal to it, in ascending position order.
constexpr int kWarpRowsPerCta = 8;
constexpr int kWarpSample = 256;

struct WarpTopkSmem {
  uint32_t hist[kSelBins];
  uint32_t cand[kSelCandCap + 4];
};

// f(key) for every score of src[0 .. n) (16-byte loads when vec4, else 4-byte);
// lanes call f different numbers of times.
template <typename F>
__device__ __forceinline__ void visit_row_keys(const float* src, int n, bool vec4, F f) {
  const int lane = (int)(threadIdx.x & 31u);
  if (vec4) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    const int n4 = n >> 2;
    constexpr int kU = 4;
    for (int g0 = 0; g0 < n4; g0 += 32 * kU) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int g = g0 + u * 32 + lane;
        v[u] = g < n4 ? __ldg(s4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (g0 + u * 32 + lane < n4) {
          f(score_to_key(v[u].x));
          f(score_to_key(v[u].y));
          f(score_to_key(v[u].z));
          f(score_to_key(v[u].w));
        }
      }
    }
    for (int s = (n4 << 2) + lane; s < n; s += 32) f(score_to_key(__ldg(src + s)));
  } else {
    constexpr int kU = 8;
    for (int s0 = 0; s0 < n; s0 += 32 * kU) {
      float v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int s = s0 + u * 32 + lane;
        v[u] = s < n ? __ldg(src + s) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (s0 + u * 32 + lane < n) f(score_to_key(v[u]));
    }
  }
}

__global__ void __launch_bounds__(32 * kWarpRowsPerCta, 4) topk_warp_kernel(const TopkParams p) {
  griddep_launch_dependents();
  griddep_wait();                                   // the scores are complete
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int lane = (int)(threadIdx.x & 31u), warp = (int)(threadIdx.x >> 5);
  WarpTopkSmem& sh = reinterpret_cast<WarpTopkSmem*>(smem_raw)[warp];
  const long long row = (long long)blockIdx.x * kWarpRowsPerCta + warp;   // b * Lq + i
  if (row >= (long long)p.B * p.Lq) return;                             // whole warp
  const int i = (int)(row % p.Lq);
  const long long t = (long long)p.q_offset + i;
  const int n = (int)((t + 1 < p.Lk) ? t + 1 : p.Lk);
  const uint32_t k = (uint32_t)p.k;
  int32_t* out = p.indices + (size_t)row * k;
  float* sel_out = p.sel_scores ? p.sel_scores + (size_t)row * k : nullptr;
  const float* src = p.scores + (size_t)row * p.Lk;
  if ((uint32_t)n <= k) {                           // everything up to t is selected
    for (uint32_t x = lane; x < k; x += 32) {
      out[x] = (x < (uint32_t)n) ? (int32_t)x : -1;
      if (sel_out) sel_out[x] = (x < (uint32_t)n) ? key_to_score(score_to_key(__ldg(src + x))) : -INFINITY;
    }
    return;
  }
  const bool vec4 = p.vec4 != 0;

  // ---- 1. key range of a strided sample
  uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
  for (int u = 0; u < kWarpSample / 32; ++u) {
    const int j = u * 32 + lane;
    const uint32_t key = score_to_key(__ldg(src + (int)(((long long)j * n) / kWarpSample)));
    lo = min(lo, key);
    hi = max(hi, key);
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  const int shift = sel_shift(hi - lo);

  // ---- 2. clamped histogram of the whole row and the boundary bin
  for (int x = lane; x < kSelBins / 4; x += 32) reinterpret_cast<uint4*>(sh.hist)[x] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  visit_row_keys(src, n, vec4, [&](uint32_t key) {
    const uint32_t d = key < lo ? 0u : min((uint32_t)(kSelBins - 1), (key - lo) >> shift);
    atomicAdd(&sh.hist[d], 1u);
  });
  __syncwarp();
  constexpr int kPer = kSelBins / 32;                // bins per lane
  uint32_t mine = 0;
#pragma unroll
  for (int x = 0; x < kPer / 4; ++x) {
    const uint4 v = reinterpret_cast<const uint4*>(sh.hist + lane * kPer)[x];
    mine += v.x + v.y + v.z + v.w;
  }
  uint32_t suffix = mine;                            // bins of lanes >= this lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suffix, o);
    if (lane + o < 32) suffix += y;
  }
  const uint32_t above_lane = suffix - mine;
  const uint32_t owner = __ffs(__ballot_sync(0xffffffffu, above_lane < k && suffix >= k)) - 1;
  uint32_t b = 0, above = 0;
  if ((uint32_t)lane == owner) {
    uint32_t acc = above_lane;
    for (int x = kPer - 1; x >= 0; --x) {
      const uint32_t c = sh.hist[lane * kPer + x];
      if (acc + c >= k) { b = lane * kPer + x; above = acc; break; }
      acc += c;
    }
  }
  b = __shfl_sync(0xffffffffu, b, owner);
  above = __shfl_sync(0xffffffffu, above, owner);
  __syncwarp();

  // ---- 3. exact threshold among the keys of bin b's window
  const uint32_t wlo = b == 0 ? 0u : lo + (b << shift);
  uint32_t whi = 0xffffffffu;
  if (b + 1 < (uint32_t)kSelBins) {
    const unsigned long long top = (unsigned long long)lo + ((unsigned long long)(b + 1) << shift) - 1ull;
    whi = top < 0xffffffffull ? (uint32_t)top : 0xffffffffu;
  }
  uint32_t thr, gt_w;
  auto visit = [&](auto&& f) { visit_row_keys(src, n, vec4, f); };
  warp_find_threshold(sh.hist, sh.cand, visit, k - above, wlo, whi, thr, gt_w, sh.hist[b]);
  const uint32_t eq_take = k - above - gt_w;

  // ---- 4. ordered output: every key above thr and the first eq_take equal to it.
  // Scores are compared as floats with thr's float value: the key order is the
  // float order with -0.0 equal to +0.0, so no key is formed per score.
  const float thr_f = key_to_score(thr);
  uint32_t w = 0, eq_seen = 0;
  // v[] are the scores at positions s .. s + cnt - 1 of this lane (cnt <= 4), lanes in position order
  auto emit_group = [&](int s, const float (&v)[4], int cnt) {
    uint32_t gtm = 0, eqm = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      gtm |= (j < cnt && v[j] > thr_f) ? (1u << j) : 0u;
      eqm |= (j < cnt && v[j] == thr_f) ? (1u << j) : 0u;
    }
    uint32_t eq_tot = 0, take = gtm;
    if (__any_sync(0xffffffffu, eqm != 0u)) {           // most groups hold no key equal to thr
      const uint32_t eq_rank = eq_seen + warp_exclusive_sum(__popc(eqm), eq_tot);
      uint32_t e = eqm;
      for (uint32_t r = eq_rank; e && r < eq_take; ++r) {   // equal keys taken in position order
        take |= e & (0u - e);
        e &= e - 1u;
      }
    }
    uint32_t kept;
    uint32_t at = w + warp_exclusive_sum(__popc(take), kept);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (take & (1u << j)) {
        out[at] = s + j;
        if (sel_out) sel_out[at] = v[j] == 0.f ? 0.f : v[j];   // -0.0 as +0.0, as the selection saw it
        ++at;
      }
    }
    w += kept;
    eq_seen += eq_tot;
  };
  if (vec4) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    const int n4 = (n + 3) >> 2;                     // the last group may run past n (masked below)
    constexpr int kU = 4;
    for (int g0 = 0; g0 < n4; g0 += 32 * kU) {
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int g = g0 + u * 32 + lane;
        v[u] = g < (n >> 2) ? __ldg(s4 + g) : make_float4(0.f, 0.f, 0.f, 0.f);
        if (g == (n >> 2) && (n & 3)) {               // ragged tail: scalar loads inside the row
          v[u].x = __ldg(src + 4 * g);
          if ((n & 3) > 1) v[u].y = __ldg(src + 4 * g + 1);
          if ((n & 3) > 2) v[u].z = __ldg(src + 4 * g + 2);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (g0 + u * 32 < n4) {
          const int g = g0 + u * 32 + lane;
          const float sv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
          emit_group(4 * g, sv, max(0, min(4, n - 4 * g)));
        }
      }
    }
  } else {
    constexpr int kU = 8;
    for (int s0 = 0; s0 < n; s0 += 32 * kU) {
      float v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int s = s0 + u * 32 + lane;
        v[u] = s < n ? __ldg(src + s) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int s = s0 + u * 32 + lane;
        if (s0 + u * 32 < n) {
          const float sv[4] = {v[u], 0.f, 0.f, 0.f};
          emit_group(s, sv, s < n ? 1 : 0);
        }
      }
    }
  }
}

}  // namespace

size_t topk_smem_bytes(int cache_cap, int bit_words, int cand_cap, bool cluster) {
  static_assert(sizeof(TopkShared) % 16 == 0, "arrays that follow must stay 16-byte aligned");
  static_assert(sizeof(TopkClusterShared) % 16 == 0, "arrays that follow must stay 16-byte aligned");
  if (cluster)
    return sizeof(TopkClusterShared) + 2 * (size_t)bit_words * 4 + (size_t)cand_cap * 8 + (size_t)kClusterGatherCap * 4;
  return sizeof(TopkShared) + ((size_t)cache_cap + 2 * (size_t)bit_words) * 4 + (size_t)cand_cap * 8;
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t stream) {
  const int rows = p.B * p.Lq;
  if (p.warp_rows) {
    const size_t wsmem = sizeof(WarpTopkSmem) * kWarpRowsPerCta;
    cudaError_t e = cudaFuncSetAttribute(topk_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wsmem);
    if (e != cudaSuccess) return e;
    if (rows == 0) return cudaSuccess;
    return launch_pdl(topk_warp_kernel, dim3((rows + kWarpRowsPerCta - 1) / kWarpRowsPerCta),
                      dim3(32 * kWarpRowsPerCta), wsmem, stream, p);
  }
  const size_t smem = topk_smem_bytes(p.cache_cap, p.bit_words, p.cand_cap, p.cluster != 0);
  if (p.cluster) {
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (rows == 0) return cudaSuccess;
    return launch_pdl(topk_cluster_kernel, dim3(rows * kClusterCtas), dim3(kThreads), smem, stream, p);
  }
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (rows == 0) return cudaSuccess;
  return launch_pdl(topk_kernel, dim3(rows), dim3(kThreads), smem, stream, p);
}

cudaError_t read_topk_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
