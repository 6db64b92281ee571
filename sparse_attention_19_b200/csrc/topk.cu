// topk.cu -- per-query top-k over the indexer scores (radix select).
//
// Row (b, i) sits at position t = q_offset + i and selects, among the n =
// min(t+1, Lk) scores I[t, 0..n), the m = min(k, n) largest, ties to the smaller
// position ("Отбор и основное внимание": the k KV entries with the largest
// I_{t,s}).  The result is written in ascending position order, -1 padded.
//
// Method: fp32 scores become order-preserving 32-bit keys (-0.0 is first
// canonicalised to +0.0).  The key of the m-th largest element is found digit by
// digit (11 + 11 + 10 bits) from shared-memory histograms; after the first digit
// only the elements of the boundary bin (copied to a candidate list) are
// visited.  A final pass in position order takes every key above the threshold
// and the first (m - #above) keys equal to it, placing each selected element at
// (number of selected elements before it) via a block-wide prefix sum, so the
// output is sorted and ties resolve to smaller positions.
// One CTA per row; the row is cached in shared memory when it fits.
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;                       // -0.0 -> +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// 16-byte multiple, so the row cache and the 8-byte candidate pairs that follow
// it in dynamic shared memory stay aligned.
struct alignas(16) TopkShared {
  uint32_t hist[2048];
  uint32_t warp_tot[kWarps];
  uint32_t bin, above, ncand;
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
// reaches `need`; records b and the count strictly above it.
__device__ void find_bin(TopkShared& sh, int nbins, uint32_t need) {
  const int per = nbins / kThreads;                 // bins per thread (4 or 2)
  const int lo = threadIdx.x * per;
  uint32_t mine = 0;
  for (int x = 0; x < per; ++x) mine += sh.hist[lo + x];
  uint32_t total;
  const uint32_t incl = block_inclusive_scan(mine, sh.warp_tot, total);
  uint32_t acc = total - incl;                      // count in bins above this thread's range
  for (int x = per - 1; x >= 0; --x) {
    const uint32_t c = sh.hist[lo + x];
    if (acc < need && acc + c >= need) {
      sh.bin = (uint32_t)(lo + x);
      sh.above = acc;
    }
    acc += c;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* cache = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));
  uint2* cand = reinterpret_cast<uint2*>(cache + (p.cache_cap + 3) / 4 * 4);

  const int row = blockIdx.x;                       // b * Lq + i
  const int i = row % p.Lq;
  const long long t = (long long)p.q_offset + i;
  const int n = (int)((t + 1 < p.Lk) ? t + 1 : p.Lk);
  const int k = p.k;
  int32_t* out = p.indices + (size_t)row * k;
  const float* src = p.scores + (size_t)row * p.Lk;

  if (n <= k) {                                     // everything up to t is selected
    for (int x = threadIdx.x; x < k; x += kThreads) out[x] = (x < n) ? x : -1;
    return;
  }
  const bool cached = n <= p.cache_cap;

  // ---- digit 1: bits 31..21, over the whole row (also fills the cache)
  for (int x = threadIdx.x; x < 2048; x += kThreads) sh.hist[x] = 0u;
  if (threadIdx.x == 0) sh.ncand = 0u;
  __syncthreads();
  for (int s = threadIdx.x; s < n; s += kThreads) {
    const uint32_t key = score_key(__ldcs(src + s));
    if (cached) cache[s] = key;
    atomicAdd(&sh.hist[key >> 21], 1u);
  }
  __syncthreads();
  find_bin(sh, 2048, (uint32_t)k);
  const uint32_t b1 = sh.bin;
  uint32_t need = (uint32_t)k - sh.above;           // still to take inside bin b1
  auto key_at = [&](int s) -> uint32_t { return cached ? cache[s] : score_key(__ldcs(src + s)); };

  // ---- compact the boundary bin
  for (int s = threadIdx.x; s < n; s += kThreads) {
    const uint32_t key = key_at(s);
    if ((key >> 21) == b1) {
      const uint32_t pos = atomicAdd(&sh.ncand, 1u);
      if (pos < (uint32_t)p.cand_cap) cand[pos] = make_uint2(key, (uint32_t)s);
    }
  }
  __syncthreads();
  const uint32_t ncand = sh.ncand;
  const bool use_cand = ncand <= (uint32_t)p.cand_cap;
  const int scan_n = use_cand ? (int)ncand : n;

  // ---- digits 2 (bits 20..10) and 3 (bits 9..0) over the candidates
  uint32_t prefix = b1;                              // known high bits of the threshold key
  int known = 11;                                    // how many high bits are known
  const int widths[2] = {11, 10};
  for (int d = 0; d < 2; ++d) {
    const int wbits = widths[d];
    const int shift = 32 - known - wbits;
    const int nbins = 1 << wbits;
    for (int x = threadIdx.x; x < 2048; x += kThreads) sh.hist[x] = 0u;
    __syncthreads();
    for (int x = threadIdx.x; x < scan_n; x += kThreads) {
      const uint32_t key = use_cand ? cand[x].x : key_at(x);
      if ((key >> (32 - known)) == prefix) atomicAdd(&sh.hist[(key >> shift) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_bin(sh, nbins < 2048 ? 2048 : nbins, need);   // unused upper bins are zero
    prefix = (prefix << wbits) | sh.bin;
    need -= sh.above;
    known += wbits;
  }
  const uint32_t thr = prefix;                       // exact key of the m-th largest
  const uint32_t eq_take = need;                     // how many keys == thr to take

  // ---- ordered output pass
  constexpr int E = 4;                               // consecutive elements per thread
  uint32_t gt_off = 0, eq_off = 0;
  for (int base = 0; base < n; base += kThreads * E) {
    const int s0 = base + threadIdx.x * E;
    uint32_t keys[E];
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int s = s0 + e;
      keys[e] = (s < n) ? key_at(s) : 0u;
      if (s < n) { gt += keys[e] > thr; eq += keys[e] == thr; }
    }
    uint32_t total;
    const uint32_t incl = block_inclusive_scan(gt | (eq << 16), sh.warp_tot, total);
    const uint32_t excl = incl - (gt | (eq << 16));
    uint32_t g = gt_off + (excl & 0xFFFFu), q = eq_off + (excl >> 16);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int s = s0 + e;
      if (s >= n) break;
      if (keys[e] > thr) {
        const uint32_t pos = g + min(q, eq_take);
        if (pos < (uint32_t)k) out[pos] = s;
        ++g;
      } else if (keys[e] == thr) {
        if (q < eq_take && g + q < (uint32_t)k) out[g + q] = s;
        ++q;
      }
    }
    gt_off += total & 0xFFFFu;
    eq_off += total >> 16;
  }
}

}  // namespace

size_t topk_smem_bytes(int cache_cap, int cand_cap) {
  static_assert(sizeof(TopkShared) % 16 == 0, "candidate pairs must stay 8-byte aligned");
  return sizeof(TopkShared) + (size_t)((cache_cap + 3) / 4 * 4) * 4 + (size_t)cand_cap * 8;
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t stream) {
  const size_t smem = topk_smem_bytes(p.cache_cap, p.cand_cap);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = p.B * p.Lq;
  if (rows == 0) return cudaSuccess;
  topk_kernel<<<rows, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t read_topk_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
