// warp_select.cuh -- exact top-k selection by one warp over candidate lists kept in
// global memory (L2), for the fused indexer + top-k.
//
// A candidate is (key, position): key is the order-preserving 32-bit image of an
// fp32 indexer score (larger key = larger score, -0.0 folded onto +0.0) and
// position the key token's index s.  Lists are kept in increasing position order.
// The selection order is "key descending, then position ascending" (ties go to
// the smaller position), the reading of the top-k step ("Отбор и основное
// внимание") that makes index sets unique.
//
// The top-m of a list is described by a threshold key thr and a count eq_take:
// every candidate with key > thr, plus the first eq_take candidates (in position
// order) with key == thr.  warp_find_threshold() finds (thr, gt = #{key > thr})
// by histogram refinement over the list's key range; warp_compact() then walks
// the list once, in order, and keeps exactly those candidates, so the output stays
// in position order.
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

namespace dsa {

constexpr int kSelBins = 1024;          // histogram bins per refinement level
constexpr int kSelBinBits = 10;
constexpr int kSelCandCap = 512;        // boundary-bin keys gathered into shared memory

__device__ __forceinline__ uint32_t score_to_key(float f) {
  // f + 0.0f turns -0.0 into +0.0 (round-to-nearest) and leaves every other value
  // as it is; then negatives are complemented and positives get the top bit set.
  const uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
  return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
}
__device__ __forceinline__ float key_to_score(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Right shift mapping a key window of width range+1 onto at most kSelBins bins.
__device__ __forceinline__ int sel_shift(uint32_t range) {
  return range == 0u ? 0 : max(0, 32 - __clz(range) - kSelBinBits);
}

// A run of candidates in global memory (keys[i], pos[i]), i < n.
struct CandSeg {
  const uint32_t* key;
  const uint32_t* pos;
  int n;
};

// One refinement level: histogram of the keys in [lo, lo + (kSelBins << shift)) that
// `visit` produces, then the bin b (from the top) where the running count first
// reaches `need`, and the count strictly above bin b.  `hist` is this warp's
// shared-memory histogram.
template <typename Visit>
__device__ __forceinline__ void sel_level(uint32_t* hist, Visit visit, uint32_t lo, uint32_t hi, int shift,
                                          uint32_t need, uint32_t& bin, uint32_t& above) {
  const uint32_t lane = threadIdx.x & 31u;
  for (int i = (int)lane; i < kSelBins / 4; i += 32) reinterpret_cast<uint4*>(hist)[i] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  visit([&](uint32_t key) {
    if (key >= lo && key <= hi) atomicAdd(&hist[(key - lo) >> shift], 1u);
  });
  __syncwarp();
  // Lane j owns bins [kPer j, kPer (j + 1)).  Counts from the top: suffix sums over lanes.
  constexpr int kPer = kSelBins / 32;
  uint32_t mine = 0;
  const uint4* h4 = reinterpret_cast<const uint4*>(hist + lane * kPer);
#pragma unroll
  for (int i = 0; i < kPer / 4; ++i) {
    const uint4 v = h4[i];
    mine += v.x + v.y + v.z + v.w;
  }
  uint32_t suffix = mine;                              // bins of lanes >= this lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, suffix, o);
    if (lane + o < 32) suffix += y;
  }
  const uint32_t above_lane = suffix - mine;           // bins of lanes > this lane
  const bool here = above_lane < need && suffix >= need;
  const uint32_t owner = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
  uint32_t b = 0, ab = 0;
  if (lane == owner) {
    uint32_t acc = above_lane;
    for (int i = kPer - 1; i >= 0; --i) {
      const uint32_t c = hist[lane * kPer + i];
      if (acc + c >= need) { b = lane * kPer + i; ab = acc; break; }
      acc += c;
    }
  }
  bin = __shfl_sync(0xffffffffu, b, owner);
  above = __shfl_sync(0xffffffffu, ab, owner);
  __syncwarp();
}

// Threshold of the top-`m` of the keys in [lo, hi] that `visit` produces (keys
// outside the window are ignored), of which there are at least m.  Returns thr and
// gt = #{lo <= key <= hi, key > thr} (so m - gt keys equal to thr are taken, the
// first ones in position order).  `cand` holds up to kSelCandCap keys of the
// boundary bin.  `count`, when not 0xffffffff, is the number of keys in the window,
// known to the caller: at most kSelCandCap of them go straight to the candidates.
template <typename Visit>
__device__ __forceinline__ void warp_find_threshold(uint32_t* hist, uint32_t* cand, Visit visit, uint32_t m, uint32_t lo,
                                    uint32_t hi, uint32_t& thr, uint32_t& gt, uint32_t count = 0xffffffffu) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t need = m, got = 0;
  // Levels over the list itself until the boundary bin is small enough to copy.
  for (; count > (uint32_t)kSelCandCap;) {
    const int shift = sel_shift(hi - lo);
    uint32_t b, above;
    sel_level(hist, visit, lo, hi, shift, need, b, above);
    got += above;
    need -= above;
    if (shift == 0) { thr = lo + b; gt = got; return; }
    const uint32_t nb = hist[b];
    lo = lo + (b << shift);
    const unsigned long long top = (unsigned long long)lo + (1ull << shift) - 1ull;
    hi = top < (unsigned long long)hi ? (uint32_t)top : hi;
    __syncwarp();
    if (nb <= (uint32_t)kSelCandCap) break;
  }
  // Copy the boundary bin's keys (at most kSelCandCap) to shared memory and refine there.
  uint32_t* ncand = cand + kSelCandCap;                // counter word after the keys
  if (lane == 0) *ncand = 0u;
  __syncwarp();
  visit([&](uint32_t key) {
    if (key >= lo && key <= hi) {
      const uint32_t at = atomicAdd(ncand, 1u);
      if (at < (uint32_t)kSelCandCap) cand[at] = key;
    }
  });
  __syncwarp();
  const int nc = (int)*ncand;
  auto visit_cand = [&](auto&& f) {
    for (int i = (int)lane; i < nc; i += 32) f(cand[i]);
  };
  for (;;) {
    const int shift = sel_shift(hi - lo);
    uint32_t b, above;
    sel_level(hist, visit_cand, lo, hi, shift, need, b, above);
    got += above;
    need -= above;
    if (shift == 0) { thr = lo + b; gt = got; return; }
    lo = lo + (b << shift);
    const unsigned long long top = (unsigned long long)lo + (1ull << shift) - 1ull;
    hi = top < (unsigned long long)hi ? (uint32_t)top : hi;
    __syncwarp();
  }
}

// Calls f(key) for the keys[0 .. n) of a list, read as 16-byte groups with kVisitU
// groups in flight per lane.  A list in global memory (kGlobal) is read through L2
// only (its writers may be other CTAs), where latency rather than bytes would
// otherwise set the pace; a list in shared memory is read directly.  The list must
// start 16-byte aligned and be readable up to n rounded up to a multiple of four
// (list capacities are multiples of 32).  Lanes call f different numbers of
// times: f must not contain warp-collective operations.
constexpr int kVisitU = 4;
constexpr int kCompactU = 2;          // (key, position) group pairs in flight per lane when compacting

template <bool kGlobal>
__device__ __forceinline__ uint4 load_group(const uint4* p) {
  if constexpr (kGlobal) return __ldcg(p);
  else return *p;
}

template <bool kGlobal, typename F>
__device__ __forceinline__ void visit_list_keys(const uint32_t* key, int n, F f) {
  const int lane = (int)(threadIdx.x & 31u);
  const uint4* k4 = reinterpret_cast<const uint4*>(key);
  const int n4 = (n + 3) >> 2;
  for (int g0 = 0; g0 < n4; g0 += 32 * kVisitU) {
    uint4 v[kVisitU];
#pragma unroll
    for (int u = 0; u < kVisitU; ++u) {
      const int g = g0 + u * 32 + lane;
      v[u] = g < n4 ? load_group<kGlobal>(k4 + g) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kVisitU; ++u) {
      const int i = (g0 + u * 32 + lane) * 4;
      if (i + 0 < n) f(v[u].x);
      if (i + 1 < n) f(v[u].y);
      if (i + 2 < n) f(v[u].z);
      if (i + 3 < n) f(v[u].w);
    }
  }
}

// Exclusive prefix sum of v over the lanes of the warp; `total` receives the sum.
__device__ __forceinline__ uint32_t warp_exclusive_sum(uint32_t v, uint32_t& total) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= (uint32_t)o) x += y;
  }
  total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// Stable selection pass: walks the segments get_seg(0 .. nseg-1) in order and
// hands every kept candidate to emit(index, key, pos) with consecutive indices from
// `base`: all keys > thr and the first eq_take keys == thr.  Returns the count.
// Entries are read as 16-byte groups (lane l holds entries 4l .. 4l+3 of each 128),
// kCompactU groups per lane in flight; every group of a block is read before any of
// the block is emitted, so emitting into the list being read (at an index not
// above the one read) is safe.
template <bool kGlobal, typename GetSeg, typename Emit>
__device__ __forceinline__ uint32_t warp_compact(GetSeg get_seg, int nseg, uint32_t thr, uint32_t eq_take,
                                                 uint32_t base, Emit emit) {
  const int lane = (int)(threadIdx.x & 31u);
  uint32_t w = base, eq_seen = 0;
  for (int g = 0; g < nseg; ++g) {
    const CandSeg sg = get_seg(g);
    const uint4* k4 = reinterpret_cast<const uint4*>(sg.key);
    const uint4* p4 = reinterpret_cast<const uint4*>(sg.pos);
    const int n4 = (sg.n + 3) >> 2;
    for (int g0 = 0; g0 < n4; g0 += 32 * kCompactU) {
      uint4 kv[kCompactU], pv[kCompactU];
#pragma unroll
      for (int u = 0; u < kCompactU; ++u) {
        const int q = g0 + u * 32 + lane;
        kv[u] = q < n4 ? load_group<kGlobal>(k4 + q) : make_uint4(0u, 0u, 0u, 0u);
        pv[u] = q < n4 ? load_group<kGlobal>(p4 + q) : make_uint4(0u, 0u, 0u, 0u);
      }
      __syncwarp();
#pragma unroll
      for (int u = 0; u < kCompactU; ++u) {
        const int i = (g0 + u * 32 + lane) * 4;
        const int nv = min(4, max(0, sg.n - i));          // valid entries of this lane's group
        const uint32_t vmask = (1u << nv) - 1u;
        const uint32_t gt = vmask & ((kv[u].x > thr ? 1u : 0u) | (kv[u].y > thr ? 2u : 0u) |
                                     (kv[u].z > thr ? 4u : 0u) | (kv[u].w > thr ? 8u : 0u));
        const uint32_t eq = vmask & ((kv[u].x == thr ? 1u : 0u) | (kv[u].y == thr ? 2u : 0u) |
                                     (kv[u].z == thr ? 4u : 0u) | (kv[u].w == thr ? 8u : 0u));
        uint32_t eq_total;
        const uint32_t eq_rank = eq_seen + warp_exclusive_sum(__popc(eq), eq_total);
        // equal keys are taken in order while fewer than eq_take have been taken
        const uint32_t room = eq_take > eq_rank ? eq_take - eq_rank : 0u;   // equal keys this lane may take
        uint32_t take = 0, e = eq;
        for (uint32_t t = 0; e && t < room; ++t) {
          take |= e & (0u - e);                             // lowest remaining equal entry
          e &= e - 1u;
        }
        const uint32_t keep = gt | take;
        uint32_t keep_total;
        uint32_t at = w + warp_exclusive_sum(__popc(keep), keep_total);
        if (keep & 1u) emit(at++, kv[u].x, pv[u].x);
        if (keep & 2u) emit(at++, kv[u].y, pv[u].y);
        if (keep & 4u) emit(at++, kv[u].z, pv[u].z);
        if (keep & 8u) emit(at++, kv[u].w, pv[u].w);
        w += keep_total;
        eq_seen += eq_total;
      }
      __syncwarp();
    }
  }
  return w - base;
}

}  // namespace dsa
