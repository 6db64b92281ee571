// indexer_loss.cu -- forward of the lightning indexer's training loss.
//
// DeepSeek-V3.2 technical-report summary, section "Как учили индексатор": the
// indexer is trained towards the main attention.  For query row r (batch b,
// selection S_r) and head h, the main attention's probabilities over S_r are
//   a_h[s] = exp(scale * q[r,h,:] . kv[b,s,:] - lse[r,h]),
// their head sum P[s] = sum_h a_h[s] is L1-normalised into the target
//   p[s] = P[s] / sum_s P[s],
// and the loss of the row is the KL divergence of the indexer's softmax from it,
//   KL_r = sum_{s in S_r} p[s] (log p[s] - log softmax_{S_r}(I[r,:])[s]),
// restricted to the selected positions as in the sparse training stage (item 2
// of that section).  lse is the log-sum-exp the attention kernel returns for the
// same selection, so the logits are recomputed but never renormalised here.
//
// One CTA per query row at a time (persistent over rows), no cluster:
//   * Q (128 head rows x d_qk bf16, 9 planes of 128 x 64 columns) stays in shared
//     memory for the row; keys come in tiles of 64 selected positions, gathered
//     in 64-column chunks (TMA tile::gather4, 128-byte swizzle) through a ring.
//   * S = Q K^T per tile is a chain of tcgen05.mma (M = 128 heads, N = 64 keys,
//     K = 16), issued by one thread, double-buffered in TMEM (2 x 64 columns).
//   * Eight epilogue warps read S: warp w holds heads 32(w%4)..+31 (its TMEM lane
//     quarter) for keys 32(w/4)..+31.  Each lane turns its 32 logits into
//     probabilities with the row's lse, then the warp sums them over its 32 heads
//     by a butterfly transpose-reduction (31 shuffles leave lane i holding key
//     i's sum); the four head quarters meet in shared memory.
//   * Warps 0-1 then own one key each: they fold P into the row's running sums
//     (sum P, sum P log P, sum P (I - m), and the indexer log-sum-exp with a
//     running maximum m), write P to the target, and at the row's end combine
//     the sums into KL and rescale the target row by 1 / sum P.
// Warp roles (800 threads): 0-7 epilogue, 8 TMEM owner + MMA issuer, 9-22 key
// loaders (two warps per ring slot, each issuing half of a chunk's 16 gathers),
// 23-24 stage each row's selected positions one row ahead.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kTileKeys = 64;          // selected positions per S tile
constexpr int kStages = 7;             // key-chunk ring depth (8 KB stages)
constexpr int kWarpsPerSlot = 2;
constexpr int kEpiWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp0 = 9;
constexpr int kLoadWarps = kStages * kWarpsPerSlot;   // 14
constexpr int kStageWarp0 = kLoadWarp0 + kLoadWarps;  // 23
constexpr int kStageWarps = 2;
constexpr int kThreads = 32 * (kStageWarp0 + kStageWarps);   // 800
constexpr int kStageBatch = 8;         // index words in flight per staging warp
constexpr int kMaxIdx = 2048;
constexpr int kMaxChunks = 9;
constexpr uint32_t kQPlane = 128 * 128;   // 128 head rows x 128 B
constexpr uint32_t kChunk = 64 * 128;     // 64 key rows x 128 B
constexpr uint32_t kTmemCols = 128;       // two S buffers of 64 columns
constexpr float kLog2e = 1.4426950408889634f;

struct KlShared {
  uint64_t q_full[kMaxChunks], q_empty[kMaxChunks];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t idx_full[2], idx_empty[2];
  uint64_t xbar;                        // rendezvous of the eight epilogue warps
  uint64_t final_mma;
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t valid_mask[2][kMaxIdx / 32]; // per 32 staged slots: bit set = valid position
  float red[2][4][kTileKeys];           // per S buffer: head-quarter partial sums per key
  float fin[2][5];                      // per key warp: (Z, A, Bs, m, s) of the row
};

// Row of kv (in the [B*Lk, d_qk] view) staged for a slot; bit 31 marks padding,
// which gathers row b*Lk (a valid row) and is masked.
__device__ __forceinline__ int gather_row(const int32_t* rows, int pos) { return rows[pos] & 0x7fffffff; }

// Running sums of one row: Z = sum P, A = sum P log P, Bs = sum P (I - m),
// m = max I, s = sum exp(I - m), over the valid selected positions seen so far.
struct RowSums {
  float Z, A, Bs, m, s;
};

__device__ __forceinline__ RowSums merge(const RowSums& x, const RowSums& y) {
  RowSums r;
  r.m = fmaxf(x.m, y.m);
  const float sx = x.m == -INFINITY ? 0.f : x.s * ex2_approx((x.m - r.m) * kLog2e);
  const float sy = y.m == -INFINITY ? 0.f : y.s * ex2_approx((y.m - r.m) * kLog2e);
  r.s = sx + sy;
  // Bs is referenced to each side's own maximum: move both to the common one.
  const float bx = x.Z > 0.f ? fmaf(x.Z, x.m - r.m, x.Bs) : 0.f;
  const float by = y.Z > 0.f ? fmaf(y.Z, y.m - r.m, y.Bs) : 0.f;
  r.Bs = bx + by;
  r.Z = x.Z + y.Z;
  r.A = x.A + y.A;
  return r;
}

template <int NC>
__global__ void __launch_bounds__(kThreads, 1)
indexer_kl_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                  const KlParams p) {
  static_assert(NC <= kMaxChunks, "d_qk");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  KlShared& S = *reinterpret_cast<KlShared*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t area_off = ((raw_addr + sizeof(KlShared) + 1023u) & ~1023u) - raw_addr;
  uint8_t* q_sm = smem_raw + area_off;                              // NC planes
  uint8_t* k_sm = q_sm + NC * kQPlane;                              // kStages chunks
  int32_t* idx_sm = reinterpret_cast<int32_t*>(k_sm + kStages * kChunk);   // 2 x kMaxIdx

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  volatile uint32_t* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxChunks; ++i) { mbar_init(&S.q_full[i], 1); mbar_init(&S.q_empty[i], 1); }
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.k_full[i], 1); mbar_init(&S.k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], kEpiWarps);
      mbar_init(&S.idx_full[i], kStageWarps);
      mbar_init(&S.idx_empty[i], kLoadWarps + kEpiWarps);
    }
    mbar_init(&S.xbar, kEpiWarps);
    mbar_init(&S.final_mma, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  bool ok = true;

  if (warp >= kStageWarp0) {
    // ------------------------------------------------------------------ index staging
    // Row ordinal n goes to buffer n % 2 as kv rows to gather (batch offset applied,
    // bit 31 on padding and out-of-range entries) plus one validity ballot per 32
    // slots.  Slots past k are padding.
    const int sw = (int)warp - kStageWarp0;
    const int nwords = p.n_tiles * (kTileKeys / 32);
    uint32_t ucount = 0;
    for (int row = blockIdx.x; row < p.n_rows && ok; row += gridDim.x, ++ucount) {
      const uint32_t buf = ucount & 1u, ph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_empty[buf], ph ^ 1u, abort_flag);
      if (!ok) break;
      const int b = row / p.Lq;
      int32_t* dst = idx_sm + buf * kMaxIdx;
      const int32_t* src = p.indices + (size_t)row * p.k;
      for (int w0 = sw; w0 < nwords; w0 += kStageWarps * kStageBatch) {
        int sidx[kStageBatch];
#pragma unroll
        for (int e = 0; e < kStageBatch; ++e) {
          const int w = w0 + e * kStageWarps, x = w * 32 + (int)lane;
          sidx[e] = (w < nwords && x < p.k) ? __ldg(src + x) : -1;
        }
#pragma unroll
        for (int e = 0; e < kStageBatch; ++e) {
          const int w = w0 + e * kStageWarps;
          if (w >= nwords) break;                     // warp-uniform
          const bool valid = sidx[e] >= 0 && sidx[e] < p.Lk;
          const int grow = b * p.Lk + (valid ? sidx[e] : 0);
          dst[w * 32 + (int)lane] = valid ? grow : (int)((uint32_t)grow | 0x80000000u);
          const uint32_t bal = __ballot_sync(0xffffffffu, valid);
          if (lane == 0) S.valid_mask[buf][w] = bal;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_full[buf]);
    }
  } else if (warp >= kLoadWarp0) {
    // ------------------------------------------------------------------ key loaders
    // Per row: the Q planes (plane c from loader c % kLoadWarps), then for each
    // tile its NC key chunks (64 keys x 64 columns).  Chunk kc goes to ring slot
    // kc % kStages; the slot's two warps issue its 16 four-row gathers, groups
    // g = part, part + 2, ...
    const int pw = (int)warp - kLoadWarp0;
    const uint32_t my_slot = (uint32_t)(pw / kWarpsPerSlot);
    const int part = pw % kWarpsPerSlot;
    uint32_t ucount = 0, kc = 0;
    if (pw == 0 && lane == 0) { prefetch_tmap(&tmap_q); prefetch_tmap(&tmap_kv); }
    for (int row = blockIdx.x; row < p.n_rows && ok; row += gridDim.x, ++ucount) {
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      if (lane == 0) {
        for (int c = pw; c < NC && ok; c += kLoadWarps) {
          ok = mbar_wait(&S.q_empty[c], (ucount & 1u) ^ 1u, abort_flag);
          if (!ok) break;
          mbar_arrive_expect_tx(&S.q_full[c], kQPlane);
          tma_load_2d(q_sm + c * kQPlane, &tmap_q, &S.q_full[c], c * 64, row * p.H);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      const int32_t* idx = idx_sm + ib * kMaxIdx;
      for (int j = 0; j < p.n_tiles && ok; ++j) {
        for (int c = 0; c < NC; ++c, ++kc) {
          const uint32_t st = kc % kStages, ph = (kc / kStages) & 1u;
          if (st != my_slot) continue;
          bool w_ok = true;
          if (lane == 0) {
            w_ok = mbar_wait(&S.k_empty[st], ph ^ 1u, abort_flag);
            if (w_ok && part == 0) mbar_arrive_expect_tx(&S.k_full[st], kChunk);
          }
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
          const int g = part + kWarpsPerSlot * (int)lane;         // 4-key group of this lane
          if (g < kTileKeys / 4) {
            const int base = j * kTileKeys + g * 4;
            tma_gather4(k_sm + st * kChunk + g * 512, &tmap_kv, &S.k_full[st], c * 64, gather_row(idx, base + 0),
                        gather_row(idx, base + 1), gather_row(idx, base + 2), gather_row(idx, base + 3));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // S = Q K^T for each tile into TMEM buffer (tile ordinal % 2): per key chunk,
    // 4 MMAs of K = 16 (descriptor start addresses advance 32 B, encoded 2).
    if (elect_one()) {
      constexpr uint32_t idesc = make_idesc(1, 1, 128, kTileKeys, 0, 0);   // bf16, K-major x K-major
      const uint64_t q_desc = make_smem_desc(smem_u32(q_sm), 16, 1024, LAYOUT_SW128);
      const uint64_t k_desc = make_smem_desc(smem_u32(k_sm), 16, 1024, LAYOUT_SW128);
      uint32_t ucount = 0, kc = 0, sc = 0;
      for (int row = blockIdx.x; row < p.n_rows && ok; row += gridDim.x, ++ucount) {
        for (int j = 0; j < p.n_tiles && ok; ++j, ++sc) {
          const uint32_t sb = sc & 1u;
          ok = mbar_wait(&S.s_empty[sb], ((sc >> 1) & 1u) ^ 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem_base + sb * kTileKeys;
          for (int c = 0; c < NC; ++c, ++kc) {
            if (j == 0 && !mbar_wait(&S.q_full[c], ucount & 1u, abort_flag)) { ok = false; break; }
            const uint32_t st = kc % kStages, ph = (kc / kStages) & 1u;
            if (!mbar_wait(&S.k_full[st], ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = q_desc + (uint64_t)(c * (kQPlane >> 4));
            const uint64_t bd = k_desc + (uint64_t)(st * (kChunk >> 4));
            mma_bf16_ss(d, ad + 0, bd + 0, idesc, c ? 1u : 0u);
            mma_bf16_ss(d, ad + 2, bd + 2, idesc, 1u);
            mma_bf16_ss(d, ad + 4, bd + 4, idesc, 1u);
            mma_bf16_ss(d, ad + 6, bd + 6, idesc, 1u);
            mma_commit(&S.k_empty[st]);
            if (j == p.n_tiles - 1) mma_commit(&S.q_empty[c]);   // plane free for the next row
          }
          if (!ok) break;
          mma_commit(&S.s_full[sb]);
        }
      }
      // Every MMA this thread issued completes before the TMEM is released.
      mma_commit(&S.final_mma);
      mbar_wait(&S.final_mma, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3u;            // TMEM lane quarter = head group
    const int c0 = (int)(warp >> 2) * 32;          // this warp's 32 keys of the tile
    const int head = (int)quarter * 32 + (int)lane;
    const bool head_ok = head < p.H;
    const uint32_t lane_addr = (quarter * 32u) << 16;
    const bool keyer = warp < 2;                   // owns key `key` of every tile
    const int key = (int)warp * 32 + (int)lane;
    const float2 scl = make_float2(p.scale_log2, p.scale_log2);
    uint32_t ucount = 0, sc = 0, xph = 0;
    for (int row = blockIdx.x; row < p.n_rows && ok; row += gridDim.x, ++ucount) {
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      const int32_t* idx = idx_sm + ib * kMaxIdx;
      const int bLk = (row / p.Lq) * p.Lk;
      const float* srow = p.scores + (size_t)row * p.Lk;
      float* trow = p.target ? p.target + (size_t)row * p.k : nullptr;
      // exponent offset: a_h[s] = 2^(z * scale * log2 e - lse * log2 e)
      const float nl = head_ok ? -p.lse[(size_t)row * p.H + head] * kLog2e : 0.f;
      const float2 nl2 = make_float2(nl, nl);
      RowSums acc{0.f, 0.f, 0.f, -INFINITY, 0.f};
      for (int j = 0; j < p.n_tiles && ok; ++j, ++sc) {
        // The key warps fetch this tile's indexer scores before waiting for S.
        const int slot = j * kTileKeys + key;
        bool kvalid = false;
        float iv = 0.f;
        if (keyer) {
          const int32_t gr = idx[slot];
          kvalid = gr >= 0;
          if (kvalid) iv = __ldg(srow + (gr - bLk));
        }
        const uint32_t sb = sc & 1u;
        ok = mbar_wait_warp(&S.s_full[sb], (sc >> 1) & 1u, abort_flag);
        if (!ok) break;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_addr + sb * kTileKeys + c0, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.s_empty[sb]);
        const uint32_t vm = head_ok ? S.valid_mask[ib][(j * kTileKeys + c0) >> 5] : 0u;
        float pr[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), scl, nl2);
          pr[e] = ((vm >> e) & 1u) ? ex2_approx(x.x) : 0.f;
          pr[e + 1] = ((vm >> (e + 1)) & 1u) ? ex2_approx(x.y) : 0.f;
        }
        // Butterfly transpose-reduction over the warp's 32 heads: at each step a lane
        // keeps the half of its columns selected by one bit of its lane number and
        // adds the partner's copy of that half.  Lane i ends with key c0 + i.
#pragma unroll
        for (int half = 16; half >= 1; half >>= 1) {
          const bool up = (lane & (uint32_t)half) != 0u;
#pragma unroll
          for (int e = 0; e < half; ++e) {
            const float lo = pr[e], hi = pr[e + half];
            const float send = up ? lo : hi;
            const float keep = up ? hi : lo;
            pr[e] = keep + __shfl_xor_sync(0xffffffffu, send, half);
          }
        }
        S.red[sb][quarter][c0 + (int)lane] = pr[0];
        ok = warps_rendezvous(&S.xbar, xph, abort_flag);
        if (!ok) break;
        if (keyer) {
          const float P = (S.red[sb][0][key] + S.red[sb][1][key]) + (S.red[sb][2][key] + S.red[sb][3][key]);
          if (kvalid) {
            if (iv > acc.m) {                          // move the references to the new maximum
              if (acc.Z > 0.f) acc.Bs = fmaf(-acc.Z, iv - acc.m, acc.Bs);
              acc.s = acc.m == -INFINITY ? 0.f : acc.s * ex2_approx((acc.m - iv) * kLog2e);
              acc.m = iv;
            }
            if (iv != -INFINITY) acc.s += ex2_approx((iv - acc.m) * kLog2e);
            acc.Z += P;
            if (P > 0.f) {
              acc.Bs = fmaf(P, iv - acc.m, acc.Bs);
              acc.A = fmaf(P, __logf(P), acc.A);
            }
          }
          if (trow && slot < p.k) trow[slot] = P;      // rescaled once the row's sum is known
        }
      }
      if (!ok) break;
      // ---- end of the row: combine the key warps' sums into KL and normalise the target
      if (keyer) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          RowSums o;
          o.Z = __shfl_xor_sync(0xffffffffu, acc.Z, off);
          o.A = __shfl_xor_sync(0xffffffffu, acc.A, off);
          o.Bs = __shfl_xor_sync(0xffffffffu, acc.Bs, off);
          o.m = __shfl_xor_sync(0xffffffffu, acc.m, off);
          o.s = __shfl_xor_sync(0xffffffffu, acc.s, off);
          acc = merge(acc, o);
        }
        if (lane == 0) {
          S.fin[warp][0] = acc.Z; S.fin[warp][1] = acc.A; S.fin[warp][2] = acc.Bs;
          S.fin[warp][3] = acc.m; S.fin[warp][4] = acc.s;
        }
      }
      ok = warps_rendezvous(&S.xbar, xph, abort_flag);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
      if (!ok) break;
      if (keyer) {
        const RowSums r0{S.fin[0][0], S.fin[0][1], S.fin[0][2], S.fin[0][3], S.fin[0][4]};
        const RowSums r1{S.fin[1][0], S.fin[1][1], S.fin[1][2], S.fin[1][3], S.fin[1][4]};
        const RowSums r = merge(r0, r1);
        // KL = sum p log p - sum p (I - lse_I) with p = P / Z:
        //    = (A - Bs) / Z - log Z + log s    (lse_I = m + log s; Bs is relative to m)
        if (warp == 0 && lane == 0)
          p.kl[row] = r.Z > 0.f ? (r.A - r.Bs) / r.Z - logf(r.Z) + logf(r.s) : 0.f;
        if (trow && r.Z > 0.f) {
          const float inv = 1.f / r.Z;
          for (int x = key; x < p.k; x += kTileKeys) trow[x] *= inv;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int NC>
cudaError_t launch_t(const KlParams& p, const CUtensorMap& tq, const CUtensorMap& tkv, int grid,
                     cudaStream_t stream) {
  const size_t smem = indexer_kl_smem_bytes(NC * 64);
  auto kern = indexer_kl_kernel<NC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tq, tkv, p);
  return cudaGetLastError();
}

}  // namespace

size_t indexer_kl_smem_bytes(int d_qk) {
  const int nc = d_qk / 64;
  size_t b = sizeof(KlShared) + 1024;              // shared state + alignment slack
  b += (size_t)nc * kQPlane;                       // Q
  b += (size_t)kStages * kChunk;                   // key ring
  b += 2 * (size_t)kMaxIdx * sizeof(int32_t);      // staged positions, two rows
  return b;
}

cudaError_t launch_indexer_kl(const KlParams& p, int d_qk, const CUtensorMap& tq, const CUtensorMap& tkv, int grid,
                              cudaStream_t stream) {
  if (d_qk == 576) return launch_t<9>(p, tq, tkv, grid, stream);
  if (d_qk == 192) return launch_t<3>(p, tq, tkv, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t read_kl_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
