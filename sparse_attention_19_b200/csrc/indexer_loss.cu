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
// Mapping onto a pair of SMs (a 2-CTA cluster, tcgen05 .cta_group::2), one query
// row at a time per pair:
//   * Each CTA holds 64 of the 128 heads' Q rows (64 x d_qk bf16) in shared
//     memory, so most of the shared memory is left for keys in flight: a ring of
//     16 chunks of 64 gathered latent rows x 64 columns per CTA (TMA
//     tile::gather4, 128-byte swizzle).  Eight loader warps own two ring slots
//     each and issue all 16 gathers of their chunks, one per lane.
//   * Keys come in tiles of 128 selected positions; S^T = K Q^T is one pair-MMA
//     chain (M = 128 keys, 64 per CTA: the CTA's own gathered rows; N = 128 heads,
//     64 per CTA: its own Q rows; K = 16 per instruction) issued by one thread of
//     the leader CTA, into four S buffers in TMEM.  Each CTA's TMEM holds its 64
//     keys against all 128 heads: lane l holds key l % 64 and heads
//     64 (l / 64) .. 64 (l / 64) + 63 in its 64 columns.  So a key's head sum is
//     a per-thread sum over columns, with no exchange between threads.
//   * Eight reduction warps per CTA read S: warp w holds TMEM lane quarter w % 4
//     (32 keys, one head half) and 32 of the half's 64 heads.  Each thread turns
//     its key's 32 logits into probabilities with the heads' lse and sums them,
//     then posts the sum to a 3-tile ring in the leader's shared memory: the
//     leader's warps with plain stores and an arrive, the other CTA's with
//     st.async, whose bytes complete the same barrier.
//   * Four loss warps of the leader own one key each: per tile they add the four
//     head-quarter sums into P, fold it into the row's running sums (sum P,
//     sum P log P, sum P (I - m), and the indexer log-sum-exp with a running
//     maximum m) and write P to the target; at the row's end they combine the
//     sums into KL and rescale the target row by 1 / sum P.  The ring keeps this
//     chain off the path of the TMEM reads.
// A row's tiles end at the last one holding a valid position (for top-k output,
// which is valid-first, the all-padding tail of short rows is skipped).
// Warp roles (768 threads per CTA): 0-7 reduction, 8-11 loss (leader), 12 TMEM
// owner + MMA issuer (leader), 13-14 stage each row's selected positions one row
// ahead, 16-23 key loaders (each owning two ring slots).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kTileKeys = 128;         // selected positions per S tile (pair)
constexpr int kHalfKeys = 64;          // keys per CTA in B, and per TMEM lane half
constexpr int kStages = 16;            // key-chunk ring depth (8 KB stages)
constexpr int kRedWarps = 8;           // reduction warps (warpgroups 0-1)
constexpr int kLossWarp0 = 8;          // loss warps (warpgroup 2, leader)
constexpr int kLossWarps = kTileKeys / 32;
constexpr int kMmaWarp = 12;
constexpr int kStageWarp0 = 13;
constexpr int kStageWarps = 2;
constexpr int kLoadWarp0 = 16;
// Eight loader warps, each owning two ring slots and issuing all 16 gathers of
// their chunks (lanes 0-15): measured faster than teams of two or four warps per
// chunk (fewer waits and index loads for the same gather rate).
constexpr int kTeamWarps = 1;          // loader warps sharing each chunk's 16 gathers
constexpr int kTeamSlots = 2;          // consecutive ring slots a team owns
constexpr int kLoadWarps = kStages / kTeamSlots * kTeamWarps;   // 8
constexpr int kThreads = 32 * (kLoadWarp0 + kLoadWarps);   // 768
constexpr int kRedSlots = 3;           // tiles of head sums in flight to the loss warps
constexpr uint32_t kPeerBytes = kRedWarps * 32 * 4;       // the other CTA's sums per tile
constexpr int kStageBatch = 8;         // index words in flight per staging warp
constexpr int kMaxIdx = 2048;
constexpr int kMaxChunks = 9;
constexpr uint32_t kPlane = 64 * 128;  // 64 rows x 128 B (Q plane, key chunk)
constexpr int kSBufs = 4;              // S buffers in TMEM (64 columns each per CTA)
constexpr uint32_t kTmemCols = kSBufs * 64;
constexpr float kLog2e = 1.4426950408889634f;

struct KlShared {
  uint64_t q_full[kMaxChunks], q_empty[kMaxChunks];
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t s_full[kSBufs], s_empty[kSBufs];
  uint64_t idx_full[2], idx_empty[2];
  uint64_t red_full[kRedSlots];          // leader: its reduction warps + the other CTA's bytes
  uint64_t red_empty[kRedSlots];         // both CTAs: the leader's loss warps
  uint64_t lbar;                         // rendezvous of the loss warps
  uint64_t final_mma;
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t valid_mask[2][kMaxIdx / 32];  // per 32 staged slots: bit set = valid position
  int32_t last_word[2][kStageWarps];     // per staging warp: last 32-slot word with a valid position
  float red[kRedSlots][4][kTileKeys];    // leader: per tile, 32-head sums (head quarter), per key
  alignas(16) float nl[kRedWarps][32];   // per reduction warp: -lse * log2 e of its 32 heads (row)
  float fin[kLossWarps][5];              // leader: per loss warp (Z, A, Bs, m, s) of the row
};

// Rows of kv (in the [B*Lk, d_qk] view) staged for four consecutive slots; padding
// was staged as row b*Lk (a valid row) and is masked through valid_mask.
__device__ __forceinline__ int4 gather_rows4(const int32_t* rows, int pos) {
  return *reinterpret_cast<const int4*>(rows + pos);   // four consecutive slots, pos a multiple of 4
}

// Tiles of the staged row in buffer `buf`: up to the last one that holds a valid
// position (top-k output is valid-first, so this skips its all-padding tail).
__device__ __forceinline__ int row_tiles(const volatile int32_t (*last_word)[kStageWarps], uint32_t buf) {
  int last = -1;
#pragma unroll
  for (int w = 0; w < kStageWarps; ++w) last = max(last, (int)last_word[buf][w]);
  return (last + 1 + (kTileKeys / 32) - 1) / (kTileKeys / 32);
}

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
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
indexer_kl_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                  const KlParams p) {
  static_assert(NC <= kMaxChunks, "d_qk");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  KlShared& S = *reinterpret_cast<KlShared*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t area_off = ((raw_addr + sizeof(KlShared) + 1023u) & ~1023u) - raw_addr;
  uint8_t* q_sm = smem_raw + area_off;                              // NC planes
  uint8_t* k_sm = q_sm + NC * kPlane;                               // kStages chunks
  int32_t* idx_sm = reinterpret_cast<int32_t*>(k_sm + kStages * kPlane);   // 2 x kMaxIdx

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  volatile uint32_t* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxChunks; ++i) { mbar_init(&S.q_full[i], 1); mbar_init(&S.q_empty[i], 1); }
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.k_full[i], 1); mbar_init(&S.k_empty[i], 1); }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 2 * kRedWarps);           // both CTAs' reduction warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.idx_full[i], kStageWarps);
      // readers of the staged positions: loaders, reduction warps, and the leader's loss
      // warps and MMA issuer
      mbar_init(&S.idx_empty[i], kLoadWarps + kRedWarps + (leader ? kLossWarps + 1 : 0));
    }
    for (int i = 0; i < kRedSlots; ++i) {
      mbar_init(&S.red_full[i], kRedWarps);              // + kPeerBytes of transaction count
      mbar_init(&S.red_empty[i], kLossWarps);
    }
    mbar_init(&S.lbar, kLossWarps);
    mbar_init(&S.final_mma, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&S.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = S.tmem_base;
  const uint16_t kBoth = 0x3;
  griddep_launch_dependents();
  griddep_wait();                                      // the previous kernel's writes are visible
  bool ok = true;

  if (warp >= kLoadWarp0) {
    // ------------------------------------------------------------------ key loaders
    // Per row with tiles: this CTA's Q planes (plane c from loader c % kLoadWarps),
    // then for each tile its NC key chunks (this CTA's 64 keys x 64 columns).  Chunk
    // kc goes to ring slot kc % kStages; the team of kTeamWarps warps that owns that
    // slot splits its 16 four-row gathers (groups g = part, part + kTeamWarps, ...).
    // Both CTAs' loads complete on the leader's barriers.
    const int pw = (int)warp - kLoadWarp0;
    const uint32_t my_team = (uint32_t)(pw / kTeamWarps);
    const int part = pw % kTeamWarps;
    uint32_t ucount = 0, qcount = 0, kc = 0;
    if (pw == 0 && lane == 0) { prefetch_tmap(&tmap_q); prefetch_tmap(&tmap_kv); }
    for (int row = cluster_id; row < p.n_rows && ok; row += n_clusters, ++ucount) {
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      const int nt = row_tiles(S.last_word, ib);
      if (nt > 0) {
        if (lane == 0) {
          const int qrow = row * p.H + (int)rank * 64;
          for (int c = pw; c < NC && ok; c += kLoadWarps) {
            ok = mbar_wait(&S.q_empty[c], (qcount & 1u) ^ 1u, abort_flag);
            if (!ok) break;
            if (leader) mbar_arrive_expect_tx(&S.q_full[c], 2u * kPlane);
            tma_load_2d_pair(q_sm + c * kPlane, &tmap_q, mapa_shared(smem_u32(&S.q_full[c]), 0), c * 64, qrow);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        ++qcount;
      }
      const int32_t* idx = idx_sm + ib * kMaxIdx;
      // This row's chunks are kc0 .. kc0 + nt*NC - 1; visit only the team's slots.
      const uint32_t kc0 = kc, kc_end = kc0 + (uint32_t)(nt * NC);
      while (kc < kc_end && (kc % kStages) / kTeamSlots != my_team) ++kc;
      for (; kc < kc_end && ok;
           kc += ((kc % kTeamSlots) == kTeamSlots - 1) ? (uint32_t)(kStages - kTeamSlots + 1) : 1u) {
        {
          const uint32_t st = kc % kStages, ph = (kc / kStages) & 1u;
          const int j = (int)((kc - kc0) / NC), c = (int)((kc - kc0) % NC);
          bool w_ok = true;
          if (lane == 0) {
            w_ok = mbar_wait(&S.k_empty[st], ph ^ 1u, abort_flag);
            if (w_ok && leader && part == 0) mbar_arrive_expect_tx(&S.k_full[st], 2u * kPlane);
          }
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
          const int g = part + kTeamWarps * (int)lane;             // 4-key group of this lane
          if (g < kHalfKeys / 4) {
            const int4 r4 = gather_rows4(idx, j * kTileKeys + (int)rank * kHalfKeys + g * 4);
            tma_gather4_pair(k_sm + st * kPlane + g * 512, &tmap_kv, mapa_shared(smem_u32(&S.k_full[st]), 0),
                             c * 64, r4.x, r4.y, r4.z, r4.w);
          }
        }
      }
      kc = kc_end;                                     // every warp's count moves past the row
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
    }
  } else if (warp >= kStageWarp0 && warp < kStageWarp0 + kStageWarps) {
    // ------------------------------------------------------------------ index staging
    // Row ordinal n goes to buffer n % 2 as kv rows to gather (batch offset applied;
    // padding and out-of-range entries gather row b*Lk) plus one validity ballot
    // per 32 slots.  Slots past k are padding.  Both CTAs stage the whole row.
    const int sw = (int)warp - kStageWarp0;
    const int nwords = p.n_tiles * (kTileKeys / 32);
    uint32_t ucount = 0;
    for (int row = cluster_id; row < p.n_rows && ok; row += n_clusters, ++ucount) {
      const uint32_t buf = ucount & 1u, ph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_empty[buf], ph ^ 1u, abort_flag);
      if (!ok) break;
      const int b = row / p.Lq;
      int last = -1;
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
          dst[w * 32 + (int)lane] = grow;              // validity: the ballot below
          const uint32_t bal = __ballot_sync(0xffffffffu, valid);
          if (lane == 0) S.valid_mask[buf][w] = bal;
          if (bal) last = w;                          // words are visited in increasing order
        }
      }
      if (lane == 0) S.last_word[buf][sw] = last;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_full[buf]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    // S^T = K Q^T for each tile into TMEM buffer (tile ordinal % kSBufs): per key
    // chunk, 4 pair-MMAs of K = 16 (descriptor start addresses advance 32 B, encoded 2).
    if (leader && elect_one()) {
      constexpr uint32_t idesc = make_idesc(1, 1, 128, kTileKeys, 0, 0);   // bf16, K-major x K-major
      const uint64_t q_desc = make_smem_desc(smem_u32(q_sm), 16, 1024, LAYOUT_SW128);
      const uint64_t k_desc = make_smem_desc(smem_u32(k_sm), 16, 1024, LAYOUT_SW128);
      uint32_t ucount = 0, qcount = 0, kc = 0, sc = 0;
      for (int row = cluster_id; row < p.n_rows && ok; row += n_clusters, ++ucount) {
        const uint32_t ib = ucount & 1u;
        ok = mbar_wait(&S.idx_full[ib], (ucount >> 1) & 1u, abort_flag);
        if (!ok) break;
        const int nt = row_tiles(S.last_word, ib);
        for (int j = 0; j < nt && ok; ++j, ++sc) {
          const uint32_t sb = sc % kSBufs;
          ok = mbar_wait(&S.s_empty[sb], ((sc / kSBufs) & 1u) ^ 1u, abort_flag, true);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d = tmem_base + sb * kHalfKeys;
          for (int c = 0; c < NC; ++c, ++kc) {
            if (j == 0 && !mbar_wait(&S.q_full[c], qcount & 1u, abort_flag)) { ok = false; break; }
            const uint32_t st = kc % kStages, ph = (kc / kStages) & 1u;
            if (!mbar_wait(&S.k_full[st], ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            // A = this tile's key chunk (keys on M), B = the Q plane (heads on N)
            const uint64_t ad = k_desc + (uint64_t)(st * (kPlane >> 4));
            const uint64_t bd = q_desc + (uint64_t)(c * (kPlane >> 4));
            mma_bf16_ss_pair(d, ad + 0, bd + 0, idesc, c ? 1u : 0u);
            mma_bf16_ss_pair(d, ad + 2, bd + 2, idesc, 1u);
            mma_bf16_ss_pair(d, ad + 4, bd + 4, idesc, 1u);
            mma_bf16_ss_pair(d, ad + 6, bd + 6, idesc, 1u);
            mma_commit_pair_mc(&S.k_empty[st], kBoth);
            if (j == nt - 1) mma_commit_pair_mc(&S.q_empty[c], kBoth);   // plane free for the next row
          }
          if (!ok) break;
          mma_commit_pair_mc(&S.s_full[sb], kBoth);
        }
        if (nt > 0) ++qcount;
        mbar_arrive(&S.idx_empty[ib]);
      }
      // Every MMA this thread issued completes before the TMEM is released.
      mma_commit(&S.final_mma);
      mbar_wait(&S.final_mma, 0, nullptr);
    }
  } else if (warp < (uint32_t)kRedWarps) {
    // ------------------------------------------------------------------ reduction warps
    const uint32_t quarter = warp & 3u;            // TMEM lane quarter
    const int hh = (int)(quarter >> 1);            // head half held by these lanes
    const int key_c = (int)(quarter & 1u) * 32 + (int)lane;   // this thread's key among the CTA's 64
    const int key = (int)rank * kHalfKeys + key_c; // and within the tile
    const int c0 = (int)(warp >> 2) * 32;          // this warp's 32 of the half's 64 heads (columns)
    const int hq = hh * 2 + (int)(warp >> 2);      // head quarter: heads 32 hq .. 32 hq + 31
    const uint32_t lane_addr = (quarter * 32u) << 16;
    const float2 scl = make_float2(p.scale_log2, p.scale_log2);
    // where this thread's sum goes in the leader's ring, and the barrier that counts them
    const uint32_t red_dst = mapa_shared(smem_u32(&S.red[0][hq][key]), 0);
    const uint32_t red_full0 = mapa_shared(smem_u32(&S.red_full[0]), 0);
    const float4* nl4 = reinterpret_cast<const float4*>(S.nl[warp]);
    uint32_t ucount = 0, sc = 0;
    for (int row = cluster_id; row < p.n_rows && ok; row += n_clusters, ++ucount) {
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      const int nt = row_tiles(S.last_word, ib);
      // exponent offsets of this warp's 32 heads: a_h[s] = 2^(z * scale * log2 e - lse_h * log2 e);
      // heads past H get -inf (probability 0)
      {
        const int head = hq * 32 + (int)lane;
        __syncwarp();                                // the previous row's reads are done
        S.nl[warp][lane] = (head < p.H && nt > 0) ? -p.lse[(size_t)row * p.H + head] * kLog2e : -INFINITY;
        __syncwarp();
      }
      for (int j = 0; j < nt && ok; ++j, ++sc) {
        const uint32_t sb = sc % kSBufs;
        ok = mbar_wait_warp(&S.s_full[sb], (sc / kSBufs) & 1u, abort_flag);
        if (!ok) break;
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_addr + sb * kHalfKeys + c0, v);
        tmem_ld_wait();
        tmem_regs_ready(v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.s_empty[sb]), 0));
        const bool kvalid = (S.valid_mask[ib][(j * kTileKeys + key) >> 5] >> (key & 31)) & 1u;
        // sum over the 32 heads of 2^(z * scale * log2 e + nl_h)
        float2 acc_a = make_float2(0.f, 0.f), acc_b = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 n4 = nl4[e / 4];
          const float2 xa = ffma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), scl,
                                  make_float2(n4.x, n4.y));
          const float2 xb = ffma2(make_float2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])), scl,
                                  make_float2(n4.z, n4.w));
          acc_a = fadd2(acc_a, make_float2(ex2_approx(xa.x), ex2_approx(xa.y)));
          acc_b = fadd2(acc_b, make_float2(ex2_approx(xb.x), ex2_approx(xb.y)));
        }
        const float2 t2 = fadd2(acc_a, acc_b);
        const float psum = kvalid ? t2.x + t2.y : 0.f;
        // Post to ring slot sc % kRedSlots once the loss warps are done with it.
        const uint32_t slot = sc % kRedSlots, rph = (sc / kRedSlots) & 1u;
        ok = mbar_wait_warp(&S.red_empty[slot], rph ^ 1u, abort_flag, true);
        if (!ok) break;
        const uint32_t off = slot * (uint32_t)sizeof(S.red[0]);
        if (leader) {
          S.red[slot][hq][key] = psum;
          __syncwarp();
          if (lane == 0) {
            if (warp == 0) mbar_arrive_expect_tx(&S.red_full[slot], kPeerBytes);
            else mbar_arrive(&S.red_full[slot]);
          }
        } else {
          st_async_f32(red_dst + off, psum, red_full0 + slot * 8u);
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
    }
  } else if (warp >= (uint32_t)kLossWarp0 && warp < (uint32_t)(kLossWarp0 + kLossWarps) && leader) {
    // ------------------------------------------------------------------ loss warps (leader)
    const int key = ((int)warp - kLossWarp0) * 32 + (int)lane;   // key of every tile this thread owns
    uint32_t ucount = 0, sc = 0, lph = 0;
    const uint32_t peer_empty0 = mapa_shared(smem_u32(&S.red_empty[0]), 1);
    for (int row = cluster_id; row < p.n_rows && ok; row += n_clusters, ++ucount) {
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      const int32_t* idx = idx_sm + ib * kMaxIdx;
      const int nt = row_tiles(S.last_word, ib);
      const int bLk = (row / p.Lq) * p.Lk;
      const float* srow = p.scores ? p.scores + (size_t)row * p.Lk : nullptr;
      float* trow = p.target ? p.target + (size_t)row * p.k : nullptr;
      RowSums acc{0.f, 0.f, 0.f, -INFINITY, 0.f};
      // The indexer score of this thread's key in tile j (0 for padding or past the
      // row's tiles); fetched four tiles before it is used, so that its DRAM latency
      // stays off the chain.
      const float* selrow = p.sel_scores ? p.sel_scores + (size_t)row * p.k : nullptr;
      auto fetch = [&](int j) -> float {
        if (j >= nt) return 0.f;
        const int slot = j * kTileKeys + key;
        if (!((S.valid_mask[ib][slot >> 5] >> (slot & 31)) & 1u)) return 0.f;
        return selrow ? __ldg(selrow + slot) : __ldg(srow + (idx[slot] - bLk));
      };
      auto consume = [&](int j, float iv) -> bool {
        const int slot_x = j * kTileKeys + key;
        const bool kvalid = (S.valid_mask[ib][slot_x >> 5] >> (slot_x & 31)) & 1u;
        const uint32_t slot = sc % kRedSlots, rph = (sc / kRedSlots) & 1u;
        ++sc;
        if (!mbar_wait_warp(&S.red_full[slot], rph, abort_flag, true)) return false;
        const float P = (S.red[slot][0][key] + S.red[slot][1][key]) + (S.red[slot][2][key] + S.red[slot][3][key]);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.red_empty[slot]);
          mbar_arrive_cluster(peer_empty0 + slot * 8u);
        }
        if (kvalid) {
          if (iv > acc.m) {                            // move the references to the new maximum
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
        if (trow && slot_x < p.k) trow[slot_x] = P;    // rescaled once the row's sum is known
        return true;
      };
      float iv0 = fetch(0), iv1 = fetch(1), iv2 = fetch(2), iv3 = fetch(3);
      for (int j = 0; j < nt && ok; j += 4) {
        ok = consume(j, iv0);
        iv0 = fetch(j + 4);
        if (ok && j + 1 < nt) { ok = consume(j + 1, iv1); iv1 = fetch(j + 5); }
        if (ok && j + 2 < nt) { ok = consume(j + 2, iv2); iv2 = fetch(j + 6); }
        if (ok && j + 3 < nt) { ok = consume(j + 3, iv3); iv3 = fetch(j + 7); }
      }
      if (!ok) break;
      // ---- end of the row: combine the loss warps' sums into KL and normalise the target
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        RowSums y;
        y.Z = __shfl_xor_sync(0xffffffffu, acc.Z, o);
        y.A = __shfl_xor_sync(0xffffffffu, acc.A, o);
        y.Bs = __shfl_xor_sync(0xffffffffu, acc.Bs, o);
        y.m = __shfl_xor_sync(0xffffffffu, acc.m, o);
        y.s = __shfl_xor_sync(0xffffffffu, acc.s, o);
        acc = merge(acc, y);
      }
      const int lw = (int)warp - kLossWarp0;
      if (lane == 0) {
        S.fin[lw][0] = acc.Z; S.fin[lw][1] = acc.A; S.fin[lw][2] = acc.Bs;
        S.fin[lw][3] = acc.m; S.fin[lw][4] = acc.s;
      }
      ok = warps_rendezvous(&S.lbar, lph, abort_flag);
      if (!ok) break;
      RowSums r{S.fin[0][0], S.fin[0][1], S.fin[0][2], S.fin[0][3], S.fin[0][4]};
#pragma unroll
      for (int w = 1; w < kLossWarps; ++w)
        r = merge(r, RowSums{S.fin[w][0], S.fin[w][1], S.fin[w][2], S.fin[w][3], S.fin[w][4]});
      ok = warps_rendezvous(&S.lbar, lph, abort_flag);   // fin is rewritten at the next row's end
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
      if (!ok) break;
      // KL = sum p log p - sum p (I - lse_I) with p = P / Z:
      //    = (A - Bs) / Z - log Z + log s    (lse_I = m + log s; Bs is relative to m)
      if (lw == 0 && lane == 0) p.kl[row] = r.Z > 0.f ? (r.A - r.Bs) / r.Z - logf(r.Z) + logf(r.s) : 0.f;
      if (trow) {
        // loads in batches of eight, then their stores: two round trips per row;
        // slots past the processed tiles are padding and get 0
        const float inv = r.Z > 0.f ? 1.f / r.Z : 0.f;
        const int done = nt * kTileKeys;
        constexpr int kBatch = 8;
        for (int i0 = 0; i0 < kMaxIdx / kTileKeys; i0 += kBatch) {
          float t[kBatch];
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            const int x = key + (i0 + i) * kTileKeys;
            t[i] = (x < p.k && x < done) ? trow[x] : 0.f;
          }
#pragma unroll
          for (int i = 0; i < kBatch; ++i) {
            const int x = key + (i0 + i) * kTileKeys;
            if (x < p.k) trow[x] = t[i] * inv;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int NC>
cudaError_t launch_t(const KlParams& p, const CUtensorMap& tq, const CUtensorMap& tkv, int grid_clusters,
                     cudaStream_t stream) {
  const size_t smem = indexer_kl_smem_bytes(NC * 64);
  auto kern = indexer_kl_kernel<NC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid_clusters * 2), dim3(kThreads), smem, stream, tq, tkv, p);
}

}  // namespace

size_t indexer_kl_smem_bytes(int d_qk) {
  const int nc = d_qk / 64;
  size_t b = sizeof(KlShared) + 1024;              // shared state + alignment slack
  b += (size_t)nc * kPlane;                        // this CTA's Q rows
  b += (size_t)kStages * kPlane;                   // key ring
  b += 2 * (size_t)kMaxIdx * sizeof(int32_t);      // staged positions, two rows
  return b;
}

cudaError_t launch_indexer_kl(const KlParams& p, int d_qk, const CUtensorMap& tq, const CUtensorMap& tkv,
                              int grid_clusters, cudaStream_t stream) {
  if (d_qk == 576) return launch_t<9>(p, tq, tkv, grid_clusters, stream);
  if (d_qk == 192) return launch_t<3>(p, tq, tkv, grid_clusters, stream);
  return cudaErrorInvalidValue;
}

cudaError_t read_kl_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
