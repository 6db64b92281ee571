// sparse_attn.cu -- sparse MQA / MLA-absorbed attention over the selected latent rows.
//
// For query row r (batch b, position t) and head h, over the selected positions s:
//   z_s = scale * q[r,h,:] . kv[b,s,:]        (all d_qk columns: latent + rope)
//   out[r,h,:] = sum_s softmax(z)_s * kv[b,s,:d_v]
// (DeepSeek-V3.2 technical-report summary, "Отбор и основное внимание", equation
// for u_t: attention only over the top-k latent entries c_s; MLA in MQA mode, one
// KV row serves every query head.)
//
// Mapping onto a pair of SMs (a 2-CTA cluster, tcgen05 .cta_group::2):
//   * Each CTA owns 64 of the 128 query heads; its Q rows (64 x d_qk bf16) stay in
//     shared memory for the whole query.  MMA M = 128 heads across the pair.
//   * Keys come in tiles of 128 selected positions.  S = Q K^T is one pair-MMA
//     chain with N = 128 keys: each CTA gathers 64 of the tile's key rows, in
//     64-column chunks (TMA tile::gather4, 128-byte swizzle), streamed through a
//     ring.  S lands in TMEM as 64 columns per CTA (lanes 0-63: keys 0-63,
//     lanes 64-127: keys 64-127 of the tile, for that CTA's 64 heads).
//   * Four softmax warps per CTA turn S into P (bf16, in shared memory, the A
//     operand of the next MMA) with an online softmax whose reference maximum
//     only moves when a new maximum exceeds it by 2^8 (the accumulator is then
//     rescaled in TMEM); the two lanes that hold one head's two key halves swap
//     their maxima through shared memory.
//   * O += P V is a pair-MMA with N = 256 value columns per instruction; V is
//     the same gathered rows read as an MN-major operand, each CTA holding 128
//     value columns of all 128 keys.  O for 64 heads x 512 columns fits in 256
//     TMEM columns per CTA (the pair layout puts half of N in lanes 64-127), so
//     S double-buffers beside it.
//   * The leader CTA (rank 0) issues every MMA; both CTAs' TMA loads complete on
//     the leader's barriers, and MMA completion is multicast to both CTAs.  The
//     softmax warps of both CTAs signal the leader's barriers directly (after a
//     fence.proxy.async for the P tile they wrote).  P is double-buffered, so the
//     softmax of tile j+1 overlaps the P.V of tile j.
//   * S = Q K^T and O += P V are issued by two threads (warps 4 and 5 of the
//     leader): at these shapes one thread's issue rate, not the tensor core, would
//     bound the MMAs, and P.V(j) then never waits behind the key chunks of S(j+1).
//   * Loads: TMA requests from one warp are served in order, so the gather rate
//     grows with the number of issuing warps.  Key chunks come from 9 warps and
//     value stages from 9 others (each group walks its own ring, so a value slot
//     that is still in use never holds back the next tile's keys); the value
//     loaders also stage each unit's selected positions, one unit ahead.
// Warp roles (768 threads per CTA): warps 0-3 softmax/epilogue (TMEM lane quarter
// = warp), warp 4 TMEM owner + S issuer (leader), warp 5 P.V issuer (leader),
// warps 6-14 key loaders, warps 15-23 value loaders + index staging.  The softmax
// warpgroup holds 120 registers per thread, the others 72 (setmaxnreg).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kTileKeys = 128;       // keys per tile (pair)
constexpr int kHalfKeys = 64;        // keys per CTA in S, and keys per V stage
constexpr int kKStages = 6;          // K-chunk ring depth (8 KB stages)
constexpr int kVStages = 3;          // V ring depth (64 keys x this CTA's value planes)
constexpr int kPBufs = 2;            // P buffers (2 planes each: keys 0-63, 64-127)
constexpr int kMaxIdx = 2048;        // selected positions per unit (staged in shared memory)
constexpr int kMmaWarp = 4;           // TMEM owner + S issuer
constexpr int kPvWarp = 5;            // P.V issuer
// Loaders own ring slots, so a warp waits only on its own slots (in ring order)
// and the stages of different slots are issued in parallel.  Key chunks: a team
// of kKTeamWarps warps owns kKTeamSlots consecutive slots and splits each chunk's
// 16 gathers; value stages: kVWarpsPerSlot warps per slot split its gathers.
constexpr int kKTeamWarps = 3;
constexpr int kKTeamSlots = 2;
constexpr int kVWarpsPerSlot = 3;
constexpr int kKWarp0 = 6;           // key-chunk loaders
constexpr int kKWarps = kKStages / kKTeamSlots * kKTeamWarps;
constexpr int kVWarp0 = kKWarp0 + kKWarps;   // value-stage loaders
constexpr int kVWarps = kVStages * kVWarpsPerSlot;
constexpr int kThreads = 32 * (kVWarp0 + kVWarps);   // 768
constexpr int kStageBatch = 8;       // index words in flight per warp while staging
// Register split: the CTA launches with 80 registers per thread (6 warps per SM
// sub-partition); the softmax warpgroup then takes 120 and the other warpgroups
// (MMA issuers, loaders) keep 72.
constexpr uint32_t kRegsLaunch = 80;
constexpr uint32_t kRegsSoftmax = 120;
constexpr uint32_t kRegsOther = 72;
static_assert(128 * kRegsSoftmax + (kThreads - 128) * kRegsOther <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kPlane64 = 64 * 128;    // 64 rows x 128 B  (Q plane, K stage, V plane, P plane)
constexpr uint32_t kTmemS = 0;             // S buffers: columns [0, 128)
constexpr uint32_t kTmemO = 128;           // O: columns [128, 128 + d_v/2)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxChunks = 9;

struct AttnBarriers {
  uint64_t q_full[kMaxChunks], q_empty[kMaxChunks];
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[kPBufs], p_empty[kPBufs];
  uint64_t o_full, o_empty, final_s, final_pv;
  uint64_t idx_full[2], idx_empty[2];
  uint32_t valid_mask[2][kMaxIdx / 32];   // per 32 staged positions: bit set = valid entry
  uint64_t xbar[2];          // rendezvous of softmax warps w and w ^ 2 (same heads, other key half)
  uint32_t tmem_base;
  uint32_t abort_flag;
  float red_max[2][128];
  float red_sum[128];
};

template <int DV>
struct VShape {
  static constexpr int kNpv = DV >= 256 ? DV / 256 : 1;   // PV instructions per tile
  static constexpr int kN = DV >= 256 ? 256 : DV;         // N of one PV instruction
  static constexpr int kPlanes = kN / 128;                // 64-column planes per CTA per instruction
  static constexpr uint32_t kStageBytes = kPlanes * kPlane64;   // 64 keys x planes
};

// A unit is one query row's key-tile range [j0, j1) (the whole row without split-k).
struct Unit {
  int row, b, t, j0, j1, split;
};

__device__ __forceinline__ Unit decode_unit(const AttnParams& p, int u) {
  Unit U;
  const int n_rows = p.B * p.Lq;
  U.row = n_rows - 1 - u / p.splits;       // longest rows first (top-k output is valid-first)
  U.split = u % p.splits;
  U.b = U.row / p.Lq;
  U.t = p.q_offset + U.row % p.Lq;
  int nt = p.n_tiles;
  if (p.compact) {
    const int nvalid = min(p.k, U.t + 1);
    nt = (nvalid + kTileKeys - 1) / kTileKeys;
  }
  U.j0 = min(nt, U.split * p.tiles_per_split);
  U.j1 = min(nt, (U.split + 1) * p.tiles_per_split);
  return U;
}

// First unit at or after u (stepping by the cluster count) that has key tiles;
// returns p.n_units when there is none.
__device__ __forceinline__ int next_unit(const AttnParams& p, int u, int step, Unit& U) {
  for (; u < p.n_units; u += step) {
    U = decode_unit(p, u);
    if (U.j0 < U.j1) return u;
  }
  return p.n_units;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Rows of kv (in the [B*Lk, d_qk] view) of four consecutive staged positions
// (pos a multiple of 4), one 16-byte shared-memory load; padding and out-of-range
// entries were staged as row b*Lk (a valid row), masked in the softmax.
__device__ __forceinline__ int4 gather_rows4(const int32_t* rows, int pos) {
  return *reinterpret_cast<const int4*>(rows + pos);
}

template <int NC, int DV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_kv,
                   const __grid_constant__ CUtensorMap tmap_kv_tile, const AttnParams p) {
  using VS = VShape<DV>;
  static_assert(NC <= kMaxChunks, "d_qk");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  AttnBarriers& S = *reinterpret_cast<AttnBarriers*>(smem_raw);
  // 1024-byte aligned operand area (the 128-byte swizzle is address based).
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t area_off = ((raw_addr + sizeof(AttnBarriers) + 1023u) & ~1023u) - raw_addr;
  uint8_t* area = smem_raw + area_off;
  uint8_t* q_sm = area;                                             // NC planes
  uint8_t* k_sm = q_sm + NC * kPlane64;                             // kKStages planes
  uint8_t* v_sm = k_sm + kKStages * kPlane64;                       // kVStages x kPlanes planes
  uint8_t* p_sm = v_sm + kVStages * VS::kStageBytes;                // kPBufs x 2 planes
  int32_t* idx_sm = reinterpret_cast<int32_t*>(p_sm + kPBufs * 2 * kPlane64);  // 2 x kMaxIdx

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  volatile uint32_t* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxChunks; ++i) { mbar_init(&S.q_full[i], 1); mbar_init(&S.q_empty[i], 1); }
    for (int i = 0; i < kKStages; ++i) { mbar_init(&S.k_full[i], 1); mbar_init(&S.k_empty[i], 1); }
    for (int i = 0; i < kVStages; ++i) { mbar_init(&S.v_full[i], 1); mbar_init(&S.v_empty[i], 1); }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&S.p_full[i], 8);      // 4 softmax warps x 2 CTAs
      mbar_init(&S.p_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 8);     // 4 softmax warps x 2 CTAs
      mbar_init(&S.idx_full[i], kVWarps);   // the value loaders stage the indices
      mbar_init(&S.idx_empty[i], 4 + kKWarps + kVWarps);   // softmax warps + loader warps
    }
    mbar_init(&S.o_full, 1);
    mbar_init(&S.o_empty, 8);
    mbar_init(&S.final_s, 1);
    mbar_init(&S.final_pv, 1);
    mbar_init(&S.xbar[0], 2);
    mbar_init(&S.xbar[1], 2);
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

  if (warp >= 4) {
    regs_decrease<kRegsOther>();
    if (warp >= kKWarp0 && warp < kVWarp0) {
      // ------------------------------------------------------------------ key loaders
      // Per unit: the Q planes (plane c from warp c % kKWarps), then for each tile
      // its NC key chunks (this CTA's 64 keys x 64 columns).  Chunk kc goes to
      // ring slot kc % kKStages; the team that owns that slot issues its 16
      // four-row gathers, groups g = part, part + kKTeamWarps, ...
      const int pw = (int)warp - kKWarp0;
      const uint32_t my_team = (uint32_t)(pw / kKTeamWarps);
      const int part = pw % kKTeamWarps;
      uint32_t ucount = 0, kc = 0;
      bool ok = true;
      if (pw == 0 && lane == 0) {
        prefetch_tmap(&tmap_q);
        prefetch_tmap(p.dense ? &tmap_kv_tile : &tmap_kv);
      }
      Unit U;
      for (int u = next_unit(p, cluster_id, n_clusters, U); u < p.n_units && ok;
           u = next_unit(p, u + n_clusters, n_clusters, U)) {
        const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
        if (lane == 0) {
          const int qrow = U.row * p.H + (int)rank * 64;
          for (int c = pw; c < NC && ok; c += kKWarps) {
            ok = mbar_wait(&S.q_empty[c], (ucount & 1u) ^ 1u, abort_flag);
            if (!ok) break;
            if (leader) mbar_arrive_expect_tx(&S.q_full[c], 2u * kPlane64);
            tma_load_2d_pair(q_sm + c * kPlane64, &tmap_q, mapa_shared(smem_u32(&S.q_full[c]), 0), c * 64, qrow);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
        if (!ok) break;
        const int32_t* idx = idx_sm + ib * kMaxIdx;
        // The unit's chunks are kc_u .. kc_u + nk - 1; chunk x goes to slot x % kKStages.
        // The team visits only the chunks of its own slots (lo .. lo + kKTeamSlots - 1)
        // rather than stepping through all of them.
        const uint32_t kc_u = kc, nk = (uint32_t)(U.j1 - U.j0) * NC, lo = my_team * kKTeamSlots;
        uint32_t x = kc_u;
        {
          const uint32_t r = x % kKStages;
          if (r < lo) x += lo - r;
          else if (r >= lo + kKTeamSlots) x += kKStages - r + lo;
        }
        for (; x < kc_u + nk && ok; x += (x % kKStages + 1 < lo + kKTeamSlots) ? 1u : kKStages - kKTeamSlots + 1u) {
          const uint32_t st = x % kKStages, ph = (x / kKStages) & 1u;
          const int j = U.j0 + (int)((x - kc_u) / NC), c = (int)((x - kc_u) % NC);
          // Dense mode: one box per chunk from the team's first warp; the others
          // have nothing to load and must not wait either (a waiter that adds
          // nothing to a phase can fall two phases behind, where its parity test
          // would no longer see the phase it waits for).
          if (p.dense && part != 0) continue;
          bool w_ok = true;
          if (lane == 0) {
            w_ok = mbar_wait(&S.k_empty[st], ph ^ 1u, abort_flag);
            if (w_ok && leader && part == 0) mbar_arrive_expect_tx(&S.k_full[st], 2u * kPlane64);
          }
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
          const uint32_t full_l = mapa_shared(smem_u32(&S.k_full[st]), 0);
          if (p.dense) {
            // keys 0..t are contiguous: this CTA's 64 rows of the tile in one box
            if (part == 0 && lane == 0)
              tma_load_2d_pair(k_sm + st * kPlane64, &tmap_kv_tile, full_l, c * 64,
                               U.b * p.Lk + j * kTileKeys + (int)rank * kHalfKeys);
            continue;
          }
          const int g = part + kKTeamWarps * (int)lane;            // 4-key group of this lane
          if (g < kHalfKeys / 4) {
            const int4 r4 = gather_rows4(idx, (j - U.j0) * kTileKeys + (int)rank * kHalfKeys + g * 4);
            tma_gather4_pair(k_sm + st * kPlane64 + g * 512, &tmap_kv, full_l, c * 64, r4.x, r4.y, r4.z, r4.w);
          }
        }
        kc = kc_u + nk;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
        ++ucount;
      }
    } else if (warp >= kVWarp0) {
      // ------------------------------------------------------------------ value loaders
      // Index staging: the value loaders also stage each unit's selected positions
      // [j0*128, j1*128) into buffer (unit ordinal % 2), one unit ahead, as the kv
      // row to gather -- batch offset applied; padding and out-of-range entries
      // gather row b*Lk and are masked -- plus one validity ballot per 32
      // positions for the softmax.  Warp pw stages the
      // 32-position words pw, pw + kVWarps, ...  A buffer is free again once the
      // loaders and the softmax warps are done with the unit two back.
      // Value stages: per tile, 2 x kNpv stages of 64 keys (kh) x this CTA's kN/2
      // columns of value block h, i.e. all 128 keys of the tile across the two halves.
      const int pw = (int)warp - kVWarp0;
      const uint32_t my_slot = (uint32_t)(pw / kVWarpsPerSlot);
      const int part = pw % kVWarpsPerSlot;
      uint32_t ucount = 0, vc = 0;
      bool ok = true;
      auto stage = [&](const Unit& V, uint32_t buf) {
        int32_t* dst = idx_sm + buf * kMaxIdx;
        uint32_t* vmask = S.valid_mask[buf];
        const int x_begin = V.j0 * kTileKeys, nwords = (V.j1 - V.j0) * (kTileKeys / 32);
        if (p.dense) {
          // Row t selects every position 0..t (in slot order); the loads need no
          // staged rows, only the validity words.  The leader also writes the
          // row's index list, and the first split its tail of -1 slots.
          int32_t* io = p.idx_out + (size_t)V.row * p.k;
          for (int w = pw; w < nwords; w += kVWarps) {
            const int x = x_begin + w * 32 + (int)lane;
            const bool valid = x <= V.t && x < p.k;
            const uint32_t bal = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) vmask[w] = bal;
            if (leader && x < p.k) io[x] = valid ? x : -1;
          }
          if (leader && V.split == 0) {
            const int nt_row = (min(p.k, V.t + 1) + kTileKeys - 1) / kTileKeys;
            for (int x = nt_row * kTileKeys + pw * 32 + (int)lane; x < p.k; x += kVWarps * 32) io[x] = -1;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.idx_full[buf]);
          return;
        }
        const int32_t* src = p.indices + (size_t)V.row * p.k;
        for (int w0 = pw; w0 < nwords; w0 += kVWarps * kStageBatch) {
          int sidx[kStageBatch];
#pragma unroll
          for (int e = 0; e < kStageBatch; ++e) {
            const int w = w0 + e * kVWarps, x = x_begin + w * 32 + (int)lane;
            sidx[e] = (w < nwords && x < p.k) ? __ldg(src + x) : -1;
          }
#pragma unroll
          for (int e = 0; e < kStageBatch; ++e) {
            const int w = w0 + e * kVWarps;
            if (w >= nwords) break;                       // warp-uniform
            const bool valid = (sidx[e] >= 0) && (sidx[e] < p.Lk);
            dst[w * 32 + (int)lane] = V.b * p.Lk + (valid ? sidx[e] : 0);   // validity: the ballot below
            const uint32_t bal = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) vmask[w] = bal;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.idx_full[buf]);
      };
      Unit U, Un;
      int u = next_unit(p, cluster_id, n_clusters, U);
      if (u < p.n_units) stage(U, 0);                    // buffer 0 starts free
      while (u < p.n_units && ok) {
        const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
        const int un = next_unit(p, u + n_clusters, n_clusters, Un);
        if (un < p.n_units) {
          const uint32_t nb = (ucount + 1) & 1u, nph = ((ucount + 1) >> 1) & 1u;
          ok = mbar_wait_warp(&S.idx_empty[nb], nph ^ 1u, abort_flag);
          if (!ok) break;
          stage(Un, nb);
        }
        ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
        if (!ok) break;
        const int32_t* idx = idx_sm + ib * kMaxIdx;
        // The unit's value stages are vc_u .. vc_u + nv - 1 (per tile: key half kh,
        // then value block h); stage x goes to slot x % kVStages, and this warp visits
        // only its own slot's stages.
        constexpr uint32_t kPerTile = 2u * VS::kNpv;
        const uint32_t vc_u = vc, nv = (uint32_t)(U.j1 - U.j0) * kPerTile;
        for (uint32_t x = vc_u + (my_slot + kVStages - vc_u % kVStages) % kVStages; x < vc_u + nv && ok;
             x += kVStages) {
          const uint32_t st = my_slot, ph = (x / kVStages) & 1u;
          const uint32_t rem = (x - vc_u) % kPerTile;
          const int j = U.j0 + (int)((x - vc_u) / kPerTile), kh = (int)(rem / VS::kNpv), h = (int)(rem % VS::kNpv);
          if (p.dense && part != 0) continue;         // one issuing warp per slot (see the key loaders)
          bool w_ok = true;
          if (lane == 0) {
            w_ok = mbar_wait(&S.v_empty[st], ph ^ 1u, abort_flag);
            if (w_ok && leader && part == 0) mbar_arrive_expect_tx(&S.v_full[st], 2u * VS::kStageBytes);
          }
          if (!__shfl_sync(0xffffffffu, w_ok, 0)) { ok = false; break; }
          const uint32_t full_l = mapa_shared(smem_u32(&S.v_full[st]), 0);
          if (p.dense) {
            // 64 contiguous keys x this CTA's value columns: one box per plane
            if (part == 0 && lane < (uint32_t)VS::kPlanes) {
              const int col = h * VS::kN + (int)rank * (VS::kN / 2) + (int)lane * 64;
              tma_load_2d_pair(v_sm + st * VS::kStageBytes + lane * kPlane64, &tmap_kv_tile, full_l, col,
                               U.b * p.Lk + j * kTileKeys + kh * kHalfKeys);
            }
            continue;
          }
          const int g = part + kVWarpsPerSlot * (int)lane;
          if (g < 16 * VS::kPlanes) {
            const int pl = g / 16, kg = g % 16;
            const int4 r4 = gather_rows4(idx, (j - U.j0) * kTileKeys + kh * kHalfKeys + kg * 4);
            const int col = h * VS::kN + (int)rank * (VS::kN / 2) + pl * 64;
            tma_gather4_pair(v_sm + st * VS::kStageBytes + pl * kPlane64 + kg * 512, &tmap_kv, full_l, col,
                             r4.x, r4.y, r4.z, r4.w);
          }
        }
        vc = vc_u + nv;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
        ++ucount;
        u = un;
        U = Un;
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ S issuer
      // S = Q K^T for each tile into TMEM buffer (tile ordinal % 2), one key chunk
      // (4 MMAs of K = 16) per ring stage.  S and P.V come from two threads so that
      // the single-thread issue rate bounds neither.
      if (leader && elect_one()) {
        constexpr uint32_t idesc_s = make_idesc(1, 1, 128, kTileKeys, 0, 0);       // bf16, K-major x K-major
        const uint64_t q_desc = make_smem_desc(smem_u32(q_sm), 16, 1024, LAYOUT_SW128);
        const uint64_t k_desc = make_smem_desc(smem_u32(k_sm), 16, 1024, LAYOUT_SW128);
        uint32_t ucount = 0, kc = 0, sc = 0;
        bool ok = true;
        Unit U;
        for (int u = next_unit(p, cluster_id, n_clusters, U); u < p.n_units && ok;
             u = next_unit(p, u + n_clusters, n_clusters, U)) {
          for (int j = U.j0; j < U.j1 && ok; ++j) {
            const uint32_t sb = sc & 1u;
            ok = mbar_wait(&S.s_empty[sb], ((sc >> 1) & 1u) ^ 1u, abort_flag, true);
            if (!ok) break;
            tc_fence_after();
            const uint32_t d = tmem_base + kTmemS + sb * kHalfKeys;
            for (int c = 0; c < NC; ++c) {
              if (j == U.j0 && !mbar_wait(&S.q_full[c], ucount & 1u, abort_flag)) { ok = false; break; }
              const uint32_t st = kc % kKStages, ph = (kc / kKStages) & 1u;
              if (!mbar_wait(&S.k_full[st], ph, abort_flag)) { ok = false; break; }
              tc_fence_after();
              // descriptor start addresses advance 32 B (encoded 2) per K step of 16
              const uint64_t ad = q_desc + (uint64_t)(c * (kPlane64 >> 4));
              const uint64_t bd = k_desc + (uint64_t)(st * (kPlane64 >> 4));
              mma_bf16_ss_pair(d, ad + 0, bd + 0, idesc_s, c ? 1u : 0u);
              mma_bf16_ss_pair(d, ad + 2, bd + 2, idesc_s, 1u);
              mma_bf16_ss_pair(d, ad + 4, bd + 4, idesc_s, 1u);
              mma_bf16_ss_pair(d, ad + 6, bd + 6, idesc_s, 1u);
              mma_commit_pair_mc(&S.k_empty[st], kBoth);
              if (j == U.j1 - 1) mma_commit_pair_mc(&S.q_empty[c], kBoth);   // Q plane free for the next unit
              ++kc;
            }
            if (!ok) break;
            mma_commit_pair_mc(&S.s_full[sb], kBoth);
            ++sc;
          }
          ++ucount;
        }
        // Wait until every MMA this thread issued has completed before teardown.
        mma_commit(&S.final_s);
        mbar_wait(&S.final_s, 0, nullptr);
      }
    } else if (warp == kPvWarp) {
      // ------------------------------------------------------------------ P.V issuer
      // O += P V per tile: for each value stage (64 keys x kN value columns across
      // the pair), 4 MMAs of K = 16 keys reading P buffer (tile ordinal % 2).
      if (leader && elect_one()) {
        constexpr uint32_t idesc_pv = make_idesc(1, 1, 128, VS::kN, 0, 1);         // P K-major, V MN-major
        const uint64_t p_desc = make_smem_desc(smem_u32(p_sm), 16, 1024, LAYOUT_SW128);
        const uint64_t v_desc = make_smem_desc(smem_u32(v_sm), kPlane64, 1024, LAYOUT_SW128);
        uint32_t vc = 0, pc = 0, oc = 0;
        bool ok = true;
        Unit U;
        for (int u = next_unit(p, cluster_id, n_clusters, U); u < p.n_units && ok;
             u = next_unit(p, u + n_clusters, n_clusters, U)) {
          for (int j = U.j0; j < U.j1 && ok; ++j) {
            const bool first = (j == U.j0);
            ok = mbar_wait(&S.p_full[pc & 1u], (pc >> 1) & 1u, abort_flag, true);
            if (ok && first) ok = mbar_wait(&S.o_empty, (oc & 1u) ^ 1u, abort_flag, true);
            if (!ok) break;
            tc_fence_after();
            for (int kh = 0; kh < 2 && ok; ++kh) {
              for (int h = 0; h < VS::kNpv; ++h) {
                const uint32_t st = vc % kVStages, ph = (vc / kVStages) & 1u;
                if (!mbar_wait(&S.v_full[st], ph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + kTmemO + h * (VS::kN / 2);
                // P advances 32 B (encoded 2) and V 16 keys = 2048 B (encoded 128) per K step
                const uint64_t ad = p_desc + (uint64_t)(((pc & 1u) * 2 + kh) * (kPlane64 >> 4));
                const uint64_t bd = v_desc + (uint64_t)(st * (VS::kStageBytes >> 4));
                mma_bf16_ss_pair(d, ad + 0, bd + 0, idesc_pv, (first && kh == 0) ? 0u : 1u);
                mma_bf16_ss_pair(d, ad + 2, bd + 128, idesc_pv, 1u);
                mma_bf16_ss_pair(d, ad + 4, bd + 256, idesc_pv, 1u);
                mma_bf16_ss_pair(d, ad + 6, bd + 384, idesc_pv, 1u);
                mma_commit_pair_mc(&S.v_empty[st], kBoth);
                ++vc;
              }
            }
            if (!ok) break;
            mma_commit_pair_mc(&S.p_empty[pc & 1u], kBoth);
            if (j == U.j1 - 1) { mma_commit_pair_mc(&S.o_full, kBoth); ++oc; }
            ++pc;
          }
        }
        mma_commit(&S.final_pv);
        mbar_wait(&S.final_pv, 0, nullptr);
      }
    }
  } else {
    regs_increase<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax / epilogue
    const uint32_t l = warp * 32 + lane;          // TMEM lane = (key half, head)
    const uint32_t h = l & 63u;                   // head within this CTA
    const uint32_t half = l >> 6;                 // which 64 keys of the tile this lane holds
    const int head = (int)rank * 64 + (int)h;
    const uint32_t lane_addr = (warp * 32u) << 16;
    uint32_t ucount = 0, sc = 0, pc = 0, oc = 0, xph = 0;
    bool ok = true;
    for (int u = cluster_id; u < p.n_units && ok; u += n_clusters) {
      const Unit U = decode_unit(p, u);
      if (U.j0 >= U.j1) {
        // An empty split: no keys.  Partial result is (O = 0, lse = -inf).
        if (p.splits > 1 && half == 0 && head < p.H) {
          const size_t prow = ((size_t)U.row * p.splits + U.split) * p.H + head;
          p.part_lse[prow] = -INFINITY;
          float4* o4 = reinterpret_cast<float4*>(p.part_o + prow * DV);
          for (int x = 0; x < DV / 4; ++x) o4[x] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      const uint32_t ib = ucount & 1u, uph = (ucount >> 1) & 1u;
      ok = mbar_wait_warp(&S.idx_full[ib], uph, abort_flag);
      if (!ok) break;
      float m = -INFINITY, lsum = 0.f;
      for (int j = U.j0; j < U.j1 && ok; ++j) {
        const uint32_t sb = sc & 1u;
        ok = mbar_wait_warp(&S.s_full[sb], (sc >> 1) & 1u, abort_flag);
        if (!ok) break;
        tc_fence_after();
        // This lane's 64 logits, read from TMEM once.  Invalid entries (padding,
        // out-of-range) become -inf; whole groups are valid except in a row's last tile.
        const uint32_t s_addr = tmem_base + lane_addr + kTmemS + sb * kHalfKeys;
        const uint32_t* vm = &S.valid_mask[ib][((j - U.j0) * kTileKeys + (int)half * kHalfKeys) / 32];
        const uint32_t vmask0 = vm[0], vmask1 = vm[1];   // warp-uniform
        uint32_t v[64];
        tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        if ((vmask0 & vmask1) != 0xffffffffu) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!((((c < 32) ? vmask0 : vmask1) >> (c & 31)) & 1u)) v[c] = __float_as_uint(-INFINITY);
        }
        float smax = -INFINITY;                       // maximum of the raw logits (scale > 0)
#pragma unroll
        for (int c = 0; c < 64; ++c) smax = fmaxf(smax, __uint_as_float(v[c]));
        float tmax = smax * p.scale_log2;
        const uint32_t rb = sc & 1u;
        S.red_max[rb][l] = tmax;
        ok = warps_rendezvous(&S.xbar[warp & 1u], xph, abort_flag);
        if (!ok) break;
        tmax = fmaxf(tmax, S.red_max[rb][l ^ 64u]);
        const float m_new = fmaxf(m, tmax);
        const bool first = (j == U.j0);
        const bool need = first || (m_new > m + kRescaleThreshold);
        const float m_ref = need ? m_new : m;
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        // P buffer pc % 2 is free once the P.V two tiles back is done.
        const uint32_t pbuf = pc & 1u;
        ok = mbar_wait_warp(&S.p_empty[pbuf], ((pc >> 1) & 1u) ^ 1u, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (!first && __any_sync(0xffffffffu, need)) {
          // Rescaling O needs the previous tile's P.V to be complete.
          ok = mbar_wait_warp(&S.p_empty[pbuf ^ 1u], ((pc - 1u) >> 1) & 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const float alpha = need ? exp2f(m - m_new) : 1.f;
          for (int c0 = 0; c0 < VS::kNpv * (VS::kN / 2); c0 += 16) {
            uint32_t ov[16];
            tmem_ld16(tmem_base + lane_addr + kTmemO + c0, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st16(tmem_base + lane_addr + kTmemO + c0, ov);
          }
          tmem_st_wait();
          if (need) lsum *= alpha;
        }
        if (need) m = m_new;
        // Probabilities 2^(z*scale*log2e - m), packed to bf16 straight into P (row h of
        // this lane's key-half plane, 128-byte swizzle); the row sum is kept in fp32.
        uint8_t* prow = p_sm + (pbuf * 2 + half) * kPlane64 + (h >> 3) * 1024 + (h & 7) * 128;
        const float2 scl = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm = make_float2(-m_use, -m_use);
        float2 sum2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {                   // 16-byte chunk q: keys 8q .. 8q+7
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c0 = q * 8 + 2 * e;
            const float2 x = ffma2(make_float2(__uint_as_float(v[c0]), __uint_as_float(v[c0 + 1])), scl, nm);
            const float2 pr = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            sum2 = fadd2(sum2, pr);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(pr.x, pr.y);
            w4[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(prow + ((q ^ (h & 7)) * 16)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        const float psum = sum2.x + sum2.y;
        lsum += psum;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.s_empty[sb]), 0));
        ++sc;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.p_full[pbuf]), 0));
        ++pc;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.idx_empty[ib]);
      ++ucount;
      // ---- epilogue of the unit
      ok = mbar_wait_warp(&S.o_full, oc & 1u, abort_flag);
      ++oc;
      if (!ok) break;
      tc_fence_after();
      S.red_sum[l] = lsum;
      ok = warps_rendezvous(&S.xbar[warp & 1u], xph, abort_flag);
      if (!ok) break;
      const float total = lsum + S.red_sum[l ^ 64u];
      ok = warps_rendezvous(&S.xbar[warp & 1u], xph, abort_flag);   // red_sum may be rewritten next unit
      if (!ok) break;
      const float inv = total > 0.f ? 1.f / total : 0.f;
      const float lse_v = total > 0.f ? (m + log2f(total)) * kLn2 : -INFINITY;
      const bool write = head < p.H;
      for (int hi = 0; hi < VS::kNpv; ++hi) {
        for (int c0 = 0; c0 < VS::kN / 2; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem_base + lane_addr + kTmemO + hi * (VS::kN / 2) + c0, ov);
          tmem_ld_wait();
          const int dv0 = hi * VS::kN + (int)half * (VS::kN / 2) + c0;
          if (!write) continue;
          if (p.splits == 1) {
            __nv_bfloat16* dst = p.out + ((size_t)U.row * p.H + head) * DV + dv0;
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(ov[e + 0]) * inv, __uint_as_float(ov[e + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + e) = w;
            }
          } else {
            float* dst = p.part_o + (((size_t)U.row * p.splits + U.split) * p.H + head) * DV + dv0;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) =
                  make_float4(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv,
                              __uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
          }
        }
      }
      if (write && half == 0) {
        if (p.splits == 1) {
          if (p.lse) p.lse[(size_t)U.row * p.H + head] = lse_v;
        } else {
          p.part_lse[((size_t)U.row * p.splits + U.split) * p.H + head] = lse_v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&S.o_empty), 0));
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

// Merge split-k partials: lse = log sum_i exp(lse_i); out = sum_i exp(lse_i - lse) o_i.
template <int DV>
__global__ void __launch_bounds__(128) attn_combine_kernel(const AttnParams p) {
  griddep_launch_dependents();
  griddep_wait();                                      // the partials are complete
  const int warps = blockDim.x / 32;
  const int gw = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int n = p.B * p.Lq * p.H;
  if (gw >= n) return;
  const int row = gw / p.H, head = gw % p.H;
  float mx = -INFINITY;
  for (int sp = 0; sp < p.splits; ++sp)
    mx = fmaxf(mx, p.part_lse[((size_t)row * p.splits + sp) * p.H + head]);
  float wsum = 0.f;
  float acc[DV / 32];
#pragma unroll
  for (int e = 0; e < DV / 32; ++e) acc[e] = 0.f;
  if (mx > -INFINITY) {
    for (int sp = 0; sp < p.splits; ++sp) {
      const size_t prow = ((size_t)row * p.splits + sp) * p.H + head;
      const float wgt = expf(p.part_lse[prow] - mx);
      wsum += wgt;
      const float* src = p.part_o + prow * DV;
#pragma unroll
      for (int e = 0; e < DV / 32; ++e) acc[e] = fmaf(wgt, src[e * 32 + lane], acc[e]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = p.out + ((size_t)row * p.H + head) * DV;
#pragma unroll
  for (int e = 0; e < DV / 32; ++e) dst[e * 32 + lane] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0 && p.lse) p.lse[(size_t)row * p.H + head] = (wsum > 0.f) ? mx + logf(wsum) : -INFINITY;
}

template <int NC, int DV>
cudaError_t launch_t(const AttnParams& p, const CUtensorMap& tq, const CUtensorMap& tkv,
                     const CUtensorMap& tkv_tile, int grid_clusters, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes(NC * 64, DV);
  auto kern = sparse_attn_kernel<NC, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // The register split must fit in what the CTA launches with, or the increase
  // would wait forever: refuse to launch a build where it does not.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(grid_clusters * 2), dim3(kThreads), smem, stream, tq, tkv, tkv_tile, p);
}

}  // namespace

size_t attn_smem_bytes(int d_qk, int d_v) {
  const int nc = d_qk / 64;
  const int n = d_v >= 256 ? 256 : d_v;
  const size_t v_stage = (size_t)(n / 128) * kPlane64;
  size_t b = sizeof(AttnBarriers) + 1024;          // barriers + alignment slack
  b += (size_t)nc * kPlane64;                      // Q
  b += (size_t)kKStages * kPlane64;                // K ring
  b += (size_t)kVStages * v_stage;                 // V ring
  b += (size_t)kPBufs * 2 * kPlane64;              // P buffers (keys 0-63, 64-127 each)
  b += 2 * (size_t)kMaxIdx * sizeof(int32_t);      // staged indices, two units
  return b;
}

cudaError_t launch_sparse_attn(const AttnParams& p, int d_qk, int d_v, const CUtensorMap& tq,
                               const CUtensorMap& tkv, const CUtensorMap& tkv_tile, int grid_clusters,
                               cudaStream_t stream) {
  if (d_qk == 576 && d_v == 512) return launch_t<9, 512>(p, tq, tkv, tkv_tile, grid_clusters, stream);
  if (d_qk == 192 && d_v == 128) return launch_t<3, 128>(p, tq, tkv, tkv_tile, grid_clusters, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_combine(const AttnParams& p, int d_v, cudaStream_t stream) {
  const int n = p.B * p.Lq * p.H;
  const int grid = (n + 3) / 4;
  if (d_v == 512) return launch_pdl(attn_combine_kernel<512>, dim3(grid), dim3(128), 0, stream, p);
  if (d_v == 128) return launch_pdl(attn_combine_kernel<128>, dim3(grid), dim3(128), 0, stream, p);
  return cudaErrorInvalidValue;
}

cudaError_t read_attn_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
