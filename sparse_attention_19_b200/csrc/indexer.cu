// indexer.cu -- the lightning indexer on sm_100a tensor cores.
//
// Computes I[t,s] = q_scale[t] * k_scale[s] * sum_{j<H_I} w[t,j] * ReLU(q8[t,j] . k8[s])
// (DeepSeek-V3.2 technical-report summary, "Молниеносный индексатор", equation for
// I_{t,s}; FP8 per its third bullet).  The per-token scales are positive, so they
// factor out of the ReLU and are applied after the head sum.
//
// Mapping.  One tcgen05.mma (kind::f8f6f4, fp32 accumulate in TMEM) multiplies a
// tile of 128 keys (M, the A operand, K-major: one key row of d_I e4m3 bytes) by
// QB queries x H_I heads (N = QB*H_I <= 256, the B operand).  With keys on the M
// axis, TMEM lane = key and the H_I columns of one query sit in that lane, so the
// ReLU, the weighting and the head sum are a per-thread loop in the epilogue with
// no cross-thread reduction.  Each CTA keeps NSUB query sub-blocks resident in
// shared memory and streams key tiles through a TMA ring; 512 / N TMEM
// accumulators (up to 8) let the epilogue of one sub-block overlap the MMAs of the
// next ones.  Prefill with H_I = 64 uses QB = 4 (N = 256, two accumulators, two
// sub-blocks; fewer, larger steps measured faster than QB = 2 with four); decode
// uses QB = 1 (N = 64) with a deeper key ring, the key scales staged through a TMA
// ring, and the two epilogue warp halves taking alternate accumulators.
//
// Two modes.  Scores mode writes I[t,s] to a [B, Lq, Lk] array.  Fused mode (the
// forward pass) selects every row's top-k on chip instead ("Отбор и основное
// внимание": only the k positions with the largest I[t,s] go on to attention), so
// no score matrix reaches global memory:
//   * the epilogue compares each score with its row's current threshold and
//     ballot-compacts the survivors of each (tile, query) into a shared-memory
//     staging ring;
//   * three selector warps append the staged candidates to a per-row list kept
//     in global memory (L2-resident, in position order) and, when a list fills,
//     cut it to the row's exact top-k by histogram refinement (warp_select.cuh),
//     which raises the row's threshold: later scores must beat the k-th best so
//     far (a tie loses, since every later position is larger);
//   * at the end of a row the list is cut to its final top-k and written out in
//     ascending position order, with the selected scores.  A row split over
//     several units (decode) is finished by whichever unit ends last, over the
//     units' lists.
// Warp roles (768 threads): warps 0..15 epilogue (warp w reads TMEM lanes
// 32(w%4) .. 32(w%4)+31 of the 64-column groups w/4, w/4 + 4, ...), warp 16 TMEM
// owner + MMA issuer, warps 17..19 selectors (fused mode), warps 20..23 TMA
// loaders.  Four epilogue warps per SM sub-partition hide the latency of the
// per-element ReLU / weighting / head sum.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "dsa_internal.h"
#include "ptx.cuh"
#include "warp_select.cuh"

namespace dsa {

namespace {

constexpr int kKeysPerTile = 128;
constexpr int kMaxStages = 12;
constexpr int kEpiWarps = 16;        // four per TMEM lane quarter ("quads" of four warps)
constexpr int kQuads = kEpiWarps / 4;
constexpr int kMmaWarp = kEpiWarps;  // warp 16: MMA issuer
constexpr int kSelWarp0 = kMmaWarp + 1;   // warps 17-19: selectors (fused mode)
constexpr int kSelWarps = 3;
constexpr int kLoaders = 4;          // TMA requests from one warp are served in order, so each
                                     // key tile is loaded as four 32-row boxes from four warps
constexpr int kLoaderWarp0 = kMmaWarp + 4;
constexpr int kThreads = 32 * (kLoaderWarp0 + kLoaders);   // 768
// Register split: 80 per thread at launch (6 warps per SM sub-partition); the four
// epilogue warpgroups take 88, the MMA / selector warpgroup keeps the 80 it
// launched with, and the loader warpgroup (TMA issue only) gives up to 48.
constexpr uint32_t kRegsLaunch = 80, kRegsEpi = 88, kRegsLoader = 48;
static_assert(32 * kEpiWarps * kRegsEpi + 128 * kRegsLaunch + 128 * kRegsLoader <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
static_assert(kThreads == 32 * kEpiWarps + 256, "one MMA/selector warpgroup and one loader warpgroup");

constexpr int kTmemCols = 512;
constexpr int kScaleSlots = 16;      // key-scale ring: 128 fp32 per tile, released by the epilogue
constexpr int kMaxStage = 32;        // staging slots (fused mode)
constexpr int kMaxRows = 32;         // rows (queries) per unit in fused mode

// Fused mode: shared-memory areas after the weights, as byte offsets from `base`.
struct FusedLayout {
  uint32_t stg_key, stg_pos, stg_cnt;      // [n_stage][qb][128], same, [n_stage][qb][4]
  uint32_t theta;                          // [kMaxRows] u64: (unit ordinal << 32) | threshold key
  uint32_t row_n, row_thr, row_min, row_max;   // [kMaxRows] each, selector-owned
  uint32_t hist, cand;                     // [kSelWarps][kSelBins], [kSelWarps][kSelCandCap + 4]
  uint32_t lkey, lpos;                     // candidate lists: [rows][cap] keys, [rows][cap] positions
  uint32_t end;
};
__host__ __device__ constexpr uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline FusedLayout fused_layout(uint32_t base, int qb, int n_stage, int rows, int cap) {
  FusedLayout L{};
  const uint32_t entries = (uint32_t)n_stage * qb * 128u;
  L.stg_key = align_up(base, 16);
  L.stg_pos = L.stg_key + entries * 4;
  L.stg_cnt = L.stg_pos + entries * 4;
  L.theta = align_up(L.stg_cnt + (uint32_t)n_stage * qb * 16u, 16);
  L.row_n = L.theta + kMaxRows * 8;
  L.row_thr = L.row_n + kMaxRows * 4;
  L.row_min = L.row_thr + kMaxRows * 4;
  L.row_max = L.row_min + kMaxRows * 4;
  L.hist = align_up(L.row_max + kMaxRows * 4, 16);
  L.cand = L.hist + kSelWarps * kSelBins * 4;
  L.lkey = align_up(L.cand + kSelWarps * (kSelCandCap + 4) * 4, 16);
  L.lpos = L.lkey + (uint32_t)rows * cap * 4;
  L.end = L.lpos + (uint32_t)rows * cap * 4;
  return L;
}

struct IndexerSmem {
  // Barriers and small per-unit data first; big tiles follow at a 1024-byte boundary.
  uint64_t q_full[2], q_empty[2];         // query block buffers (two when the block is small)
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];
  uint64_t acc_full[8], acc_empty[8];     // TMEM accumulators: 512 / N of them (at most 8)
  uint64_t sc_full[kScaleSlots], sc_empty[kScaleSlots];
  uint64_t stg_full[kMaxStage], stg_empty[kMaxStage];   // staging ring (fused mode)
  uint64_t final_bar;
  uint64_t epi_bar;          // rendezvous of the epilogue warps
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Query-block buffers: two (the next unit's block loads while this one runs) when a
// block is small, as in decode; one for the large prefill blocks.
__host__ __device__ constexpr uint32_t query_buffers(uint32_t q_bytes) { return q_bytes < 32768u ? 2u : 1u; }

struct UnitInfo {
  int b, i0, kt0, kt1;  // batch, first query, key-tile range [kt0, kt1)
};

__device__ __forceinline__ UnitInfo decode_unit(const IndexerParams& p, int u) {
  // Longest work first: query blocks are visited from the last one down.
  const int per_block = p.B * p.kchunks;
  const int qblk = p.n_qblocks - 1 - u / per_block;
  const int rem = u % per_block;
  const int b = rem / p.kchunks;
  const int kc = rem % p.kchunks;
  UnitInfo info;
  info.b = b;
  info.i0 = qblk * p.queries_per_unit;
  const int i_last = min(p.Lq, info.i0 + p.queries_per_unit) - 1;
  const int t_last = p.q_offset + i_last;                       // <= Lk - 1
  const int ntiles = t_last / kKeysPerTile + 1;
  const int per_chunk = (ntiles + p.kchunks - 1) / p.kchunks;
  info.kt0 = min(ntiles, kc * per_chunk);
  info.kt1 = min(ntiles, (kc + 1) * per_chunk);
  return info;
}

template <int H_I, int D_I, int kStages, bool kFused, int kQB, int kNSub>
__global__ void __launch_bounds__(kThreads, 1)
indexer_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
               const __grid_constant__ CUtensorMap tmap_s, const IndexerParams p) {
  static_assert(D_I == 64 || D_I == 128, "d_I");
  static_assert(kStages % kLoaders == 0 && kStages <= kMaxStages, "loaders own whole residues of the ring");
  static_assert(kScaleSlots % kLoaders == 0, "a scale slot always belongs to the same loader");
  constexpr uint32_t kRowBytes = D_I;                  // one e4m3 row
  constexpr uint32_t kLayout = (D_I == 128) ? LAYOUT_SW128 : LAYOUT_SW64;
  constexpr uint32_t kAtomBytes = 8 * kRowBytes;       // 8-row swizzle atom
  constexpr int kKSteps = D_I / 32;                    // MMA K = 32 bytes of e4m3
  // Units of one query sub-block: every fused launch, and the deep-ring launch,
  // which serves decode-sized query blocks (the launcher checks nsub == 1).
  constexpr bool kOneSubBlock = kFused || kStages == kMaxStages;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IndexerSmem& S = *reinterpret_cast<IndexerSmem*>(smem_raw);
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* tiles = smem_raw + (((raw_addr + (uint32_t)sizeof(IndexerSmem) + 1023u) & ~1023u) - raw_addr);
  // Query-block shape: compile-time in the builds specialised for the common
  // prefill and decode shapes (kQB, kNSub > 0), else the launch's values.
  const int qb = kQB > 0 ? kQB : p.qb;
  const int nsub = kNSub > 0 ? kNSub : p.nsub;
  const int N = qb * H_I;                              // MMA N (queries x heads)
  const uint32_t nslot = min(8, kTmemCols / N);        // accumulators in flight (more when N is small)
  // Epilogue quads work on accumulators in groups of `span`: the groups take
  // accumulators in turn (group g gets seq = g mod ngroups), and within a group quad
  // q reads the 64-column groups (q mod span) * 64, + span * 64, ...  Two quads per
  // accumulator (prefill, N = 256): two accumulators are read at once, each warp
  // reading two queries, so one group's fixed per-accumulator costs overlap the
  // other group's arithmetic.  One quad per accumulator when N <= 64 (decode).
  const int span = N <= 64 ? 1 : 2;
  const uint32_t ngroups = (uint32_t)(kQuads / span);
  const int warps_per_acc = 4 * span;
  const int QU = p.queries_per_unit;                   // = qb * nsub
  const uint32_t q_bytes = (uint32_t)(nsub * N) * kRowBytes;   // one query block
  const uint32_t n_qbuf = query_buffers(q_bytes);
  uint8_t* q_smem = tiles;                             // n_qbuf x (nsub * N rows)
  uint8_t* k_smem = tiles + n_qbuf * (size_t)q_bytes;
  float* sc_smem = reinterpret_cast<float*>(k_smem + (size_t)kStages * kKeysPerTile * kRowBytes);
  float* w_smem = sc_smem + (p.scale_ring ? kScaleSlots * kKeysPerTile : 0);   // 2 x QU * H_I (double-buffered)
  float* sq_smem = w_smem + 2 * QU * H_I;                  // 2 x QU
  // fused mode: staging ring, per-row thresholds, selector state and candidate lists
  const FusedLayout FL = fused_layout((uint32_t)(reinterpret_cast<uint8_t*>(sq_smem + 2 * QU) - tiles), qb,
                                      p.n_stage, p.rows_per_unit, p.cap);
  uint32_t* stg_key = reinterpret_cast<uint32_t*>(tiles + FL.stg_key);
  uint32_t* stg_pos = reinterpret_cast<uint32_t*>(tiles + FL.stg_pos);
  uint32_t* stg_cnt = reinterpret_cast<uint32_t*>(tiles + FL.stg_cnt);
  volatile unsigned long long* theta = reinterpret_cast<volatile unsigned long long*>(tiles + FL.theta);
  uint32_t* row_n = reinterpret_cast<uint32_t*>(tiles + FL.row_n);
  uint32_t* row_thr = reinterpret_cast<uint32_t*>(tiles + FL.row_thr);
  uint32_t* row_min = reinterpret_cast<uint32_t*>(tiles + FL.row_min);
  uint32_t* row_max = reinterpret_cast<uint32_t*>(tiles + FL.row_max);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  volatile uint32_t* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.k_full[s], 1);
      mbar_init(&S.k_empty[s], 1);
    }
    for (int s = 0; s < 8; ++s) {
      mbar_init(&S.acc_full[s], 1);
      mbar_init(&S.acc_empty[s], warps_per_acc);
    }
    // A tile's key scales are read by the warps of the groups that process one of
    // its sub-blocks' accumulators (consecutive accumulators go to consecutive groups).
    const int sc_readers = warps_per_acc * min(nsub, (int)ngroups);
    for (int s = 0; s < kScaleSlots; ++s) {
      mbar_init(&S.sc_full[s], 1);
      mbar_init(&S.sc_empty[s], sc_readers);
    }
    if (kFused) {
      for (int s = 0; s < p.n_stage; ++s) {
        mbar_init(&S.stg_full[s], warps_per_acc);
        mbar_init(&S.stg_empty[s], min(kSelWarps, p.rows_per_unit));   // selectors that own a row
      }
      // No unit owns a threshold yet (unit ordinals start at 0).
      for (int r = 0; r < kMaxRows; ++r) theta[r] = 0xffffffff00000000ull;
    }
    mbar_init(&S.final_bar, 1);
    mbar_init(&S.epi_bar, kEpiWarps);
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
  griddep_launch_dependents();
  griddep_wait();                                      // the previous kernel's writes are visible

  if (warp >= (uint32_t)kEpiWarps) {
  if (warp >= kLoaderWarp0) {
    regs_decrease<kRegsLoader>();
    // ------------------------------------------------------------ TMA loaders
    // Loader 0 also loads the query block.  Loader pw owns the ring stages
    // congruent to pw (mod kLoaders): it waits only for those, and fills each with
    // one 128-key box and, when staged, the tile's key scales.
    const int pw = (int)warp - kLoaderWarp0;
    if (elect_one()) {
      if (pw == 0) { prefetch_tmap(&tmap_q); prefetch_tmap(&tmap_k); if (p.scale_ring) prefetch_tmap(&tmap_s); }
      uint32_t ucount = 0, kstage = 0, kphase = 0, sc_use = 0;
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++ucount) {
        const UnitInfo U = decode_unit(p, u);
        if (pw == 0) {
          // query block of this unit into buffer ucount % n_qbuf (free once the unit
          // n_qbuf back is done)
          const uint32_t qb_i = ucount % n_qbuf;
          if (!mbar_wait(&S.q_empty[qb_i], ((ucount / n_qbuf) & 1u) ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&S.q_full[qb_i], q_bytes);
          for (int sb = 0; sb < nsub; ++sb) {
            const int row = ((U.b * p.Lq) + U.i0 + sb * qb) * H_I;
            tma_load_2d(q_smem + qb_i * q_bytes + (size_t)sb * N * kRowBytes, &tmap_q, &S.q_full[qb_i], 0, row);
          }
        }
        bool ok = true;
        for (int kt = U.kt0; kt < U.kt1; ++kt) {
          if (kstage % kLoaders == (uint32_t)pw) {
            if (!mbar_wait(&S.k_empty[kstage], kphase ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&S.k_full[kstage], kKeysPerTile * kRowBytes);
            tma_load_2d(k_smem + (size_t)kstage * kKeysPerTile * kRowBytes, &tmap_k, &S.k_full[kstage], 0,
                        U.b * p.Lk + kt * kKeysPerTile);
            if (p.scale_ring) {
              // the tile's 128 key scales (zero-filled past Lk) into the scale ring
              const uint32_t ss = sc_use % kScaleSlots;
              if (!mbar_wait(&S.sc_empty[ss], ((sc_use / kScaleSlots) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
              mbar_arrive_expect_tx(&S.sc_full[ss], kKeysPerTile * 4);
              tma_load_2d(sc_smem + ss * kKeysPerTile, &tmap_s, &S.sc_full[ss], kt * kKeysPerTile, U.b);
            }
          }
          if (p.scale_ring) ++sc_use;
          if (++kstage == kStages) { kstage = 0; kphase ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc = make_idesc(0, 0, 128, (uint32_t)N, 0, 0);  // e4m3 x e4m3 -> f32
      uint32_t ucount = 0, kstage = 0, kphase = 0, slot = 0, use = 0;
      const uint32_t k_base = smem_u32(k_smem);
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++ucount) {
        const UnitInfo U = decode_unit(p, u);
        const uint32_t qb_i = ucount % n_qbuf;
        const uint32_t q_base = smem_u32(q_smem) + qb_i * q_bytes;
        if (!mbar_wait(&S.q_full[qb_i], (ucount / n_qbuf) & 1u, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = U.kt0; kt < U.kt1 && ok; ++kt) {
          if (!mbar_wait(&S.k_full[kstage], kphase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = k_base + kstage * kKeysPerTile * kRowBytes;
          for (int sb = 0; sb < nsub; ++sb) {
            if (!mbar_wait(&S.acc_empty[slot], (use & 1u) ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + slot * (uint32_t)N;
            const uint32_t b_addr = q_base + (uint32_t)(sb * N) * kRowBytes;
#pragma unroll
            for (int ks = 0; ks < kKSteps; ++ks) {
              const uint64_t ad = make_smem_desc(a_addr + ks * 32, 16, kAtomBytes, kLayout);
              const uint64_t bd = make_smem_desc(b_addr + ks * 32, 16, kAtomBytes, kLayout);
              mma_f8_ss(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
            mma_commit(&S.acc_full[slot]);
            if (++slot == nslot) { slot = 0; ++use; }
          }
          mma_commit(&S.k_empty[kstage]);
          if (++kstage == kStages) { kstage = 0; kphase ^= 1; }
        }
        mma_commit(&S.q_empty[qb_i]);
        if (!ok) break;
      }
      // Every MMA issued here completes before the TMEM is released.
      mma_commit(&S.final_bar);
      mbar_wait(&S.final_bar, 0, nullptr);
    }
  } else if (kFused && warp >= (uint32_t)kSelWarp0 && warp < (uint32_t)(kSelWarp0 + kSelWarps)) {
    // ------------------------------------------------------------ selectors
    // Selector `me` owns the unit's rows r with r % kSelWarps == me.  It consumes
    // every staging slot in order (releasing it for the epilogue) and appends its
    // rows' staged candidates to their lists, which live in shared memory.
    const int me = (int)warp - kSelWarp0;
    const int RPU = p.rows_per_unit;
    const bool active = me < RPU;            // a unit with fewer rows than selectors leaves some idle
    const uint32_t k = (uint32_t)p.k;
    const uint32_t lt = (1u << lane) - 1u;
    uint32_t* hist = reinterpret_cast<uint32_t*>(tiles + FL.hist) + me * kSelBins;
    uint32_t* cand = reinterpret_cast<uint32_t*>(tiles + FL.cand) + me * (kSelCandCap + 4);
    uint32_t* lkey = reinterpret_cast<uint32_t*>(tiles + FL.lkey);
    uint32_t* lpos = reinterpret_cast<uint32_t*>(tiles + FL.lpos);
    // Rows split over units leave their per-unit top-k in global memory.
    auto glist_key = [&](int unit, int r) { return p.xkey + ((size_t)unit * RPU + r) * p.cap; };
    auto glist_pos = [&](int unit, int r) { return p.xpos + ((size_t)unit * RPU + r) * p.cap; };
    // Cut a row's shared-memory list to its top-k in place and raise its threshold.
    auto cut = [&](int r, uint32_t ucount) {
      uint32_t* xk = lkey + (size_t)r * p.cap;
      uint32_t* xp = lpos + (size_t)r * p.cap;
      const uint32_t n = row_n[r];
      uint32_t thr, gt;
      auto visit = [&](auto&& f) { visit_list_keys<false>(xk, (int)n, f); };
      warp_find_threshold(hist, cand, visit, k, row_min[r], row_max[r], thr, gt);
      auto seg = [&](int) { return CandSeg{xk, xp, (int)n}; };
      warp_compact<false>(seg, 1, thr, k - gt, 0, [&](uint32_t at, uint32_t key, uint32_t pos) {
        xk[at] = key;
        xp[at] = pos;
      });
      __syncwarp();
      if (lane == 0) {
        row_n[r] = k;
        row_thr[r] = thr;
        row_min[r] = thr;
        theta[r] = ((unsigned long long)ucount << 32) | thr;
      }
      __syncwarp();
    };
    // Final output of one row from the concatenated segments get_seg(0 .. nseg-1)
    // (position order), holding `total` candidates with keys in [lo, hi].
    auto emit_row = [&](auto global, size_t row, auto get_seg, int nseg, uint32_t total, uint32_t lo,
                        uint32_t hi) {
      constexpr bool kG = decltype(global)::value;
      int32_t* oi = p.indices + row * (size_t)p.k;
      float* os = p.sel_scores ? p.sel_scores + row * (size_t)p.k : nullptr;
      auto emit = [&](uint32_t at, uint32_t key, uint32_t pos) {
        oi[at] = (int32_t)pos;
        if (os) os[at] = key_to_score(key);
      };
      uint32_t m;
      if (total > k) {
        uint32_t thr, gt;
        auto visit = [&](auto&& f) {
          for (int g = 0; g < nseg; ++g) {
            const CandSeg sg = get_seg(g);
            visit_list_keys<kG>(sg.key, sg.n, f);
          }
        };
        warp_find_threshold(hist, cand, visit, k, lo, hi, thr, gt);
        m = warp_compact<kG>(get_seg, nseg, thr, k - gt, 0, emit);
      } else {
        m = warp_compact<kG>(get_seg, nseg, 0u, 0u, 0, emit);   // every candidate (all keys > 0)
      }
      for (uint32_t j = m + lane; j < k; j += 32) {
        oi[j] = -1;
        if (os) os[j] = -INFINITY;
      }
    };

    uint32_t seq = 0, ucount = 0;
    for (int u = blockIdx.x; active && u < p.n_units; u += gridDim.x, ++ucount) {
      const UnitInfo U = decode_unit(p, u);
      if (lane == 0)
        for (int r = me; r < RPU; r += kSelWarps) {
          row_n[r] = 0;
          row_thr[r] = 0;
          row_min[r] = 0xffffffffu;
          row_max[r] = 0;
        }
      __syncwarp();
      bool ok = true;
      for (int kt = U.kt0; kt < U.kt1 && ok; ++kt) {
        for (int sb = 0; sb < nsub; ++sb, ++seq) {
          const uint32_t gs = seq % (uint32_t)p.n_stage;
          if (!mbar_wait_warp(&S.stg_full[gs], (seq / (uint32_t)p.n_stage) & 1u, abort_flag)) { ok = false; break; }
          for (int qi = 0; qi < qb; ++qi) {
            const int r = sb * qb + qi;
            if (r % kSelWarps != me || U.i0 + r >= p.Lq) continue;
            const uint32_t* cnt = stg_cnt + (gs * qb + qi) * 4;
            const uint32_t c0 = cnt[0], c1 = cnt[1], c2 = cnt[2], c3 = cnt[3];
            if (row_n[r] + c0 + c1 + c2 + c3 > (uint32_t)p.cap) cut(r, ucount);
            uint32_t* xk = lkey + (size_t)r * p.cap;
            uint32_t* xp = lpos + (size_t)r * p.cap;
            uint32_t n = row_n[r];
            const uint32_t th = row_thr[r];
            const uint32_t* sk = stg_key + (gs * qb + qi) * 128;
            const uint32_t* sp = stg_pos + (gs * qb + qi) * 128;
            uint32_t mn = 0xffffffffu, mx = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t cq = q == 0 ? c0 : q == 1 ? c1 : q == 2 ? c2 : c3;
              uint32_t key = 0, pos = 0;
              if (lane < cq) {
                key = sk[q * 32 + lane];
                pos = sp[q * 32 + lane];
              }
              const bool keep = lane < cq && key > th;
              const uint32_t bal = __ballot_sync(0xffffffffu, keep);
              if (keep) {
                const uint32_t at = n + __popc(bal & lt);
                xk[at] = key;
                xp[at] = pos;
                mn = min(mn, key);
                mx = max(mx, key);
              }
              n += __popc(bal);
            }
            mn = __reduce_min_sync(0xffffffffu, mn);
            mx = __reduce_max_sync(0xffffffffu, mx);
            __syncwarp();
            if (lane == 0) {
              row_n[r] = n;
              row_min[r] = min(row_min[r], mn);
              row_max[r] = max(row_max[r], mx);
            }
            __syncwarp();
          }
          if (lane == 0) mbar_arrive(&S.stg_empty[gs]);
        }
      }
      if (!ok) break;
      // ---- the unit's rows are complete: output them, or hand them to the last chunk
      for (int r = me; r < RPU; r += kSelWarps) {
        if (U.i0 + r >= p.Lq) continue;
        const size_t row = (size_t)U.b * p.Lq + U.i0 + r;
        uint32_t* xk = lkey + (size_t)r * p.cap;
        uint32_t* xp = lpos + (size_t)r * p.cap;
        if (p.kchunks == 1) {
          const uint32_t n = row_n[r];
          auto seg = [&](int) { return CandSeg{xk, xp, (int)n}; };
          emit_row(std::false_type{}, row, seg, 1, n, row_min[r], row_max[r]);
          __syncwarp();
          continue;
        }
        if (row_n[r] > k) cut(r, ucount);
        // this unit's top-k of the row (position order) to global memory
        const uint32_t n = row_n[r];
        uint32_t* gk = glist_key(u, r);
        uint32_t* gp = glist_pos(u, r);
        for (uint32_t i = lane * 4; i < n; i += 128) {
          __stcg(reinterpret_cast<uint4*>(gk + i), *reinterpret_cast<const uint4*>(xk + i));
          __stcg(reinterpret_cast<uint4*>(gp + i), *reinterpret_cast<const uint4*>(xp + i));
        }
        if (lane == 0) __stcg(p.xmeta + (size_t)u * RPU + r, make_uint4(n, row_min[r], row_max[r], 0u));
        __threadfence();
        __syncwarp();
        uint32_t prev = 0;
        if (lane == 0) prev = atomicAdd(p.done + row, 1u);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev != (uint32_t)p.kchunks - 1) continue;
        // Last chunk of this row: select over every chunk's list, in chunk (= position) order.
        __threadfence();
        const int u0 = u - u % p.kchunks;
        auto seg = [&](int c) {
          const uint4 m = __ldcg(p.xmeta + (size_t)(u0 + c) * RPU + r);
          return CandSeg{glist_key(u0 + c, r), glist_pos(u0 + c, r), (int)m.x};
        };
        uint32_t total = 0, lo = 0xffffffffu, hi = 0;
        for (int c = 0; c < p.kchunks; ++c) {
          const uint4 m = __ldcg(p.xmeta + (size_t)(u0 + c) * RPU + r);
          total += m.x;
          if (m.x) { lo = min(lo, m.y); hi = max(hi, m.z); }
        }
        emit_row(std::true_type{}, row, seg, p.kchunks, total, lo, hi);
        __syncwarp();
      }
    }
  }
  } else {
    regs_increase<kRegsEpi>();
    // ------------------------------------------------------------ epilogue
    const uint32_t quarter = warp & 3u;              // TMEM lane quarter this warp may read
    const uint32_t quad = warp >> 2;
    const uint32_t group = quad / (uint32_t)span;    // reads accumulators seq = group mod ngroups
    // this warp's 64-column groups of such an accumulator: g_first, g_first + g_step, ...
    const int g_first = (int)(quad % (uint32_t)span) * 64, g_step = 64 * span;
    const uint32_t row = quarter * 32 + lane;        // key row within the tile
    const int et = threadIdx.x;                      // 0 .. 32 * kEpiWarps - 1
    uint32_t seq = 0, epi_phase = 0, sc_use = 0, ucount = 0, acc_slot = 0, acc_use = 0;
    // A unit's weights and query scales sit in smem buffer (unit ordinal % 2).  The
    // next unit's values are read into registers when a unit starts and stored when
    // it ends, so their memory latency hides under the unit's work.
    constexpr int kWPerThread = 512 / (32 * kEpiWarps);       // QU * H_I <= 512 (host-checked)
    float wr[kWPerThread], sr = 0.f;
    auto fetch = [&](const UnitInfo& V) {
#pragma unroll
      for (int e = 0; e < kWPerThread; ++e) {
        const int x = et + e * 32 * kEpiWarps, qq = x / H_I, i = V.i0 + qq;
        wr[e] = (x < QU * H_I && i < p.Lq)
                    ? __bfloat162float(p.w[((size_t)V.b * p.Lq + i) * H_I + x % H_I]) : 0.f;
      }
      const int i = V.i0 + et;
      sr = (et < QU && i < p.Lq) ? (p.q_scale ? p.q_scale[(size_t)V.b * p.Lq + i] : 1.f) : 0.f;
    };
    auto store = [&](uint32_t buf) {
#pragma unroll
      for (int e = 0; e < kWPerThread; ++e) {
        const int x = et + e * 32 * kEpiWarps;
        if (x < QU * H_I) w_smem[buf * QU * H_I + x] = wr[e];
      }
      if (et < QU) sq_smem[buf * QU + et] = sr;
    };
    if ((int)blockIdx.x < p.n_units) {
      fetch(decode_unit(p, blockIdx.x));
      store(0);
    }
    for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++ucount) {
      const UnitInfo U = decode_unit(p, u);
      // this unit's buffer is complete and the other one is no longer read
      if (!warps_rendezvous(&S.epi_bar, epi_phase, abort_flag)) break;
      const bool has_next = u + (int)gridDim.x < p.n_units;
      if (has_next) fetch(decode_unit(p, u + gridDim.x));
      const float* wbuf = w_smem + (ucount & 1u) * QU * H_I;
      const float* sqbuf = sq_smem + (ucount & 1u) * QU;
      bool ok = true;
      // Key scales: from the TMA-filled ring when staged (scale_ring), else loaded
      // one tile ahead, so their memory latency overlaps the current tile's epilogue.
      auto key_scale = [&](int kt) -> float {
        const int s = kt * kKeysPerTile + (int)row;
        if (kt >= U.kt1 || s >= p.Lk) return 0.f;
        return p.k_scale ? __ldg(p.k_scale + (size_t)U.b * p.Lk + s) : 1.f;
      };
      // With one sub-block per tile (decode, fused mode) a group owns every
      // ngroups-th tile: the warp visits only those, stepping the tile, accumulator
      // and scale-slot counters over the others instead of looping through them
      // (each skipped pass cost as much as a few hundred instructions of issue).
      constexpr bool stride = kOneSubBlock;
      const uint32_t seq_u = seq, sc_u = sc_use;
      const int kt_first = stride ? U.kt0 + (int)((group - seq_u) & (ngroups - 1u)) : U.kt0;
      const int kt_step = stride ? (int)ngroups : 1;
      float sk_next = p.scale_ring ? 0.f : key_scale(kt_first);
      for (int kt = kt_first; kt < U.kt1 && ok; kt += kt_step) {
        if (stride) {
          seq = seq_u + (uint32_t)(kt - U.kt0);
          sc_use = sc_u + (uint32_t)(kt - U.kt0);
          acc_slot = seq % nslot;
          acc_use = seq / nslot;
        }
        const int s = kt * kKeysPerTile + (int)row;
        float sk = 0.f;
        const uint32_t ss = sc_use % kScaleSlots;
        // This warp reads the tile only if its group owns one of the tile's
        // accumulators (seq .. seq + nsub - 1).
        bool reads_tile = false;
        for (int sb = 0; sb < nsub; ++sb) reads_tile |= ((seq + (uint32_t)sb) & (ngroups - 1u)) == group;
        if (p.scale_ring) {
          if (reads_tile) {
            if (!mbar_wait_warp(&S.sc_full[ss], (sc_use / kScaleSlots) & 1u, abort_flag)) { ok = false; break; }
            sk = sc_smem[ss * kKeysPerTile + row];
          }
        } else {
          sk = sk_next;
          sk_next = key_scale(kt + kt_step);
        }
        for (int sb = 0; sb < nsub; ++sb, ++seq) {
          const uint32_t slot = acc_slot, use = acc_use;
          if (++acc_slot == nslot) { acc_slot = 0; ++acc_use; }
          if ((seq & (ngroups - 1u)) != group) continue;
          if (!mbar_wait_warp(&S.acc_full[slot], use & 1u, abort_flag)) { ok = false; break; }
          uint32_t gs = 0;                                   // staging slot (fused mode)
          if constexpr (kFused) {
            gs = seq % (uint32_t)p.n_stage;
            if (!mbar_wait_warp(&S.stg_empty[gs], ((seq / (uint32_t)p.n_stage) & 1u) ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t t_base = tmem_base + ((quarter * 32u) << 16) + slot * (uint32_t)N;
          // One query's score for this lane's key: ReLU, weighting and head sum over its
          // H_I columns (two interleaved partial sums, packed FMA), then the scales and
          // the causal mask.  Scores mode stores it; fused mode stages it (warp-wide
          // call) if it beats the row's current threshold.
          auto finish = [&](int qi, float acc) {
            const int qq = sb * qb + qi;
            const int i = U.i0 + qq;
            if constexpr (kFused) {
              const bool valid = i < p.Lq && s < p.Lk && s <= p.q_offset + i;
              const uint32_t key = score_to_key(acc * sqbuf[qq] * sk);
              const unsigned long long tv = theta[qq];
              const uint32_t th = (uint32_t)(tv >> 32) == ucount ? (uint32_t)tv : 0u;
              const bool pass = valid && key > th;
              const uint32_t bal = __ballot_sync(0xffffffffu, pass);
              const uint32_t base = (gs * (uint32_t)qb + (uint32_t)qi) * 128u + quarter * 32u;
              if (pass) {
                const uint32_t at = base + __popc(bal & ((1u << lane) - 1u));
                stg_key[at] = key;
                stg_pos[at] = (uint32_t)s;
              }
              if (lane == 0) stg_cnt[(gs * (uint32_t)qb + (uint32_t)qi) * 4u + quarter] = __popc(bal);
            } else if (i < p.Lq && s < p.Lk) {
              const int t = p.q_offset + i;
              float* dst = p.scores + ((size_t)U.b * p.Lq + i) * (size_t)p.Lk + s;
              if (s <= t)
                __stcs(dst, acc * sqbuf[qq] * sk);
              else if (p.fill_upper)
                __stcs(dst, -INFINITY);
            }
          };
          // sum_j w_j ReLU(x_j): packed FMAs, two independent chains.
          auto relu_dot = [&](const uint32_t* v, const float4* wq, int n, float2 acc2) -> float2 {
            float2 acc_b = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < n; e += 4) {
              const float4 w4 = wq[e / 4];       // weights as 16-byte loads
              acc2 = ffma2(make_float2(fmaxf(__uint_as_float(v[e]), 0.f), fmaxf(__uint_as_float(v[e + 1]), 0.f)),
                           make_float2(w4.x, w4.y), acc2);
              acc_b = ffma2(make_float2(fmaxf(__uint_as_float(v[e + 2]), 0.f), fmaxf(__uint_as_float(v[e + 3]), 0.f)),
                            make_float2(w4.z, w4.w), acc_b);
            }
            return fadd2(acc2, acc_b);
          };
          // The accumulator is handed back to the MMA issuer as soon as this warp's
          // last TMEM load of it has completed.
          auto release = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acc_empty[slot]);
          };
          if constexpr (H_I == 64) {
            // This warp's 64-column groups (one query each).  Two of them (prefill:
            // each warp holds two queries of the accumulator) are read together, 16
            // columns of each per TMEM load, so the two reductions interleave; the
            // accumulator goes back to the MMA issuer once the last load is in.
            if (g_first + g_step < N) {
              const int qa = g_first / 64, qb2 = (g_first + g_step) / 64;   // queries within the sub-block
              const float4* wa = reinterpret_cast<const float4*>(wbuf + (size_t)(sb * qb + qa) * H_I);
              const float4* wb = reinterpret_cast<const float4*>(wbuf + (size_t)(sb * qb + qb2) * H_I);
              float2 acc_a = make_float2(0.f, 0.f), acc_b = make_float2(0.f, 0.f);
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                uint32_t va[16], vb[16];
                tmem_ld16(t_base + (uint32_t)(g_first + c * 16), va);
                tmem_ld16(t_base + (uint32_t)(g_first + g_step + c * 16), vb);
                tmem_ld_wait();
                tmem_regs_ready(va);
                tmem_regs_ready(vb);
                if (c == 3) release();
                acc_a = relu_dot(va, wa + c * 4, 16, acc_a);
                acc_b = relu_dot(vb, wb + c * 4, 16, acc_b);
              }
              finish(qa, acc_a.x + acc_a.y);
              finish(qb2, acc_b.x + acc_b.y);
            } else
            for (int g0 = g_first; g0 < N; g0 += g_step) {
              const int qi = g0 / 64;                            // query within the sub-block
              const float4* wq = reinterpret_cast<const float4*>(wbuf + (size_t)(sb * qb + qi) * H_I);
              uint32_t v[32];
              tmem_ld32(t_base + (uint32_t)g0, v);
              tmem_ld_wait();
              tmem_regs_ready(v);
              float2 acc2 = relu_dot(v, wq, 32, make_float2(0.f, 0.f));
              tmem_ld32(t_base + (uint32_t)g0 + 32, v);
              tmem_ld_wait();
              tmem_regs_ready(v);
              if (g0 + g_step >= N) release();
              acc2 = relu_dot(v, wq + 8, 32, acc2);
              finish(qi, acc2.x + acc2.y);
            }
            if (g_first >= N) release();
          } else {
            // Small H_I: each 64-column group holds 64 / H_I queries, 32 / H_I per load.
            constexpr int QPL = 32 / H_I;
            for (int g0 = g_first; g0 < N; g0 += g_step) {
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                uint32_t v[32];
                tmem_ld32(t_base + (uint32_t)(g0 + part * 32), v);
                tmem_ld_wait();
                tmem_regs_ready(v);
#pragma unroll
                for (int a = 0; a < QPL; ++a) {
                  const int qi = (g0 + part * 32) / H_I + a;
                  const float4* wq = reinterpret_cast<const float4*>(wbuf + (size_t)(sb * qb + qi) * H_I);
                  const float2 acc2 = relu_dot(v + a * H_I, wq, H_I, make_float2(0.f, 0.f));
                  finish(qi, acc2.x + acc2.y);
                }
              }
            }
            release();
          }
          if (kFused) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.stg_full[gs]);
          }
        }
        if (p.scale_ring) {
          __syncwarp();
          if (reads_tile && lane == 0) mbar_arrive(&S.sc_empty[ss]);
          ++sc_use;
        }
      }
      if (!ok) break;
      if (stride) {
        // counters past the unit's last tile, whichever tile this warp saw last
        const uint32_t nt = (uint32_t)(U.kt1 - U.kt0);
        seq = seq_u + nt;
        if (p.scale_ring) sc_use = sc_u + nt;
        acc_slot = seq % nslot;
        acc_use = seq / nslot;
      }
      // Full-matrix output: positions beyond this unit's causal tiles are -inf.
      if (!kFused && p.fill_upper && p.kchunks == 1) {
        const int nt_all = (p.Lk + kKeysPerTile - 1) / kKeysPerTile;
        for (int kt = U.kt1; kt < nt_all; ++kt) {
          const int s = kt * kKeysPerTile + (int)row;
          if (s >= p.Lk) continue;
          for (int qq = (int)quad; qq < QU; qq += kQuads) {
            const int i = U.i0 + qq;
            if (i < p.Lq)
              __stcs(p.scores + ((size_t)U.b * p.Lq + i) * (size_t)p.Lk + s, -INFINITY);
          }
        }
      }
      if (has_next) store((ucount + 1) & 1u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int H_I, int D_I, int kStages, bool kFused, int kQB = 0, int kNSub = 0>
cudaError_t launch_indexer_t(const IndexerParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& ts, int grid, cudaStream_t stream) {
  if ((kQB > 0 && p.qb != kQB) || (kNSub > 0 && p.nsub != kNSub)) return cudaErrorInvalidValue;
  const size_t smem = indexer_smem_bytes(p.nsub * p.qb * H_I, D_I, p.queries_per_unit * H_I, p.queries_per_unit,
                                         kStages, p.scale_ring != 0, kFused, p.qb, p.n_stage, p.rows_per_unit,
                                         p.cap);
  auto kern = indexer_kernel<H_I, D_I, kStages, kFused, kQB, kNSub>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // The register split must fit in what the CTA launches with, or the increase
  // would wait forever: refuse to launch a build where it does not.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, tq, tk, ts, p);
}

}  // namespace

size_t indexer_smem_bytes(int q_rows, int d_I, int w_floats, int sq_floats, int stages, bool scale_ring,
                          bool fused, int qb, int n_stage, int rows_per_unit, int cap) {
  size_t t = query_buffers((uint32_t)(q_rows * d_I)) * (size_t)q_rows * d_I;   // query block buffers
  t += (size_t)stages * kKeysPerTile * d_I;                    // key ring
  if (scale_ring) t += (size_t)kScaleSlots * kKeysPerTile * sizeof(float);   // key-scale ring
  t += 2 * (size_t)(w_floats + sq_floats) * sizeof(float);     // weights / query scales, double-buffered
  if (fused) t = fused_layout((uint32_t)t, qb, n_stage, rows_per_unit, cap).end;   // staging, selectors, lists
  const size_t b = sizeof(IndexerSmem) + 1024 + t;             // barriers + alignment slack
  // At least ~116 KB so that one CTA (and its 512 TMEM columns) owns each SM.
  return b < 118784 ? 118784 : b;
}

int indexer_fused_max_rows() { return kMaxRows; }
int indexer_fused_max_stage() { return kMaxStage; }

cudaError_t launch_indexer(const IndexerParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& ts, int grid, cudaStream_t stream) {
  // A small resident query block (decode) leaves room for a deeper key ring.
  const bool deep = p.nsub * p.qb * p.H_I <= 128;
  const bool fused = p.scores == nullptr;
  // Accumulators go to the epilogue's quad groups in turn (four groups of one quad
  // when N <= 64, else two of two); each staging slot must stay with one group (see
  // the staging ring), so n_stage is a multiple of the group count.
  const int ngroups = p.qb * p.H_I <= 64 ? kQuads : kQuads / 2;
  if (fused && p.nsub != 1) return cudaErrorInvalidValue;   // fused units hold one sub-block
  if (fused && (p.rows_per_unit > kMaxRows || p.n_stage > kMaxStage || p.n_stage < 1 || p.cap < p.k + 128 ||
                p.cap % 32 != 0 || p.n_stage % ngroups != 0))
    return cudaErrorInvalidValue;
  if (p.H_I == 64 && p.d_I == 128) {
    if (fused) {
      // Specialised for the prefill (4 queries) and decode (one query) blocks.
      if (!deep && p.qb == 4) return launch_indexer_t<64, 128, 4, true, 4, 1>(p, tq, tk, ts, grid, stream);
      if (deep && p.qb == 1) return launch_indexer_t<64, 128, 8, true, 1, 1>(p, tq, tk, ts, grid, stream);
      // Any other block (two queries: the deeper ring and the lists of two rows do
      // not fit together) takes the 4-stage ring.
      return launch_indexer_t<64, 128, 4, true>(p, tq, tk, ts, grid, stream);
    }
    if (deep && p.nsub != 1) return cudaErrorInvalidValue;   // the deep-ring build visits tiles by group
    // Builds specialised for the prefill block (4 queries x 2 sub-blocks) and the
    // decode block (one query).
    if (!deep && p.qb == 4 && p.nsub == 2) return launch_indexer_t<64, 128, 4, false, 4, 2>(p, tq, tk, ts, grid, stream);
    if (deep && p.qb == 1) return launch_indexer_t<64, 128, 12, false, 1, 1>(p, tq, tk, ts, grid, stream);
    // Two queries per block: two 16 KB query buffers leave room for 8 key stages, not 12.
    if (deep && p.qb == 2) return launch_indexer_t<64, 128, 8, false>(p, tq, tk, ts, grid, stream);
    return deep ? launch_indexer_t<64, 128, 12, false>(p, tq, tk, ts, grid, stream)
                : launch_indexer_t<64, 128, 4, false>(p, tq, tk, ts, grid, stream);
  }
  if (p.H_I == 4 && p.d_I == 64)
    return fused ? launch_indexer_t<4, 64, 4, true>(p, tq, tk, ts, grid, stream)
                 : launch_indexer_t<4, 64, 4, false>(p, tq, tk, ts, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t read_indexer_error(uint32_t* value, bool clear) { return read_unit_error(value, clear); }

}  // namespace dsa
