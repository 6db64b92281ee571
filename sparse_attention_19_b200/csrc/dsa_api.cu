// dsa_api.cu -- the C ABI of libdsa.so (declared in include/dsa.h): argument
// checks, TMA descriptor set-up, workspace layout and kernel dispatch for the
// DeepSeek Sparse Attention forward pass.  Every step of the computation runs in
// the kernels of indexer.cu, topk.cu, sparse_attn.cu and indexer_loss.cu; this
// file only checks, describes and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "dsa.h"
#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kMaxK = 2048;
constexpr int kAttnTile = 128;
constexpr long long kTopkCacheMax = 8192;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem_bytes`-byte elements, box [box_rows, box_cols].
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, int elem_bytes, const void* base, uint64_t rows,
               uint64_t cols, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

dsa_status check_indexer(const dsa_indexer_args* a) {
  if (!a || !a->q_I || !a->w || !a->k_I) return DSA_ERR_INVALID_ARG;
  if (a->B <= 0 || a->Lq <= 0 || a->Lk <= 0 || a->q_offset < 0) return DSA_ERR_INVALID_ARG;
  if ((long long)a->q_offset + a->Lq > a->Lk) return DSA_ERR_INVALID_ARG;
  if (!aligned16(a->q_I) || !aligned16(a->k_I) || !aligned16(a->w)) return DSA_ERR_INVALID_ARG;
  if (a->q_scale && !aligned16(a->q_scale)) return DSA_ERR_INVALID_ARG;
  if (a->k_scale && !aligned16(a->k_scale)) return DSA_ERR_INVALID_ARG;
  const bool shape_ok = (a->H_I == 64 && a->d_I == 128) || (a->H_I == 4 && a->d_I == 64);
  if (!shape_ok) return DSA_ERR_UNSUPPORTED;
  if ((long long)a->B * a->Lk >= (1LL << 31) || (long long)a->B * a->Lq * a->H_I >= (1LL << 31))
    return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status check_attn(const dsa_attn_args* a, int B, int Lq, int Lk) {
  if (!a || !a->q || !a->kv) return DSA_ERR_INVALID_ARG;
  if (B <= 0 || Lq <= 0 || Lk <= 0) return DSA_ERR_INVALID_ARG;
  if (!aligned16(a->q) || !aligned16(a->kv)) return DSA_ERR_INVALID_ARG;
  if (!(a->scale > 0.f) || !std::isfinite(a->scale)) return DSA_ERR_INVALID_ARG;
  const bool shape_ok = (a->H == 128 && a->d_qk == 576 && a->d_v == 512) ||
                        (a->H == 16 && a->d_qk == 192 && a->d_v == 128);
  if (!shape_ok) return DSA_ERR_UNSUPPORTED;
  if ((long long)B * Lk >= (1LL << 31) || (long long)B * Lq * 128 >= (1LL << 31)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// Split-k factor for the attention: each row's key tiles are spread over s units
// (s a power of two).  Cost model in units of one tile's pipelined time on a CTA
// pair (measured ~2.5 us): a unit costs its tiles plus about 1.8 tiles of fill,
// drain and partial-result traffic; units run in waves over the pairs; merging
// split partials adds about one tile.  Few rows (decode) get split, many do not.
int attn_splits(int rows, int n_tiles) {
  constexpr double kUnitOverheadTiles = 1.8, kCombineTiles = 1.0;
  const long long pairs = sm_count() / 2;
  int best_s = 1;
  double best = 1e300;
  for (int s = 1; s <= n_tiles; s *= 2) {
    const long long units = (long long)rows * s;
    const long long waves = (units + pairs - 1) / pairs;
    const int tiles = (n_tiles + s - 1) / s;
    const double cost = (double)waves * (tiles + kUnitOverheadTiles) + (s > 1 ? kCombineTiles : 0.0);
    if (cost < best) { best = cost; best_s = s; }
  }
  return best_s;
}

size_t attn_ws_bytes(int B, int Lq, int k, int H, int d_v) {
  const int n_tiles = (k + kAttnTile - 1) / kAttnTile;
  const int rows = B * Lq;
  const int splits = attn_splits(rows, n_tiles);
  if (splits <= 1) return 0;
  const size_t per = (size_t)rows * splits * H;
  return per * (size_t)d_v * 4 + per * 4 + 256;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch shape of the indexer for these sizes: query block, sub-blocks, key-tile
// chunks per block and, in the fused top-k mode, the candidate lists and the
// staging ring.  The same plan sizes the workspace and drives the launch.
IndexerParams plan_indexer(const dsa_indexer_args* a, bool fused, int k) {
  IndexerParams p{};
  p.B = a->B; p.Lq = a->Lq; p.Lk = a->Lk; p.q_offset = a->q_offset;
  p.H_I = a->H_I; p.d_I = a->d_I;
  if (a->H_I == 64) {
    p.qb = a->Lq >= 4 ? 4 : a->Lq;
  } else if (fused) {
    p.qb = 16;                                   // N = 64: one 64-column accumulator per sub-block
  } else {
    const int r4 = (a->Lq + 3) / 4 * 4;
    p.qb = r4 < 64 ? r4 : 64;
  }
  // The fused mode keeps each unit's rows' candidate lists in shared memory, so its
  // units hold one sub-block (four rows in prefill).
  p.nsub = (a->Lq > p.qb && !fused) ? 2 : 1;
  p.queries_per_unit = p.qb * p.nsub;
  p.n_qblocks = (a->Lq + p.queries_per_unit - 1) / p.queries_per_unit;
  const int sms = sm_count();
  const long long base_units = (long long)p.n_qblocks * a->B;
  const int max_tiles = (a->q_offset + a->Lq - 1) / 128 + 1;
  // Few query blocks (decode): split each sequence's key tiles over kchunks units
  // (at least ~8 tiles each).
  int kch = 1;
  if (base_units < 4LL * sms) {
    int cap = (max_tiles + 7) / 8;
    if (fused || p.n_qblocks > 1) {
      // Cost in key tiles per CTA: waves of units over the SMs, each unit its tiles
      // plus ~two of start-up (the causal query blocks of a long prefill chunk, and
      // the fused mode, whose last unit of a row also selects over every chunk's
      // list of up to k candidates, so its chunks are capped at 16).
      constexpr double kUnitOverheadTiles = 2.0;
      if (fused && cap > 16) cap = 16;
      double best = 1e300;
      for (int c = 1; c <= cap; ++c) {
        const long long waves = (base_units * c + sms - 1) / sms;
        const double cost = (double)waves * ((double)(max_tiles + c - 1) / c + kUnitOverheadTiles);
        if (cost < best) { best = cost; kch = c; }
      }
    } else {
      // One query block per sequence (decode).  Key tiles of the busiest CTA:
      // waves of units over the SMs times the tiles of a unit.  Many splits come
      // within a few percent of the fewest; among those, units nearest 32 tiles
      // (4096 keys) measured fastest on B200 (decode, 64 x 131072 keys: 9 units a
      // sequence 194 us, 16: 196, 23: 187, 32: 183, 37: 182, 48: 184, 64: 183,
      // 74: 186).
      constexpr int kPreferTiles = 32;
      auto cost = [&](int c) {
        return ((base_units * c + sms - 1) / sms) * (long long)((max_tiles + c - 1) / c);
      };
      long long best = cost(1);
      for (int c = 2; c <= cap; ++c) best = cost(c) < best ? cost(c) : best;
      int best_gap = 1 << 30;
      for (int c = 1; c <= cap; ++c) {
        if (cost(c) * 50 > best * 51) continue;           // more than 2 % above the fewest
        const int tiles = (max_tiles + c - 1) / c;
        const int gap = tiles > kPreferTiles ? tiles - kPreferTiles : kPreferTiles - tiles;
        if (gap <= best_gap) { best_gap = gap; kch = c; }   // ties: the finer split
      }
    }
  }
  p.kchunks = kch;
  p.n_units = (int)(base_units * kch);
  p.scale_ring = (a->k_scale && a->Lk % 4 == 0 && p.nsub * p.qb * a->H_I <= 128) ? 1 : 0;
  if (fused) {
    const int k32 = (k + 31) / 32 * 32;
    p.k = k;
    // List capacity: k plus room for several tiles' candidates (at least one tile,
    // 128, must fit after every cut to k); more room means fewer cuts.
    const int room = k32 < 256 ? 256 : (k32 > 512 ? 512 : k32);
    p.cap = k32 + room;
    p.rows_per_unit = p.queries_per_unit;
    const int slot_bytes = p.qb * 128 * 8;
    int ns = 16384 / slot_bytes;
    ns = ns < 2 ? 2 : (ns > indexer_fused_max_stage() ? indexer_fused_max_stage() : ns);
    // The epilogue's quad groups take accumulators (and so staging slots) in turn:
    // four groups when an accumulator is one 64-column group, else two.  A slot must
    // always belong to the same group, since an mbarrier's parity only tells its
    // current phase from the one before: a group that could run two uses of a slot
    // ahead of the selector would pass its wait early.  So the slot count is a
    // multiple of the group count.
    const int ngroups = p.qb * a->H_I <= 64 ? 4 : 2;
    ns = ns < ngroups ? ngroups : ns / ngroups * ngroups;
    p.n_stage = ns;
  }
  return p;
}

int indexer_grid(const IndexerParams& p) {
  const int sms = sm_count();
  return p.n_units < sms ? p.n_units : sms;
}

// Workspace of the fused indexer + top-k: the candidate lists (per CTA, or per
// unit when rows are split over several units), then the per-(unit, row) list
// summaries and the per-row chunk counters of split rows.
struct FusedWs {
  size_t key_off, pos_off, meta_off, done_off, bytes;
};
FusedWs fused_ws_layout(const IndexerParams& p) {
  FusedWs w{};
  // Lists live in shared memory; only rows split over units leave one per unit here.
  const size_t slots = p.kchunks == 1 ? 0 : (size_t)p.n_units;
  const size_t list = slots * p.rows_per_unit * (size_t)p.cap * 4;
  w.key_off = 0;
  w.pos_off = round_up(list, 256);
  w.meta_off = w.pos_off + round_up(list, 256);
  const size_t meta = p.kchunks > 1 ? (size_t)p.n_units * p.rows_per_unit * 16 : 0;
  w.done_off = w.meta_off + round_up(meta, 256);
  const size_t done = p.kchunks > 1 ? (size_t)p.B * p.Lq * 4 : 0;
  w.bytes = w.done_off + round_up(done, 256);
  if (w.bytes == 0) w.bytes = 256;             // a non-empty workspace keeps the argument checks uniform
  return w;
}

// The staged forward's score matrix (fp32 [B, Lq, Lk]; only s <= t is written and read).
size_t scores_ws_bytes(const dsa_indexer_args* a) {
  return round_up((size_t)a->B * a->Lq * a->Lk * sizeof(float), 256);
}

size_t indexer_topk_ws_bytes(const dsa_indexer_args* a, int k) {
  const IndexerParams p = plan_indexer(a, true, k);
  if (p.queries_per_unit * a->H_I > 512 || p.rows_per_unit > indexer_fused_max_rows()) return 0;
  return fused_ws_layout(p).bytes;
}

bool make_indexer_maps(const dsa_indexer_args* a, const IndexerParams& p, CUtensorMap* tq, CUtensorMap* tk,
                       CUtensorMap* ts) {
  const CUtensorMapSwizzle swz = (a->d_I == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_tmap(tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a->q_I, (uint64_t)a->B * a->Lq * a->H_I, a->d_I,
                 a->d_I, (uint32_t)(p.qb * a->H_I), swz))
    return false;
  if (!make_tmap(tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a->k_I, (uint64_t)a->B * a->Lk, a->d_I, a->d_I, 128,
                 swz))                                     // one 128-key tile per box
    return false;
  *ts = *tk;                                               // unused unless scale_ring
  if (p.scale_ring && !make_tmap(ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a->k_scale, (uint64_t)a->B, a->Lk,
                                 128, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return false;
  return true;
}

dsa_status run_indexer(const dsa_indexer_args* a, float* scores, bool fill_upper, cudaStream_t st) {
  IndexerParams p = plan_indexer(a, false, 0);
  if (p.queries_per_unit * a->H_I > 512) return DSA_ERR_UNSUPPORTED;   // epilogue staging limit
  p.fill_upper = fill_upper ? 1 : 0;
  p.q_scale = a->q_scale;
  p.w = reinterpret_cast<const __nv_bfloat16*>(a->w);
  p.k_scale = a->k_scale;
  p.scores = scores;
  CUtensorMap tq, tk, ts;
  if (!make_indexer_maps(a, p, &tq, &tk, &ts)) return DSA_ERR_CUDA;
  return launch_indexer(p, tq, tk, ts, indexer_grid(p), st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// The indexer with top-k selection fused into it: per row the k positions with the
// largest scores (ties to the smaller position), ascending, -1 padded, and their
// scores; no score matrix is written.
dsa_status run_indexer_topk(const dsa_indexer_args* a, int k, int32_t* indices, float* sel_scores, void* ws,
                            size_t ws_bytes, cudaStream_t st) {
  IndexerParams p = plan_indexer(a, true, k);
  if (p.queries_per_unit * a->H_I > 512 || p.rows_per_unit > indexer_fused_max_rows()) return DSA_ERR_UNSUPPORTED;
  const FusedWs w = fused_ws_layout(p);
  if (!ws || ws_bytes < w.bytes || !aligned16(ws)) return DSA_ERR_WORKSPACE;
  char* base = static_cast<char*>(ws);
  p.q_scale = a->q_scale;
  p.w = reinterpret_cast<const __nv_bfloat16*>(a->w);
  p.k_scale = a->k_scale;
  p.scores = nullptr;
  p.indices = indices;
  p.sel_scores = sel_scores;
  p.xkey = reinterpret_cast<uint32_t*>(base + w.key_off);
  p.xpos = reinterpret_cast<uint32_t*>(base + w.pos_off);
  p.xmeta = reinterpret_cast<uint4*>(base + w.meta_off);
  p.done = reinterpret_cast<uint32_t*>(base + w.done_off);
  if (p.kchunks > 1 && cudaMemsetAsync(p.done, 0, (size_t)p.B * p.Lq * 4, st) != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap tq, tk, ts;
  if (!make_indexer_maps(a, p, &tq, &tk, &ts)) return DSA_ERR_CUDA;
  return launch_indexer(p, tq, tk, ts, indexer_grid(p), st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status run_topk(const float* scores, int B, int Lq, int Lk, int q_offset, int k, int32_t* idx,
                    float* sel_scores, cudaStream_t st) {
  TopkParams p{};
  p.scores = scores; p.B = B; p.Lq = Lq; p.Lk = Lk; p.q_offset = q_offset; p.k = k; p.indices = idx;
  p.sel_scores = sel_scores;
  const long long nmax = (long long)q_offset + Lq < Lk ? (long long)q_offset + Lq : Lk;   // longest row
  // Rows up to kTopkCacheMax scores stay in shared memory between passes; longer
  // ones are re-read from L2 (measured faster at 32K: the small CTA lets more rows
  // share an SM, and their second pass still hits L2).
  p.cache_cap = nmax <= kTopkCacheMax ? (int)round_up((size_t)nmax, 4) : 0;
  p.bit_words = (int)round_up((size_t)(nmax + 31) / 32, 4);
  p.cand_cap = 4096;
  // Too few rows to fill the GPU (decode) and long ones: a cluster of CTAs per row,
  // each CTA owning a 32-aligned segment of it.
  const long long rows = (long long)B * Lq;
  if (rows * kTopkClusterCtas <= 2LL * sm_count() && nmax > 16384) {
    const long long seg = ((nmax + kTopkClusterCtas - 1) / kTopkClusterCtas + 31) / 32 * 32;
    p.cluster = 1;
    p.cache_cap = 0;
    p.bit_words = (int)round_up((size_t)(seg / 32), 4);
    p.sampled = 1;            // one pass with a sampled threshold first (see the cluster kernel)
  }
  p.vec4 = (aligned16(scores) && Lk % 4 == 0) ? 1 : 0;
  // Many rows of moderate length (prefill up to 32K): one warp per row, rows
  // streamed from L2 / HBM with no block-wide steps; enough of them to give every
  // SM several CTAs of rows.
  p.warp_rows = (!p.cluster && rows >= 16LL * sm_count() && nmax <= 32768) ? 1 : 0;
  // Longer rows (a 128K prefill's chunks) are read once: a sampled threshold keeps
  // the few thousand keys that can be in the top-k (the candidate buffer grows to
  // 8192 entries for them), with the two-pass selection as the fallback.
  if (!p.cluster && !p.warp_rows && p.cache_cap == 0) {
    p.sampled = 1;
    p.cand_cap = 8192;
  }
  return launch_topk(p, st) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Sparse attention over `idx`; or, when `dense_idx_out` is given (short sequence:
// q_offset + Lq <= k), dense causal attention over keys 0..t read as contiguous
// tiles, with the index lists 0..t written to dense_idx_out by the same kernel.
dsa_status run_attn(const dsa_attn_args* a, int B, int Lq, int Lk, int q_offset, bool compact,
                    const int32_t* idx, int k, void* out, float* lse, void* ws, size_t ws_bytes,
                    cudaStream_t st, int32_t* dense_idx_out = nullptr) {
  AttnParams p{};
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.H = a->H; p.k = k;
  p.dense = dense_idx_out ? 1 : 0;
  p.idx_out = dense_idx_out;
  if (p.dense) compact = true;
  p.n_tiles = (k + kAttnTile - 1) / kAttnTile;
  const int rows = B * Lq;
  p.splits = attn_splits(rows, p.n_tiles);
  p.tiles_per_split = (p.n_tiles + p.splits - 1) / p.splits;
  p.n_units = rows * p.splits;
  p.compact = compact ? 1 : 0;
  p.q_offset = q_offset;
  p.scale_log2 = a->scale * 1.4426950408889634f;
  p.indices = idx;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  if (p.splits > 1) {
    const size_t need = attn_ws_bytes(B, Lq, k, a->H, a->d_v);
    if (!ws || ws_bytes < need || !aligned16(ws)) return DSA_ERR_WORKSPACE;
    const size_t per = (size_t)rows * p.splits * a->H;
    p.part_o = reinterpret_cast<float*>(ws);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(ws) + round_up(per * a->d_v * 4, 256));
  }
  CUtensorMap tq, tkv;
  if (!make_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->q, (uint64_t)rows * a->H, a->d_qk, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (!make_tmap(&tkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->kv, (uint64_t)B * Lk, a->d_qk, 64, 1,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  CUtensorMap tkv_tile = tkv;                               // 64 contiguous rows per box (dense mode)
  if (p.dense && !make_tmap(&tkv_tile, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->kv, (uint64_t)B * Lk, a->d_qk, 64,
                            64, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  const int pairs = sm_count() / 2;
  const int grid = p.n_units < pairs ? p.n_units : pairs;
  if (launch_sparse_attn(p, a->d_qk, a->d_v, tq, tkv, tkv_tile, grid, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (p.splits > 1 && launch_attn_combine(p, a->d_v, st) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status run_indexer_kl(const dsa_attn_args* a, int B, int Lq, int Lk, const int32_t* indices, int k,
                          const float* lse, const float* scores, const float* sel_scores, float* target, float* kl,
                          cudaStream_t st) {
  KlParams p{};
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.H = a->H; p.k = k;
  p.n_rows = B * Lq;
  p.n_tiles = (k + 127) / 128;
  p.scale_log2 = a->scale * 1.4426950408889634f;
  p.indices = indices;
  p.lse = lse;
  p.scores = scores;
  p.sel_scores = sel_scores;
  p.target = target;
  p.kl = kl;
  CUtensorMap tq, tkv;
  if (!make_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->q, (uint64_t)p.n_rows * a->H, a->d_qk, 64, 64,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (!make_tmap(&tkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a->kv, (uint64_t)B * Lk, a->d_qk, 64, 1,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  const int pairs = sm_count() / 2;
  const int grid = p.n_rows < pairs ? p.n_rows : pairs;
  if (launch_indexer_kl(p, a->d_qk, tq, tkv, grid, st) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

__global__ void wait_selftest_kernel(uint32_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t a = smem_u32(&bar);
    bool done = false;
    for (uint32_t i = 0; i < limit && !done; ++i) done = mbar_test_wait(a, 0);
    if (!done) atomicExch(&g_device_error, DEV_ERR_TIMEOUT);
    mbar_arrive(&bar);          // complete the phase so the barrier is left idle
  }
}

}  // namespace

cudaError_t read_device_error(uint32_t* value, bool clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  // Every unit's word holds DEV_ERR_NONE or the one code a failed wait records.
  uint32_t words[5] = {0, 0, 0, 0, 0};
  if ((e = read_unit_error(&words[0], clear)) != cudaSuccess) return e;
  if ((e = read_indexer_error(&words[1], clear)) != cudaSuccess) return e;
  if ((e = read_topk_error(&words[2], clear)) != cudaSuccess) return e;
  if ((e = read_attn_error(&words[3], clear)) != cudaSuccess) return e;
  if ((e = read_kl_error(&words[4], clear)) != cudaSuccess) return e;
  *value = words[0] | words[1] | words[2] | words[3] | words[4];
  return cudaSuccess;
}

cudaError_t launch_wait_selftest(uint32_t spin_limit, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(spin_limit);
  return cudaGetLastError();
}

}  // namespace dsa

using namespace dsa;

extern "C" {

dsa_status dsa_indexer_scores(const dsa_indexer_args* args, float* scores, void* stream) {
  dsa_status s = check_indexer(args);
  if (s != DSA_OK) return s;
  if (!scores || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  return run_indexer(args, scores, true, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk(const float* scores, int B, int Lq, int Lk, int q_offset, int k, int32_t* indices,
                    void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!scores || !indices || B <= 0 || Lq <= 0 || Lk <= 0 || q_offset < 0) return DSA_ERR_INVALID_ARG;
  if ((long long)q_offset + Lq > Lk) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(indices)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  if ((long long)B * Lq >= (1LL << 31)) return DSA_ERR_UNSUPPORTED;
  return run_topk(scores, B, Lq, Lk, q_offset, k, indices, nullptr, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_attn(const dsa_attn_args* args, int B, int Lq, int Lk, const int32_t* indices, int k,
                           void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status s = check_attn(args, B, Lq, Lk);
  if (s != DSA_OK) return s;
  if (!indices || !out || !aligned16(indices) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (lse && !aligned16(lse)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  return run_attn(args, B, Lq, Lk, 0, false, indices, k, out, lse, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

dsa_status dsa_indexer_kl_loss(const dsa_attn_args* args, int B, int Lq, int Lk, const int32_t* indices, int k,
                               const float* lse, const float* scores, float* target, float* kl, void* stream) {
  dsa_status s = check_attn(args, B, Lq, Lk);
  if (s != DSA_OK) return s;
  if (!indices || !lse || !scores || !kl) return DSA_ERR_INVALID_ARG;
  if (!aligned16(indices) || !aligned16(lse) || !aligned16(scores) || !aligned16(kl)) return DSA_ERR_INVALID_ARG;
  if (target && !aligned16(target)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  return run_indexer_kl(args, B, Lq, Lk, indices, k, lse, scores, nullptr, target, kl,
                        static_cast<cudaStream_t>(stream));
}

dsa_status dsa_indexer_kl_loss_selected(const dsa_attn_args* args, int B, int Lq, int Lk, const int32_t* indices,
                                        int k, const float* lse, const float* sel_scores, float* target, float* kl,
                                        void* stream) {
  dsa_status s = check_attn(args, B, Lq, Lk);
  if (s != DSA_OK) return s;
  if (!indices || !lse || !sel_scores || !kl) return DSA_ERR_INVALID_ARG;
  if (!aligned16(indices) || !aligned16(lse) || !aligned16(sel_scores) || !aligned16(kl)) return DSA_ERR_INVALID_ARG;
  if (target && !aligned16(target)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  return run_indexer_kl(args, B, Lq, Lk, indices, k, lse, nullptr, sel_scores, target, kl,
                        static_cast<cudaStream_t>(stream));
}

size_t dsa_workspace_size_args(dsa_op op, const dsa_indexer_args* iargs, int k, int H, int d_v) {
  if (!iargs || check_indexer(iargs) != DSA_OK || k < 1 || k > kMaxK) return 0;
  switch (op) {
    case DSA_OP_TOPK:
      return 0;
    case DSA_OP_SPARSE_ATTN:
      return H > 0 && d_v > 0 ? attn_ws_bytes(iargs->B, iargs->Lq, k, H, d_v) : 0;
    case DSA_OP_INDEXER_TOPK:
      return indexer_topk_ws_bytes(iargs, k);
    case DSA_OP_FORWARD:
      if (H <= 0 || d_v <= 0) return 0;
      return scores_ws_bytes(iargs) + attn_ws_bytes(iargs->B, iargs->Lq, k, H, d_v);
    case DSA_OP_FORWARD_LOWMEM: {
      if (H <= 0 || d_v <= 0) return 0;
      const size_t sel = indexer_topk_ws_bytes(iargs, k);
      return sel ? round_up(sel, 256) + attn_ws_bytes(iargs->B, iargs->Lq, k, H, d_v) : 0;
    }
  }
  return 0;
}

size_t dsa_workspace_size(dsa_op op, int B, int Lq, int Lk, int k, int H, int d_v) {
  if (B <= 0 || Lq <= 0 || Lk <= 0 || Lq > Lk || k < 1 || k > kMaxK || H <= 0 || d_v <= 0) return 0;
  switch (op) {
    case DSA_OP_TOPK:
      return 0;
    case DSA_OP_SPARSE_ATTN:
      return attn_ws_bytes(B, Lq, k, H, d_v);
    case DSA_OP_INDEXER_TOPK:
    case DSA_OP_FORWARD:
    case DSA_OP_FORWARD_LOWMEM: {
      // The documented convention: H_I = 64, d_I = 128, q_offset = Lk - Lq.
      alignas(16) static const uint8_t dummy[16] = {};
      dsa_indexer_args a{B, Lq, Lk, Lk - Lq, 64, 128, dummy, nullptr, dummy, dummy, nullptr};
      return dsa_workspace_size_args(op, &a, k, H, d_v);
    }
  }
  return 0;
}

dsa_status dsa_indexer_topk(const dsa_indexer_args* args, int k, int32_t* indices, float* sel_scores,
                            void* workspace, size_t workspace_bytes, void* stream) {
  dsa_status s = check_indexer(args);
  if (s != DSA_OK) return s;
  if (!indices || !aligned16(indices)) return DSA_ERR_INVALID_ARG;
  if (sel_scores && !aligned16(sel_scores)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  return run_indexer_topk(args, k, indices, sel_scores, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(stream));
}

dsa_status dsa_forward_timed(const dsa_indexer_args* iargs, const dsa_attn_args* aargs, int k, int32_t* indices,
                             float* sel_scores, void* out, float* lse, void* workspace, size_t workspace_bytes,
                             void* stream, void* const* stage_events) {
  dsa_status s = check_indexer(iargs);
  if (s != DSA_OK) return s;
  s = check_attn(aargs, iargs->B, iargs->Lq, iargs->Lk);
  if (s != DSA_OK) return s;
  if (!indices || !out || !aligned16(indices) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (lse && !aligned16(lse)) return DSA_ERR_INVALID_ARG;
  if (sel_scores && !aligned16(sel_scores)) return DSA_ERR_INVALID_ARG;
  if (k < 1 || k > kMaxK) return DSA_ERR_UNSUPPORTED;
  const size_t attn_need = attn_ws_bytes(iargs->B, iargs->Lq, k, aargs->H, aargs->d_v);
  if (!workspace || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  // Staged selection when the workspace holds the score matrix (the faster path),
  // else the fused indexer + top-k with its candidate lists.
  const size_t staged_bytes = scores_ws_bytes(iargs);
  const size_t fused_sel = indexer_topk_ws_bytes(iargs, k);
  const size_t fused_bytes = fused_sel ? round_up(fused_sel, 256) : 0;
  bool staged;
  if (workspace_bytes >= staged_bytes + attn_need) staged = true;
  else if (fused_bytes && workspace_bytes >= fused_bytes + attn_need) staged = false;
  else return DSA_ERR_WORKSPACE;
  const size_t sel_bytes = staged ? staged_bytes : fused_bytes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> bool {
    return !stage_events || cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), st) == cudaSuccess;
  };
  char* attn_ws = static_cast<char*>(workspace) + sel_bytes;
  const size_t attn_ws_size = workspace_bytes - sel_bytes;
  if (!mark(0)) return DSA_ERR_CUDA;
  // Short sequences: when every row's causal range fits in k (q_offset + Lq <= k),
  // every position is selected whatever the scores, and the pass is dense causal
  // attention.  Unless the selected scores are asked for, the indexer is skipped
  // and the attention kernel writes the index lists 0..t.
  const bool dense = (long long)iargs->q_offset + iargs->Lq <= k && !sel_scores;
  if (!dense && staged) {
    // Scores of s <= t only (the top-k reads no others), then the selection.
    float* scores = static_cast<float*>(workspace);
    s = run_indexer(iargs, scores, false, st);
    if (s != DSA_OK) return s;
    if (!mark(1)) return DSA_ERR_CUDA;
    s = run_topk(scores, iargs->B, iargs->Lq, iargs->Lk, iargs->q_offset, k, indices, sel_scores, st);
    if (s != DSA_OK) return s;
    if (!mark(2)) return DSA_ERR_CUDA;
  } else {
    if (!dense) {
      // Indexer with the top-k fused into it: no score matrix is written.
      s = run_indexer_topk(iargs, k, indices, sel_scores, workspace, sel_bytes, st);
      if (s != DSA_OK) return s;
    }
    if (!mark(1) || !mark(2)) return DSA_ERR_CUDA;
  }
  // Dense mode: the attention kernel reads keys 0..t as contiguous tiles and writes
  // the index lists itself (no top-k launch, no gathers).
  s = run_attn(aargs, iargs->B, iargs->Lq, iargs->Lk, iargs->q_offset, true, indices, k, out, lse, attn_ws,
               attn_ws_size, st, dense ? indices : nullptr);
  if (s != DSA_OK) return s;
  if (!mark(3)) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status dsa_forward(const dsa_indexer_args* iargs, const dsa_attn_args* aargs, int k, int32_t* indices,
                       void* out, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  return dsa_forward_timed(iargs, aargs, k, indices, nullptr, out, lse, workspace, workspace_bytes, stream,
                           nullptr);
}

const char* dsa_status_string(dsa_status status) {
  switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: invalid argument";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED: shape outside the supported set";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace too small";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA: CUDA call or kernel launch failed";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT: a device-side wait gave up";
  }
  return "DSA_ERR_UNKNOWN";
}

dsa_status dsa_device_status(int clear) {
  uint32_t v = 0;
  if (read_device_error(&v, clear != 0) != cudaSuccess) return DSA_ERR_CUDA;
  return v == DEV_ERR_NONE ? DSA_OK : DSA_ERR_TIMEOUT;
}

dsa_status dsa_selftest_wait_timeout(uint32_t spin_limit, void* stream) {
  uint32_t v = 0;
  if (read_device_error(&v, true) != cudaSuccess) return DSA_ERR_CUDA;
  if (launch_wait_selftest(spin_limit, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSA_ERR_CUDA;
  if (read_device_error(&v, true) != cudaSuccess) return DSA_ERR_CUDA;
  return v == DEV_ERR_TIMEOUT ? DSA_ERR_TIMEOUT : DSA_OK;
}

int dsa_version(void) { return 100; }

}  // extern "C"
