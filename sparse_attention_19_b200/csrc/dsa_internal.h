// dsa_internal.h -- parameter blocks and launchers shared by the kernels and the
// C-ABI layer of libdsa.so.  Not part of the public interface (include/dsa.h is).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

namespace dsa {

// Launches a kernel with programmatic stream serialization: it may be scheduled
// while the previous kernel in the stream finishes, and waits for it inside
// (griddep_wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- indexer
struct IndexerParams {
  int B, Lq, Lk, q_offset;
  int H_I, d_I;
  int qb;                 // queries per MMA (N = qb * H_I <= 256)
  int nsub;               // query sub-blocks resident per unit
  int queries_per_unit;   // qb * nsub
  int n_qblocks;          // ceil(Lq / queries_per_unit)
  int kchunks;            // key-tile ranges per query block (>1 splits long rows across CTAs)
  int n_units;            // n_qblocks * B * kchunks
  int fill_upper;         // write -inf for s > t (full-matrix output)
  int scale_ring;         // key scales staged per tile by TMA (k_scale set, Lk % 4 == 0)
  const float* q_scale;   // [B, Lq] or null
  const __nv_bfloat16* w; // [B, Lq, H_I]
  const float* k_scale;   // [B, Lk] or null
  float* scores;          // [B, Lq, Lk] (scores mode)
  // ---- fused top-k mode (scores == nullptr): every row's k largest scores are
  // selected on chip; no score reaches global memory except the selected ones.
  int k;                  // positions selected per row
  int cap;                // candidate-list capacity per row (multiple of 32, >= k + 128)
  int n_stage;            // staging slots (one per accumulator use) in shared memory
  int rows_per_unit;      // queries_per_unit
  int32_t* indices;       // [B, Lq, k]
  float* sel_scores;      // [B, Lq, k] or null
  uint32_t* xkey;         // kchunks > 1: each unit's top-k per row, keys:  [unit][rows_per_unit][cap]
  uint32_t* xpos;         // kchunks > 1: the same, positions
  uint4* xmeta;           // kchunks > 1: per (unit, row) {count, min key, max key, 0}
  uint32_t* done;         // kchunks > 1: per row, chunks finished (zeroed before the launch)
};
// Shared-memory bytes of the indexer kernel for a query block of q_rows (query,
// head) rows, `stages` key stages and, in the fused mode, the staging and
// selection areas.
size_t indexer_smem_bytes(int q_rows, int d_I, int w_floats, int sq_floats, int stages, bool scale_ring,
                          bool fused, int qb, int n_stage, int rows_per_unit, int cap);
cudaError_t launch_indexer(const IndexerParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& ts, int grid, cudaStream_t stream);
int indexer_fused_max_rows();    // rows per unit the fused mode supports
int indexer_fused_max_stage();   // staging slots the fused mode supports

// ---------------------------------------------------------------- top-k
struct TopkParams {
  const float* scores;    // [B, Lq, Lk]
  int B, Lq, Lk, q_offset, k;
  int32_t* indices;       // [B, Lq, k]
  float* sel_scores;      // [B, Lq, k] or null: score of each selected position (-0.0 as +0.0), -inf padding
  int cache_cap;          // row elements cached in shared memory (0 = re-read from global); multiple of 4
  int bit_words;          // 32-bit words of each position bitmap (>= ceil(row length / 32)); multiple of 4
  int cand_cap;           // candidate (key, position) pairs held in shared memory
  int vec4;               // rows start 16-byte aligned (scores aligned, Lk % 4 == 0): 16-byte loads
  int cluster;            // each row spread over a cluster of kTopkClusterCtas CTAs (few long rows);
                          // bit_words then covers one CTA's segment
  int warp_rows;          // one warp per row (many rows): no block-wide steps, rows streamed from L2
  int sampled;            // long rows: try the single-pass selection above a sampled threshold first
};
constexpr int kTopkClusterCtas = 4;
size_t topk_smem_bytes(int cache_cap, int bit_words, int cand_cap, bool cluster);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- sparse attention
struct AttnParams {
  int B, Lq, Lk, H, k;
  int n_tiles;            // ceil(k / 128)
  int splits;             // key-tile ranges per query (split-k); 1 = direct output
  int tiles_per_split;
  int n_units;            // B * Lq * splits
  int compact;            // indices are valid-first (top-k output): skip all-padding tiles
  int dense;              // short sequence (q_offset + Lq <= k): row t attends to keys 0..t, read as
                          // contiguous tiles; the kernel writes those positions to idx_out
  int q_offset;           // only used when compact or dense
  int32_t* idx_out;       // dense: [B, Lq, k] receives 0..t then -1
  float scale_log2;       // softmax scale * log2(e)
  const int32_t* indices; // [B, Lq, k]
  __nv_bfloat16* out;     // [B, Lq, H, d_v] (splits == 1)
  float* lse;             // [B, Lq, H] or null (splits == 1)
  float* part_o;          // [B*Lq, splits, H, d_v] fp32 (splits > 1)
  float* part_lse;        // [B*Lq, splits, H] fp32 (splits > 1)
};
size_t attn_smem_bytes(int d_qk, int d_v);
cudaError_t launch_sparse_attn(const AttnParams& p, int d_qk, int d_v, const CUtensorMap& tq,
                               const CUtensorMap& tkv, const CUtensorMap& tkv_tile, int grid_clusters,
                               cudaStream_t stream);
cudaError_t launch_attn_combine(const AttnParams& p, int d_v, cudaStream_t stream);

// ---------------------------------------------------------------- indexer training loss
struct KlParams {
  int B, Lq, Lk, H, k;
  int n_rows;             // B * Lq
  int n_tiles;            // ceil(k / 128)
  float scale_log2;       // softmax scale * log2(e)
  const int32_t* indices; // [B, Lq, k]
  const float* lse;       // [B, Lq, H], natural log
  const float* scores;    // [B, Lq, Lk], or null when sel_scores is given
  const float* sel_scores;  // [B, Lq, k]: the score of each index slot (or null)
  float* target;          // [B, Lq, k] or null
  float* kl;              // [B, Lq]
};
size_t indexer_kl_smem_bytes(int d_qk);
cudaError_t launch_indexer_kl(const KlParams& p, int d_qk, const CUtensorMap& tq, const CUtensorMap& tkv,
                              int grid_clusters, cudaStream_t stream);

// ---------------------------------------------------------------- misc
// Error words of the kernel units (one per translation unit), and their union.
cudaError_t read_indexer_error(uint32_t* value, bool clear);
cudaError_t read_topk_error(uint32_t* value, bool clear);
cudaError_t read_attn_error(uint32_t* value, bool clear);
cudaError_t read_kl_error(uint32_t* value, bool clear);
cudaError_t read_device_error(uint32_t* value, bool clear);
cudaError_t launch_wait_selftest(uint32_t spin_limit, cudaStream_t stream);

}  // namespace dsa
