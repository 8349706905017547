// Argument blocks and host launchers of the sm_100a kernels (one translation unit per stage).
#pragma once

#include <atomic>
#include <utility>
#include "common.cuh"

namespace dsa {

struct IndexerArgs {
  int B, n_q;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  const float* q_scale;
  const float* head_w;
  const float* k_scale;
  float* scores;
  int64_t L_max;
  const int32_t* tile_prefix;  // [B+1] exclusive prefix of query groups x ceil(len / tile tokens),
                               // or null: the kernel builds it (B <= indexer_prefix_rows())
  unsigned int* err;
};

struct TopkArgs {
  int n_q;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  const float* scores;
  int64_t L_max;
  int top_k;
  int32_t* logical;   // may be null
  int32_t* physical;  // may be null
  unsigned int* err;
  // long-row gather (chunks > 1): per-query candidate count, largest key - threshold,
  // threshold, and candidate buffers [Bq, cand_cap]; counts and maxima start at zero
  int chunks;
  int pair;   // > 1: each row over a cluster of that many CTAs (chunks == 1 only)
  int cand_cap;
  uint32_t* g_cnt;
  uint32_t* g_rmax;
  uint32_t* g_thr;
  uint32_t* g_key;
  int32_t* g_idx;
};

// The step before the path (append.cu): each query's new token at position q_pos[q] (or
// seq_lens[b] - 1). Inputs are bf16 bit patterns; kvf is one of kKvBf16 / kKvFp8 /
// kKvFp8Packed (declared below).
struct AppendArgs {
  int n_q;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  const int32_t* block_table;
  int max_pages;
  int num_pages;
  const uint16_t* idx_q;    // [Bq, 64, 128]
  const uint16_t* idx_k;    // [Bq, 128]
  const uint16_t* latent;   // [Bq, 576]
  uint16_t* q_mla;          // [Bq, 64, 576] (rope columns rotated in place) or null
  double theta[32];         // rope_base^(-2i/64), formed on the host in fp64
  uint8_t* q_out;           // [Bq, 64, 128] e4m3
  float* q_scale_out;       // [Bq, 64]
  uint8_t* k_cache;         // [num_pages * 64, 128] e4m3
  float* k_scale;           // [num_pages * 64]
  void* kv_cache;
  int kvf;
  float* kv_scale;          // [num_pages * 64, 5] (kKvFp8 only)
  unsigned int* err;
};

// Per-(query, split, head) partial statistics: m, l, then one normaliser per value group.
constexpr int kPartStats = 6;

struct MlaArgs {
  const void* q;        // [Bq, 64, 576] bf16 queries
  int Bq;
  int top_k;
  int nsplit;
  int keys_per_split;   // multiple of mla_tile_keys()
  const uint8_t* kv;    // [num_slots, 576] fp8 codes or bf16 values
  const float* kv_scale;
  int64_t num_slots;
  const int32_t* physical;
  float scale_log2;     // softmax_scale * log2(e)
  void* out;
  int out_fp32;
  float* lse;
  float* part_ml;       // [Bq, nsplit, 64, kPartStats]: running max (log2 units), sum of p, and
                        // the normaliser of each 128-column value group (see mla_combine_kernel)
  float* part_o;        // [Bq, nsplit, 64, 512]
  unsigned int* err;
  long long wait_limit; // bound of every wait, in SM cycles (kWaitLimitCycles unless a test shortens it)
  int stall;            // test hook: the softmax warps wait on a barrier nothing arrives on
  int pair;             // nsplit == 2 launched as clusters of two: the splits merge in the kernel
};

// Raises kernel K's dynamic shared-memory limit once per device (a host-side cost that
// would otherwise be paid on every launch). One flag word per kernel.
template <auto K>
inline cudaError_t set_smem_once(int bytes) {
  static std::atomic<uint64_t> done{0};   // one bit per device ordinal < 64
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_release);
  return e;
}

// Launches `kernel` on `stream` with programmatic stream serialisation, so that it may
// start while the previous kernel in the stream is still running (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
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

// launch_pdl for a grid of thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t stream, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Each returns the launch error (cudaSuccess when queued) and adds the number of
// kernels it queued to *launches.
// Tokens per indexer tile for this cache type and query count (the plan's tile unit).
int indexer_tile_tokens(bool fp8, int n_q);
// Rows up to which the indexer builds its work-item prefix itself (no plan kernel).
int indexer_prefix_rows();
cudaError_t launch_plan(const int32_t* seq_lens, const int32_t* q_pos, int B, int n_q, int max_pages, int tile_tok,
                        int32_t* tile_prefix, unsigned int* err, cudaStream_t stream, int* launches);
cudaError_t launch_indexer(bool fp8, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q, const IndexerArgs& a,
                           int grid, cudaStream_t stream, int* launches);
// Chunks per row of the long-row top-k (1 = one CTA per query) and its candidate capacity.
int topk_chunks(int Bq, int64_t L_max, int sms);
// CTAs per row's cluster (2, 4 or 8) when each row's gather is split over a cluster (all
// clusters in one wave), else 0.
int topk_pairs(int Bq, int64_t L_max, int sms);
int topk_candidate_capacity();
cudaError_t launch_topk(const TopkArgs& a, int Bq, cudaStream_t stream, int* launches);
cudaError_t launch_pagemap(int n_q, int top_k, int64_t total, const int32_t* block_table, int max_pages,
                           int num_pages, const int32_t* logical, int32_t* physical, unsigned int* err,
                           cudaStream_t stream, int* launches);
// Latent cache layouts of the MLA decode: bf16 rows; E4M3 rows with a [rows, 5] fp32 scale
// plane; packed 656-byte rows (512 E4M3 codes, four fp32 scales, 64 bf16 rope values).
constexpr int kKvBf16 = 0, kKvFp8 = 1, kKvFp8Packed = 2;
constexpr int kPackedRowBytes = kDimV + 4 * 4 + 2 * (kDimK - kDimV);
cudaError_t launch_mla(int kvf, const CUtensorMap& tmap_q, const MlaArgs& a, cudaStream_t stream, int* launches);
cudaError_t launch_rope_quantize_append(const AppendArgs& a, int Bq, cudaStream_t stream, int* launches);
int mla_tile_keys();  // index-list entries per MLA tile (splits are whole tiles)

// Token-sharded decode (shard.cu).
struct ShardCandArgs {
  int Bq, n_q, top_k;
  const float* scores;           // [Bq, L_max] this rank's indexer scores
  int64_t L_max;
  const int32_t* logical;        // [Bq, top_k] this rank's local selection (-1 unused)
  const int32_t* token_offset;   // [B] global token of each row's local token 0
  float* cand_score;             // [Bq, top_k] out: score, -inf where unused
  int32_t* cand_token;           // [Bq, top_k] out: global token, -1 where unused
  unsigned int* err;
};
struct ShardSelectArgs {
  int Bq, n_q, top_k, n_ranks, rank;
  const float* all_score;        // [n_ranks, Bq, top_k] every rank's candidates
  const int32_t* all_token;
  const int32_t* token_offset;   // [B] this rank's offsets
  const int32_t* seq_lens;       // [B] this rank's local lengths
  const int32_t* block_table;    // [B, max_pages] this rank's block table
  int max_pages, num_pages;
  int32_t* physical;             // [Bq, top_k] out: this rank's winners' slots, then -1
  int32_t* logical;              // [Bq, top_k] out (or null): the global selection
  unsigned int* err;
  int in_smem;                   // the candidates of a row are staged in shared memory
};
struct ShardMergeArgs {
  int Bq, n_ranks;
  const float* all_out;          // [n_ranks, Bq, 64, 512] every rank's normalised output
  const float* all_lse;          // [n_ranks, Bq, 64]
  void* out;                     // [Bq, 64, 512] bf16 or fp32
  int out_fp32;
  float* lse;                    // [Bq, 64] or null
};
constexpr int kShardSelectSmemCap = 227 * 1024;
// Dynamic shared memory of the select kernel with a row's n_cand candidates staged, or 0
// when they do not fit (the kernel then reads them from global memory on every pass).
int shard_select_smem_bytes(int n_cand);
cudaError_t launch_shard_candidates(const ShardCandArgs& a, cudaStream_t stream, int* launches);
cudaError_t launch_shard_select(const ShardSelectArgs& a, cudaStream_t stream, int* launches);
cudaError_t launch_shard_merge(const ShardMergeArgs& a, cudaStream_t stream, int* launches);

}  // namespace dsa
