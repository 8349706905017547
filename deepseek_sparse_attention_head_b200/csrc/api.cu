// C ABI of the DSA decode library (declared in include/dsa.h): argument checks,
// workspace layout, TMA tensor maps and kernel launches. No allocation, no host
// synchronisation except in dsa_get_error.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "kernels.cuh"

using namespace dsa;

namespace {

thread_local int g_launches = 0;
// test hooks of dsa_test_set_wait_hooks (this host thread's later MLA launches)
thread_local long long g_test_wait_limit = 0;
thread_local int g_test_stall = 0;

// ------------------------------------------------------------------ device facts

int device_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] with swizzled boxes of box_cols x box_rows.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------------ checks

dsa_status check_paging(const dsa_paging* pg) {
  if (pg == nullptr || pg->seq_lens == nullptr || pg->block_table == nullptr) return DSA_ERR_INVALID_ARG;
  if (pg->B < 1 || pg->n_q < 1 || pg->max_pages_per_seq < 1 || pg->num_pages < 1) return DSA_ERR_INVALID_ARG;
  if (pg->page_size != kPage) return DSA_ERR_UNSUPPORTED;
  const int64_t Bq = static_cast<int64_t>(pg->B) * pg->n_q;
  if (Bq * kHeads >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(pg->num_pages) * kPage >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(pg->max_pages_per_seq) * kPage >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// KV splits of the MLA decode for Bq queries of top_k keys. The count minimises an
// estimate of the time, (waves of CTAs over the SMs) x (tiles per CTA + the CTA's fixed
// cost in tiles, + one for the combine when split), over counts that keep Bq x splits
// within max_ctas (the caller's budget for partial buffers; 0: four waves). One CTA per SM.
int mla_splits_for(int Bq, int top_k, int* keys_per_split, int max_ctas = 0) {
  constexpr int kFixedTiles = 4;   // prologue + epilogue, about four 64-key tiles
  const int sms = device_sms() > 0 ? device_sms() : 1;
  const int tile = mla_tile_keys();
  const int ntiles = (top_k + tile - 1) / tile;
  const int64_t bq = Bq > 0 ? Bq : 1;
  const int64_t cap = max_ctas > 0 ? std::max<int64_t>(max_ctas, bq) : std::max<int64_t>(4LL * sms, bq);
  int best_tiles = ntiles;
  int64_t best_cost = -1;
  for (int s = 1; s <= ntiles; ++s) {
    const int tps = (ntiles + s - 1) / s;           // tiles per split
    const int se = (ntiles + tps - 1) / tps;        // splits actually used
    if (se != s) continue;                          // the same layout as a smaller count
    if (bq * se > cap) break;
    const int64_t waves = (bq * se + sms - 1) / sms;
    const int64_t cost = waves * (tps + kFixedTiles + (se > 1 ? 1 : 0));
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_tiles = tps;
    }
  }
  const int kps = best_tiles * tile;
  if (keys_per_split) *keys_per_split = kps;
  return (top_k + kps - 1) / kps;
}

struct Layout {
  size_t prefix = 0, scores = 0, logical = 0, physical = 0, part_ml = 0, part_o = 0, total = 0;
  // long-row top-k: per-query count / max / threshold words and candidate buffers
  int tk_chunks = 1;
  size_t tk_meta = 0, tk_key = 0, tk_idx = 0;
};

// op: DSA_OP_* or -1 for the MLA call alone.
Layout layout_for(int B, int64_t Bq, int64_t L_max, int top_k, int op, int nsplit) {
  Layout l;
  size_t off = 256;  // header
  if (op == DSA_OP_INDEXER || op == DSA_OP_LAYER) {
    l.prefix = off;
    off += up256(static_cast<size_t>(B + 1) * 4);
  }
  if (op == DSA_OP_LAYER) {
    l.scores = off;
    off += up256(static_cast<size_t>(Bq) * static_cast<size_t>(L_max) * 4);
    l.logical = off;
    off += up256(static_cast<size_t>(Bq) * top_k * 4);
    l.physical = off;
    off += up256(static_cast<size_t>(Bq) * top_k * 4);
  }
  if (op == DSA_OP_SHARD_LOCAL) {
    l.logical = off;
    off += up256(static_cast<size_t>(Bq) * top_k * 4);
  }
  if (op == DSA_OP_TOPK || op == DSA_OP_LAYER || op == DSA_OP_SHARD_LOCAL) {
    const int ch = topk_chunks(static_cast<int>(Bq), L_max, device_sms());
    if (ch > 1) {
      const size_t cap = static_cast<size_t>(topk_candidate_capacity());
      l.tk_chunks = ch;
      l.tk_meta = off;
      off += up256(static_cast<size_t>(Bq) * 3 * 4);
      l.tk_key = off;
      off += up256(static_cast<size_t>(Bq) * cap * 4);
      l.tk_idx = off;
      off += up256(static_cast<size_t>(Bq) * cap * 4);
    }
  }
  if ((op == DSA_OP_LAYER || op == -1) && nsplit > 1) {
    l.part_ml = off;
    off += up256(static_cast<size_t>(Bq) * nsplit * kHeads * kPartStats * 4);
    l.part_o = off;
    off += up256(static_cast<size_t>(Bq) * nsplit * kHeads * kDimV * 4);
  }
  l.total = off;
  return l;
}

dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

unsigned int* err_word(void* ws) { return reinterpret_cast<unsigned int*>(ws); }

// ------------------------------------------------------------------ stage bodies

dsa_status run_indexer(const dsa_paging* pg, const void* q_idx, dsa_dtype dt, const float* q_scale,
                       const float* head_w, const void* k_cache, const float* k_scale, float* scores, int64_t L_max,
                       uint8_t* ws, const Layout& lay, cudaStream_t st) {
  const bool fp8 = dt == DSA_FP8_E4M3;
  const int64_t Bq = static_cast<int64_t>(pg->B) * pg->n_q;
  CUtensorMap tk, tq;
  const CUtensorMapDataType cdt = fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int es = fp8 ? 1 : 2;
  const uint32_t box_cols = fp8 ? 128 : 64;
  if (!make_map(&tk, k_cache, cdt, es, kDimIdx, static_cast<uint64_t>(pg->num_pages) * kPage, box_cols, kPage) ||
      !make_map(&tq, q_idx, cdt, es, kDimIdx, static_cast<uint64_t>(Bq) * kHeads, box_cols, kHeads))
    return DSA_ERR_CUDA;
  unsigned int* err = err_word(ws);
  int32_t* prefix = nullptr;   // up to indexer_prefix_rows() rows the indexer builds it itself
  if (pg->B > indexer_prefix_rows()) {
    prefix = reinterpret_cast<int32_t*>(ws + lay.prefix);
    cudaError_t e = launch_plan(pg->seq_lens, pg->q_pos, pg->B, pg->n_q, pg->max_pages_per_seq,
                                indexer_tile_tokens(fp8, pg->n_q), prefix, err, st, &g_launches);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  IndexerArgs a;
  a.B = pg->B;
  a.n_q = pg->n_q;
  a.seq_lens = pg->seq_lens;
  a.q_pos = pg->q_pos;
  a.block_table = pg->block_table;
  a.max_pages = pg->max_pages_per_seq;
  a.num_pages = pg->num_pages;
  a.q_scale = q_scale;
  a.head_w = head_w;
  a.k_scale = k_scale;
  a.scores = scores;
  a.L_max = L_max;
  a.tile_prefix = prefix;
  a.err = err;
  const int grid = device_sms();
  if (grid <= 0) return DSA_ERR_CUDA;
  return cuda_status(launch_indexer(fp8, tk, tq, a, grid, st, &g_launches));
}

// Zeroes the long-row top-k counters (count, max, threshold per query) of a layout.
dsa_status clear_topk_counters(const Layout& lay, int64_t Bq, uint8_t* ws, cudaStream_t st) {
  if (lay.tk_chunks <= 1) return DSA_OK;
  return cuda_status(cudaMemsetAsync(ws + lay.tk_meta, 0, static_cast<size_t>(Bq) * 3 * 4, st));
}

// `counters_clear`: the long-row counters were zeroed earlier on this stream.
dsa_status run_topk(const dsa_paging* pg, const float* scores, int64_t L_max, int top_k, int32_t* logical,
                    int32_t* physical, uint8_t* ws, const Layout& lay, bool counters_clear, cudaStream_t st) {
  const int64_t Bq = static_cast<int64_t>(pg->B) * pg->n_q;
  TopkArgs a;
  a.n_q = pg->n_q;
  a.seq_lens = pg->seq_lens;
  a.q_pos = pg->q_pos;
  a.block_table = pg->block_table;
  a.max_pages = pg->max_pages_per_seq;
  a.num_pages = pg->num_pages;
  a.scores = scores;
  a.L_max = L_max;
  a.top_k = top_k;
  a.logical = logical;
  a.physical = physical;
  a.err = err_word(ws);
  a.chunks = lay.tk_chunks;
  a.pair = lay.tk_chunks <= 1 ? topk_pairs(static_cast<int>(Bq), L_max, device_sms()) : 0;
  a.cand_cap = topk_candidate_capacity();
  a.g_cnt = a.g_rmax = a.g_thr = a.g_key = nullptr;
  a.g_idx = nullptr;
  if (lay.tk_chunks > 1) {
    uint32_t* meta = reinterpret_cast<uint32_t*>(ws + lay.tk_meta);
    a.g_cnt = meta;
    a.g_rmax = meta + Bq;
    a.g_thr = meta + 2 * Bq;
    a.g_key = reinterpret_cast<uint32_t*>(ws + lay.tk_key);
    a.g_idx = reinterpret_cast<int32_t*>(ws + lay.tk_idx);
    if (!counters_clear) {
      const dsa_status s = clear_topk_counters(lay, Bq, ws, st);
      if (s != DSA_OK) return s;
    }
  }
  return cuda_status(launch_topk(a, static_cast<int>(Bq), st, &g_launches));
}

dsa_status run_mla(int Bq, const void* q, const void* kv, dsa_dtype kv_dtype, const float* kv_scale,
                   int64_t num_slots, const int32_t* physical, int top_k, float softmax_scale, void* out,
                   dsa_dtype out_dtype, float* lse, uint8_t* ws, const Layout& lay, int nsplit, int kps,
                   cudaStream_t st) {
  CUtensorMap tq;
  if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kDimK, static_cast<uint64_t>(Bq) * kHeads, 64, 64))
    return DSA_ERR_CUDA;
  MlaArgs a;
  a.q = q;
  a.Bq = Bq;
  a.top_k = top_k;
  a.nsplit = nsplit;
  a.keys_per_split = kps;
  a.kv = static_cast<const uint8_t*>(kv);
  a.kv_scale = kv_scale;
  a.num_slots = num_slots;
  a.physical = physical;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.out = out;
  a.out_fp32 = out_dtype == DSA_FP32 ? 1 : 0;
  a.lse = lse;
  a.part_ml = nsplit > 1 ? reinterpret_cast<float*>(ws + lay.part_ml) : nullptr;
  a.part_o = nsplit > 1 ? reinterpret_cast<float*>(ws + lay.part_o) : nullptr;
  a.err = err_word(ws);
  a.wait_limit = g_test_wait_limit > 0 ? g_test_wait_limit : kWaitLimitCycles;
  a.stall = g_test_stall;
  a.pair = a.nsplit == 2 ? 1 : 0;
  const int kvf = kv_dtype == DSA_FP8_E4M3 ? kKvFp8 : kv_dtype == DSA_FP8_E4M3_ROPE_BF16 ? kKvFp8Packed : kKvBf16;
  return cuda_status(launch_mla(kvf, tq, a, st, &g_launches));
}

dsa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < need) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

dsa_status check_index_inputs(const void* q_idx, dsa_dtype q_dtype, const float* q_scale, const float* head_w,
                              const void* k_cache, dsa_dtype k_dtype, const float* k_scale) {
  if (q_idx == nullptr || head_w == nullptr || k_cache == nullptr) return DSA_ERR_INVALID_ARG;
  if (q_dtype != k_dtype) return DSA_ERR_INVALID_ARG;
  if (q_dtype == DSA_FP8_E4M3) {
    if (q_scale == nullptr || k_scale == nullptr) return DSA_ERR_INVALID_ARG;
  } else if (q_dtype == DSA_BF16) {
    if (q_scale != nullptr || k_scale != nullptr) return DSA_ERR_INVALID_ARG;
  } else {
    return DSA_ERR_INVALID_ARG;
  }
  if (!aligned(q_idx, 16) || !aligned(k_cache, 16) || !aligned(head_w, 4)) return DSA_ERR_INVALID_ARG;
  if (k_scale != nullptr && !aligned(k_scale, 16)) return DSA_ERR_INVALID_ARG;   // copied per page in bulk
  return DSA_OK;
}

dsa_status check_mla_inputs(int Bq, const void* q, const void* kv, dsa_dtype kv_dtype, const float* kv_scale,
                            int64_t num_slots, const int32_t* physical, int top_k, float scale, const void* out,
                            dsa_dtype out_dtype) {
  if (Bq < 1 || q == nullptr || kv == nullptr || physical == nullptr || out == nullptr) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(Bq) * kHeads >= (int64_t(1) << 31)) return DSA_ERR_UNSUPPORTED;
  if (top_k < 1 || top_k > 16384 || num_slots < 1) return DSA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return DSA_ERR_INVALID_ARG;
  if (kv_dtype == DSA_FP8_E4M3) {
    if (kv_scale == nullptr) return DSA_ERR_INVALID_ARG;
  } else if (kv_dtype == DSA_BF16 || kv_dtype == DSA_FP8_E4M3_ROPE_BF16) {
    if (kv_scale != nullptr) return DSA_ERR_INVALID_ARG;   // no scale plane (packed rows carry theirs)
  } else {
    return DSA_ERR_INVALID_ARG;
  }
  if (out_dtype != DSA_BF16 && out_dtype != DSA_FP32) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv, 16)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

size_t dsa_workspace_size(const dsa_paging* paging, int64_t L_max, int32_t top_k, int32_t op) {
  if (check_paging(paging) != DSA_OK) return 0;
  if (op < DSA_OP_INDEXER || op > DSA_OP_SHARD_SELECT) return 0;
  const int64_t Bq = static_cast<int64_t>(paging->B) * paging->n_q;
  int nsplit = 1;
  if (op == DSA_OP_SHARD_LOCAL && (top_k < 1 || top_k > 16384)) return 0;
  if (op == DSA_OP_LAYER) {
    if (top_k < 1 || top_k > 16384) return 0;
    nsplit = mla_splits_for(static_cast<int>(Bq), top_k, nullptr);
    L_max = static_cast<int64_t>(paging->max_pages_per_seq) * kPage;
  }
  return layout_for(paging->B, Bq, L_max, top_k, op, nsplit).total;
}

size_t mla_workspace_size(int32_t Bq, int32_t top_k) {
  if (Bq < 1 || top_k < 1 || top_k > 16384) return 0;
  const int nsplit = mla_splits_for(Bq, top_k, nullptr);
  return layout_for(0, Bq, 0, top_k, -1, nsplit).total;
}

int32_t mla_num_splits(int32_t Bq, int32_t top_k) {
  if (Bq < 1 || top_k < 1) return 0;
  return mla_splits_for(Bq, top_k, nullptr);
}

dsa_status dsa_indexer_scores(const dsa_paging* paging, const void* q_idx, dsa_dtype q_dtype, const float* q_scale,
                              const float* head_w, const void* k_cache, dsa_dtype k_dtype, const float* k_scale,
                              float* scores, int64_t L_max, void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(paging);
  if (s != DSA_OK) return s;
  s = check_index_inputs(q_idx, q_dtype, q_scale, head_w, k_cache, k_dtype, k_scale);
  if (s != DSA_OK) return s;
  if (scores == nullptr || L_max < 1) return DSA_ERR_INVALID_ARG;
  const Layout lay = layout_for(paging->B, 0, L_max, 0, DSA_OP_INDEXER, 1);
  s = check_ws(workspace, ws_bytes, lay.total);
  if (s != DSA_OK) return s;
  return run_indexer(paging, q_idx, q_dtype, q_scale, head_w, k_cache, k_scale, scores, L_max,
                     static_cast<uint8_t*>(workspace), lay, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_topk_pagemap(const dsa_paging* paging, const float* scores, int64_t L_max, int32_t top_k,
                            int32_t* logical_out, int32_t* physical_out, void* workspace, size_t ws_bytes,
                            void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(paging);
  if (s != DSA_OK) return s;
  if (scores == nullptr || L_max < 1 || top_k < 1 || top_k > 16384) return DSA_ERR_INVALID_ARG;
  if (logical_out == nullptr && physical_out == nullptr) return DSA_ERR_INVALID_ARG;
  const int64_t Bq = static_cast<int64_t>(paging->B) * paging->n_q;
  const Layout lay = layout_for(paging->B, Bq, L_max, top_k, DSA_OP_TOPK, 1);
  s = check_ws(workspace, ws_bytes, lay.total);
  if (s != DSA_OK) return s;
  return run_topk(paging, scores, L_max, top_k, logical_out, physical_out, static_cast<uint8_t*>(workspace), lay,
                  false, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_pagemap(const dsa_paging* paging, const int32_t* logical, int32_t top_k, int32_t* physical,
                       void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(paging);
  if (s != DSA_OK) return s;
  if (logical == nullptr || physical == nullptr || top_k < 1) return DSA_ERR_INVALID_ARG;
  s = check_ws(workspace, ws_bytes, layout_for(paging->B, 0, 0, top_k, DSA_OP_PAGEMAP, 1).total);
  if (s != DSA_OK) return s;
  const int64_t total = static_cast<int64_t>(paging->B) * paging->n_q * top_k;
  return cuda_status(launch_pagemap(paging->n_q, top_k, total, paging->block_table, paging->max_pages_per_seq,
                                    paging->num_pages, logical, physical, err_word(workspace),
                                    static_cast<cudaStream_t>(stream), &g_launches));
}

dsa_status mla_sparse_decode(int32_t Bq, const void* q, const void* kv_cache, dsa_dtype kv_dtype,
                             const float* kv_scale, int64_t num_slots, const int32_t* physical, int32_t top_k,
                             float softmax_scale, void* out, dsa_dtype out_dtype, float* lse, void* workspace,
                             size_t ws_bytes, void* stream) {
  g_launches = 0;
  dsa_status s = check_mla_inputs(Bq, q, kv_cache, kv_dtype, kv_scale, num_slots, physical, top_k, softmax_scale,
                                  out, out_dtype);
  if (s != DSA_OK) return s;
  int kps = 0;
  const int nsplit = mla_splits_for(Bq, top_k, &kps);
  const Layout lay = layout_for(0, Bq, 0, top_k, -1, nsplit);
  s = check_ws(workspace, ws_bytes, lay.total);
  if (s != DSA_OK) return s;
  return run_mla(Bq, q, kv_cache, kv_dtype, kv_scale, num_slots, physical, top_k, softmax_scale, out, out_dtype, lse,
                 static_cast<uint8_t*>(workspace), lay, nsplit, kps, static_cast<cudaStream_t>(stream));
}

dsa_status dsa_decode_layer(const dsa_paging* paging, const void* q_idx, dsa_dtype idx_dtype, const float* q_scale,
                            const float* head_w, const void* k_cache, const float* k_scale, const void* q_mla,
                            const void* kv_cache, dsa_dtype kv_dtype, const float* kv_scale, int32_t top_k,
                            float softmax_scale, void* out, dsa_dtype out_dtype, float* lse, int32_t* logical_out,
                            int32_t* physical_out, void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(paging);
  if (s != DSA_OK) return s;
  s = check_index_inputs(q_idx, idx_dtype, q_scale, head_w, k_cache, idx_dtype, k_scale);
  if (s != DSA_OK) return s;
  const int64_t Bq = static_cast<int64_t>(paging->B) * paging->n_q;
  const int64_t num_slots = static_cast<int64_t>(paging->num_pages) * kPage;
  s = check_mla_inputs(static_cast<int>(Bq), q_mla, kv_cache, kv_dtype, kv_scale, num_slots, paging->block_table,
                       top_k, softmax_scale, out, out_dtype);
  if (s != DSA_OK) return s;
  int kps = 0;
  const int nsplit = mla_splits_for(static_cast<int>(Bq), top_k, &kps);
  const int64_t L_layer = static_cast<int64_t>(paging->max_pages_per_seq) * kPage;
  const Layout lay = layout_for(paging->B, Bq, L_layer, top_k, DSA_OP_LAYER, nsplit);
  s = check_ws(workspace, ws_bytes, lay.total);
  if (s != DSA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = reinterpret_cast<float*>(ws + lay.scores);
  int32_t* logical = logical_out ? logical_out : reinterpret_cast<int32_t*>(ws + lay.logical);
  int32_t* physical = physical_out ? physical_out : reinterpret_cast<int32_t*>(ws + lay.physical);
  // cleared here, ahead of the first kernel, so the top-k follows the indexer directly
  s = clear_topk_counters(lay, Bq, ws, st);
  if (s != DSA_OK) return s;
  s = run_indexer(paging, q_idx, idx_dtype, q_scale, head_w, k_cache, k_scale, scores, L_layer, ws, lay, st);
  if (s != DSA_OK) return s;
  s = run_topk(paging, scores, L_layer, top_k, logical, physical, ws, lay, true, st);
  if (s != DSA_OK) return s;
  return run_mla(static_cast<int>(Bq), q_mla, kv_cache, kv_dtype, kv_scale, num_slots, physical, top_k,
                 softmax_scale, out, out_dtype, lse, ws, lay, nsplit, kps, st);
}

dsa_status dsa_shard_local_topk(const dsa_paging* local, const float* scores, int64_t L_max, int32_t top_k,
                                const int32_t* token_offset, float* cand_score, int32_t* cand_token,
                                void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(local);
  if (s != DSA_OK) return s;
  if (local->q_pos != nullptr) return DSA_ERR_UNSUPPORTED;
  if (scores == nullptr || L_max < 1 || top_k < 1 || top_k > 16384) return DSA_ERR_INVALID_ARG;
  if (token_offset == nullptr || cand_score == nullptr || cand_token == nullptr) return DSA_ERR_INVALID_ARG;
  const int64_t Bq = static_cast<int64_t>(local->B) * local->n_q;
  const Layout lay = layout_for(local->B, Bq, L_max, top_k, DSA_OP_SHARD_LOCAL, 1);
  s = check_ws(workspace, ws_bytes, lay.total);
  if (s != DSA_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* logical = reinterpret_cast<int32_t*>(ws + lay.logical);
  s = run_topk(local, scores, L_max, top_k, logical, nullptr, ws, lay, false, st);
  if (s != DSA_OK) return s;
  ShardCandArgs a;
  a.Bq = static_cast<int>(Bq);
  a.n_q = local->n_q;
  a.top_k = top_k;
  a.scores = scores;
  a.L_max = L_max;
  a.logical = logical;
  a.token_offset = token_offset;
  a.cand_score = cand_score;
  a.cand_token = cand_token;
  a.err = err_word(ws);
  return cuda_status(launch_shard_candidates(a, st, &g_launches));
}

dsa_status dsa_shard_select(const dsa_paging* local, int32_t n_ranks, int32_t rank, const float* all_score,
                            const int32_t* all_token, int32_t top_k, const int32_t* token_offset,
                            int32_t* physical_out, int32_t* logical_out, void* workspace, size_t ws_bytes,
                            void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(local);
  if (s != DSA_OK) return s;
  if (local->q_pos != nullptr) return DSA_ERR_UNSUPPORTED;
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || top_k < 1 || top_k > 16384) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(n_ranks) * top_k >= (int64_t(1) << 30)) return DSA_ERR_UNSUPPORTED;
  if (all_score == nullptr || all_token == nullptr || token_offset == nullptr || physical_out == nullptr)
    return DSA_ERR_INVALID_ARG;
  s = check_ws(workspace, ws_bytes, layout_for(local->B, 0, 0, top_k, DSA_OP_SHARD_SELECT, 1).total);
  if (s != DSA_OK) return s;
  ShardSelectArgs a;
  a.Bq = local->B * local->n_q;
  a.n_q = local->n_q;
  a.top_k = top_k;
  a.n_ranks = n_ranks;
  a.rank = rank;
  a.all_score = all_score;
  a.all_token = all_token;
  a.token_offset = token_offset;
  a.seq_lens = local->seq_lens;
  a.block_table = local->block_table;
  a.max_pages = local->max_pages_per_seq;
  a.num_pages = local->num_pages;
  a.physical = physical_out;
  a.logical = logical_out;
  a.err = err_word(workspace);
  a.in_smem = shard_select_smem_bytes(n_ranks * top_k) > 0 ? 1 : 0;
  return cuda_status(launch_shard_select(a, static_cast<cudaStream_t>(stream), &g_launches));
}

dsa_status dsa_shard_merge(int32_t Bq, int32_t n_ranks, const float* all_out, const float* all_lse, void* out,
                           dsa_dtype out_dtype, float* lse, void* stream) {
  g_launches = 0;
  if (Bq < 1 || n_ranks < 1 || all_out == nullptr || all_lse == nullptr || out == nullptr) return DSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(Bq) * kHeads >= (int64_t(1) << 31) / n_ranks) return DSA_ERR_UNSUPPORTED;
  if (out_dtype != DSA_BF16 && out_dtype != DSA_FP32) return DSA_ERR_INVALID_ARG;
  if (!aligned(all_out, 16) || !aligned(out, out_dtype == DSA_FP32 ? 16 : 8) || !aligned(all_lse, 4))
    return DSA_ERR_INVALID_ARG;
  ShardMergeArgs a;
  a.Bq = Bq;
  a.n_ranks = n_ranks;
  a.all_out = all_out;
  a.all_lse = all_lse;
  a.out = out;
  a.out_fp32 = out_dtype == DSA_FP32 ? 1 : 0;
  a.lse = lse;
  return cuda_status(launch_shard_merge(a, static_cast<cudaStream_t>(stream), &g_launches));
}

dsa_status dsa_get_error(void* workspace, void* stream) {
  if (workspace == nullptr) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned int word[2] = {0, 0};
  if (cudaMemcpy(word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (word[0] != 0) {
    const unsigned int zero[2] = {0, 0};
    if (cudaMemcpy(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  }
  return static_cast<dsa_status>(word[0]);
}

const char* dsa_status_string(dsa_status status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case DSA_ERR_CUDA: return "CUDA runtime error";
    case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSA_ERR_DEVICE_BOUNDS: return "device-side index or length out of range (clamped)";
    case DSA_ERR_TIMEOUT: return "device-side bounded wait ran out";
  }
  return "unknown status";
}

int32_t dsa_last_launch_count(void) { return g_launches; }

dsa_status dsa_test_set_wait_hooks(int64_t wait_limit_cycles, int32_t stall) {
  if (wait_limit_cycles < 0 || (stall != 0 && stall != 1)) return DSA_ERR_INVALID_ARG;
  g_test_wait_limit = wait_limit_cycles;
  g_test_stall = stall;
  return DSA_OK;
}

}  // extern "C"

// ====================================================================== MLA decode without allocation
//
// mla_sparse_decode_noalloc: the split-KV MLA decode with its partials (and error words)
// kept in one file-scope device array instead of a caller-provided workspace, for callers
// that cannot allocate device memory themselves (a plugin inside an engine that owns the
// GPU's memory, or a loop that must not pay for cudaMalloc).

namespace {

// Largest layout mla_sparse_decode ever needs on a 148-SM GPU: 148 (query, split) pairs of
// 64 x 512 fp32 partial outputs plus 64 x 2 (max, sum) floats, and the 256-byte header.
constexpr size_t kMlaStaticScratchBytes = size_t(20) << 20;

}  // namespace

// One copy per device that loads this library, held until the process exits.
static __device__ __align__(256) uint8_t g_mla_static_scratch[kMlaStaticScratchBytes];

namespace {

// Device address of g_mla_static_scratch on the current device. In host code the array's
// name is only a handle, so the address is looked up once per device, with that device
// current, on the first call made there.
uint8_t* mla_static_scratch() {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_static_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  return addr[dev];
}

}  // namespace

extern "C" dsa_status mla_sparse_decode_noalloc(int32_t Bq, const void* q, const void* kv_cache,
                                                dsa_dtype kv_dtype, const float* kv_scale, int64_t num_slots,
                                                const int32_t* physical, int32_t top_k, float softmax_scale,
                                                void* out, dsa_dtype out_dtype, float* lse, unsigned int* status,
                                                void* stream) {
  g_launches = 0;
  dsa_status s = check_mla_inputs(Bq, q, kv_cache, kv_dtype, kv_scale, num_slots, physical, top_k, softmax_scale,
                                  out, out_dtype);
  if (s != DSA_OK) return s;
  if (status != nullptr && !aligned(status, 8)) return DSA_ERR_INVALID_ARG;
  int kps = 0;
  // at most one (query, split) pair per SM, which the static scratch is sized for
  const int nsplit = mla_splits_for(Bq, top_k, &kps, device_sms());
  const Layout lay = layout_for(0, Bq, 0, top_k, -1, nsplit);
  if (lay.total > kMlaStaticScratchBytes) return DSA_ERR_WORKSPACE;
  uint8_t* scratch = mla_static_scratch();
  if (scratch == nullptr) return DSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The error words must read zero when the kernels start; the partials are always
  // written in full before the combine reads them.
  if (cudaMemsetAsync(scratch, 0, 8, st) != cudaSuccess) return DSA_ERR_CUDA;
  s = run_mla(Bq, q, kv_cache, kv_dtype, kv_scale, num_slots, physical, top_k, softmax_scale, out, out_dtype, lse,
              scratch, lay, nsplit, kps, st);
  if (s != DSA_OK || status == nullptr) return s;
  return cuda_status(cudaMemcpyAsync(status, scratch, 8, cudaMemcpyDeviceToDevice, st));
}

// ====================================================================== the step before the path

extern "C" dsa_status dsa_rope_quantize_append(const dsa_paging* paging, const void* idx_q, const void* idx_k,
                                               const void* latent, void* q_mla, float rope_base, void* q_idx_out,
                                               float* q_scale_out, void* k_cache, float* k_scale, void* kv_cache,
                                               dsa_dtype kv_dtype, float* kv_scale, unsigned int* status,
                                               void* stream) {
  g_launches = 0;
  dsa_status s = check_paging(paging);
  if (s != DSA_OK) return s;
  if (idx_q == nullptr || idx_k == nullptr || latent == nullptr || q_idx_out == nullptr || q_scale_out == nullptr ||
      k_cache == nullptr || k_scale == nullptr || kv_cache == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!(rope_base > 1.0f) || !std::isfinite(rope_base)) return DSA_ERR_INVALID_ARG;
  int kvf = kKvBf16;
  if (kv_dtype == DSA_FP8_E4M3) {
    if (kv_scale == nullptr || !aligned(kv_scale, 4)) return DSA_ERR_INVALID_ARG;
    kvf = kKvFp8;
  } else if (kv_dtype == DSA_FP8_E4M3_ROPE_BF16 || kv_dtype == DSA_BF16) {
    if (kv_scale != nullptr) return DSA_ERR_INVALID_ARG;
    kvf = kv_dtype == DSA_BF16 ? kKvBf16 : kKvFp8Packed;
  } else {
    return DSA_ERR_INVALID_ARG;
  }
  if (!aligned(idx_q, 16) || !aligned(idx_k, 16) || !aligned(latent, 16) || !aligned(q_idx_out, 16) ||
      !aligned(q_scale_out, 4) || !aligned(k_cache, 16) || !aligned(k_scale, 4) || !aligned(kv_cache, 16) ||
      (q_mla != nullptr && !aligned(q_mla, 16)) || (status != nullptr && !aligned(status, 8)))
    return DSA_ERR_INVALID_ARG;
  AppendArgs a;
  a.n_q = paging->n_q;
  a.seq_lens = paging->seq_lens;
  a.q_pos = paging->q_pos;
  a.block_table = paging->block_table;
  a.max_pages = paging->max_pages_per_seq;
  a.num_pages = paging->num_pages;
  a.idx_q = static_cast<const uint16_t*>(idx_q);
  a.idx_k = static_cast<const uint16_t*>(idx_k);
  a.latent = static_cast<const uint16_t*>(latent);
  a.q_mla = static_cast<uint16_t*>(q_mla);
  for (int i = 0; i < 32; ++i) a.theta[i] = std::pow(static_cast<double>(rope_base), -2.0 * i / 64.0);
  a.q_out = static_cast<uint8_t*>(q_idx_out);
  a.q_scale_out = q_scale_out;
  a.k_cache = static_cast<uint8_t*>(k_cache);
  a.k_scale = k_scale;
  a.kv_cache = kv_cache;
  a.kvf = kvf;
  a.kv_scale = kv_scale;
  a.err = status;
  const int Bq = paging->B * paging->n_q;
  return cuda_status(launch_rope_quantize_append(a, Bq, static_cast<cudaStream_t>(stream), &g_launches));
}
