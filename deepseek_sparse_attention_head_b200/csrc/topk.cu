// Stage 2 of the DSA decode step: top-k selection with the fused page-mapping
// transform ("GLM-52 Runs on RTX 4090", kernel list item 2; glm-5.2-4090 README,
// usage: SGLANG_NSA_FUSE_TOPK=1 fuses the page-mapping transform into top-k).
//
// One CTA per query. Scores are mapped to order-preserving 32-bit keys and the
// k-th largest key is found exactly by a three-digit radix select (12 + 12 + 8 bits)
// over shared-memory histograms; a last pass emits every key above it plus the
// needed number of keys equal to it, and maps each logical token through the
// block table to its physical slot. A query that sees no more than top_k tokens
// takes all of them (the dense path).
#include "kernels.cuh"

namespace dsa {

// Larger float -> larger unsigned key (negative values bit-flipped, positives get the top bit).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTopkThreads = 1024;
constexpr int kHistBins = 4096;

__global__ void __launch_bounds__(kTopkThreads) topk_pagemap_kernel(const TopkArgs a) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t wsum[32];
  __shared__ uint32_t sel_bin, sel_rem, cnt_gt, cnt_eq;

  const int tid = threadIdx.x;
  const int q = blockIdx.x;
  const int b = q / a.n_q;
  const int L = row_len(a.seq_lens, b, a.max_pages);
  int vis = query_vis(a.q_pos, q, L);
  if (vis > a.L_max) vis = static_cast<int>(a.L_max);
  const int K = a.top_k;
  int32_t* lo = a.logical ? a.logical + static_cast<int64_t>(q) * K : nullptr;
  int32_t* po = a.physical ? a.physical + static_cast<int64_t>(q) * K : nullptr;

  auto emit = [&](int pos, int s) {
    if (lo) lo[pos] = s;
    if (po) {
      int slot = -1;
      if (s >= 0) slot = checked_page(a.block_table, b, s >> 6, a.max_pages, a.num_pages, a.err) * kPage + (s & 63);
      po[pos] = slot;
    }
  };

  if (vis <= K) {  // dense path: every visible token
    for (int i = tid; i < K; i += kTopkThreads) emit(i, i < vis ? i : -1);
    return;
  }

  const float* row = a.scores + static_cast<int64_t>(q) * a.L_max;
  uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(K);
  const int lane = tid & 31, warp = tid >> 5;

#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int sh = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
    const uint32_t dm = pass == 2 ? 0xFFu : 0xFFFu;
    for (int i = tid; i < kHistBins; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int s = tid; s < vis; s += kTopkThreads) {
      const uint32_t u = order_key(row[s]);
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> sh) & dm], 1u);
    }
    __syncthreads();
    // thread t owns bins [4t, 4t+4); count the keys in all higher bins (suffix scan)
    uint32_t c0 = hist[4 * tid], c1 = hist[4 * tid + 1], c2 = hist[4 * tid + 2], c3 = hist[4 * tid + 3];
    const uint32_t mine = c0 + c1 + c2 + c3;
    uint32_t v = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n = __shfl_down_sync(0xffffffffu, v, off);
      if (lane + off < 32) v += n;
    }
    if (lane == 0) wsum[warp] = v;
    __syncthreads();
    uint32_t above = v - mine;
    for (int w = warp + 1; w < 32; ++w) above += wsum[w];
    const uint32_t cs[4] = {c0, c1, c2, c3};
#pragma unroll
    for (int i = 3; i >= 0; --i) {
      if (above < remaining && above + cs[i] >= remaining) {
        sel_bin = static_cast<uint32_t>(4 * tid + i);
        sel_rem = remaining - above;
      }
      above += cs[i];
    }
    __syncthreads();
    prefix |= sel_bin << sh;
    pmask |= dm << sh;
    remaining = sel_rem;
    __syncthreads();
  }

  // `prefix` is now the exact key of the k-th largest score; take every larger key and
  // `remaining` of the keys equal to it.
  if (tid == 0) {
    cnt_gt = 0;
    cnt_eq = 0;
  }
  __syncthreads();
  const uint32_t kth = prefix;
  const uint32_t take_eq = remaining;
  const uint32_t n_gt = static_cast<uint32_t>(K) - take_eq;
  for (int s = tid; s < vis; s += kTopkThreads) {
    const uint32_t u = order_key(row[s]);
    if (u > kth) {
      const uint32_t p = atomicAdd(&cnt_gt, 1u);
      if (p < n_gt) emit(static_cast<int>(p), s);
    } else if (u == kth) {
      const uint32_t e = atomicAdd(&cnt_eq, 1u);
      if (e < take_eq) emit(static_cast<int>(n_gt + e), s);
    }
  }
}

// The page-mapping transform alone: physical = table[b, i/64]*64 + i%64, -1 -> -1.
__global__ void pagemap_kernel(int n_q, int top_k, int64_t total, const int32_t* block_table, int max_pages,
                               int num_pages, const int32_t* logical, int32_t* physical, unsigned int* err) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int q = static_cast<int>(i / top_k);
    const int b = q / n_q;
    const int s = logical[i];
    int out = -1;
    if (s >= 0) {
      int p = s >> 6;
      if (p >= max_pages) {
        record_error(err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(s));
        p = 0;
      }
      out = checked_page(block_table, b, p, max_pages, num_pages, err) * kPage + (s & 63);
    } else if (s != -1) {
      record_error(err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(s));
    }
    physical[i] = out;
  }
}

cudaError_t launch_topk(const TopkArgs& a, int Bq, cudaStream_t stream, int* launches) {
  topk_pagemap_kernel<<<Bq, kTopkThreads, 0, stream>>>(a);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t launch_pagemap(int n_q, int top_k, int64_t total, const int32_t* block_table, int max_pages,
                           int num_pages, const int32_t* logical, int32_t* physical, unsigned int* err,
                           cudaStream_t stream, int* launches) {
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  pagemap_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(n_q, top_k, total, block_table, max_pages, num_pages,
                                                               logical, physical, err);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace dsa
