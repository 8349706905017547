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
constexpr int kCand = 6144;   // candidates kept in shared memory after the first digit

struct TopkSmem {
  uint32_t hist[kHistBins];
  uint32_t cand_key[kCand];
  int32_t cand_idx[kCand];
  uint32_t wsum[32];
  uint32_t sel_bin, sel_rem, n_cand, cnt_out, cnt_eq;
};

// Visits keys[0..n) of a row with 16-byte loads (4 in flight per thread) where the
// row is 16-byte aligned; `f(key, index)` is called for every element.
template <typename F>
__device__ __forceinline__ void for_each_key(const float* row, int n, F f) {
  const int tid = threadIdx.x;
  if ((reinterpret_cast<uintptr_t>(row) & 15) == 0) {
    const int n4 = n >> 2;
    const float4* r4 = reinterpret_cast<const float4*>(row);
    int i = tid;
    for (; i + 3 * kTopkThreads < n4; i += 4 * kTopkThreads) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(r4 + i + u * kTopkThreads);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = 4 * (i + u * kTopkThreads);
        f(order_key(v[u].x), s);
        f(order_key(v[u].y), s + 1);
        f(order_key(v[u].z), s + 2);
        f(order_key(v[u].w), s + 3);
      }
    }
    for (; i < n4; i += kTopkThreads) {
      const float4 v = __ldg(r4 + i);
      f(order_key(v.x), 4 * i);
      f(order_key(v.y), 4 * i + 1);
      f(order_key(v.z), 4 * i + 2);
      f(order_key(v.w), 4 * i + 3);
    }
    for (int s = 4 * n4 + tid; s < n; s += kTopkThreads) f(order_key(row[s]), s);
  } else {
    for (int s = tid; s < n; s += kTopkThreads) f(order_key(row[s]), s);
  }
}

// Picks the bin holding the `remaining`-th largest key: sets sm.sel_bin and
// sm.sel_rem = remaining - (keys in higher bins). Thread t owns bins [4t, 4t+4).
__device__ __forceinline__ void select_bin(TopkSmem& sm, uint32_t remaining) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t c0 = sm.hist[4 * tid], c1 = sm.hist[4 * tid + 1], c2 = sm.hist[4 * tid + 2],
                 c3 = sm.hist[4 * tid + 3];
  const uint32_t mine = c0 + c1 + c2 + c3;
  uint32_t v = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_down_sync(0xffffffffu, v, off);
    if (lane + off < 32) v += n;
  }
  if (lane == 0) sm.wsum[warp] = v;
  __syncthreads();
  uint32_t above = v - mine;
  for (int w = warp + 1; w < 32; ++w) above += sm.wsum[w];
  const uint32_t cs[4] = {c0, c1, c2, c3};
#pragma unroll
  for (int i = 3; i >= 0; --i) {
    if (above < remaining && above + cs[i] >= remaining) {
      sm.sel_bin = static_cast<uint32_t>(4 * tid + i);
      sm.sel_rem = remaining - above;
    }
    above += cs[i];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_pagemap_kernel(const TopkArgs a) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);

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

  // ---- digit 1 (key bits 31..20) over the whole row
  for (int i = tid; i < kHistBins; i += kTopkThreads) sm.hist[i] = 0;
  if (tid == 0) {
    sm.n_cand = 0;
    sm.cnt_out = 0;
    sm.cnt_eq = 0;
  }
  __syncthreads();
  for_each_key(row, vis, [&](uint32_t u, int) { atomicAdd(&sm.hist[u >> 20], 1u); });
  __syncthreads();
  select_bin(sm, static_cast<uint32_t>(K));
  const uint32_t bin1 = sm.sel_bin;
  uint32_t remaining = sm.sel_rem;
  const uint32_t n_above = static_cast<uint32_t>(K) - remaining;   // keys in bins above bin1

  // ---- second pass: emit keys above bin1, gather bin1's keys as candidates
  for_each_key(row, vis, [&](uint32_t u, int s) {
    const uint32_t d = u >> 20;
    if (d > bin1) {
      const uint32_t p = atomicAdd(&sm.cnt_out, 1u);
      if (p < n_above) emit(static_cast<int>(p), s);
    } else if (d == bin1) {
      const uint32_t c = atomicAdd(&sm.n_cand, 1u);
      if (c < kCand) {
        sm.cand_key[c] = u;
        sm.cand_idx[c] = s;
      }
    }
  });
  __syncthreads();
  const uint32_t n_cand = sm.n_cand;
  const bool in_smem = n_cand <= static_cast<uint32_t>(kCand);

  // ---- digits 2 (bits 19..8) and 3 (bits 7..0) among the candidates
  uint32_t prefix = bin1 << 20, pmask = 0xFFF00000u;
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    const int sh = pass == 0 ? 8 : 0;
    const uint32_t dm = pass == 0 ? 0xFFFu : 0xFFu;
    for (int i = tid; i < kHistBins; i += kTopkThreads) sm.hist[i] = 0;
    __syncthreads();
    if (in_smem) {
      for (int c = tid; c < static_cast<int>(n_cand); c += kTopkThreads) {
        const uint32_t u = sm.cand_key[c];
        if ((u & pmask) == prefix) atomicAdd(&sm.hist[(u >> sh) & dm], 1u);
      }
    } else {
      for_each_key(row, vis, [&](uint32_t u, int) {
        if ((u & pmask) == prefix) atomicAdd(&sm.hist[(u >> sh) & dm], 1u);
      });
    }
    __syncthreads();
    select_bin(sm, remaining);
    prefix |= sm.sel_bin << sh;
    pmask |= dm << sh;
    remaining = sm.sel_rem;
  }

  // `prefix` is the exact key of the k-th largest score: take the candidates above it and
  // `remaining` of those equal to it.
  const uint32_t kth = prefix;
  const uint32_t take_eq = remaining;
  const uint32_t n_gt = static_cast<uint32_t>(K) - take_eq;
  auto final_pick = [&](uint32_t u, int s) {
    if ((u >> 20) != bin1) return;   // keys above bin1 were emitted already
    if (u > kth) {
      const uint32_t p = atomicAdd(&sm.cnt_out, 1u);
      if (p < n_gt) emit(static_cast<int>(p), s);
    } else if (u == kth) {
      const uint32_t e = atomicAdd(&sm.cnt_eq, 1u);
      if (e < take_eq) emit(static_cast<int>(n_gt + e), s);
    }
  };
  if (in_smem) {
    for (int c = tid; c < static_cast<int>(n_cand); c += kTopkThreads) final_pick(sm.cand_key[c], sm.cand_idx[c]);
  } else {
    for_each_key(row, vis, final_pick);
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
  const int smem = static_cast<int>(sizeof(TopkSmem));
  cudaError_t e = cudaFuncSetAttribute(topk_pagemap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  topk_pagemap_kernel<<<Bq, kTopkThreads, smem, stream>>>(a);
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
