// Stage 1 of the DSA decode step: the lightning indexer ("GLM-52 Runs on RTX 4090",
// kernel list item 1, "Lightning-indexer GEMM"):
//
//   score[q, s] = k_scale[slot(s)] * sum_h (w[q,h] * q_scale[q,h]) * ReLU(<q8[q,h], k8[slot(s)]>)
//
// Design (sm_100a): one persistent CTA per SM walks a contiguous range of 128-token
// tiles (two 64-token pages) of the paged key cache.
//   warp 0  TMA producer: one 64 x 128 B box per page straight from the block table,
//           128-byte swizzled, into an 8-deep ring; query tiles into a 2-slot ring.
//   warp 1  tcgen05 issuer: D[128 tokens, 64*g heads] = K_tile x Q_group^T, fp8 x fp8
//           (kind::f8f6f4) or bf16 x bf16 (kind::f16), fp32 in TMEM, 2 accumulators.
//   warps 2-5  epilogue: one thread per token (its TMEM lane) applies ReLU, the head
//           weights and the key scale, and writes the fp32 score row.
// Decode (n_q = 1) loads a row's query once per row; chunked prefill streams groups
// of up to 4 queries (N = 256) past every key tile.
#include "kernels.cuh"

namespace dsa {

template <int KC>
struct IdxCfg {
  static constexpr int kStages = KC == 1 ? 8 : 2;
  static constexpr int kBSlots = 2;
  static constexpr int kAStage = KC * 16384;   // 128 tokens x 128 B per K-chunk
  static constexpr int kBSlot = KC * 32768;    // 4 queries x 64 heads x 128 B per K-chunk
  static constexpr int kWBytes = 4 * 2 * 256 * 4;  // per-warp double-buffered head weights
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kAStage;
  static constexpr int kOffW = kOffB + kBSlots * kBSlot;
  static constexpr int kOffBar = kOffW + kWBytes;
  static constexpr int kNumBars = 2 * kStages + 2 * kBSlots + 4 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 64 + 1024;  // + slack to align the base to 1024
};

constexpr int kTileTok = 128;
constexpr int kQGroup = 4;
constexpr uint32_t kIdxTmemCols = 512;  // 2 accumulators x 256 columns

// Walks the CTA's contiguous range of global tile ids, yielding (row, tile-in-row).
struct TileWalker {
  const int32_t* prefix;
  int b, gt, end;
  __device__ void init(const int32_t* p, int B, int begin, int stop) {
    prefix = p;
    gt = begin;
    end = stop;
    int lo = 0, hi = B;  // largest b with prefix[b] <= begin
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= begin) lo = mid; else hi = mid;
    }
    b = lo;
  }
  __device__ bool next(int& row, int& tile) {
    if (gt >= end) return false;
    while (gt >= prefix[b + 1]) ++b;
    row = b;
    tile = gt - prefix[b];
    ++gt;
    return true;
  }
};

// A query group contributes to a tile when one of its queries sees a token of it.
__device__ __forceinline__ bool group_active(const IndexerArgs& a, int b, int g, int tok0, int L) {
  if (a.q_pos == nullptr) return true;
  const int q0 = b * a.n_q + g * kQGroup;
  const int nqg = min(kQGroup, a.n_q - g * kQGroup);
  for (int j = 0; j < nqg; ++j)
    if (query_vis(a.q_pos, q0 + j, L) > tok0) return true;
  return false;
}

__device__ __forceinline__ void bounded_drain(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) break;
  }
}

template <int KC>
__global__ void __launch_bounds__(192, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                   const IndexerArgs a) {
  using C = IdxCfg<KC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::kOffA;
  uint8_t* sB = smem + C::kOffB;
  float* sW = reinterpret_cast<float*>(smem + C::kOffW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + C::kStages;
  uint64_t* b_full = a_empty + C::kStages;
  uint64_t* b_empty = b_full + C::kBSlots;
  uint64_t* acc_full = b_empty + C::kBSlots;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < C::kBSlots; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kIdxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int total = a.tile_prefix[a.B];
  const int per = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int t_begin = min(total, static_cast<int>(blockIdx.x) * per);
  const int t_end = min(total, t_begin + per);
  const int ngroups = (a.n_q + kQGroup - 1) / kQGroup;

  if (t_begin < t_end) {
    TileWalker walk;
    walk.init(a.tile_prefix, a.B, t_begin, t_end);

    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_map(&tmap_k);
        tma_prefetch_map(&tmap_q);
        int it = 0, bit = -1, cur_q0 = -1;
        bool ok = true;
        int b, t;
        while (ok && walk.next(b, t)) {
          const int L = row_len(a.seq_lens, b, a.max_pages);
          const int npages = (L + kPage - 1) / kPage;
          const int s = it % C::kStages;
          if (!wait_one(&a_empty[s], ((it / C::kStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
          const int p0 = checked_page(a.block_table, b, 2 * t, a.max_pages, a.num_pages, a.err);
          const bool has1 = 2 * t + 1 < npages;
          const int p1 = has1 ? checked_page(a.block_table, b, 2 * t + 1, a.max_pages, a.num_pages, a.err) : 0;
          mbar_arrive_expect_tx(&a_full[s], (has1 ? 2u : 1u) * KC * 8192u);
          uint8_t* dst = sA + s * C::kAStage;
#pragma unroll
          for (int kc = 0; kc < KC; ++kc) {
            tma_load_2d(dst + kc * 16384, &tmap_k, kc * 64, p0 * kPage, &a_full[s]);
            if (has1) tma_load_2d(dst + kc * 16384 + 8192, &tmap_k, kc * 64, p1 * kPage, &a_full[s]);
          }
          ++it;
          const int tok0 = t * kTileTok;
          for (int g = 0; g < ngroups; ++g) {
            if (!group_active(a, b, g, tok0, L)) continue;
            const int q0 = b * a.n_q + g * kQGroup;
            if (q0 == cur_q0) continue;
            const int nqg = min(kQGroup, a.n_q - g * kQGroup);
            ++bit;
            const int bs = bit % C::kBSlots;
            if (!wait_one(&b_empty[bs], ((bit / C::kBSlots) & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&b_full[bs], static_cast<uint32_t>(nqg) * KC * 8192u);
            for (int j = 0; j < nqg; ++j)
#pragma unroll
              for (int kc = 0; kc < KC; ++kc)
                tma_load_2d(sB + bs * C::kBSlot + kc * 32768 + j * 8192, &tmap_q, kc * 64, (q0 + j) * kHeads,
                            &b_full[bs]);
            cur_q0 = q0;
          }
        }
        if (!ok) {
          record_error(a.err, DSA_ERR_TIMEOUT, 1);
          *abort_flag = 1;
          for (int i = max(0, it - C::kStages); i < it; ++i) bounded_drain(&a_full[i % C::kStages], (i / C::kStages) & 1);
          for (int i = max(0, bit - C::kBSlots + 1); i <= bit; ++i)
            bounded_drain(&b_full[i % C::kBSlots], (i / C::kBSlots) & 1);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ tcgen05 issuer
      if (lane == 0) {
        const uint32_t fmt = KC == 1 ? 0u : 1u;  // e4m3 (kind::f8f6f4) or bf16 (kind::f16)
        int it = 0, bit = -1, cur_q0 = -1, acc_it = 0;
        bool ok = true;
        int b, t;
        while (ok && walk.next(b, t)) {
          const int L = row_len(a.seq_lens, b, a.max_pages);
          const int s = it % C::kStages;
          if (!wait_one(&a_full[s], (it / C::kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const int tok0 = t * kTileTok;
          const uint32_t a_base = smem_u32(sA + s * C::kAStage);
          for (int g = 0; g < ngroups && ok; ++g) {
            if (!group_active(a, b, g, tok0, L)) continue;
            const int q0 = b * a.n_q + g * kQGroup;
            const int nqg = min(kQGroup, a.n_q - g * kQGroup);
            if (q0 != cur_q0) {
              if (bit >= 0) tc_commit(&b_empty[bit % C::kBSlots]);
              ++bit;
              if (!wait_one(&b_full[bit % C::kBSlots], (bit / C::kBSlots) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              cur_q0 = q0;
            }
            const int ab = acc_it & 1;
            if (!wait_one(&acc_empty[ab], ((acc_it >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + static_cast<uint32_t>(ab * 256);
            const uint32_t idesc = idesc_make(fmt, fmt, false, false, 128, kHeads * nqg);
            const uint32_t b_base = smem_u32(sB + (bit % C::kBSlots) * C::kBSlot);
#pragma unroll
            for (int kc = 0; kc < KC; ++kc)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t ad = sdesc_sw128(a_base + kc * 16384 + ks * 32, 16, 1024);
                const uint64_t bd = sdesc_sw128(b_base + kc * 32768 + ks * 32, 16, 1024);
                if (KC == 1) mma_f8(d, ad, bd, idesc, (kc | ks) != 0);
                else mma_f16(d, ad, bd, idesc, (kc | ks) != 0);
              }
            tc_commit(&acc_full[ab]);
            ++acc_it;
          }
          if (!ok) break;
          tc_commit(&a_empty[s]);
          ++it;
        }
        if (!ok) {
          record_error(a.err, DSA_ERR_TIMEOUT, 2);
          *abort_flag = 1;
        }
        // every MMA this thread issued has finished before the CTA frees TMEM
        tc_commit(drain);
        bounded_drain(drain, 0);
      }
      __syncwarp();
    } else {
      // ------------------------------------------------------------ epilogue (warps 2..5)
      const int quarter = warp & 3;            // TMEM lanes [32*quarter, 32*quarter + 32)
      const int row_in_tile = quarter * 32 + lane;
      float* wmine = sW + (warp - 2) * 512;    // two 256-entry buffers per warp
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      int acc_it = 0, cur_q0 = -1, wb = 1;
      bool ok = true;
      int b, t;
      while (ok && walk.next(b, t)) {
        const int L = row_len(a.seq_lens, b, a.max_pages);
        const int tok0 = t * kTileTok;
        const int tok = tok0 + row_in_tile;
        float kscale = 1.0f;
        if (a.k_scale != nullptr && tok < L) {
          const int pg = checked_page(a.block_table, b, tok >> 6, a.max_pages, a.num_pages, a.err);
          kscale = a.k_scale[static_cast<int64_t>(pg) * kPage + (tok & 63)];
        }
        for (int g = 0; g < ngroups; ++g) {
          if (!group_active(a, b, g, tok0, L)) continue;
          const int q0 = b * a.n_q + g * kQGroup;
          const int nqg = min(kQGroup, a.n_q - g * kQGroup);
          if (q0 != cur_q0) {
            wb ^= 1;
            __syncwarp();
            for (int i = lane; i < nqg * kHeads; i += 32) {
              float w = a.head_w[static_cast<int64_t>(q0) * kHeads + i];
              if (a.q_scale != nullptr) w *= a.q_scale[static_cast<int64_t>(q0) * kHeads + i];
              wmine[wb * 256 + i] = w;
            }
            __syncwarp();
            cur_q0 = q0;
          }
          const int ab = acc_it & 1;
          if (!wait_warp(&acc_full[ab], (acc_it >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          for (int j = 0; j < nqg; ++j) {
            float acc[32];
            float sc = 0.0f;
            const float* wq = wmine + wb * 256 + j * kHeads;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              tmem_ld32(lane_addr + static_cast<uint32_t>(ab * 256 + j * kHeads + half * 32), acc);
#pragma unroll
              for (int h = 0; h < 32; ++h) sc = fmaf(wq[half * 32 + h], fmaxf(acc[h], 0.0f), sc);
            }
            const int q = q0 + j;
            int vis = query_vis(a.q_pos, q, L);
            if (vis > a.L_max) vis = static_cast<int>(a.L_max);
            if (tok < vis) a.scores[static_cast<int64_t>(q) * a.L_max + tok] = sc * kscale;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          ++acc_it;
        }
      }
      if (!ok && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 3);
        *abort_flag = 1;
      }
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kIdxTmemCols);
}

// Tile prefix over rows (single CTA) plus validation of lengths and causal positions.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* seq_lens, const int32_t* q_pos, int B, int n_q,
                                                    int max_pages, int32_t* tile_prefix, unsigned int* err) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x;
  if (tid == 0) {
    carry = 0;
    tile_prefix[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int b = base + tid;
    int tiles = 0;
    if (b < B) {
      const int raw = seq_lens[b];
      if (raw < 0 || raw > max_pages * kPage) record_error(err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(raw));
      tiles = (row_len(seq_lens, b, max_pages) + kTileTok - 1) / kTileTok;
    }
    int v = tiles;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, off);
      if ((tid & 31) >= off) v += n;
    }
    if ((tid & 31) == 31) warp_sums[tid >> 5] = v;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < (tid >> 5); ++w) before += warp_sums[w];
    if (b < B) tile_prefix[b + 1] = carry + before + v;
    __syncthreads();
    if (tid == 0) {
      int tot = 0;
      for (int w = 0; w < 32; ++w) tot += warp_sums[w];
      carry += tot;
    }
    __syncthreads();
  }
  if (q_pos != nullptr) {
    for (int q = tid; q < B * n_q; q += 1024) {
      const int L = row_len(seq_lens, q / n_q, max_pages);
      const int p = q_pos[q];
      if (p < 0 || p >= L) record_error(err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(p));
    }
  }
}

template __global__ void indexer_kernel<1>(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                                           const IndexerArgs);
template __global__ void indexer_kernel<2>(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,
                                           const IndexerArgs);

cudaError_t launch_plan(const int32_t* seq_lens, const int32_t* q_pos, int B, int n_q, int max_pages,
                        int32_t* tile_prefix, unsigned int* err, cudaStream_t stream, int* launches) {
  plan_kernel<<<1, 1024, 0, stream>>>(seq_lens, q_pos, B, n_q, max_pages, tile_prefix, err);
  ++*launches;
  return cudaGetLastError();
}

template <int KC>
static cudaError_t launch_indexer_kc(const CUtensorMap& tk, const CUtensorMap& tq, const IndexerArgs& a, int grid,
                                     cudaStream_t stream) {
  constexpr int smem = IdxCfg<KC>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(indexer_kernel<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  indexer_kernel<KC><<<grid, 192, smem, stream>>>(tk, tq, a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(bool fp8, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q, const IndexerArgs& a,
                           int grid, cudaStream_t stream, int* launches) {
  ++*launches;
  return fp8 ? launch_indexer_kc<1>(tmap_k, tmap_q, a, grid, stream)
             : launch_indexer_kc<2>(tmap_k, tmap_q, a, grid, stream);
}

}  // namespace dsa
