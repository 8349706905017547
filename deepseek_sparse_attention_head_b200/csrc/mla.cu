// Stage 3 of the DSA decode step: MLA sparse decode ("GLM-52 Runs on RTX 4090", kernel
// list item 3). For query q, head h and its selected latent rows j:
//
//   z[h, j] = scale * <q[h, 0:576], KV[slot_j, 0:576]>,  out[h, :] = sum_j softmax_j(z) KV[slot_j, 0:512]
//
// (576 = 512 latent + 64 rope columns; "Show HN: colibri", features.)
//
// Design (sm_100a): grid = (query, split); each CTA walks 64-row tiles of its share of
// the index list.
//   * fp8 rows (576 B) are fetched with one bulk async copy each into a 2-deep ring,
//     then dequantised (code x per-group scale -> bf16) into a 128-byte-swizzled tile
//     that serves both as the K operand of QK and the (MN-major) V operand of PV.
//   * QK:  S[heads, keys] = Q[64 (+64 unused rows), 576] x KV^T    (tcgen05 kind::f16, M=128)
//   * softmax per head (one thread per head, row in TMEM), lazily rescaled: the
//     running max only moves when a tile's max exceeds it by more than 8 (log2 units).
//   * PV:  O^T[512 dims, 64 heads] += V^T x P^T                    (4 x M=128, N=64)
// Splits write (m, l, o) partials; a combine kernel merges them with log-sum-exp.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {

constexpr int kMlaTile = 64;
constexpr int kMlaThreads = 128;
constexpr uint32_t kMlaTmemCols = 512;   // S: cols [0,64); O^T: cols [64, 320)
constexpr int kOffQ = 0;                 // 9 x 8 KB, K-major SW128
constexpr int kOffKV = 73728;            // 9 x 8 KB, K-major SW128 (rows = keys)
constexpr int kOffP = 147456;            // 64 heads x 128 B
constexpr int kOffStage = 155648;        // 2 x 64 x 576 B fp8 staging
constexpr int kStageBytes = kMlaTile * kDimK;
constexpr int kOffIdx = kOffStage + 2 * kStageBytes;   // 2 x 64 int32
constexpr int kOffAlpha = kOffIdx + 512;               // 64 f32
constexpr int kOffInvL = kOffAlpha + 256;              // 64 f32
constexpr int kOffMisc = kOffInvL + 256;               // vmask (u64), tmem holder, abort
constexpr int kOffBars = kOffMisc + 64;                // q_full, stage_full[2], s_done, o_done
constexpr int kMlaSmem = kOffBars + 64 + 1024;

__device__ __forceinline__ void store_swizzled(uint8_t* tile, int row, int chunk16, uint4 v) {
  // row-major [rows][128 B] block of one 64-element K chunk, 16-byte unit swizzled by row % 8
  *reinterpret_cast<uint4*>(tile + row * 128 + ((chunk16 ^ (row & 7)) << 4)) = v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Four E4M3 codes (one 32-bit word) times `sc` -> two bf16x2 words.
__device__ __forceinline__ void dequant4(uint32_t w, float sc, uint32_t& o0, uint32_t& o1) {
  const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
  const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
  o0 = pack_bf16x2(f01.x * sc, f01.y * sc);
  o1 = pack_bf16x2(f23.x * sc, f23.y * sc);
}

__device__ __forceinline__ void bounded_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) break;
  }
}

template <bool FP8>
__global__ void __launch_bounds__(kMlaThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const MlaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  uint8_t* sStage = smem + kOffStage;
  int32_t* sIdx = reinterpret_cast<int32_t*>(smem + kOffIdx);
  float* sAlpha = reinterpret_cast<float*>(smem + kOffAlpha);
  float* sInvL = reinterpret_cast<float*>(smem + kOffInvL);
  unsigned long long* sVmask = reinterpret_cast<unsigned long long*>(smem + kOffMisc);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 12);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* q_full = bars;
  uint64_t* stage_full = bars + 1;  // [2]
  uint64_t* s_done = bars + 3;
  uint64_t* o_done = bars + 4;
  uint64_t* drain = bars + 5;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int q = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int k0 = split * a.keys_per_split;
  const int k1 = min(a.top_k, k0 + a.keys_per_split);
  const int nkeys = max(0, k1 - k0);
  const int ntiles = (nkeys + kMlaTile - 1) / kMlaTile;
  const int32_t* phys = a.physical + static_cast<int64_t>(q) * a.top_k;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(&stage_full[0], 1);
    mbar_init(&stage_full[1], 1);
    mbar_init(s_done, 1);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, kMlaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tmem_S = tmem;
  const uint32_t tmem_O = tmem + 64;

  // Reads tile T's slot list into sIdx[st] (invalid -> -1) and, for fp8, starts one
  // bulk copy per valid row into staging buffer st. Executed by warp 3.
  auto issue_tile = [&](int T, int st) {
    int32_t* idx = sIdx + st * kMlaTile;
    int slots[2];
    unsigned valid = 0;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int j = lane + 32 * r;
      const int k = k0 + T * kMlaTile + j;
      int slot = k < k1 ? phys[k] : -1;
      if (slot < -1 || slot >= a.num_slots) {
        record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(slot));
        slot = -1;
      }
      slots[r] = slot;
      idx[j] = slot;
      valid += slot >= 0 ? 1u : 0u;
    }
    if (FP8) {
      unsigned nvalid = valid;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) nvalid += __shfl_xor_sync(0xffffffffu, nvalid, off);
      if (lane == 0) mbar_arrive_expect_tx(&stage_full[st], nvalid * kDimK);
      __syncwarp();
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int j = lane + 32 * r;
        if (slots[r] >= 0)
          bulk_load(sStage + st * kStageBytes + j * kDimK, a.kv + static_cast<int64_t>(slots[r]) * kDimK, kDimK,
                    &stage_full[st]);
      }
    }
    __syncwarp();
  };

  if (tid == 0 && ntiles > 0) {
    tma_prefetch_map(&tmap_q);
    mbar_arrive_expect_tx(q_full, 9u * 8192u);
#pragma unroll 1
    for (int c = 0; c < 9; ++c) tma_load_2d(sQ + c * 8192, &tmap_q, c * 64, q * kHeads, q_full);
  }
  if (warp == 3) {
    if (ntiles > 0) issue_tile(0, 0);
    if (ntiles > 1) issue_tile(1, 1);
  }

  float m_run = -INFINITY, l_run = 0.0f;   // per head (threads 0..63)
  bool ok = true;
  int issued = min(ntiles, 2);             // tiles whose rows have been requested
  int T = 0;
  if (ntiles > 0) ok = wait_warp(q_full, 0, abort_flag);
  __syncthreads();

  const uint32_t idesc_qk = idesc_make(1, 1, false, false, 128, 64);
  const uint32_t idesc_pv = idesc_make(1, 1, true, false, 128, 64);

#pragma unroll 1
  for (; T < ntiles; ++T) {
    const int st = T & 1;
    if (FP8) {
      const bool got = wait_warp(&stage_full[st], (T >> 1) & 1, abort_flag);
      ok = __syncthreads_and(got && ok);
      if (!ok) break;
    }
    // ---- dequantise the tile into the swizzled bf16 KV tile
    const int32_t* idx = sIdx + st * kMlaTile;
    if (FP8) {
      const uint8_t* stage = sStage + st * kStageBytes;
#pragma unroll 2
      for (int c = tid; c < kMlaTile * 36; c += kMlaThreads) {
        const int j = c / 36, cc = c - j * 36;
        const int slot = idx[j];
        uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
        if (slot >= 0) {
          const uint4 raw = *reinterpret_cast<const uint4*>(stage + j * kDimK + cc * 16);
          const float sc = a.kv_scale[static_cast<int64_t>(slot) * kKvGroups + (cc >> 3)];
          dequant4(raw.x, sc, o0.x, o0.y);
          dequant4(raw.y, sc, o0.z, o0.w);
          dequant4(raw.z, sc, o1.x, o1.y);
          dequant4(raw.w, sc, o1.z, o1.w);
        }
        uint8_t* blk = sKV + (cc >> 2) * 8192;
        store_swizzled(blk, j, (cc & 3) * 2, o0);
        store_swizzled(blk, j, (cc & 3) * 2 + 1, o1);
      }
    } else {
      for (int c = tid; c < kMlaTile * 72; c += kMlaThreads) {
        const int j = c / 72, cc = c - j * 72;
        const int slot = idx[j];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (slot >= 0) v = *reinterpret_cast<const uint4*>(a.kv + static_cast<int64_t>(slot) * (2 * kDimK) + cc * 16);
        store_swizzled(sKV + (cc >> 3) * 8192, j, cc & 7, v);
      }
    }
    if (warp == 0) {
      const unsigned lo = __ballot_sync(0xffffffffu, idx[lane] >= 0);
      const unsigned hi = __ballot_sync(0xffffffffu, idx[32 + lane] >= 0);
      if (lane == 0) *sVmask = (static_cast<unsigned long long>(hi) << 32) | lo;
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- refill this staging buffer; issue QK
    if (warp == 3 && T + 2 < ntiles) issue_tile(T + 2, st);
    if (T + 2 < ntiles) issued = T + 3;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t q_base = smem_u32(sQ), kv_base = smem_u32(sKV);
#pragma unroll 1
      for (int kc = 0; kc < 9; ++kc)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem_S, sdesc_sw128(q_base + kc * 8192 + ks * 32, 16, 1024),
                  sdesc_sw128(kv_base + kc * 8192 + ks * 32, 16, 1024), idesc_qk, (kc | ks) != 0);
      tc_commit(s_done);
    }

    // ---- softmax: thread h < 64 owns head h (TMEM lane h)
    int need_rescale = 0;
    bool got = true;
    if (warp < 2) {
      got = wait_warp(s_done, T & 1, abort_flag);
      if (got) {
        tc_fence_after();
        const unsigned long long vm = *sVmask;
        const int h = tid;
        float z[64];
        {
          float tmp[32];
          tmem_ld32(tmem_S + (static_cast<uint32_t>(warp * 32) << 16), tmp);
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = tmp[i];
          tmem_ld32(tmem_S + (static_cast<uint32_t>(warp * 32) << 16) + 32, tmp);
#pragma unroll
          for (int i = 0; i < 32; ++i) z[32 + i] = tmp[i];
        }
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          z[i] = ((vm >> i) & 1ull) ? z[i] * a.scale_log2 : -INFINITY;
          mt = fmaxf(mt, z[i]);
        }
        float alpha = 1.0f;
        if (m_run == -INFINITY) {
          m_run = mt;                       // first tile with a valid key (O is still zero)
        } else if (mt > m_run + 8.0f) {
          alpha = exp2f(m_run - mt);
          l_run *= alpha;
          m_run = mt;
          need_rescale = 1;
        }
        sAlpha[h] = alpha;
        float lsum = 0.0f;
        uint8_t* prow = sP + h * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = m_run == -INFINITY ? 0.0f : exp2f(z[8 * c + 2 * e] - m_run);
            const float p1 = m_run == -INFINITY ? 0.0f : exp2f(z[8 * c + 2 * e + 1] - m_run);
            const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
            const float2 pr = __bfloat1622float2(pb);   // the weights PV will use
            lsum += pr.x + pr.y;
            w[e] = *reinterpret_cast<const uint32_t*>(&pb);
          }
          *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_run += lsum;
        fence_proxy_async_smem();
      }
    }
    tc_fence_before();
    const int any_rescale = __syncthreads_or(need_rescale);
    ok = __syncthreads_and(got && ok);
    if (!ok) break;

    // ---- rare: rescale O^T columns by alpha[head]
    if (any_rescale) {
      tc_fence_after();
      const uint32_t lane_base = tmem_O + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
      for (int d = 0; d < 4; ++d)
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float v[32];
          const uint32_t addr = lane_base + d * 64 + half * 32;
          tmem_ld32(addr, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= sAlpha[half * 32 + i];
          tmem_st32(addr, v);
        }
      tc_fence_before();
      __syncthreads();
    }

    // ---- PV
    if (tid == 0) {
      tc_fence_after();
      const uint32_t kv_base = smem_u32(sKV), p_base = smem_u32(sP);
#pragma unroll
      for (int d = 0; d < 4; ++d)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_f16(tmem_O + d * 64, sdesc_sw128(kv_base + (2 * d) * 8192 + ks * 2048, 8192, 1024),
                  sdesc_sw128(p_base + ks * 32, 16, 1024), idesc_pv, (T > 0 || ks > 0) ? 1u : 0u);
      tc_commit(o_done);
    }
    got = wait_warp(o_done, T & 1, abort_flag);
    tc_fence_after();
    ok = __syncthreads_and(got && ok);
    if (!ok) break;
  }

  if (!ok) {
    if (tid == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 4);
      *abort_flag = 1;
      // let this CTA's in-flight work land (bounded): its MMAs and its row copies
      tc_commit(drain);
      bounded_wait(drain, 0);
      if (FP8)
        for (int t = T; t < issued; ++t) bounded_wait(&stage_full[t & 1], (t >> 1) & 1);
    }
    __syncthreads();
  } else {
    // ---- epilogue
    const bool split_out = a.nsplit > 1;
    if (tid < kHeads) {
      const float l = l_run;
      sInvL[tid] = l > 0.0f ? 1.0f / l : 0.0f;
      if (split_out) {
        float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + tid) * 2;
        ml[0] = l > 0.0f ? m_run : -INFINITY;
        ml[1] = l;
      } else if (a.lse != nullptr) {
        a.lse[static_cast<int64_t>(q) * kHeads + tid] =
            l > 0.0f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
    __syncthreads();
    const int dim_in_tile = warp * 32 + lane;
#pragma unroll 1
    for (int d = 0; d < 4; ++d) {
      const int dim = d * 128 + dim_in_tile;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float v[32];
        if (ntiles > 0) {
          tmem_ld32(tmem_O + (static_cast<uint32_t>(warp * 32) << 16) + d * 64 + half * 32, v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        }
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const int h = half * 32 + i;
          if (split_out) {
            a.part_o[((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * kDimV + dim] = v[i];
          } else {
            const float o = v[i] * sInvL[h];
            const int64_t off = (static_cast<int64_t>(q) * kHeads + h) * kDimV + dim;
            if (a.out_fp32) static_cast<float*>(a.out)[off] = o;
            else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(o);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kMlaTmemCols);
}

// Log-sum-exp merge of the split partials: M = max_s m_s, a_s = 2^(m_s - M),
// out = sum_s a_s o_s / sum_s a_s l_s, lse = (M + log2 sum_s a_s l_s) * ln 2.
__global__ void __launch_bounds__(128) mla_combine_kernel(const MlaArgs a) {
  const int q = blockIdx.x;
  const int h = blockIdx.y;
  const int S = a.nsplit;
  const float* ml = a.part_ml + static_cast<int64_t>(q) * S * kHeads * 2;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, ml[(s * kHeads + h) * 2]);
  float Lsum = 0.0f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < S; ++s) {
    const float m = ml[(s * kHeads + h) * 2];
    if (m == -INFINITY) continue;
    const float w = exp2f(m - M);
    Lsum += w * ml[(s * kHeads + h) * 2 + 1];
    const float* o = a.part_o + ((static_cast<int64_t>(q) * S + s) * kHeads + h) * kDimV;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] += w * o[threadIdx.x + 128 * i];
  }
  const float inv = Lsum > 0.0f ? 1.0f / Lsum : 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t off = (static_cast<int64_t>(q) * kHeads + h) * kDimV + threadIdx.x + 128 * i;
    const float o = acc[i] * inv;
    if (a.out_fp32) static_cast<float*>(a.out)[off] = o;
    else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(o);
  }
  if (threadIdx.x == 0 && a.lse != nullptr)
    a.lse[static_cast<int64_t>(q) * kHeads + h] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

template <bool FP8>
static cudaError_t launch_mla_t(const CUtensorMap& tq, const MlaArgs& a, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMlaSmem);
  if (e != cudaSuccess) return e;
  mla_decode_kernel<FP8><<<a.Bq * a.nsplit, kMlaThreads, kMlaSmem, stream>>>(tq, a);
  return cudaGetLastError();
}

cudaError_t launch_mla(bool fp8, const CUtensorMap& tmap_q, const MlaArgs& a, cudaStream_t stream, int* launches) {
  cudaError_t e = fp8 ? launch_mla_t<true>(tmap_q, a, stream) : launch_mla_t<false>(tmap_q, a, stream);
  ++*launches;
  if (e != cudaSuccess || a.nsplit == 1) return e;
  mla_combine_kernel<<<dim3(a.Bq, kHeads), 128, 0, stream>>>(a);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace dsa
