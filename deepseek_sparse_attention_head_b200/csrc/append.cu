// The step before the DSA decode path, for each query's new token: partial interleaved
// RoPE ("Show HN: colibri", features: MLA attention with partial interleaved RoPE) on the
// 64 rope columns of the projected indexer query (the first 64 of each head's 128), the
// indexer key (the first 64 of 128) and the latent row (the last 64 of 576); E4M3
// quantisation with amax/448 fp32 scales (one per (query, head), one per key, one per
// 128-column latent group); and the key and latent rows written into the paged caches at
// the token's slot. The absorbed MLA query's rope columns are rotated in place as well.
//
// One CTA of 256 threads per new token. Pair i of the rope columns turns by
// pos * base^(-2i/64): the frequencies come from the host in fp64, each angle is formed and
// reduced to [-pi, pi] in fp64 (positions reach 1M), and its cosine and sine are taken in
// fp32 from there, like every later step of the rotation.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {
namespace {

constexpr int kAppThreads = 256;
constexpr int kRopePairs = 32;

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
}

__device__ __forceinline__ uint32_t float2_to_bf16x2(float x, float y) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__device__ __forceinline__ uint8_t e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ void rotate(float& x, float& y, float c, float s) {
  const float a = x * c - y * s;
  const float b = x * s + y * c;
  x = a;
  y = b;
}

__global__ void __launch_bounds__(kAppThreads) rope_quantize_append_kernel(const AppendArgs a) {
  __shared__ float cs[kRopePairs], sn[kRopePairs];
  __shared__ unsigned int gmax[6];            // latent group amax bits (5), key amax (1)
  __shared__ float kmax_w[2];
  const int q = blockIdx.x;
  const int t = threadIdx.x;
  const int b = q / a.n_q;
  pdl_trigger();
  pdl_wait();

  // ---- every row this thread reads, issued before the position -> page lookup so that the
  // loads and that dependent pair of reads overlap
  int pos = a.q_pos != nullptr ? a.q_pos[q] : a.seq_lens[b] - 1;
  const int h = t >> 2, part = t & 3;
  uint4 qw[4];
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.idx_q + (static_cast<int64_t>(q) * kHeads + h) * kDimIdx +
                                                      32 * part);
#pragma unroll
    for (int i = 0; i < 4; ++i) qw[i] = src[i];
  }
  const uint32_t kw = t < 64 ? reinterpret_cast<const uint32_t*>(a.idx_k + static_cast<int64_t>(q) * kDimIdx)[t] : 0u;
  uint32_t lw[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int p = t + kAppThreads * k;
    lw[k] = p < kDimK / 2 ? reinterpret_cast<const uint32_t*>(a.latent + static_cast<int64_t>(q) * kDimK)[p] : 0u;
  }
  uint32_t mw[8];
  if (a.q_mla != nullptr) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int j = t + kAppThreads * k;          // (head, pair)
      mw[k] = reinterpret_cast<const uint32_t*>(a.q_mla + (static_cast<int64_t>(q) * kHeads + (j >> 5)) * kDimK +
                                                kDimV)[j & 31];
    }
  }

  // ---- the token's position and slot (no cache write when either is out of range)
  int page = -1;
  if (pos < 0 || pos >= a.max_pages * kPage) {
    if (t == 0) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(pos));
    pos = 0;
  } else {
    page = a.block_table[static_cast<int64_t>(b) * a.max_pages + (pos >> 6)];
    if (page < 0 || page >= a.num_pages) {
      if (t == 0) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(page));
      page = -1;
    }
  }
  const int64_t slot = page >= 0 ? static_cast<int64_t>(page) * kPage + (pos & 63) : -1;

  if (t < kRopePairs) {
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    const double ang = static_cast<double>(pos) * a.theta[t];
    const float r = static_cast<float>(ang - rint(ang / kTwoPi) * kTwoPi);
    float s, c;
    sincosf(r, &s, &c);
    cs[t] = c;
    sn[t] = s;
  }
  if (t < 6) gmax[t] = 0u;
  __syncthreads();

  // ---- indexer query: four threads per head, 32 columns each (columns < 64 rotate)
  {
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 w = qw[i];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = bf16x2_to_float2(ws[j]);
        v[8 * i + 2 * j] = f.x;
        v[8 * i + 2 * j + 1] = f.y;
      }
    }
    if (part < 2) {
#pragma unroll
      for (int j = 0; j < 16; ++j) rotate(v[2 * j], v[2 * j + 1], cs[16 * part + j], sn[16 * part + j]);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      c[i] = static_cast<uint32_t>(e4m3(v[4 * i] / scale)) | (static_cast<uint32_t>(e4m3(v[4 * i + 1] / scale)) << 8) |
             (static_cast<uint32_t>(e4m3(v[4 * i + 2] / scale)) << 16) |
             (static_cast<uint32_t>(e4m3(v[4 * i + 3] / scale)) << 24);
    uint4* dst = reinterpret_cast<uint4*>(a.q_out + (static_cast<int64_t>(q) * kHeads + h) * kDimIdx + 32 * part);
    dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
    dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
    if (part == 0) a.q_scale_out[static_cast<int64_t>(q) * kHeads + h] = scale;
  }

  // ---- indexer key: threads 0..63, one column pair each (pairs < 32 rotate)
  float kx = 0.0f, ky = 0.0f;
  if (t < 64) {
    const float2 f = bf16x2_to_float2(kw);
    kx = f.x;
    ky = f.y;
    if (t < kRopePairs) rotate(kx, ky, cs[t], sn[t]);
    float m = fmaxf(fabsf(kx), fabsf(ky));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0) kmax_w[t >> 5] = m;
  }

  // ---- latent row: pairs p = t and t + 256 (p < 288); pairs >= 256 are the rope columns
  float lx[2] = {0.0f, 0.0f}, ly[2] = {0.0f, 0.0f};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int p = t + kAppThreads * k;
    if (p < kDimK / 2) {
      const float2 f = bf16x2_to_float2(lw[k]);
      lx[k] = f.x;
      ly[k] = f.y;
      if (p >= kDimV / 2) rotate(lx[k], ly[k], cs[p - kDimV / 2], sn[p - kDimV / 2]);
      atomicMax(&gmax[min(2 * p / 128, 4)], __float_as_uint(fmaxf(fabsf(lx[k]), fabsf(ly[k]))));
    }
  }

  // ---- the absorbed MLA query's rope columns, in place
  if (a.q_mla != nullptr) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int j = t + kAppThreads * k;          // (head, pair)
      const int h = j >> 5, i = j & 31;
      uint32_t* w = reinterpret_cast<uint32_t*>(a.q_mla + (static_cast<int64_t>(q) * kHeads + h) * kDimK + kDimV) + i;
      const float2 f = bf16x2_to_float2(mw[k]);
      float x = f.x, y = f.y;
      rotate(x, y, cs[i], sn[i]);
      *w = float2_to_bf16x2(x, y);
    }
  }
  __syncthreads();

  // ---- write the key and the latent row at the token's slot
  if (slot < 0) return;
  if (t < 64) {
    const float m = fmaxf(kmax_w[0], kmax_w[1]);
    const float scale = m > 0.0f ? m / 448.0f : 1.0f;
    const uint32_t c2 = static_cast<uint32_t>(e4m3(kx / scale)) | (static_cast<uint32_t>(e4m3(ky / scale)) << 8);
    reinterpret_cast<uint16_t*>(a.k_cache + slot * kDimIdx)[t] = static_cast<uint16_t>(c2);
    if (t == 0) a.k_scale[slot] = scale;
  }
  float gscale[5];
#pragma unroll
  for (int g = 0; g < 5; ++g) {
    const float m = __uint_as_float(gmax[g]);
    gscale[g] = m > 0.0f ? m / 448.0f : 1.0f;
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int p = t + kAppThreads * k;
    if (p >= kDimK / 2) continue;
    const int g = min(2 * p / 128, 4);
    if (a.kvf == kKvBf16) {
      reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(a.kv_cache) + slot * kDimK)[p] = float2_to_bf16x2(lx[k], ly[k]);
    } else if (a.kvf == kKvFp8) {
      const uint32_t c2 =
          static_cast<uint32_t>(e4m3(lx[k] / gscale[g])) | (static_cast<uint32_t>(e4m3(ly[k] / gscale[g])) << 8);
      reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(a.kv_cache) + slot * kDimK)[p] = static_cast<uint16_t>(c2);
    } else {
      uint8_t* row = static_cast<uint8_t*>(a.kv_cache) + slot * kPackedRowBytes;
      if (g < 4) {
        const uint32_t c2 =
            static_cast<uint32_t>(e4m3(lx[k] / gscale[g])) | (static_cast<uint32_t>(e4m3(ly[k] / gscale[g])) << 8);
        reinterpret_cast<uint16_t*>(row)[p] = static_cast<uint16_t>(c2);
      } else {
        reinterpret_cast<uint32_t*>(row + kDimV + 16)[p - kDimV / 2] = float2_to_bf16x2(lx[k], ly[k]);
      }
    }
  }
  if (t < 5) {
    if (a.kvf == kKvFp8) a.kv_scale[slot * kKvGroups + t] = gscale[t];
    else if (a.kvf == kKvFp8Packed && t < 4)
      reinterpret_cast<float*>(static_cast<uint8_t*>(a.kv_cache) + slot * kPackedRowBytes + kDimV)[t] = gscale[t];
  }
}

}  // namespace

cudaError_t launch_rope_quantize_append(const AppendArgs& a, int Bq, cudaStream_t stream, int* launches) {
  ++*launches;
  return launch_pdl(rope_quantize_append_kernel, dim3(Bq), dim3(kAppThreads), 0, stream, a);
}

}  // namespace dsa
