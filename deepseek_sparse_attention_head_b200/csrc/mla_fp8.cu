// Stage 3 of the DSA decode step for an fp8 latent cache: MLA sparse decode ("GLM-52 Runs
// on RTX 4090", kernel list item 3) over rows of 576 E4M3 codes (512 latent + 64 rope
// columns, "Show HN: colibri", features) with one fp32 scale per 128-column group and one
// for the rope columns. For query q, head h and its selected rows j:
//
//   z[h, j] = scale * sum_g s_g[j] <q[h, cols g], code[j, cols g]>
//   out[h, d] = sum_j softmax_j(z) s_g(d)[j] code[j, d]            (d < 512)
//
// Design (sm_100a), one CTA per (query, KV split), 12 warps:
//   warps 2-3  producers: cp.async (16-byte, L2-only) gathers of the selected fp8 rows
//              straight into a 3-stage ring of 64-row tiles, 128-byte swizzled (the rope
//              columns 64-byte swizzled), plus the rows' scales; zero-fill for unused
//              slots. No register staging, no conversion: the rows stay E4M3.
//   warp 0     tcgen05 issuer (kind::f8f6f4, fp32 accumulators in TMEM):
//                QK: S_g = Q2 K_g^T per scale group g (M = 128 stacked query rows,
//                    N = 64 rows of the tile), each group into one of four 64-column
//                    TMEM slots so the softmax warps apply s_g[j] per column;
//                PV: O_g^T += V_g^T P_g^T per 128-column value group (M = 128 value
//                    columns read MN-major from the same tile, N = 64 heads), the scale
//                    s_g[j] folded into P_g.
//              Issue order QK(0), QK(1), PV(0), QK(2), PV(1), ... keeps the tensor pipe on
//              the next tile's QK while the softmax warps finish the current one.
//   warps 4-11 softmax: two warps per TMEM lane quadrant, each on 32 of the tile's 64
//              rows. They reduce the five group slots to logits, keep a lazy running
//              maximum per head (rescaling O in TMEM only when a tile's maximum exceeds it
//              by more than 3 log2 units), and write P_g = p * s_g * 2^(5 - E_g) as two
//              E4M3 terms (hi + lo residual, about 8 significant bits together).
// Queries: Q2 stacks, for every head h, row 2h = e4m3(Q'_h) and row 2h+1 = e4m3(Q'_h -
// row 2h), with Q'_h = Q_h * 2^F_h a power-of-two rescale of the bf16 query into
// [128, 256), so the two rows together carry about as many significant bits as bf16.
// Value-group exponents E_g (one per 128 value columns, shared by all heads of the CTA)
// keep P_g below 256 and therefore inside E4M3's range; a tile whose scales outgrow
// 2^E_g rescales that O block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {
namespace {

constexpr int kTile = 64;
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kMmaWarp = 0;
constexpr int kProdWarp0 = 2;                  // producers: warps 2, 3 (rows 0-31, 32-63)
constexpr int kEpiWarp0 = 4;                   // softmax: warps 4 .. 11
constexpr int kEpiThreads = 256;
constexpr int kGroups = 5;                     // four 128-column latent groups + rope
constexpr uint32_t kTmemCols = 512;            // S slots: cols [0, 256); O^T: cols [256, 512)
constexpr uint32_t kTmemO = 256;
constexpr int kNoExp = -100000;
constexpr float kLazy = 3.0f;                  // rescale threshold of the running max (log2 units)
constexpr int kPShift = 5;                     // P_g = p * s_g * 2^(kPShift - E_g) < 2^3 * 2^5

// shared memory (offsets from a 1024-aligned base)
constexpr int kQChunk = 128 * 128;             // 128 stacked query rows x 128 B (one group)
constexpr int kQBytes = 4 * kQChunk + 128 * 64;   // + rope: 128 rows x 64 B
constexpr int kKvChunk = kTile * 128;          // 64 rows x 128 B
constexpr int kStageBytes = 4 * kKvChunk + kTile * 64;
constexpr int kPGroup = 64 * 128;              // 64 heads x (64 hi bytes | 64 lo bytes)
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffP = kOffStage + kStages * kStageBytes;
constexpr int kOffScale = kOffP + 4 * kPGroup;                 // [stage][group][row] fp32
constexpr int kOffMask = kOffScale + kStages * kGroups * kTile * 4;   // [stage][2] row-validity words
constexpr int kOffXch = kOffMask + 64;                         // [parity][half][head] tile maxima
constexpr int kOffGx = kOffXch + 2 * 2 * 64 * 4;               // [parity][half][group] scale maxima
constexpr int kOffHead = kOffGx + 2 * 2 * 4 * 4;               // cq[64], alpha[64]
constexpr int kOffL = kOffHead + 2 * 64 * 4;                   // [half][head][8]: l, then L_g (g < 4)
constexpr int kOffInv = kOffL + 2 * 64 * 8 * 4;                // [parity][group][row] 1 / s_g
constexpr int kOffBars = kOffInv + 2 * 4 * kTile * 4;
constexpr int kOffMisc = kOffBars + 256;
constexpr int kSmem = kOffMisc + 64 + 1024;

static_assert(kOffStage % 1024 == 0 && kStageBytes % 1024 == 0 && kOffP % 1024 == 0, "alignment");
static_assert(kSmem <= 232448, "shared memory");

// barrier indices
constexpr int kBarQReady = 0;
constexpr int kBarKvFull = 1;      // [3]
constexpr int kBarKvEmpty = 4;     // [3]
constexpr int kBarSFull = 7;       // [4]
constexpr int kBarSEmpty = 11;     // [4]
constexpr int kBarPFull = 15;
constexpr int kBarPvDone = 16;
constexpr int kBarDrain = 17;
constexpr int kBarNever = 18;      // test hook only: nothing ever arrives on it
constexpr int kProdArrivals = 64 + 2;   // 64 cp.async completions + 2 mask-word arrivals

__device__ __forceinline__ uint32_t sw128(int row, int unit) {
  return static_cast<uint32_t>(row * 128 + ((unit ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint32_t sw64(int row, int unit) {
  return static_cast<uint32_t>(row * 64 + ((unit ^ ((row >> 1) & 3)) << 4));
}

// Sixteen consecutive query columns (two uint4 of bf16) -> the 16-byte e4m3 words of the
// hi row and of the lo row, after scaling by the exact power of two `sc`.
__device__ __forceinline__ void split_hi_lo16(const uint4& a, const uint4& b, float sc, uint4& hi, uint4& lo) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t h[4] = {0, 0, 0, 0}, l[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    const float x0 = f.x * sc, x1 = f.y * sc;
    const __nv_fp8x2_storage_t h2 = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
    const __half2_raw hb = __nv_cvt_fp8x2_to_halfraw2(h2, __NV_E4M3);
    const float2 back = __half22float2(*reinterpret_cast<const __half2*>(&hb));
    const __nv_fp8x2_storage_t l2 =
        __nv_cvt_float2_to_fp8x2(make_float2(x0 - back.x, x1 - back.y), __NV_SATFINITE, __NV_E4M3);
    h[j >> 1] |= static_cast<uint32_t>(h2) << (16 * (j & 1));
    l[j >> 1] |= static_cast<uint32_t>(l2) << (16 * (j & 1));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Two values -> (hi, lo) e4m3 pairs with hi + lo ~ x (the residual is formed in fp16,
// exactly: both terms lie on x's fp16 grid). Returns hi + lo, the values the tensor core
// will actually multiply.
__device__ __forceinline__ float2 split_pair(float x0, float x1, uint32_t& hi2, uint32_t& lo2) {
  const __half2 xh = __floats2half2_rn(x0, x1);
  const __nv_fp8x2_storage_t h = __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&xh),
                                                             __NV_SATFINITE, __NV_E4M3);
  const __half2_raw hb = __nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3);
  const __half2 r = __hsub2(xh, *reinterpret_cast<const __half2*>(&hb));
  const __nv_fp8x2_storage_t l = __nv_cvt_halfraw2_to_fp8x2(*reinterpret_cast<const __half2_raw*>(&r),
                                                             __NV_SATFINITE, __NV_E4M3);
  const __half2_raw lb = __nv_cvt_fp8x2_to_halfraw2(l, __NV_E4M3);
  hi2 = h;
  lo2 = l;
  return __half22float2(__hadd2(*reinterpret_cast<const __half2*>(&hb), *reinterpret_cast<const __half2*>(&lb)));
}

__global__ void __launch_bounds__(kThreads, 1) mla_fp8_kernel(const MlaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sStage = smem + kOffStage;
  uint8_t* sP = smem + kOffP;
  float* sScale = reinterpret_cast<float*>(smem + kOffScale);
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + kOffMask);
  float* sXch = reinterpret_cast<float*>(smem + kOffXch);
  float* sGx = reinterpret_cast<float*>(smem + kOffGx);
  float* sCq = reinterpret_cast<float*>(smem + kOffHead);
  float* sAlpha = sCq + 64;
  float* sL = reinterpret_cast<float*>(smem + kOffL);
  float* sInv = reinterpret_cast<float*>(smem + kOffInv);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int q = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int k0 = split * a.keys_per_split;
  const int k1 = min(a.top_k, k0 + a.keys_per_split);
  const int nkeys = max(0, k1 - k0);
  const int ntiles = (nkeys + kTile - 1) / kTile;
  const bool split_out = a.nsplit > 1;
  const long long limit = a.wait_limit;

  if (tid == 0) {
    mbar_init(&bars[kBarQReady], 8);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bars[kBarKvFull + i], kProdArrivals);
      mbar_init(&bars[kBarKvEmpty + i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars[kBarSFull + i], 1);
      mbar_init(&bars[kBarSEmpty + i], 8);
    }
    mbar_init(&bars[kBarPFull], 8);
    mbar_init(&bars[kBarPvDone], 1);
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarNever], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (ntiles > 0 && warp >= kEpiWarp0) {
    // ================================================================ softmax warps
    const int et = tid - kEpiWarp0 * 32;
    const int quad = warp & 3;                 // TMEM lanes 32 quad .. 32 quad + 31
    const int half = (warp - kEpiWarp0) >> 2;  // this warp's 32 rows of every tile
    const int h = quad * 16 + (lane >> 1);     // head of this lane's stacked query row
    const int par = lane & 1;                  // 0: hi row, 1: lo row
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    bool good = true;
    // a failed wait raises the abort flag at once, so the other roles stop waiting too
    auto wait_or_abort = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool ok = wait_warp(bar, parity, abort_flag, limit);
      if (!ok && lane == 0) *abort_flag = 1;
      return ok;
    };

    // ---- Q: bf16 [64, 576] -> stacked e4m3 hi / lo rows (four threads per head)
    {
      const int qh = et >> 2, part = et & 3;    // columns [144 part, 144 part + 144)
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.q) +
                                                        (static_cast<int64_t>(q) * kHeads + qh) * kDimK * 2) + part * 18;
      uint4 v[18];
#pragma unroll
      for (int i = 0; i < 18; ++i) v[i] = __ldg(src + i);
      float mx = 0.0f;
#pragma unroll
      for (int i = 0; i < 18; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const int F = mx > 0.0f ? 7 - float_exponent(mx) : 0;   // |Q * 2^F| < 256
      const float sc = exp2i(F);
      if (part == 0) sCq[qh] = a.scale_log2 * exp2i(-F);
#pragma unroll
      for (int u = 0; u < 9; ++u) {
        uint4 hi, lo;
        split_hi_lo16(v[2 * u], v[2 * u + 1], sc, hi, lo);
        const int c0 = part * 144 + 16 * u;
        const int r0 = 2 * qh, r1 = 2 * qh + 1;
        uint8_t *p0, *p1;
        if (c0 < 512) {
          uint8_t* chunk = sQ + (c0 >> 7) * kQChunk;
          p0 = chunk + sw128(r0, (c0 & 127) >> 4);
          p1 = chunk + sw128(r1, (c0 & 127) >> 4);
        } else {
          uint8_t* rope = sQ + 4 * kQChunk;
          p0 = rope + sw64(r0, (c0 - 512) >> 4);
          p1 = rope + sw64(r1, (c0 - 512) >> 4);
        }
        *reinterpret_cast<uint4*>(p0) = hi;
        *reinterpret_cast<uint4*>(p1) = lo;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQReady]);
    }
    pdl_trigger();
    pdl_wait();   // outputs may still be read by the previous kernel of the stream
    if (a.stall) {
      // test hook: a wait that nothing satisfies; it runs out after `limit` cycles
      good = wait_or_abort(&bars[kBarNever], 0);
    }
    good = bar_and(1, kEpiThreads, good) != 0;   // also publishes sCq
    const float cq = sCq[h];

    float m_run = -INFINITY;                    // running max, log2 units (same in the head's 4 threads)
    float lsum = 0.0f;                          // sum of p over this thread's keys
    // per value group: sum over this thread's keys of the weight PV applies, in units of p
    // ((hi + lo) / (s_g 2^(kPShift - E_g))); each group is normalised by its own sum
    float Lg[4] = {0.f, 0.f, 0.f, 0.f};
    int Eg[4] = {kNoExp, kNoExp, kNoExp, kNoExp};   // value-group exponents (same in every thread)
    // Every softmax thread runs the same sequence of named barriers: a failed wait only
    // clears `good`, and the loop is left right after a barrier that made `good` uniform.
    for (int n = 0; n < ntiles; ++n) {
      const int s = n % kStages;
      const float* scl = sScale + s * kGroups * kTile;
      if (good) good = wait_or_abort(&bars[kBarKvFull + s], (n / kStages) & 1);
      // ---- logits of this warp half's 32 rows for this lane's stacked query row
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
      float gm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        const int i5 = kGroups * n + g, slot = i5 & 3;
        if (good) good = wait_or_abort(&bars[kBarSFull + slot], (i5 >> 2) & 1);
        float d[32];
        if (good) {
          tc_fence_after();
          tmem_ld32(tmem + lane_base + slot * 64 + 32 * half, d);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarSEmpty + slot]);
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 s4 = *reinterpret_cast<const float4*>(scl + g * kTile + 32 * half + j);
            acc[j + 0] = fmaf(s4.x, d[j + 0], acc[j + 0]);
            acc[j + 1] = fmaf(s4.y, d[j + 1], acc[j + 1]);
            acc[j + 2] = fmaf(s4.z, d[j + 2], acc[j + 2]);
            acc[j + 3] = fmaf(s4.w, d[j + 3], acc[j + 3]);
            if (g < 4) gm[g] = fmaxf(gm[g], fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w)));
          }
        }
      }
      // hi row + lo row of head h: this lane keeps 16 of the 32 rows
      float z[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float mine = par ? acc[16 + i] : acc[i];
        const float give = par ? acc[i] : acc[16 + i];
        z[i] = mine + __shfl_xor_sync(0xffffffffu, give, 1);
      }
      const uint32_t vm = (sMask[s * 2 + half] >> (16 * par)) & 0xFFFFu;
      float tmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        z[i] = ((vm >> i) & 1u) ? z[i] * cq : -INFINITY;
        tmax = fmaxf(tmax, z[i]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      float* xch = sXch + (n & 1) * 128;
      float* gx = sGx + (n & 1) * 8;
      if (par == 0) xch[half * 64 + h] = tmax;
      if (quad == 0 && lane == 0) {
#pragma unroll
        for (int g = 0; g < 4; ++g) gx[half * 4 + g] = gm[g];
      }
      good = bar_and(1, kEpiThreads, good) != 0;
      if (!good) break;
      const float m_tile = fmaxf(tmax, xch[(1 - half) * 64 + h]);
      const bool any_valid = (sMask[s * 2] | sMask[s * 2 + 1]) != 0u;
      float alpha = 1.0f;
      float beta[4] = {1.f, 1.f, 1.f, 1.f};
      int need = 0;
      if (any_valid) {
        if (m_run == -INFINITY) {
          m_run = m_tile;                       // nothing weighted yet: no rescale
        } else if (m_tile > m_run + kLazy) {
          alpha = ex2_ftz(m_run - m_tile);
          m_run = m_tile;
          lsum *= alpha;
#pragma unroll
          for (int g = 0; g < 4; ++g) Lg[g] *= alpha;
          need = 1;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float mxg = fmaxf(gm[g], gx[(1 - half) * 4 + g]);
          if (mxg > 0.0f) {
            int e = float_exponent(mxg) + 1;     // every scale of the tile lies below 2^e
            e = e < -100 ? -100 : (e > 100 ? 100 : e);
            if (Eg[g] == kNoExp) {
              Eg[g] = e;
            } else if (e > Eg[g]) {
              beta[g] = exp2i(Eg[g] - e);
              Eg[g] = e;
              need = 1;
            }
          }
        }
      }
      if (par == 0 && half == 0) sAlpha[h] = alpha;
      {
        // 1 / s_g of every row of the tile, one per softmax thread, for the normalisers
        const float sv = scl[(et >> 6) * kTile + (et & 63)];
        sInv[(n & 1) * 4 * kTile + et] = sv > 0.0f ? 1.0f / sv : 0.0f;
      }
      need = bar_or(1, kEpiThreads, need);
      bool pv_prev_done = n == 0;
      if (need) {
        // rescale O^T (lanes = value columns, columns = heads) once PV(n-1) has finished
        bool got = wait_or_abort(&bars[kBarPvDone], (n - 1) & 1);
        if (got) {
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            float v[32];
            const uint32_t addr = tmem + lane_base + kTmemO + 64 * g + 32 * half;
            tmem_ld32(addr, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= sAlpha[32 * half + i] * beta[g];
            tmem_st32(addr, v);
          }
          tc_fence_before();
        }
        good = bar_and(1, kEpiThreads, got) != 0;
        if (!good) break;
        pv_prev_done = true;
      }
      // ---- p = 2^(z - m), P_g = p * s_g * 2^(kPShift - E_g) as e4m3 hi + lo
      const float mm = m_run == -INFINITY ? 0.0f : m_run;
      float p[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        p[i] = ex2_ftz(z[i] - mm);
        lsum += p[i];
      }
      if (!pv_prev_done) {
        good = wait_or_abort(&bars[kBarPvDone], (n - 1) & 1);   // P buffer free
        tc_fence_after();
      }
      if (!good) continue;                     // the next barrier (tile or epilogue) stops every warp
      const int k16 = 32 * half + 16 * par;   // first of this lane's 16 rows
      const float* inv = sInv + (n & 1) * 4 * kTile;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float cg = Eg[g] == kNoExp ? 1.0f : exp2i(kPShift - Eg[g]);
        const float icg = Eg[g] == kNoExp ? 1.0f : exp2i(Eg[g] - kPShift);
        uint32_t hw[4], lw[4];
        float lg = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 s4 = *reinterpret_cast<const float4*>(scl + g * kTile + k16 + 4 * j);
          const float4 i4 = *reinterpret_cast<const float4*>(inv + g * kTile + k16 + 4 * j);
          uint32_t h0, l0, h1, l1;
          const float2 q0 = split_pair(p[4 * j + 0] * s4.x * cg, p[4 * j + 1] * s4.y * cg, h0, l0);
          const float2 q1 = split_pair(p[4 * j + 2] * s4.z * cg, p[4 * j + 3] * s4.w * cg, h1, l1);
          lg = fmaf(q0.x, i4.x, fmaf(q0.y, i4.y, fmaf(q1.x, i4.z, fmaf(q1.y, i4.w, lg))));
          hw[j] = h0 | (h1 << 16);
          lw[j] = l0 | (l1 << 16);
        }
        Lg[g] = fmaf(lg, icg, Lg[g]);
        uint8_t* prow = sP + g * kPGroup + h * 128;
        const int u = 2 * half + par;
        *reinterpret_cast<uint4*>(prow + ((u ^ (h & 7)) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(prow + (((4 + u) ^ (h & 7)) << 4)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarPFull]);
    }
    good = bar_and(1, kEpiThreads, good) != 0;

    // ---- epilogue: per-head normalisers, then O^T out of TMEM
    float l_head = lsum + __shfl_xor_sync(0xffffffffu, lsum, 1);
#pragma unroll
    for (int g = 0; g < 4; ++g) Lg[g] += __shfl_xor_sync(0xffffffffu, Lg[g], 1);
    if (good) {
      if (par == 0) {
        float* d = sL + (half * 64 + h) * 8;
        d[0] = l_head;
#pragma unroll
        for (int g = 0; g < 4; ++g) d[1 + g] = Lg[g];
      }
      good = bar_and(1, kEpiThreads, good) != 0;
    }
    if (good) {
      l_head = sL[h * 8] + sL[(64 + h) * 8];
      if (par == 0 && half == 0) {
        if (split_out) {
          float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * kPartStats;
          ml[0] = l_head > 0.0f ? m_run : -INFINITY;
          ml[1] = l_head;
#pragma unroll
          for (int g = 0; g < 4; ++g) ml[2 + g] = sL[h * 8 + 1 + g] + sL[(64 + h) * 8 + 1 + g];
        } else if (a.lse != nullptr) {
          a.lse[static_cast<int64_t>(q) * kHeads + h] =
              l_head > 0.0f ? (m_run + log2f(l_head)) * 0.69314718055994531f : -INFINITY;
        }
      }
      const int last = ntiles - 1;
      const bool got = wait_or_abort(&bars[kBarPvDone], last & 1);
      good = bar_and(1, kEpiThreads, got) != 0;
      if (good) {
        tc_fence_after();
        // this thread: value columns 128 g + 32 quad + lane, heads 32 half .. 32 half + 31
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float v[32];
          tmem_ld32(tmem + lane_base + kTmemO + 64 * g + 32 * half, v);
          const float og = Eg[g] == kNoExp ? 1.0f : exp2i(Eg[g] - kPShift);
          const int dim = 128 * g + 32 * quad + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int hh = 32 * half + i;
            float inv = 1.0f;
            if (!split_out) {
              const float L = sL[hh * 8 + 1 + g] + sL[(64 + hh) * 8 + 1 + g];
              inv = L > 0.0f ? 1.0f / L : 0.0f;
            }
            const float o = v[i] * og * inv;
            if (split_out) {
              a.part_o[((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + hh) * kDimV + dim] = o;
            } else {
              const int64_t off = (static_cast<int64_t>(q) * kHeads + hh) * kDimV + dim;
              if (a.out_fp32) static_cast<float*>(a.out)[off] = o;
              else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(o);
            }
          }
        }
      }
    }
    if (!good) {
      if (split_out && par == 0 && half == 0) {
        // an empty partial, so the combine skips this split instead of reading stale data
        float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * kPartStats;
        ml[0] = -INFINITY;
#pragma unroll
        for (int i = 1; i < kPartStats; ++i) ml[i] = 0.0f;
      }
      if (lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 23);
        *abort_flag = 1;
      }
    }
    __syncwarp();
  } else if (ntiles > 0 && warp == kMmaWarp) {
    // ================================================================ tcgen05 issuer
    pdl_trigger();
    const uint32_t idesc_qk = idesc_make(0, 0, false, false, 128, kTile);
    const uint32_t idesc_pv = idesc_make(0, 0, true, false, 128, 64);
    const uint32_t q0 = smem_u32(sQ);
    const uint64_t pd0 = sdesc_sw128(smem_u32(sP), 16, 1024);
    bool good = wait_warp(&bars[kBarQReady], 0, abort_flag, limit);
    tc_fence_after();
    auto issue_pv = [&](int n) -> bool {
      if (!wait_warp(&bars[kBarPFull], n & 1, abort_flag, limit)) return false;
      tc_fence_after();
      const uint32_t sb = smem_u32(sStage + (n % kStages) * kStageBytes);
      if (elect_one()) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint64_t vd = sdesc_sw128(sb + g * kKvChunk, kKvChunk, 1024);   // MN-major V^T
          const uint64_t pd = pd0 + static_cast<uint64_t>((g * kPGroup) >> 4);
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t va = vd + static_cast<uint64_t>((ks * 32 * 128) >> 4);
            mma_f8(tmem + kTmemO + 64 * g, va, pd + static_cast<uint64_t>((ks * 32) >> 4), idesc_pv,
                   (n > 0 || ks > 0) ? 1u : 0u);
            mma_f8(tmem + kTmemO + 64 * g, va, pd + static_cast<uint64_t>((64 + ks * 32) >> 4), idesc_pv, 1u);
          }
        }
        tc_commit(&bars[kBarPvDone]);
        tc_commit(&bars[kBarKvEmpty + n % kStages]);
      }
      __syncwarp();
      return true;
    };
    for (int n = 0; n < ntiles && good; ++n) {
      const int s = n % kStages;
      if (!wait_warp(&bars[kBarKvFull + s], (n / kStages) & 1, abort_flag, limit)) { good = false; break; }
      fence_proxy_async_smem();   // cp.async data (generic proxy) -> tensor-core reads
      tc_fence_after();
      const uint32_t sb = smem_u32(sStage + s * kStageBytes);
#pragma unroll 1
      for (int g = 0; g < kGroups; ++g) {
        const int i5 = kGroups * n + g, slot = i5 & 3;
        if (!wait_warp(&bars[kBarSEmpty + slot], ((i5 >> 2) & 1) ^ 1, abort_flag, limit)) { good = false; break; }
        tc_fence_after();
        if (elect_one()) {
          const uint64_t kd = g < 4 ? sdesc_sw128(sb + g * kKvChunk, 16, 1024) : sdesc_sw64(sb + 4 * kKvChunk, 16, 512);
          const uint64_t qd = g < 4 ? sdesc_sw128(q0 + g * kQChunk, 16, 1024) : sdesc_sw64(q0 + 4 * kQChunk, 16, 512);
          const int nks = g < 4 ? 4 : 2;   // K = 32 columns per MMA
          for (int ks = 0; ks < nks; ++ks)
            mma_f8(tmem + slot * 64, qd + static_cast<uint64_t>(2 * ks), kd + static_cast<uint64_t>(2 * ks),
                   idesc_qk, ks > 0 ? 1u : 0u);
          tc_commit(&bars[kBarSFull + slot]);
        }
        __syncwarp();
      }
      if (!good) break;
      if (n > 0 && !issue_pv(n - 1)) { good = false; break; }
    }
    if (good && !issue_pv(ntiles - 1)) good = false;
    if (!good && lane == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 20);
      *abort_flag = 1;
    }
    // every MMA this warp issued has finished before the CTA frees TMEM
    if (elect_one()) {
      tc_commit(&bars[kBarDrain]);
      wait_drain(&bars[kBarDrain], 0);
    }
    __syncwarp();
  } else if (ntiles > 0 && (warp == kProdWarp0 || warp == kProdWarp0 + 1)) {
    // ================================================================ producers
    pdl_trigger();
    pdl_wait();   // the slot list comes from top-k
    const int pw = warp - kProdWarp0;
    const int32_t* phys = a.physical + static_cast<int64_t>(q) * a.top_k + k0;
    const uint32_t stage0 = smem_u32(sStage);
    bool good = true;
    for (int n = 0; n < ntiles; ++n) {
      const int s = n % kStages;
      if (n >= kStages) {
        if (!wait_warp(&bars[kBarKvEmpty + s], ((n / kStages) - 1) & 1, abort_flag, limit)) { good = false; break; }
        fence_proxy_async_smem();   // tensor-core reads of the stage before these writes
      }
      const int ki = n * kTile + 32 * pw + lane;
      int slot = ki < nkeys ? phys[ki] : -1;
      if (slot < -1 || slot >= a.num_slots) {
        record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(slot));
        slot = -1;
      }
      const unsigned vm = __ballot_sync(0xffffffffu, slot >= 0);
      const uint32_t sb = stage0 + s * kStageBytes;
      // this warp's 32 rows x 36 sixteen-byte pieces; consecutive lanes take consecutive pieces
#pragma unroll 4
      for (int i = 0; i < 36; ++i) {
        const int p = lane + 32 * i;
        const int r = p / 36, u = p - r * 36;
        const int sl = __shfl_sync(0xffffffffu, slot, r);
        const int R = 32 * pw + r;
        const uint32_t dst = u < 32 ? sb + (u >> 3) * kKvChunk + sw128(R, u & 7) : sb + 4 * kKvChunk + sw64(R, u - 32);
        cp_async16(dst, a.kv + static_cast<int64_t>(max(sl, 0)) * kDimK + u * 16, sl >= 0 ? 16u : 0u);
      }
      const uint32_t sc = smem_u32(sScale + s * kGroups * kTile + 32 * pw + lane);
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
        cp_async4(sc + g * kTile * 4, a.kv_scale + static_cast<int64_t>(max(slot, 0)) * kKvGroups + g,
                  slot >= 0 ? 4u : 0u);
      if (lane == 0) sMask[s * 2 + pw] = vm;
      cp_async_arrive(&bars[kBarKvFull + s]);
      if (lane == 0) mbar_arrive(&bars[kBarKvFull + s]);
    }
    cp_async_wait_all();   // no copy may land after the CTA has exited
    if (!good && lane == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 22);
      *abort_flag = 1;
    }
    __syncwarp();
  } else {
    pdl_trigger();
  }

  if (ntiles == 0) {
    // nothing selected: zero output (or an empty partial)
    pdl_wait();
    for (int i = tid; i < kHeads * kDimV; i += kThreads) {
      const int hh = i / kDimV, dim = i % kDimV;
      if (split_out) {
        a.part_o[((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + hh) * kDimV + dim] = 0.0f;
      } else {
        const int64_t off = (static_cast<int64_t>(q) * kHeads + hh) * kDimV + dim;
        if (a.out_fp32) static_cast<float*>(a.out)[off] = 0.0f;
        else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(0.0f);
      }
    }
    if (tid < kHeads) {
      if (split_out) {
        float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + tid) * kPartStats;
        ml[0] = -INFINITY;
#pragma unroll
        for (int i = 1; i < kPartStats; ++i) ml[i] = 0.0f;
      } else if (a.lse != nullptr) {
        a.lse[static_cast<int64_t>(q) * kHeads + tid] = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_mla_fp8(const MlaArgs& a, cudaStream_t stream) {
  cudaError_t e = set_smem_once<mla_fp8_kernel>(kSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_fp8_kernel, dim3(a.Bq * a.nsplit), dim3(kThreads), kSmem, stream, a);
}

}  // namespace dsa
