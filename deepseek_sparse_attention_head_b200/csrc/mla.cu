// Stage 3 of the DSA decode step: MLA sparse decode ("GLM-52 Runs on RTX 4090", kernel
// list item 3). For query q, head h and its selected latent rows j:
//
//   z[h, j] = scale * <q[h, 0:576], KV[slot_j, 0:576]>,  out[h, :] = sum_j softmax_j(z) KV[slot_j, 0:512]
//
// (576 = 512 latent + 64 rope columns; "Show HN: colibri", features.)
//
// Design (sm_100a): grid = (query, split); a CTA walks 32-row tiles of its share of
// the index list with warp-specialised, double-buffered stages:
//   warp 1    producer: the tile's slot ids, one 576-byte bulk async copy per fp8 row
//             into a 3-deep ring, and the row's five scales folded into an exact
//             power-of-two row exponent E_j plus five fp16 multipliers s_g / 2^E_j;
//   warps 2-3 dequantisers: fp8 code -> fp16 (exact) x multiplier -> fp16 tile,
//             128-byte swizzled; the tile is the K operand of QK (K-major) and the
//             V operand of PV (MN-major) at once;
//   warp 0    tcgen05 issuer:  S = Q' K'^T (M=128, rows 64..127 unused, N=32),
//             O^T += V'^T P'^T (4 x M=128, N=64); fp32 accumulators in TMEM;
//   warps 4-5 softmax, one thread per head (its TMEM lane): running max with lazy
//             rescaling (only when a tile's max exceeds it by more than 8 in log2
//             units), exact fp32 normaliser, fp16 weights P' = p * 2^(E_j - E_ref);
//   warps 4-7 the rare O rescale and the output epilogue (all 128 TMEM lanes).
// Q is staged once per CTA and rescaled per head by a power of two into fp16. With
// a bf16 cache the same pipeline runs in bf16 without any rescaling.
// Splits write (m, l, o) partials that mla_combine_kernel merges by log-sum-exp.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {

constexpr int kMlaTile = 32;
constexpr int kMlaThreads = 256;
constexpr int kMlaStages = 3;
constexpr uint32_t kMlaTmemCols = 512;        // S[2]: cols [0,64); O^T: cols [64, 320)
constexpr int kRowBytes = kDimK;              // fp8 row
constexpr int kStageRows = kMlaTile * kRowBytes;
constexpr int kNoExp = -100000;               // "no valid row seen yet"

// shared-memory map (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;                                        // 9 x [64 x 128 B]
constexpr int kOffStage = kOffQ + 9 * 8192;                     // 3 x [32 x 576 B]
constexpr int kOffStageMeta = kOffStage + kMlaStages * kStageRows;
constexpr int kStageMetaBytes = 1024;                           // mult[32][5] u32, E[32], slot[32]
constexpr int kOffKV = kOffStageMeta + kMlaStages * kStageMetaBytes;   // 2 x 9 x [32 x 128 B]
constexpr int kKVChunk = kMlaTile * 128;
constexpr int kKVBytes = 9 * kKVChunk;
constexpr int kOffP = kOffKV + 2 * kKVBytes;                    // [64 heads x 128 B]; tile parity picks the half
constexpr int kOffKVMeta = kOffP + 8192;                        // 2 x (E[32], vmask)
constexpr int kOffHead = kOffKVMeta + 512;                      // cq[64], alpha[64], outscale[64]
constexpr int kOffIdxList = kOffHead + 768;                     // the split's slot list (<= 2048 entries)
constexpr int kIdxListCap = 2048;
constexpr int kOffBars = kOffIdxList + kIdxListCap * 4;
constexpr int kOffMisc = kOffBars + 256;
constexpr int kMlaSmem = kOffMisc + 64 + 1024;

static_assert(kOffKV % 1024 == 0 && kOffP % 1024 == 0 && kOffStage % 16 == 0, "alignment");
static_assert(kMlaSmem <= 232448, "shared memory");

// OR / AND over the 128 threads of warps 4..7 (named barrier 1).
__device__ __forceinline__ int group_or(int v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return static_cast<int>(r);
}
__device__ __forceinline__ int group_and(int v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return static_cast<int>(r);
}

__device__ __forceinline__ uint32_t swz(int row, int unit) {  // 128-byte swizzle inside an 8-row atom
  return static_cast<uint32_t>(row * 128 + ((unit ^ (row & 7)) << 4));
}

__device__ __forceinline__ int float_exponent(float s) {  // floor(log2 s) for positive normal s
  return static_cast<int>((__float_as_uint(s) >> 23) & 0xFF) - 127;
}

__device__ __forceinline__ float exp2i(int e) {  // exact 2^e, clamped to the normal fp32 range
  e = e < -126 ? -126 : (e > 127 ? 127 : e);
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// Four E4M3 codes -> four fp16 (exact) times the fp16 multiplier pair m2.
__device__ __forceinline__ void dequant4_f16(uint32_t w, __half2 m2, uint32_t& o0, uint32_t& o1) {
  const __half2_raw r01 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw r23 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w >> 16), __NV_E4M3);
  __half2 h01 = __hmul2(*reinterpret_cast<const __half2*>(&r01), m2);
  __half2 h23 = __hmul2(*reinterpret_cast<const __half2*>(&r23), m2);
  o0 = *reinterpret_cast<uint32_t*>(&h01);
  o1 = *reinterpret_cast<uint32_t*>(&h23);
}

template <bool FP8>
__global__ void __launch_bounds__(kMlaThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const MlaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sStage = smem + kOffStage;
  uint8_t* sStageMeta = smem + kOffStageMeta;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  int32_t* sKVMeta = reinterpret_cast<int32_t*>(smem + kOffKVMeta);
  float* sCq = reinterpret_cast<float*>(smem + kOffHead);
  float* sAlpha = sCq + 64;
  float* sOutScale = sCq + 128;
  int32_t* sIdxList = reinterpret_cast<int32_t*>(smem + kOffIdxList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* q_full = bars + 0;
  uint64_t* stage_full = bars + 1;    // [3]
  uint64_t* stage_empty = bars + 4;   // [3]
  uint64_t* kv_full = bars + 7;       // [2]
  uint64_t* s_full = bars + 9;        // [2]
  uint64_t* s_empty = bars + 11;      // [2]
  uint64_t* p_full = bars + 13;       // [2]
  uint64_t* pv_done = bars + 15;      // [2]
  uint64_t* drain = bars + 17;
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
  const int ntiles = (nkeys + kMlaTile - 1) / kMlaTile;
  const int32_t* phys = a.physical + static_cast<int64_t>(q) * a.top_k;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kMlaStages; ++i) {
      mbar_init(&stage_full[i], 1);
      mbar_init(&stage_empty[i], 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 2);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 2);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
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
  const uint32_t tmem_O = tmem + 64;

  // the split's slot list, staged once (invalid entries become -1)
  const bool list_in_smem = nkeys <= kIdxListCap;
  if (list_in_smem) {
    for (int i = tid; i < ntiles * kMlaTile; i += kMlaThreads) {
      int slot = i < nkeys ? phys[k0 + i] : -1;
      if (slot < -1 || slot >= a.num_slots) {
        record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(slot));
        slot = -1;
      }
      sIdxList[i] = slot;
    }
  }

  // ---------------------------------------------------------------- Q: load, rescale per head
  bool ok = true;
  if (ntiles > 0) {
    if (tid == 0) {
      tma_prefetch_map(&tmap_q);
      mbar_arrive_expect_tx(q_full, 9u * 8192u);
      for (int c = 0; c < 9; ++c) tma_load_2d(sQ + c * 8192, &tmap_q, c * 64, q * kHeads, q_full);
    }
    ok = wait_warp(q_full, 0, abort_flag);
    const int h = tid >> 2, part = tid & 3;   // 4 threads per head, 18 of its 72 16-byte units each
    int F = 0;
    if (FP8 && ok) {
      float mx = 0.0f;
      for (int u = part * 18; u < part * 18 + 18; ++u) {
        const uint4 v = *reinterpret_cast<const uint4*>(sQ + (u >> 3) * 8192 + swz(h, u & 7));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      F = mx > 0.0f ? float_exponent(mx) : 0;
      const float inv = exp2i(-F);
      for (int u = part * 18; u < part * 18 + 18; ++u) {
        uint4* p = reinterpret_cast<uint4*>(sQ + (u >> 3) * 8192 + swz(h, u & 7));
        const uint4 v = *p;
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
          __half2 hh = __floats2half2_rn(f.x * inv, f.y * inv);
          w[i] = *reinterpret_cast<uint32_t*>(&hh);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    if (part == 0) sCq[h] = a.scale_log2 * exp2i(F);
    fence_proxy_async_smem();
  }
  ok = __syncthreads_and(ok) != 0;

  // fp16 operands for an fp8 cache, bf16 for a bf16 cache
  const uint32_t fmt = FP8 ? 0u : 1u;
  const uint32_t idesc_qk = idesc_make(fmt, fmt, false, false, 128, kMlaTile);
  const uint32_t idesc_pv = idesc_make(fmt, fmt, true, false, 128, 64);

  if (ok && ntiles > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------ tcgen05 issuer (whole warp)
      // Descriptors are formed once and advanced by constants; MMAs and commits come from
      // one elected lane of the converged warp.
      bool good = true;
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kv_desc0 = sdesc_sw128(smem_u32(sKV), 16, 1024);                 // K-major view
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(sKV), kKVChunk, 1024);            // MN-major view
      const uint64_t p_desc0 = sdesc_sw128(smem_u32(sP), 16, 1024);
      auto issue_pv = [&](int T) {
        const int b = T & 1;
        if (!wait_warp(&p_full[b], (T >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t vb = v_desc0 + static_cast<uint64_t>((b * kKVBytes) >> 4);
        const uint64_t pb = p_desc0 + static_cast<uint64_t>((b * 64) >> 4);
        if (elect_one()) {
#pragma unroll
          for (int d = 0; d < 4; ++d)
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
              mma_f16(tmem_O + d * 64, vb + static_cast<uint64_t>(((2 * d) * kKVChunk + ks * 2048) >> 4),
                      pb + static_cast<uint64_t>((ks * 32) >> 4), idesc_pv, (T > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&pv_done[b]);
        }
        __syncwarp();
        return true;
      };
      for (int T = 0; T < ntiles; ++T) {
        const int b = T & 1;
        if (!wait_warp(&kv_full[b], (T >> 1) & 1, abort_flag)) { good = false; break; }
        if (!wait_warp(&s_empty[b], ((T >> 1) & 1) ^ 1, abort_flag)) { good = false; break; }
        tc_fence_after();
        const uint64_t kb = kv_desc0 + static_cast<uint64_t>((b * kKVBytes) >> 4);
        if (elect_one()) {
#pragma unroll 3
          for (int kc = 0; kc < 9; ++kc)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_f16(tmem + b * 32, q_desc0 + static_cast<uint64_t>((kc * 8192 + ks * 32) >> 4),
                      kb + static_cast<uint64_t>((kc * kKVChunk + ks * 32) >> 4), idesc_qk, (kc | ks) != 0);
          tc_commit(&s_full[b]);
        }
        __syncwarp();
        if (T >= 1 && !issue_pv(T - 1)) { good = false; break; }
      }
      if (good && !issue_pv(ntiles - 1)) good = false;
      if (!good && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 10);
        *abort_flag = 1;
      }
      if (elect_one()) {
        tc_commit(drain);
        wait_drain(drain, 0);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ producer
      // Lane j owns row j of every tile. Its slot comes from the staged list; its five
      // scales are loaded two tiles ahead into registers, so no global load sits on the
      // per-tile path.
      auto slot_of = [&](int T) {
        const int i = T * kMlaTile + lane;
        if (T >= ntiles) return -1;
        if (list_in_smem) return static_cast<int>(sIdxList[i]);
        int slot = i < nkeys ? phys[k0 + i] : -1;
        if (slot < -1 || slot >= a.num_slots) {
          record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(slot));
          slot = -1;
        }
        return slot;
      };
      float sc_a[kKvGroups], sc_b[kKvGroups];   // scales of tiles T and T+1
      auto load_scales = [&](int slot, float (&sc)[kKvGroups]) {
#pragma unroll
        for (int g = 0; g < kKvGroups; ++g)
          sc[g] = (FP8 && slot >= 0) ? a.kv_scale[static_cast<int64_t>(slot) * kKvGroups + g] : 0.0f;
      };
      int slot_a = slot_of(0), slot_b = slot_of(1);
      load_scales(slot_a, sc_a);
      load_scales(slot_b, sc_b);
      bool good = true;
      for (int T = 0; T < ntiles; ++T) {
        const int st = T % kMlaStages;
        if (!wait_warp(&stage_empty[st], ((T / kMlaStages) & 1) ^ 1, abort_flag)) { good = false; break; }
        uint8_t* meta = sStageMeta + st * kStageMetaBytes;
        uint32_t* mult = reinterpret_cast<uint32_t*>(meta);            // [32][5]
        int32_t* E = reinterpret_cast<int32_t*>(meta + 640);           // [32]
        int32_t* slots = reinterpret_cast<int32_t*>(meta + 768);       // [32]
        const int slot = slot_a;
        if (FP8 && slot >= 0)
          bulk_load(sStage + st * kStageRows + lane * kRowBytes, a.kv + static_cast<int64_t>(slot) * kRowBytes,
                    kRowBytes, &stage_full[st]);
        int Ej = 0;
        if (FP8) {
          float smax = 0.0f;
#pragma unroll
          for (int g = 0; g < kKvGroups; ++g) smax = fmaxf(smax, sc_a[g]);
          Ej = smax > 0.0f ? float_exponent(smax) : 0;
          const float inv = exp2i(-Ej);
#pragma unroll
          for (int g = 0; g < kKvGroups; ++g) {
            const __half2 m2 = __float2half2_rn(sc_a[g] * inv);
            mult[lane * kKvGroups + g] = *reinterpret_cast<const uint32_t*>(&m2);
          }
        }
        E[lane] = Ej;
        slots[lane] = slot;
        const unsigned vm = __ballot_sync(0xffffffffu, slot >= 0);
        __syncwarp();
        if (lane == 0) mbar_arrive_expect_tx(&stage_full[st], FP8 ? __popc(vm) * kRowBytes : 0u);
        // rotate the two-tile lookahead
        slot_a = slot_b;
#pragma unroll
        for (int g = 0; g < kKvGroups; ++g) sc_a[g] = sc_b[g];
        slot_b = slot_of(T + 2);
        load_scales(slot_b, sc_b);
      }
      if (!good && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 11);
        *abort_flag = 1;
      }
      // bounded drain of this warp's outstanding row copies
      if (lane == 0 && FP8)
        for (int T = max(0, ntiles - kMlaStages); T < ntiles; ++T)
          wait_drain(&stage_full[T % kMlaStages], (T / kMlaStages) & 1);
      __syncwarp();
    } else if (warp == 2 || warp == 3) {
      // ------------------------------------------------------------ dequantisers
      const int ct = tid - 64;   // 0..63
      bool good = true;
      for (int T = 0; T < ntiles; ++T) {
        const int st = T % kMlaStages, b = T & 1;
        if (!wait_warp(&stage_full[st], (T / kMlaStages) & 1, abort_flag)) { good = false; break; }
        if (T >= 2 && !wait_warp(&pv_done[b], ((T >> 1) & 1) ^ 1, abort_flag)) { good = false; break; }
        const uint8_t* meta = sStageMeta + st * kStageMetaBytes;
        const uint32_t* mult = reinterpret_cast<const uint32_t*>(meta);
        const int32_t* slots = reinterpret_cast<const int32_t*>(meta + 768);
        uint8_t* kv = sKV + b * kKVBytes;
        if (FP8) {
          const uint8_t* rows = sStage + st * kStageRows;
#pragma unroll 3
          for (int c = ct; c < kMlaTile * 36; c += 64) {
            const int j = c / 36, cc = c - j * 36;
            uint4 o0 = make_uint4(0, 0, 0, 0), o1 = make_uint4(0, 0, 0, 0);
            if (slots[j] >= 0) {
              const uint4 raw = *reinterpret_cast<const uint4*>(rows + j * kRowBytes + cc * 16);
              const uint32_t mw = mult[j * kKvGroups + (cc >> 3)];
              const __half2 m2 = *reinterpret_cast<const __half2*>(&mw);
              dequant4_f16(raw.x, m2, o0.x, o0.y);
              dequant4_f16(raw.y, m2, o0.z, o0.w);
              dequant4_f16(raw.z, m2, o1.x, o1.y);
              dequant4_f16(raw.w, m2, o1.z, o1.w);
            }
            uint8_t* blk = kv + (cc >> 2) * kKVChunk;
            *reinterpret_cast<uint4*>(blk + swz(j, (cc & 3) * 2)) = o0;
            *reinterpret_cast<uint4*>(blk + swz(j, (cc & 3) * 2 + 1)) = o1;
          }
        } else {
          for (int c = ct; c < kMlaTile * 72; c += 64) {
            const int j = c / 72, cc = c - j * 72;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (slots[j] >= 0)
              v = *reinterpret_cast<const uint4*>(a.kv + static_cast<int64_t>(slots[j]) * (2 * kDimK) + cc * 16);
            *reinterpret_cast<uint4*>(kv + (cc >> 3) * kKVChunk + swz(j, cc & 7)) = v;
          }
        }
        if (warp == 2) {   // row exponents and validity of this tile, for the softmax warps
          const int32_t* E = reinterpret_cast<const int32_t*>(meta + 640);
          int32_t* km = sKVMeta + b * 64;
          km[lane] = E[lane];
          const unsigned vm = __ballot_sync(0xffffffffu, slots[lane] >= 0);
          if (lane == 0) km[32] = static_cast<int32_t>(vm);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&kv_full[b]);
          mbar_arrive(&stage_empty[st]);
        }
      }
      if (!good && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 12);
        *abort_flag = 1;
      }
      __syncwarp();
    } else {
      // ------------------------------------------------------------ softmax group (warps 4..7)
      const bool is_sm = warp < 6;            // warps 4,5: heads 0..63 = TMEM lanes 0..63
      const int quarter = warp & 3;           // TMEM lane quarter this warp may access
      const int h = (warp - 4) * 32 + lane;   // head (meaningful for warps 4,5)
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      float m_run = -INFINITY, l_run = 0.0f, cq = 0.0f;
      int e_ref = kNoExp;                     // running max of the rows' exponents (same in every thread)
      if (is_sm) cq = sCq[h];
      bool good = true;
      for (int T = 0; T < ntiles; ++T) {
        const int b = T & 1;
        float y[kMlaTile];
        int need = 0;
        if (is_sm) {
          const bool got = wait_warp(&s_full[b], (T >> 1) & 1, abort_flag) &&
                           wait_warp(&kv_full[b], (T >> 1) & 1, abort_flag);
          if (got) {
            tc_fence_after();
            tmem_ld32(tmem + lane_base + b * 32, y);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[b]);
            const int32_t* km = sKVMeta + b * 64;
            const unsigned vm = static_cast<unsigned>(km[32]);
            float ymax = -INFINITY;
            int etile = kNoExp;
#pragma unroll
            for (int j = 0; j < kMlaTile; ++j) {
              const bool v = (vm >> j) & 1u;
              y[j] = v ? y[j] * cq * exp2i(km[j]) : -INFINITY;
              ymax = fmaxf(ymax, y[j]);
              if (v) etile = max(etile, km[j]);
            }
            float alpha = 1.0f;
            if (vm != 0u) {
              if (m_run == -INFINITY) {
                m_run = ymax;                       // first tile with a valid row: nothing accumulated yet
              } else if (ymax > m_run + 8.0f) {
                alpha = exp2f(m_run - ymax);
                l_run *= alpha;
                m_run = ymax;
              }
              if (e_ref == kNoExp) {
                e_ref = etile;
              } else if (etile > e_ref) {
                alpha *= exp2i(e_ref - etile);
                e_ref = etile;
              }
            }
            sAlpha[h] = alpha;
            need = alpha != 1.0f ? 1 : 0;
          } else {
            good = false;
          }
        }
        need = group_or(need);
        good = group_and(good) != 0;
        if (!good) break;
        if (need) {
          // rescale the O^T columns (heads) by alpha; PV(T-1) must have finished first
          const bool got = wait_warp(&pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, abort_flag);
          if (got) {
            tc_fence_after();
#pragma unroll 1
            for (int d = 0; d < 4; ++d)
#pragma unroll 1
              for (int half = 0; half < 2; ++half) {
                float v[32];
                const uint32_t addr = tmem_O + lane_base + d * 64 + half * 32;
                tmem_ld32(addr, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= sAlpha[half * 32 + i];
                tmem_st32(addr, v);
              }
          }
          good = group_and(got) != 0;
          if (!good) break;
        }
        if (is_sm) {
          // the P half this tile writes was last read by PV(T-2)
          const bool got = T < 2 || wait_warp(&pv_done[b], ((T >> 1) & 1) ^ 1, abort_flag);
          if (got) {
            const int32_t* km = sKVMeta + b * 64;
            uint8_t* prow = sP + h * 128;
            float lsum = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 8 * c + 2 * e;
                const float p0 = m_run == -INFINITY ? 0.0f : exp2f(y[j] - m_run);
                const float p1 = m_run == -INFINITY ? 0.0f : exp2f(y[j + 1] - m_run);
                lsum += p0 + p1;
                if (FP8) {
                  const float d0 = exp2i(km[j] - e_ref), d1 = exp2i(km[j + 1] - e_ref);
                  __half2 hh = __floats2half2_rn(p0 * d0, p1 * d1);
                  w[e] = *reinterpret_cast<uint32_t*>(&hh);
                } else {
                  __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
                  w[e] = *reinterpret_cast<uint32_t*>(&bb);
                }
              }
              *reinterpret_cast<uint4*>(prow + (((b * 4 + c) ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            l_run += lsum;
            fence_proxy_async_smem();
          } else {
            good = false;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        good = group_and(good) != 0;
        if (!good) break;
      }
      // ---- epilogue: warps 4..7 read O^T (lanes = dims), softmax threads supply per-head scales
      if (good) {
        const bool split_out = a.nsplit > 1;
        if (is_sm) {
          const float l = l_run;
          const float oscale = exp2i(e_ref == kNoExp ? 0 : e_ref);
          sOutScale[h] = split_out ? oscale : (l > 0.0f ? oscale / l : 0.0f);
          if (split_out) {
            float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * 2;
            ml[0] = l > 0.0f ? m_run : -INFINITY;
            ml[1] = l;
          } else if (a.lse != nullptr) {
            a.lse[static_cast<int64_t>(q) * kHeads + h] =
                l > 0.0f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
          }
        }
        const int last = ntiles - 1;
        const bool got = wait_warp(&pv_done[last & 1], (last >> 1) & 1, abort_flag);
        good = group_and(got) != 0;
        if (good) {
          tc_fence_after();
          const int dim_in_tile = quarter * 32 + lane;
#pragma unroll 1
          for (int d = 0; d < 4; ++d) {
            const int dim = d * 128 + dim_in_tile;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              float v[32];
              tmem_ld32(tmem_O + lane_base + d * 64 + half * 32, v);
#pragma unroll 4
              for (int i = 0; i < 32; ++i) {
                const int hh = half * 32 + i;
                const float o = v[i] * sOutScale[hh];
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
      }
      if (!good && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 13);
        *abort_flag = 1;
      }
      __syncwarp();
    }
  }

  if (ntiles == 0) {
    // nothing selected: zero output (or an empty partial)
    const bool split_out = a.nsplit > 1;
    for (int i = tid; i < kHeads * kDimV; i += kMlaThreads) {
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
        float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + tid) * 2;
        ml[0] = -INFINITY;
        ml[1] = 0.0f;
      } else if (a.lse != nullptr) {
        a.lse[static_cast<int64_t>(q) * kHeads + tid] = -INFINITY;
      }
    }
  }
  if (!ok && tid == 0) {
    record_error(a.err, DSA_ERR_TIMEOUT, 14);
    wait_drain(q_full, 0);   // the Q copy may still be landing
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

int mla_tile_keys() { return kMlaTile; }

}  // namespace dsa
