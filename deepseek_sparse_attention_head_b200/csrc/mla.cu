// Stage 3 of the DSA decode step: MLA sparse decode ("GLM-52 Runs on RTX 4090", kernel
// list item 3). For query q, head h and its selected latent rows j:
//
//   z[h, j] = scale * <q[h, 0:576], KV[slot_j, 0:576]>,  out[h, :] = sum_j softmax_j(z) KV[slot_j, 0:512]
//
// (576 = 512 latent + 64 rope columns; "Show HN: colibri", features.)
//
// Design (sm_100a): grid = (query, split); a CTA walks 64-row tiles of its share of the
// index list through two tile buffers, with warp-specialised roles:
//   warps 5.. loaders (8, or 12 for the fp8 cache with a scale plane), all on every tile,
//   tiles alternating between the two buffers.
//             Each thread keeps 9 sixteen-byte pieces of each of the next two tiles in
//             flight (plain global loads issued two tiles ahead), then turns fp8 codes into
//             fp16 (exact) x a per-row multiplier s_g / 2^E_j and stores them 128-byte
//             swizzled: the tile is the K operand of QK (K-major) and the V operand of PV
//             (MN-major) at once. E_j is the row's power-of-two exponent.
//   warp 4    tcgen05 issuer: S = Q' K'^T (M=64 heads, N=64 keys),
//             O^T += V'^T P'^T (4 x M=128 dims, N=64 heads); fp32 accumulators in TMEM.
//             Issue order QK(t), QK(t+1), PV(t), PV(t+1) lets one buffer refill while the
//             other tile's MMAs run.
//   warps 0-3 softmax, one thread per head (M=64 puts head h in TMEM lane
//             32 (h / 16) + h % 16, so each warp owns 16 heads): running max with lazy
//             rescaling (only when a tile's max exceeds it by more than 8 in log2 units),
//             exact fp32 normaliser, fp16 weights P' = p * 2^(E_j - E_ref) written into
//             the tile's rope chunk, which QK has finished with.
//   warps 0-3 Q rescale at the start, the rare O rescale and the output epilogue.
// Q is staged once per CTA and rescaled per head by a power of two into fp16. With
// a bf16 cache the same pipeline runs in bf16 without any rescaling.
// Splits write (m, l, o) partials that mla_combine_kernel merges by log-sum-exp.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace dsa {

constexpr int kMlaTile = 64;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp0 = 5;                 // loaders: warps 5 .. 4 + NL (NL = 8 or 12 loader warps)
// Threads of the decode kernel with NL loader warps: 4 softmax warps, the tcgen05 warp, the loaders.
__host__ __device__ constexpr int mla_threads(int nl) { return (kLoadWarp0 + nl) * 32; }
// Loader warps per cache layout: a warp keeps only so many loads in flight, so more loader
// warps pull a tile's rows faster; the 656-byte packed rows divide over 8 only.
__host__ __device__ constexpr int mla_loaders(int kvf) { return kvf != kKvFp8Packed ? 12 : 8; }
constexpr uint32_t kMlaTmemCols = 512;        // S[2]: cols [0,128); O^T: cols [128, 384)
constexpr uint32_t kTmemO = 128;
constexpr int kNoExp = -100000;               // "no valid row seen yet"
constexpr int kKVChunk = kMlaTile * 128;      // one 64-column chunk of a tile
constexpr int kKVBytes = 9 * kKVChunk;
constexpr int kPChunk = 8;                    // the rope chunk, reused for P after QK

// shared-memory map (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;                                        // 9 x [64 x 128 B]
constexpr int kOffKV = kOffQ + 9 * 8192;                        // 2 x 9 x [64 x 128 B]
constexpr int kOffKVMeta = kOffKV + 2 * kKVBytes;               // 2 x per-key tables (KVMeta)
constexpr int kKVMetaBytes = 1152;
constexpr int kOffGrpMeta = kOffKVMeta + 2 * kKVMetaBytes;      // per buffer: mult[64][5] (fp16x2)
constexpr int kGrpMetaBytes = kMlaTile * kKvGroups * 4;
constexpr int kOffHead = kOffGrpMeta + 2 * kGrpMetaBytes;       // cq[64], alpha[64], outscale[64]
constexpr int kOffBars = kOffHead + 768;
constexpr int kOffMisc = kOffBars + 256;
constexpr int kOffIdxList = kOffMisc + 64;                      // the split's slot list
constexpr int kIdxListCap = 1024;
constexpr int kMlaSmem = kOffIdxList + kIdxListCap * 4 + 1024;

static_assert(kOffKV % 1024 == 0 && kKVBytes % 1024 == 0, "alignment");
static_assert(kIdxListCap % kMlaTile == 0, "list capacity");
static_assert(kMlaSmem <= 232448, "shared memory");


__device__ __forceinline__ uint32_t swz(int row, int unit) {  // 128-byte swizzle inside an 8-row atom
  return static_cast<uint32_t>(row * 128 + ((unit ^ (row & 7)) << 4));
}

// Per-key tables of one tile buffer, written by the loaders (row j of the tile):
//   kmul[j] = 2^E_j (0 for an unused row), kadd[j] = 0 (-inf for an unused row),
//   E[j] = the row exponent, emax[w] = max E over the valid rows j in [32w, 32w+32)
//   (kNoExp when none), vmask[w] = validity bits of those rows;
// and by the softmax threads: fac[j] = 2^(E_j - E_ref) (0 for an unused row).
struct KVMeta {
  float kmul[64];
  float kadd[64];
  int32_t E[64];
  float fac[64];
  uint32_t vmask[2];
  int32_t emax[2];
};
static_assert(sizeof(KVMeta) <= 1152, "tile table size");

// Read-only global loads that write their destination only when `pred` holds (it keeps
// the value it had otherwise), so that nothing after the load has to wait for it to
// choose between the loaded value and a default. The gathered rows are used once: they do
// not allocate in L1, which is small next to this kernel's shared memory.
__device__ __forceinline__ void ldg_pred(uint4& v, const void* p, bool pred) {
  asm("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %5, 0;\n\t@q ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}\n"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "l"(p), "r"(static_cast<uint32_t>(pred)));
}
__device__ __forceinline__ void ldg_pred(float& v, const float* p, bool pred) {
  asm("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q ld.global.nc.f32 %0, [%1];\n\t}\n"
      : "+f"(v)
      : "l"(p), "r"(static_cast<uint32_t>(pred)));
}

// Packed 656-byte rows, a tile's pieces p in [0, 2560): p < 2048 is code piece p % 32 of row
// p / 32 (bytes 16 (p % 32)); the rest is rope piece (p - 2048) % 8 of row (p - 2048) / 8
// (bytes 528 + 16 ((p - 2048) % 8)).
constexpr int kPackedCodePieces = kMlaTile * 32;
__device__ __forceinline__ int packed_row(int p) {
  return p < kPackedCodePieces ? p >> 5 : (p - kPackedCodePieces) >> 3;
}
__device__ __forceinline__ int packed_byte(int p) {
  return p < kPackedCodePieces ? 16 * (p & 31) : kDimV + 16 + 16 * ((p - kPackedCodePieces) & 7);
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

// KVF: the latent cache layout, kKvBf16, kKvFp8 (576 E4M3 codes per row + a [rows, 5] fp32
// scale plane) or kKvFp8Packed (656-byte rows: 512 codes, four fp32 scales, 64 bf16 rope).
template <int KVF>
__global__ void __maxnreg__(mla_loaders(KVF) == 12 ? 96 : 128)   // 17 warps: 96 registers fit each sub-partition
    mla_decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const MlaArgs a) {
  constexpr bool FP8 = KVF != kKvBf16;            // fp16 operands from E4M3 codes
  constexpr bool PACKED = KVF == kKvFp8Packed;
  constexpr int NL = mla_loaders(KVF);
  constexpr int kMlaThreads = mla_threads(NL);
  constexpr int kLoadThreads = NL * 32;
  constexpr int kPerQuad = 1 + NL / 4;            // epilogue warps per TMEM lane quadrant
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  KVMeta* sKVMeta = reinterpret_cast<KVMeta*>(smem + kOffKVMeta);
  uint32_t* sGrpMeta = reinterpret_cast<uint32_t*>(smem + kOffGrpMeta);
  float* sCq = reinterpret_cast<float*>(smem + kOffHead);
  float* sAlpha = sCq + 64;
  float* sOutScale = sCq + 128;
  int32_t* sIdxList = reinterpret_cast<int32_t*>(smem + kOffIdxList);
  // Pair merge (a.pair), over the slot list once the tile loop is over: per head the split's
  // running max (log2 units) and sum of p, then the merge factors; kPairGood: the split's O is valid.
  float* sPair = reinterpret_cast<float*>(smem + kOffIdxList);
  constexpr int kPairM = 0, kPairL = 64, kPairMul = 128, kPairInvL = 192, kPairOn = 256, kPairGood = 320;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint64_t* q_full = bars + 0;
  uint64_t* q_ready = bars + 1;
  uint64_t* kv_full = bars + 2;       // [2]
  uint64_t* s_full = bars + 4;        // [2]
  uint64_t* s_empty = bars + 6;       // [2]
  uint64_t* p_full = bars + 8;        // [2]
  uint64_t* pv_done = bars + 10;      // [2]
  uint64_t* drain = bars + 12;
  uint64_t* never = bars + 13;        // test hook only: nothing ever arrives on it
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
    mbar_init(q_ready, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], NL);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, kMlaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (ntiles > 0 && tid == 0) tma_prefetch_map(&tmap_q);

  pdl_trigger();
  // The slot list comes from top-k, and any earlier kernel on the stream may still be
  // writing the queries (the cache append rotates their rope columns in place): nothing
  // from global memory is read before this wait.
  pdl_wait();
  if (ntiles > 0 && tid == 0) {
    mbar_arrive_expect_tx(q_full, 9u * 8192u);
    for (int c = 0; c < 9; ++c) tma_load_2d(sQ + c * 8192, &tmap_q, c * 64, q * kHeads, q_full);
  }

  // the split's slot list, staged once when it fits (invalid entries become -1)
  const bool list_in_smem = ntiles * kMlaTile <= kIdxListCap;
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
  __syncthreads();
  auto slot_at = [&](int T, int row) -> int {
    const int i = T * kMlaTile + row;
    if (list_in_smem) return sIdxList[i];
    int slot = i < nkeys ? phys[k0 + i] : -1;
    if (slot < -1 || slot >= a.num_slots) {
      record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(slot));
      slot = -1;
    }
    return slot;
  };

  // fp16 operands for an fp8 cache, bf16 for a bf16 cache
  const uint32_t fmt = FP8 ? 0u : 1u;

  // Output epilogue, shared by the softmax warps and the loaders once O is final: warp w
  // reads TMEM lanes 32 (w % 4) .. + 31 (value dims), and the three warps of a lane quadrant
  // (r = 0, 1, 2) take every third of its eight 32-head column blocks.
  auto write_out = [&](int r) {
    const bool split_out = a.nsplit > 1;
    const int quad = warp & 3;
    const uint32_t lb = static_cast<uint32_t>(quad * 32) << 16;
    tc_fence_after();
#pragma unroll 1
    for (int k = r; k < 8; k += kPerQuad) {
      const int d = k >> 1, half = k & 1;
      const int dim = d * 128 + quad * 32 + lane;
      float v[32];
      tmem_ld32(tmem + kTmemO + lb + d * 64 + half * 32, v);
#pragma unroll
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
  };
  constexpr int kEpiBar = 3, kEpiThreads = 4 * 32 + kLoadThreads;   // softmax warps + loaders

  if (ntiles > 0 && warp < 4) {
    // ---------------------------------------------------------------- Q rescale, softmax, epilogue
    bool good = wait_warp(q_full, 0, abort_flag, a.wait_limit);
    const bool q_landed = good;
    {
      const int h = tid >> 1, part = tid & 1;   // 2 threads per head, 36 of its 72 16-byte units each
      int F = 0;
      if (FP8 && good) {
        float mx = 0.0f;
        for (int u = part * 36; u < part * 36 + 36; ++u) {
          const uint4 v = *reinterpret_cast<const uint4*>(sQ + (u >> 3) * 8192 + swz(h, u & 7));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
            mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        F = mx > 0.0f ? float_exponent(mx) : 0;
        const float inv = exp2i(-F);
        for (int u = part * 36; u < part * 36 + 36; ++u) {
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
      __syncwarp();
      if (lane == 0) mbar_arrive(q_ready);
    }
    if (a.stall) {
      // test hook: a wait that nothing satisfies; it runs out after a.wait_limit cycles
      good = wait_warp(never, 0, abort_flag, a.wait_limit) && good;
    }
    good = bar_and(1, 128, good) != 0;

    // M=64 puts head h in TMEM lane 32 (h / 16) + h % 16: lanes 0..15 of warp w hold heads
    // 16w .. 16w+15. Lane l < 16 reads keys 0..31 of its head, lane l + 16 keys 32..63 of
    // the same head (one two-range TMEM load); both keep identical running statistics.
    const bool is_sm = lane < 16;           // the lane that writes per-head state
    const int h = warp * 16 + (lane & 15);
    const int jb = lane < 16 ? 0 : 32;      // this lane's keys: jb .. jb+31
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_run = -INFINITY, l_run = 0.0f;
    int e_ref = kNoExp;                     // running max of the rows' exponents (same in every thread)
    const float cq = sCq[h];
    for (int T = 0; T < ntiles && good; ++T) {
      const int b = T & 1;
      KVMeta* km = sKVMeta + b;
      float y[32];
      int need = 0;
      {
        const bool got = wait_warp(&s_full[b], (T >> 1) & 1, abort_flag, a.wait_limit) &&
                         wait_warp(&kv_full[b], (T >> 1) & 1, abort_flag, a.wait_limit);
        if (got) {
          tc_fence_after();
          tmem_ld_16x32bx2_x32(tmem + lane_base + b * kMlaTile, y);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[b]);
          // logits in log2 units: z = acc * cq * 2^E_j, -inf for unused rows
          float ymax = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 mu = *reinterpret_cast<const float4*>(&km->kmul[jb + j]);
            const float4 ad = *reinterpret_cast<const float4*>(&km->kadd[jb + j]);
            y[j + 0] = fmaf(y[j + 0], cq * mu.x, ad.x);
            y[j + 1] = fmaf(y[j + 1], cq * mu.y, ad.y);
            y[j + 2] = fmaf(y[j + 2], cq * mu.z, ad.z);
            y[j + 3] = fmaf(y[j + 3], cq * mu.w, ad.w);
            ymax = fmaxf(fmaxf(ymax, fmaxf(y[j + 0], y[j + 1])), fmaxf(y[j + 2], y[j + 3]));
          }
          ymax = fmaxf(ymax, __shfl_xor_sync(0xffffffffu, ymax, 16));
          const int etile = max(km->emax[0], km->emax[1]);
          float alpha = 1.0f;
          if ((km->vmask[0] | km->vmask[1]) != 0u) {
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
          if (is_sm) {
            // this lane also owns key h of the tile: its P' factor 2^(E_h - E_ref)
            km->fac[h] = km->kadd[h] == 0.0f ? exp2i(km->E[h] - e_ref) : 0.0f;
            sAlpha[h] = alpha;
          }
          need = (is_sm && alpha != 1.0f) ? 1 : 0;
        } else {
          good = false;
        }
      }
      need = bar_or(1, 128, need);
      good = bar_and(1, 128, good) != 0;
      if (!good) break;
      if (need) {
        // rescale the O^T columns (heads) by alpha; PV(T-1) must have finished first
        const bool got = wait_warp(&pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, abort_flag, a.wait_limit);
        if (got) {
          tc_fence_after();
#pragma unroll 1
          for (int d = 0; d < 4; ++d)
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
              float v[32];
              const uint32_t addr = tmem + kTmemO + lane_base + d * 64 + half * 32;
              tmem_ld32(addr, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= sAlpha[half * 32 + i];
              tmem_st32(addr, v);
            }
        }
        good = bar_and(1, 128, got) != 0;
        if (!good) break;
      }
      {
        // p = 2^(z - m) (fp32, summed exactly into l); P' = p * 2^(E_j - E_ref) in the
        // tile's rope chunk (K-major rows of 64 keys per head; this lane writes 32 of them)
        uint8_t* prow = sKV + b * kKVBytes + kPChunk * kKVChunk + h * 128;
        const float mm = m_run == -INFINITY ? 0.0f : m_run;
        float lsum0 = 0.0f, lsum1 = 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 f0 = *reinterpret_cast<const float4*>(&km->fac[jb + 8 * c]);
          const float4 f1 = *reinterpret_cast<const float4*>(&km->fac[jb + 8 * c + 4]);
          const float fa[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 8 * c + 2 * e;
            const float p0 = ex2_ftz(y[j] - mm);
            const float p1 = ex2_ftz(y[j + 1] - mm);
            lsum0 += p0;
            lsum1 += p1;
            if (FP8) {
              __half2 hh = __floats2half2_rn(p0 * fa[2 * e], p1 * fa[2 * e + 1]);
              w[e] = *reinterpret_cast<uint32_t*>(&hh);
            } else {
              __nv_bfloat162 bb = __floats2bfloat162_rn(p0, p1);
              w[e] = *reinterpret_cast<uint32_t*>(&bb);
            }
          }
          const int unit = (jb >> 3) + c;
          *reinterpret_cast<uint4*>(prow + ((unit ^ (h & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_run += lsum0 + lsum1;
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    // the two lanes of a head hold halves of its normaliser
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
    // ---- epilogue: per-head scales and statistics, then O^T out of TMEM with the loaders
    bool got = false;
    if (good) {
      const bool split_out = a.nsplit > 1;
      if (is_sm) {
        const float l = l_run;
        const float oscale = exp2i(e_ref == kNoExp ? 0 : e_ref);
        sOutScale[h] = split_out ? oscale : (l > 0.0f ? oscale / l : 0.0f);
        if (a.pair) {
          sPair[kPairM + h] = l > 0.0f ? m_run : -INFINITY;
          sPair[kPairL + h] = l;
        } else if (split_out) {
          float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * kPartStats;
          ml[0] = l > 0.0f ? m_run : -INFINITY;
#pragma unroll
          for (int i = 1; i < kPartStats; ++i) ml[i] = l;   // every value group shares l here
        } else if (a.lse != nullptr) {
          a.lse[static_cast<int64_t>(q) * kHeads + h] =
              l > 0.0f ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
      }
      const int last = ntiles - 1;
      got = wait_warp(&pv_done[last & 1], (last >> 1) & 1, abort_flag, a.wait_limit);
    }
    // a failure stops the other roles now, not after the loaders' next wait runs out
    if (!(good && got) && lane == 0) *abort_flag = 1;
    // O is final and the scales are published: the loaders join the readout
    good = bar_and(kEpiBar, kEpiThreads, good && got) != 0;
    if (good && !a.pair) write_out(0);
    if (a.pair) {
      if (!good && is_sm) {
        sPair[kPairM + h] = -INFINITY;
        sPair[kPairL + h] = 0.0f;
      }
      if (tid == 0) sPair[kPairGood] = good ? 1.0f : 0.0f;
    } else if (!good && a.nsplit > 1 && is_sm) {
      // an empty partial, so the combine skips this split instead of reading stale data
      float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + h) * kPartStats;
      ml[0] = -INFINITY;
#pragma unroll
      for (int i = 1; i < kPartStats; ++i) ml[i] = 0.0f;
    }
    if (!good && lane == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 13);
      *abort_flag = 1;
    }
    if (!q_landed && tid == 0) wait_drain(q_full, 0, a.wait_limit);   // the Q copy may still be landing
    __syncwarp();
  } else if (ntiles > 0 && warp == kMmaWarp) {
    // ---------------------------------------------------------------- tcgen05 issuer (whole warp)
    // Descriptors are formed once and advanced by constants; MMAs and commits come from
    // one elected lane of the converged warp.
    const uint32_t idesc_qk = idesc_make(fmt, fmt, false, false, 64, kMlaTile);
    const uint32_t idesc_pv = idesc_make(fmt, fmt, true, false, 128, 64);
    const uint64_t q_desc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t kv_desc0 = sdesc_sw128(smem_u32(sKV), 16, 1024);                 // K-major view
    const uint64_t v_desc0 = sdesc_sw128(smem_u32(sKV), kKVChunk, 1024);            // MN-major view
    const uint64_t p_desc0 = sdesc_sw128(smem_u32(sKV + kPChunk * kKVChunk), 16, 1024);
    bool good = wait_warp(q_ready, 0, abort_flag, a.wait_limit);
    tc_fence_after();
    auto issue_pv = [&](int T) {
      const int b = T & 1;
      tc_fence_after();
      const uint64_t vb = v_desc0 + static_cast<uint64_t>((b * kKVBytes) >> 4);
      const uint64_t pb = p_desc0 + static_cast<uint64_t>((b * kKVBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int d = 0; d < 4; ++d)
#pragma unroll
          for (int ks = 0; ks < kMlaTile / 16; ++ks)
            mma_f16(tmem + kTmemO + d * 64, vb + static_cast<uint64_t>(((2 * d) * kKVChunk + ks * 2048) >> 4),
                    pb + static_cast<uint64_t>((ks * 32) >> 4), idesc_pv, (T > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&pv_done[b]);
      }
      __syncwarp();
    };
    auto issue_qk = [&](int T) {
      const int b = T & 1;
      tc_fence_after();
      const uint64_t kb = kv_desc0 + static_cast<uint64_t>((b * kKVBytes) >> 4);
      if (elect_one()) {
#pragma unroll 3
        for (int kc = 0; kc < 9; ++kc)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_f16(tmem + b * kMlaTile, q_desc0 + static_cast<uint64_t>((kc * 8192 + ks * 32) >> 4),
                    kb + static_cast<uint64_t>((kc * kKVChunk + ks * 32) >> 4), idesc_qk, (kc | ks) != 0);
        tc_commit(&s_full[b]);
      }
      __syncwarp();
    };
    // Whichever is ready first: QK of the next tile (its buffer converted, its S slot read
    // by the softmax) or PV of the oldest tile whose weights are written. PV(T) then follows
    // the softmax at once instead of waiting for tile T + 1's conversion, and the loaders,
    // who refill a buffer after its PV, start sooner.
    int nq = 0, np = 0;   // next QK tile, next PV tile (np <= nq)
    long long t_idle = clock64();
    for (uint32_t spin = 0; good && np < ntiles;) {
      if (nq < ntiles && __all_sync(0xffffffffu, mbar_test_wait(&kv_full[nq & 1], (nq >> 1) & 1) &&
                                                     mbar_test_wait(&s_empty[nq & 1], ((nq >> 1) & 1) ^ 1))) {
        issue_qk(nq++);
      } else if (np < nq && __all_sync(0xffffffffu, mbar_test_wait(&p_full[np & 1], (np >> 1) & 1))) {
        issue_pv(np++);
      } else {
        if ((++spin & 255u) == 0u && (*abort_flag || clock64() - t_idle > a.wait_limit)) good = false;
        continue;
      }
      spin = 0;
      t_idle = clock64();
    }
    if (!good && lane == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 10);
      *abort_flag = 1;
    }
    // every MMA this warp issued has finished before the CTA frees TMEM
    if (elect_one()) {
      tc_commit(drain);
      wait_drain(drain, 0);
    }
    __syncwarp();
  } else if (ntiles > 0 && warp >= kLoadWarp0) {
    // ---------------------------------------------------------------- loaders
    // All eight loader warps (two per SM sub-partition, which balances the fp8 -> fp16
    // conversions) work on every tile. Piece p of a tile is 16 bytes of row p / R at column
    // byte (p % R) * 16, R = 36 (fp8) or 72 (bf16) pieces per row; thread t owns pieces
    // t + 256 i. Register sets A and B hold the even and the odd tiles: an fp8 tile is one
    // batch of 9 pieces per thread, loaded two tiles ahead; a bf16 tile is two batches, the
    // second loaded when it is needed.
    const int lt = tid - kLoadWarp0 * 32;
    // Packed rows: a tile's first 2048 pieces are the codes (32 per row, bytes 16 c), the
    // last 512 the bf16 rope (8 per row, bytes 528 + 16 u, past the four scales); thread t
    // owns pieces t + 256 i, so its pieces i < 8 are codes and 8, 9 rope, the same in every
    // lane of a warp.
    constexpr int kRowPieces = PACKED ? 40 : (FP8 ? 36 : 72);
    constexpr int kRowBytes = PACKED ? kPackedRowBytes : (FP8 ? kDimK : 2 * kDimK);
    constexpr int kBatches = FP8 ? 1 : 2;
    constexpr int kPieces = kMlaTile * kRowPieces / (kLoadThreads * kBatches);   // per thread and batch
    static_assert(kLoadThreads * kPieces * kBatches == kMlaTile * kRowPieces, "a tile is whole batches");
    uint4 rawA[kPieces], rawB[kPieces];
    float scA[kKvGroups], scB[kKvGroups];
    int slotA = -1, slotB = -1;   // row lt's slot (threads lt < 64)
    // all slot lookups first, then all loads, so that no lookup waits behind a load
    auto fetch = [&](uint4 (&raw)[kPieces], int T, int batch) {
      int sl[kPieces];
#pragma unroll
      for (int i = 0; i < kPieces; ++i) {
        const int p = lt + kLoadThreads * (batch * kPieces + i);
        sl[i] = slot_at(T, PACKED ? packed_row(p) : p / kRowPieces);
      }
#pragma unroll
      for (int i = 0; i < kPieces; ++i) {
        const int p = lt + kLoadThreads * (batch * kPieces + i);
        const int byte = PACKED ? packed_byte(p) : (p % kRowPieces) * 16;
        raw[i] = make_uint4(0u, 0u, 0u, 0u);
        ldg_pred(raw[i], a.kv + static_cast<int64_t>(max(sl[i], 0)) * kRowBytes + byte, sl[i] >= 0);
      }
    };
    auto fetch_meta = [&](float (&sc)[kKvGroups], int& my_slot, int T) {
      if (lt < kMlaTile) {
        my_slot = slot_at(T, lt);
#pragma unroll
        for (int k = 0; k < kKvGroups; ++k) sc[k] = 0.0f;
        if (PACKED) {
          // the four group scales sit in the row, after its 512 codes; the rope has none
          uint4 s4 = make_uint4(0u, 0u, 0u, 0u);
          ldg_pred(s4, a.kv + static_cast<int64_t>(max(my_slot, 0)) * kRowBytes + kDimV, my_slot >= 0);
          sc[0] = __uint_as_float(s4.x);
          sc[1] = __uint_as_float(s4.y);
          sc[2] = __uint_as_float(s4.z);
          sc[3] = __uint_as_float(s4.w);
        } else if (FP8) {
#pragma unroll
          for (int k = 0; k < kKvGroups; ++k)
            ldg_pred(sc[k], a.kv_scale + static_cast<int64_t>(max(my_slot, 0)) * kKvGroups + k, my_slot >= 0);
        }
      }
    };
    auto store = [&](const uint4 (&raw)[kPieces], int batch, uint8_t* kv, const uint32_t* mult, const KVMeta* km) {
      if (FP8) {
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int p = lt + kLoadThreads * (batch * kPieces + i);
          const int row = PACKED ? packed_row(p) : p / kRowPieces;
          const int c16 = PACKED ? (p < kPackedCodePieces ? (p & 31) : 32 + (p & 7)) : p - row * kRowPieces;
          if (PACKED && p >= kPackedCodePieces) {
            // eight bf16 rope values -> fp16 times 2^-E_j (the row's exponent), in fp32
            const float inv = exp2i(-km->E[row]);
            const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
              const __half2 hh = __floats2half2_rn(f.x * inv, f.y * inv);
              o[e] = *reinterpret_cast<const uint32_t*>(&hh);
            }
            *reinterpret_cast<uint4*>(kv + 8 * kKVChunk + swz(row, c16 - 32)) = make_uint4(o[0], o[1], o[2], o[3]);
            continue;
          }
          const uint32_t mwi = mult[row * kKvGroups + (c16 >> 3)];
          const __half2 m2 = *reinterpret_cast<const __half2*>(&mwi);
          uint4 o0, o1;
          dequant4_f16(raw[i].x, m2, o0.x, o0.y);
          dequant4_f16(raw[i].y, m2, o0.z, o0.w);
          dequant4_f16(raw[i].z, m2, o1.x, o1.y);
          dequant4_f16(raw[i].w, m2, o1.z, o1.w);
          uint8_t* blk = kv + (c16 >> 2) * kKVChunk;
          const int u = (c16 & 3) * 2;
          // odd chunks store their upper half first, which spreads each store instruction
          // of a warp over all eight 16-byte bank groups; chosen by selects, not a branch
          const int odd = (c16 >> 2) & 1;
          const uint4 first = odd ? o1 : o0;
          const uint4 second = odd ? o0 : o1;
          *reinterpret_cast<uint4*>(blk + swz(row, u + odd)) = first;
          *reinterpret_cast<uint4*>(blk + swz(row, u + 1 - odd)) = second;
        }
      } else {
#pragma unroll
        for (int i = 0; i < kPieces; ++i) {
          const int p = lt + kLoadThreads * (batch * kPieces + i);
          const int row = p / kRowPieces, c16 = p - row * kRowPieces;
          *reinterpret_cast<uint4*>(kv + (c16 >> 3) * kKVChunk + swz(row, c16 & 7)) = raw[i];
        }
      }
    };
    // one tile: wait for its buffer, publish the row tables, convert, hand over, prefetch T+2
    auto step = [&](uint4 (&raw)[kPieces], float (&sc)[kKvGroups], int& my_slot, int T) -> bool {
      const int b = T & 1;
      // the buffer was last read by PV(T-2)
      const bool ok = T < 2 || wait_warp(&pv_done[b], ((T >> 1) & 1) ^ 1, abort_flag, a.wait_limit);
      uint32_t* mult = sGrpMeta + b * (kGrpMetaBytes / 4);
      KVMeta* km = sKVMeta + b;
      if (ok && lt < kMlaTile) {
        // row meta: exponent E_j, multipliers s_g / 2^E_j, validity
        int Ej = 0;
        if (FP8) {
          float smax = 0.0f;
#pragma unroll
          for (int k = 0; k < kKvGroups; ++k) smax = fmaxf(smax, sc[k]);
          Ej = smax > 0.0f ? float_exponent(smax) : 0;
          const float inv = exp2i(-Ej);
#pragma unroll
          for (int k = 0; k < kKvGroups; ++k) {
            const __half2 m2 = __float2half2_rn(sc[k] * inv);
            mult[lt * kKvGroups + k] = *reinterpret_cast<const uint32_t*>(&m2);
          }
        }
        const bool valid = my_slot >= 0;
        km->kmul[lt] = valid ? exp2i(Ej) : 0.0f;
        km->kadd[lt] = valid ? 0.0f : -INFINITY;
        km->E[lt] = Ej;
        const unsigned vm = __ballot_sync(0xffffffffu, valid);
        const int em = __reduce_max_sync(0xffffffffu, valid ? Ej : kNoExp);
        if (lane == 0) {
          km->vmask[lt >> 5] = vm;
          km->emax[lt >> 5] = em;
        }
      }
      // also orders this tile's table writes after every loader's reads of tile T-2's
      if (!bar_and(2, kLoadThreads, ok)) return false;
      uint8_t* kv = sKV + b * kKVBytes;
      store(raw, 0, kv, mult, km);
      if (kBatches > 1) {
        fetch(raw, T, 1);
        store(raw, 1, kv, mult, km);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kv_full[b]);
      if (T + 2 < ntiles) {
        fetch_meta(sc, my_slot, T + 2);
        fetch(raw, T + 2, 0);
      }
      return true;
    };
    fetch_meta(scA, slotA, 0);
    fetch(rawA, 0, 0);
    if (ntiles > 1) {
      fetch_meta(scB, slotB, 1);
      fetch(rawB, 1, 0);
    }
    bool good = true;
    for (int T = 0; T < ntiles && good; T += 2) {
      good = step(rawA, scA, slotA, T);
      if (good && T + 1 < ntiles) good = step(rawB, scB, slotB, T + 1);
    }
    if (!good && lane == 0) {
      record_error(a.err, DSA_ERR_TIMEOUT, 12);
      *abort_flag = 1;
    }
    __syncwarp();
    // the output epilogue with the softmax warps (they publish the per-head scales first)
    if (bar_and(kEpiBar, kEpiThreads, good) != 0 && !a.pair) write_out(1 + (warp - kLoadWarp0) / 4);
  }

  if (ntiles == 0 && a.pair) {
    // nothing selected in this split: an empty one for the merge (no O is read from TMEM)
    if (tid < kHeads) {
      sPair[kPairM + tid] = -INFINITY;
      sPair[kPairL + tid] = 0.0f;
      sOutScale[tid] = 0.0f;
    }
    if (tid == 0) sPair[kPairGood] = 1.0f;
  } else if (ntiles == 0) {
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
        float* ml = a.part_ml + ((static_cast<int64_t>(q) * a.nsplit + split) * kHeads + tid) * kPartStats;
        ml[0] = -INFINITY;
#pragma unroll
        for (int i = 1; i < kPartStats; ++i) ml[i] = 0.0f;
      } else if (a.lse != nullptr) {
        a.lse[static_cast<int64_t>(q) * kHeads + tid] = -INFINITY;
      }
    }
  }

  if (a.pair) {
    // ---------------------------------------------------------------- merge of the two splits
    // Split s owns heads 32 s .. 32 s + 31. After the first cluster barrier each CTA reads the
    // other's (m, l), both derive the same weights, and each writes the other's head half of
    // its O (times its weight) into the other's first tile buffer, now free; after the
    // second barrier each normalises its own half. Every thread of both CTAs reaches both
    // barriers: all roles above end here, and every wait before is bounded.
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int peer = split ^ 1;
    tc_fence_before();
    cluster.sync();
    tc_fence_after();
    if (tid < kHeads) {
      const float* pp = cluster.map_shared_rank(sPair, static_cast<unsigned>(peer));
      const bool peer_good = pp[kPairGood] != 0.0f;
      const float ms = sPair[kPairM + tid], ls = sPair[kPairL + tid];
      const float mp = peer_good ? pp[kPairM + tid] : -INFINITY;
      const float lp = peer_good ? pp[kPairL + tid] : 0.0f;
      const float M = fmaxf(ms, mp);
      const float ws = ls > 0.0f ? exp2f(ms - M) : 0.0f;
      const float wp = lp > 0.0f ? exp2f(mp - M) : 0.0f;
      const float L = ws * ls + wp * lp;
      sPair[kPairMul + tid] = ws * sOutScale[tid];
      sPair[kPairInvL + tid] = L > 0.0f ? 1.0f / L : 0.0f;
      sPair[kPairOn + tid] = wp > 0.0f ? 1.0f : 0.0f;
      if ((tid >> 5) == split && a.lse != nullptr)
        a.lse[static_cast<int64_t>(q) * kHeads + tid] = L > 0.0f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
    __syncthreads();
    // a split with nothing selected sends nothing (its weight is 0) but writes its own heads
    const bool epi = (warp < 4 || warp >= kLoadWarp0) && sPair[kPairGood] != 0.0f;
    const bool send = epi && ntiles > 0;
    const int part = warp < 4 ? 0 : 1 + (warp - kLoadWarp0) / 4;   // kPerQuad warps per lane quadrant
    const int quad = warp & 3;
    const uint32_t lb = static_cast<uint32_t>(quad * 32) << 16;
    float* recv = reinterpret_cast<float*>(sKV);                        // [32 heads][512 dims]
    if (send) {
      float* precv = cluster.map_shared_rank(recv, static_cast<unsigned>(peer));
#pragma unroll 1
      for (int d = part; d < 4; d += kPerQuad) {
        const int dim = d * 128 + quad * 32 + lane;
        float v[32];
        tmem_ld32(tmem + kTmemO + lb + d * 64 + peer * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float mul = sPair[kPairMul + peer * 32 + i];
          precv[i * kDimV + dim] = mul != 0.0f ? v[i] * mul : 0.0f;
        }
      }
    }
    tc_fence_before();
    cluster.sync();
    tc_fence_after();
    if (epi) {
#pragma unroll 1
      for (int d = part; d < 4; d += kPerQuad) {
        const int dim = d * 128 + quad * 32 + lane;
        float v[32];
        tmem_ld32(tmem + kTmemO + lb + d * 64 + split * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int hh = split * 32 + i;
          const float mul = sPair[kPairMul + hh];
          const float own = mul != 0.0f ? v[i] * mul : 0.0f;
          const float other = sPair[kPairOn + hh] != 0.0f ? recv[i * kDimV + dim] : 0.0f;
          const float o = (own + other) * sPair[kPairInvL + hh];
          const int64_t off = (static_cast<int64_t>(q) * kHeads + hh) * kDimV + dim;
          if (a.out_fp32) static_cast<float*>(a.out)[off] = o;
          else static_cast<__nv_bfloat16*>(a.out)[off] = __float2bfloat16_rn(o);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kMlaTmemCols);
}

// Log-sum-exp merge of the split partials: M = max_s m_s, a_s = 2^(m_s - M),
// out[:, group g] = sum_s a_s o_s / sum_s a_s L_{g,s}, lse = (M + log2 sum_s a_s l_s) * ln 2.
// L_{g,s} is split s's normaliser for value group g (columns [128 g, 128 g + 128)): its sum
// of p for a bf16 cache, and for an fp8 cache the sum of the weights its tensor-core PV
// actually applied to that group, so that each group is normalised by the weights it used.
// Two heads per CTA: threads 128 h2 .. + 127 take head 2 blockIdx.y + h2, four consecutive
// value dims each (warp w of the half owns value group w, the 128 dims that share one
// normaliser), one 16-byte load per split.
__global__ void __launch_bounds__(256) mla_combine_kernel(const MlaArgs a) {
  pdl_trigger();
  pdl_wait();   // the partials come from the decode kernel
  const int q = blockIdx.x;
  const int h = 2 * blockIdx.y + (threadIdx.x >> 7);
  const int t = threadIdx.x & 127;
  const int g = t >> 5;                 // value group of dims 4 t .. 4 t + 3
  const int S = a.nsplit;
  const float* ml = a.part_ml + static_cast<int64_t>(q) * S * kHeads * kPartStats;
  // one pass over batches of eight splits, every load of a batch in flight together (a
  // split at a time costs one L2 round trip each); the running max M rises batch by batch
  // and what was summed so far is rescaled by 2^(M_old - M_new). A split that saw no valid
  // row (m = -inf) contributes nothing, whatever its o holds.
  constexpr int kB = 8;
  float M = -INFINITY, Lsum = 0.0f, Lg = 0.0f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < S; s0 += kB) {
    float m[kB], l1[kB], lg[kB];
    float4 o[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int s = s0 + u;
      m[u] = -INFINITY;
      l1[u] = lg[u] = 0.0f;
      o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (s < S) {
        const float* st = ml + (s * kHeads + h) * kPartStats;
        m[u] = st[0];
        l1[u] = st[1];
        lg[u] = st[2 + g];
        o[u] = reinterpret_cast<const float4*>(a.part_o + ((static_cast<int64_t>(q) * S + s) * kHeads + h) * kDimV)[t];
      }
    }
    float bm = M;
#pragma unroll
    for (int u = 0; u < kB; ++u) bm = fmaxf(bm, m[u]);
    if (bm == -INFINITY) continue;
    const float c = exp2f(M - bm);   // 0 while nothing was summed (M = -inf)
    Lsum *= c;
    Lg *= c;
    acc.x *= c;
    acc.y *= c;
    acc.z *= c;
    acc.w *= c;
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (m[u] == -INFINITY) continue;
      const float w = exp2f(m[u] - bm);
      Lsum += w * l1[u];
      Lg += w * lg[u];
      acc.x += w * o[u].x;
      acc.y += w * o[u].y;
      acc.z += w * o[u].z;
      acc.w += w * o[u].w;
    }
    M = bm;
  }
  const float inv = Lg > 0.0f ? 1.0f / Lg : 0.0f;
  const float r[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  const int64_t off = (static_cast<int64_t>(q) * kHeads + h) * kDimV + 4 * t;
  if (a.out_fp32) {
    float* o = static_cast<float*>(a.out) + off;
    if ((reinterpret_cast<uintptr_t>(a.out) & 15) == 0) {
      *reinterpret_cast<float4*>(o) = make_float4(r[0], r[1], r[2], r[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = r[i];
    }
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.out) + off;
    if ((reinterpret_cast<uintptr_t>(a.out) & 7) == 0) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(r[0], r[1]);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(r[2], r[3]);
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t*>(&lo);
      w.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(o) = w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = __float2bfloat16_rn(r[i]);
    }
  }
  if (t == 0 && a.lse != nullptr)
    a.lse[static_cast<int64_t>(q) * kHeads + h] = Lsum > 0.0f ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
}

template <int KVF>
static cudaError_t launch_mla_t(const CUtensorMap& tq, const MlaArgs& a, cudaStream_t stream) {
  constexpr int threads = mla_threads(mla_loaders(KVF));
  cudaError_t e = set_smem_once<mla_decode_kernel<KVF>>(kMlaSmem);
  if (e != cudaSuccess) return e;
  if (a.pair)
    return launch_pdl_cluster(mla_decode_kernel<KVF>, dim3(a.Bq * a.nsplit), dim3(threads), kMlaSmem, stream, 2u,
                              tq, a);
  return launch_pdl(mla_decode_kernel<KVF>, dim3(a.Bq * a.nsplit), dim3(threads), kMlaSmem, stream, tq, a);
}

cudaError_t launch_mla(int kvf, const CUtensorMap& tmap_q, const MlaArgs& a, cudaStream_t stream, int* launches) {
  cudaError_t e = kvf == kKvFp8Packed ? launch_mla_t<kKvFp8Packed>(tmap_q, a, stream)
                  : kvf == kKvFp8     ? launch_mla_t<kKvFp8>(tmap_q, a, stream)
                                      : launch_mla_t<kKvBf16>(tmap_q, a, stream);
  ++*launches;
  if (e != cudaSuccess || a.nsplit == 1 || a.pair) return e;
  ++*launches;
  return launch_pdl(mla_combine_kernel, dim3(a.Bq, kHeads / 2), dim3(256), 0, stream, a);
}

int mla_tile_keys() { return kMlaTile; }

}  // namespace dsa
