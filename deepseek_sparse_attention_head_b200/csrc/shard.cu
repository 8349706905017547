// Token-sharded decode of long sequences: each row's tokens are spread over R ranks (one
// GPU each), and one exchange step joins them (the long-context extension of the decode
// step; the pages say only that the context reaches 1M tokens, Russian news item on
// colibri). Per rank:
//   1. indexer scores and a local top-k over the rank's own tokens (the usual stages);
//   2. shard_candidates_kernel: the local winners as (score, global token) pairs, the
//      payload of the exchange;
//   3. (all ranks gather every rank's payload: a collective outside this library)
//   4. shard_select_kernel: the global top-k among all candidates, ties to the lower
//      global token, identical on every rank; the winners this rank holds are mapped to
//      its physical slots (first in the list, -1 after);
//   5. MLA sparse decode over those slots (fp32 output + lse: the rank's softmax state);
//   6. (all ranks gather every rank's state)
//   7. shard_merge_kernel: the log-sum-exp merge of the R states.
// The union of the local top-k lists holds a global top-k, and merging softmax states by
// their log-sum-exp gives the softmax over the union, so the result is the unsharded step's.
#include <cuda_bf16.h>

#include <type_traits>

#include "kernels.cuh"

namespace dsa {

constexpr int kSelThreads = 1024;
constexpr int kSelBins = 256;   // 8-bit radix digits: at most four passes per 32-bit key

// ------------------------------------------------------------------ candidates

__global__ void shard_candidates_kernel(const ShardCandArgs a) {
  pdl_trigger();
  pdl_wait();   // the local selection comes from the top-k kernel
  const int64_t total = static_cast<int64_t>(a.Bq) * a.top_k;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int q = static_cast<int>(i / a.top_k);
    const int s = a.logical[i];
    float sc = -INFINITY;
    int tok = -1;
    if (s >= 0 && s < a.L_max) {
      const int64_t g = static_cast<int64_t>(a.token_offset[q / a.n_q]) + s;
      if (a.token_offset[q / a.n_q] < 0 || g > 0x7fffffffLL) {
        record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(a.token_offset[q / a.n_q]));
      } else {
        sc = a.scores[static_cast<int64_t>(q) * a.L_max + s];
        tok = static_cast<int>(g);
      }
    }
    a.cand_score[i] = sc;
    a.cand_token[i] = tok;
  }
}

// ------------------------------------------------------------------ global select

struct SelSmem {
  uint32_t hist[kSelBins];
  uint32_t bin, rem, eq, n_valid, n_sel, n_mine, n_eq2, kmin, kmax;
};

// Candidates of query q: candidate c is entry (r = c / K, i = c % K) of the gathered
// [R, Bq, K] arrays. Two sources give every thread the same number of visits (so that
// warp-wide ballots stay converged), each visit f(c, key, token) with token -1 past the end:
//  * RegCands<P>: rows of at most P x 1024 candidates live in registers, P per thread
//    (c = tid + 1024 j), loaded once with all loads in flight;
//  * MemCands: longer rows, read from a shared-memory copy when it fits, else from global
//    memory on every visit.
__device__ __forceinline__ int64_t cand_gidx(int c, int K, int Bq, int q) {
  const int r = c / K;
  return (static_cast<int64_t>(r) * Bq + q) * K + (c - r * K);
}

// Steps (r, i) = (c / K, c % K) from candidate c to c + 1024: one conditional subtraction
// when K >= 1024, else a division.
__device__ __forceinline__ void cand_step(int& r, int& i, int c_next, int K) {
  if (K >= kSelThreads) {
    i += kSelThreads;
    if (i >= K) {
      i -= K;
      ++r;
    }
  } else {
    r = c_next / K;
    i = c_next - r * K;
  }
}

template <int P>
struct RegCands {
  uint32_t key[P];
  int32_t tok[P];
  __device__ __forceinline__ void load(const ShardSelectArgs& a, int n, int q) {
    if constexpr (P > 8) {
      // at 16 a thread (64 registers) the per-candidate form measured faster
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const int c = static_cast<int>(threadIdx.x) + j * kSelThreads;
        float sc = 0.f;
        tok[j] = -1;
        if (c < n) {
          const int64_t g = cand_gidx(c, a.top_k, a.Bq, q);
          sc = __ldg(a.all_score + g);
          tok[j] = __ldg(a.all_token + g);
        }
        key[j] = order_key(sc);
      }
      return;
    }
    // every load issued before any is used; the (rank, entry) of c = tid + 1024 j advances
    // by additions (a division per candidate costs more than the load's issue)
    const int K = a.top_k;
    int r = static_cast<int>(threadIdx.x) / K, i = static_cast<int>(threadIdx.x) - r * K;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const int c = static_cast<int>(threadIdx.x) + j * kSelThreads;
      key[j] = 0u;
      tok[j] = -1;
      if (c < n) {
        const int64_t g = (static_cast<int64_t>(r) * a.Bq + q) * K + i;
        key[j] = __float_as_uint(__ldg(a.all_score + g));
        tok[j] = __ldg(a.all_token + g);
      }
      cand_step(r, i, c + kSelThreads, K);
    }
#pragma unroll
    for (int j = 0; j < P; ++j) key[j] = order_key(__uint_as_float(key[j]));
  }
  template <typename F>
  __device__ __forceinline__ void visit(F f) const {
#pragma unroll
    for (int j = 0; j < P; ++j) f(static_cast<int>(threadIdx.x) + j * kSelThreads, key[j], tok[j]);
  }
};

struct MemCands {
  const float* sc;
  const int32_t* tk;
  const uint32_t* skey;   // shared copy (or null)
  const int32_t* stok;
  int n, K, Bq, q;
  __device__ void load(const ShardSelectArgs& a, uint8_t* smem_tail) {
    if (!a.in_smem) return;
    uint32_t* k_ = reinterpret_cast<uint32_t*>(smem_tail);
    int32_t* t_ = reinterpret_cast<int32_t*>(k_ + n);
    constexpr int kU = 8;   // eight candidates per thread in flight at once
    for (int c0 = threadIdx.x; c0 < n; c0 += kU * kSelThreads) {
      float s_[kU];
      int32_t tt[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * kSelThreads;
        if (c < n) {
          const int64_t g = cand_gidx(c, K, Bq, q);
          s_[u] = __ldg(sc + g);
          tt[u] = __ldg(tk + g);
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + u * kSelThreads;
        if (c < n) {
          k_[c] = order_key(s_[u]);
          t_[c] = tt[u];
        }
      }
    }
    skey = k_;
    stok = t_;
  }
  template <typename F>
  __device__ void visit(F f) const {
    for (int c0 = 0; c0 < n; c0 += kSelThreads) {
      const int c = c0 + static_cast<int>(threadIdx.x);
      uint32_t u = 0u;
      int32_t t = -1;
      if (c < n) {
        if (skey) {
          u = skey[c];
          t = stok[c];
        } else {
          const int64_t g = cand_gidx(c, K, Bq, q);
          u = order_key(sc[g]);
          t = tk[g];
        }
      }
      f(c, u, t);
    }
  }
};

// The k-th largest (1-based, k >= 1) of key(u, t) over the candidates with take(u, t),
// exact. The radix runs over r = key - (smallest taken key), from the highest bit in which
// the taken keys differ, in 8-bit digits (candidates gathered from every rank's top-k have
// close scores, so their keys share most leading bits). Returns the key; *need = how many
// candidates equal to it belong to the top k, *n_equal = how many there are. Whole CTA.
template <typename Src, typename Key, typename Take>
__device__ uint32_t radix_kth(SelSmem& sm, const Src& src, uint32_t k, Key key, Take take, uint32_t* need,
                              uint32_t* n_equal) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  if (tid == 0) {
    sm.kmin = 0xFFFFFFFFu;
    sm.kmax = 0u;
  }
  __syncthreads();
  {
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    src.visit([&](int, uint32_t u, int32_t t) {
      if (take(u, t)) {
        const uint32_t v = key(u, t);
        lo = v < lo ? v : lo;
        hi = v > hi ? v : hi;
      }
    });
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      atomicMin(&sm.kmin, lo);
      atomicMax(&sm.kmax, hi);
    }
  }
  __syncthreads();
  const uint32_t kmin = sm.kmin;
  const uint32_t span = sm.kmax - kmin;
  int top = span == 0u ? 0 : 32 - __clz(span);   // every r fits in bits [0, top)
  uint32_t prefix = 0u, pmask = 0u, remaining = k, eq = 0u;
#pragma unroll 1
  while (true) {
    const int lo_bit = top > 8 ? top - 8 : 0;
    const uint32_t dm = (1u << (top - lo_bit)) - 1u;   // top - lo_bit in [0, 8]
    for (int i = tid; i < kSelBins; i += kSelThreads) sm.hist[i] = 0u;
    __syncthreads();
    src.visit([&](int, uint32_t u, int32_t t) {
      if (!take(u, t)) return;
      const uint32_t r = key(u, t) - kmin;
      if ((r & pmask) == prefix) atomicAdd(&sm.hist[(r >> lo_bit) & dm], 1u);
    });
    __syncthreads();
    if (tid < 32) {
      // lane l holds bins [8 (31 - l), 8 (31 - l) + 8): lane 0 the largest digits
      const int base = 8 * (31 - lane);
      uint32_t h[8], s = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = sm.hist[base + j];
        s += h[j];
      }
      uint32_t incl = s;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      const uint32_t above = incl - s;   // keys in larger digits than this lane's
      if (above < remaining && remaining <= incl) {
        uint32_t acc = above;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (acc + h[j] >= remaining) {
            sm.bin = static_cast<uint32_t>(base + j);
            sm.rem = remaining - acc;
            sm.eq = h[j];
            break;
          }
          acc += h[j];
        }
      }
    }
    __syncthreads();
    prefix |= sm.bin << lo_bit;
    pmask |= dm << lo_bit;
    remaining = sm.rem;
    eq = sm.eq;
    __syncthreads();   // sm.bin / sm.rem are rewritten by the next pass
    if (lo_bit == 0) break;
    top = lo_bit;
  }
  *need = remaining;
  *n_equal = eq;
  return kmin + prefix;
}

// One CTA per query. P > 0: the row's candidates in registers (n <= P x 1024); P == 0:
// MemCands.
template <int P>
__global__ void __launch_bounds__(kSelThreads) shard_select_kernel(const ShardSelectArgs a) {
  extern __shared__ uint8_t sel_smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(sel_smem_raw);
  const int tid = threadIdx.x;
  const int q = blockIdx.x;
  const int b = q / a.n_q;
  const int K = a.top_k;
  const int n = a.n_ranks * K;
  pdl_trigger();
  pdl_wait();   // the gathered candidates may come from an earlier kernel on the stream

  using Src = typename std::conditional<(P > 0), RegCands<(P > 0 ? P : 1)>, MemCands>::type;
  Src src;
  if constexpr (P > 0) {
    src.load(a, n, q);
  } else {
    src = MemCands{a.all_score, a.all_token, nullptr, nullptr, n, K, a.Bq, q};
    src.load(a, sel_smem_raw + sizeof(SelSmem));
  }
  if (tid == 0) {
    sm.n_valid = 0u;
    sm.n_sel = 0u;
    sm.n_mine = 0u;
    sm.n_eq2 = 0u;
  }
  __syncthreads();
  {
    uint32_t cnt = 0u;
    src.visit([&](int, uint32_t, int32_t t) { cnt += t >= 0 ? 1u : 0u; });
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if ((tid & 31) == 0 && cnt != 0u) atomicAdd(&sm.n_valid, cnt);
  }
  __syncthreads();
  const uint32_t n_valid = sm.n_valid;
  const uint32_t k = n_valid < static_cast<uint32_t>(K) ? n_valid : static_cast<uint32_t>(K);

  // selection rule: all valid candidates (k == n_valid), else score key above kth, or equal
  // to it and among the `need` lowest global tokens of those equal
  const bool all = k == n_valid;
  uint32_t kth = 0u, need = 0u, n_equal = 0u, kth2 = 0u, need2 = 0u, n_equal2 = 0u;
  bool all_equal = true;
  if (!all) {
    kth = radix_kth(
        sm, src, k, [](uint32_t u, int32_t) { return u; }, [](uint32_t, int32_t t) { return t >= 0; }, &need,
        &n_equal);
    all_equal = need == n_equal;
    if (!all_equal) {
      // ties at the k-th score: the `need` lowest tokens (larger key = lower token)
      kth2 = radix_kth(
          sm, src, need, [](uint32_t, int32_t t) { return ~static_cast<uint32_t>(t); },
          [kth](uint32_t u, int32_t t) { return t >= 0 && u == kth; }, &need2, &n_equal2);
    }
  }

  const int off = a.token_offset[b];
  int len = a.seq_lens[b];
  len = len < 0 ? 0 : (len > a.max_pages * kPage ? a.max_pages * kPage : len);
  int32_t* lo_row = a.logical ? a.logical + static_cast<int64_t>(q) * K : nullptr;
  int32_t* ph_row = a.physical + static_cast<int64_t>(q) * K;
  auto picked = [&](uint32_t u, int32_t tok) {
    bool pick = tok >= 0;
    if (pick && !all) {
      if (u < kth) {
        pick = false;
      } else if (u == kth && !all_equal) {
        const uint32_t u2 = ~static_cast<uint32_t>(tok);
        // distinct tokens make kth2 unique; duplicates (an invalid layout) are capped
        pick = u2 > kth2 || (u2 == kth2 && atomicAdd(&sm.n_eq2, 1u) < need2);
      }
    }
    return pick;
  };
  if constexpr (P > 0 && P <= 8) {
    // register path: each thread's picks and own-rank winners are counted, one block-wide
    // exclusive scan of both counts (packed in one word) gives every thread its output
    // positions, and the stores follow with no atomic in the chain
    uint32_t pm = 0u, mm = 0u;
    {
      int r = tid / K;
      int i = tid - r * K;
#pragma unroll
      for (int j = 0; j < P; ++j) {
        if (picked(src.key[j], src.tok[j])) {
          pm |= 1u << j;
          if (r == a.rank) {
            const int s_ = src.tok[j] - off;
            if (s_ < 0 || s_ >= len) {
              record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(src.tok[j]));
            } else {
              mm |= 1u << j;
            }
          }
        }
        cand_step(r, i, tid + (j + 1) * kSelThreads, K);
      }
    }
    const uint32_t mine_v = static_cast<uint32_t>(__popc(pm)) | (static_cast<uint32_t>(__popc(mm)) << 16);
    uint32_t incl = mine_v;
    const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    __syncthreads();   // sm.hist is free once the radix passes are done
    if (lane == 31) sm.hist[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t w = sm.hist[lane];
      uint32_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += t;
      }
      sm.hist[lane] = wi - w;
      if (lane == 31) {
        sm.n_sel = wi & 0xFFFFu;
        sm.n_mine = wi >> 16;
      }
    }
    __syncthreads();
    const uint32_t base = sm.hist[warp] + incl - mine_v;
    uint32_t p = base & 0xFFFFu, m = base >> 16;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if (pm & (1u << j)) {
        if (p < k && lo_row) lo_row[p] = src.tok[j];
        ++p;
      }
      if (mm & (1u << j)) {
        if (m < static_cast<uint32_t>(K)) ph_row[m] = src.tok[j] - off;   // this rank's local token
        ++m;
      }
    }
  } else {
  // output positions come from one shared atomic per warp (ballot + popcount); at 16
  // candidates a thread this measured faster than the block scan above
  // (19.7 against 25.2 us for 16K candidates)
  const unsigned lt_mask = (1u << (tid & 31)) - 1u;
  src.visit([&](int c, uint32_t u, int32_t tok) {
    const bool pick = picked(u, tok);
    const unsigned picks = __ballot_sync(0xffffffffu, pick);
    uint32_t base = 0u;
    if ((tid & 31) == 0 && picks != 0u) base = atomicAdd(&sm.n_sel, static_cast<uint32_t>(__popc(picks)));
    const uint32_t p = __shfl_sync(0xffffffffu, base, 0) + static_cast<uint32_t>(__popc(picks & lt_mask));
    int local = -1;   // this rank's winners: local token now, its slot below
    if (pick && p < k) {
      if (lo_row) lo_row[p] = tok;
      if (c / K == a.rank) {
        const int s = tok - off;
        if (s < 0 || s >= len) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(tok));
        else local = s;
      }
    }
    const unsigned mine = __ballot_sync(0xffffffffu, local >= 0);
    uint32_t mbase = 0u;
    if ((tid & 31) == 0 && mine != 0u) mbase = atomicAdd(&sm.n_mine, static_cast<uint32_t>(__popc(mine)));
    mbase = __shfl_sync(0xffffffffu, mbase, 0);
    if (local >= 0) ph_row[mbase + __popc(mine & lt_mask)] = local;
  });
  }
  __syncthreads();
  const int n_sel = static_cast<int>(sm.n_sel < k ? sm.n_sel : k);
  const int n_mine = static_cast<int>(sm.n_mine < static_cast<uint32_t>(K) ? sm.n_mine : static_cast<uint32_t>(K));
  // page map of this rank's winners, all block-table loads of a thread in flight together
  constexpr int kU = 4;
  for (int i0 = tid; i0 < n_mine; i0 += kU * kSelThreads) {
    int s_[kU], pg[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) s_[u] = i0 + u * kSelThreads < n_mine ? ph_row[i0 + u * kSelThreads] : 0;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      pg[u] = i0 + u * kSelThreads < n_mine
                  ? checked_page(a.block_table, b, s_[u] >> 6, a.max_pages, a.num_pages, a.err)
                  : 0;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i0 + u * kSelThreads < n_mine) ph_row[i0 + u * kSelThreads] = pg[u] * kPage + (s_[u] & 63);
  }
  if (lo_row)
    for (int i = n_sel + tid; i < K; i += kSelThreads) lo_row[i] = -1;
  for (int i = n_mine + tid; i < K; i += kSelThreads) ph_row[i] = -1;
}

// ------------------------------------------------------------------ merge

// 128 threads per (query, head), four columns each; R states merged per thread.
constexpr int kMergeHeadsPerCta = 2;

__global__ void __launch_bounds__(128 * kMergeHeadsPerCta) shard_merge_kernel(const ShardMergeArgs a) {
  pdl_trigger();
  pdl_wait();
  const int hq = blockIdx.x * kMergeHeadsPerCta + static_cast<int>(threadIdx.x >> 7);   // q * 64 + h
  if (hq >= a.Bq * kHeads) return;
  const int col = 4 * static_cast<int>(threadIdx.x & 127);
  const int64_t stride_lse = static_cast<int64_t>(a.Bq) * kHeads;
  float M = -INFINITY;
  for (int r = 0; r < a.n_ranks; ++r) M = fmaxf(M, a.all_lse[r * stride_lse + hq]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < a.n_ranks; ++r) {
      const float l = a.all_lse[r * stride_lse + hq];
      if (l == -INFINITY) continue;
      const float w = expf(l - M);
      L += w;
      const float4 o = *reinterpret_cast<const float4*>(a.all_out + (r * stride_lse + hq) * kDimV + col);
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    const float inv = 1.f / L;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
  }
  const int64_t o = static_cast<int64_t>(hq) * kDimV + col;
  if (a.out_fp32) {
    *reinterpret_cast<float4*>(static_cast<float*>(a.out) + o) = acc;
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + o) = pk;
  }
  if (a.lse && col == 0) a.lse[hq] = M == -INFINITY ? -INFINITY : M + logf(L);
}

// ------------------------------------------------------------------ launches

int shard_select_smem_bytes(int n_cand) {
  const int64_t in = static_cast<int64_t>(sizeof(SelSmem)) + static_cast<int64_t>(n_cand) * 8;
  return in <= kShardSelectSmemCap ? static_cast<int>(in) : 0;
}

cudaError_t launch_shard_candidates(const ShardCandArgs& a, cudaStream_t stream, int* launches) {
  const int64_t total = static_cast<int64_t>(a.Bq) * a.top_k;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  ++*launches;
  return launch_pdl(shard_candidates_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, a);
}

cudaError_t launch_shard_select(const ShardSelectArgs& a, cudaStream_t stream, int* launches) {
  const int n = a.n_ranks * a.top_k;
  const dim3 grid(a.Bq), block(kSelThreads);
  const int small = static_cast<int>(sizeof(SelSmem));
  ++*launches;
  if (n <= 4 * kSelThreads) return launch_pdl(shard_select_kernel<4>, grid, block, small, stream, a);
  if (n <= 8 * kSelThreads) return launch_pdl(shard_select_kernel<8>, grid, block, small, stream, a);
  if (n <= 16 * kSelThreads) return launch_pdl(shard_select_kernel<16>, grid, block, small, stream, a);
  const int smem = a.in_smem ? shard_select_smem_bytes(n) : small;
  if (smem > 48 * 1024) {
    const cudaError_t e = set_smem_once<shard_select_kernel<0>>(kShardSelectSmemCap);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(shard_select_kernel<0>, grid, block, smem, stream, a);
}

cudaError_t launch_shard_merge(const ShardMergeArgs& a, cudaStream_t stream, int* launches) {
  const int64_t heads = static_cast<int64_t>(a.Bq) * kHeads;
  ++*launches;
  return launch_pdl(shard_merge_kernel, dim3(static_cast<unsigned>((heads + kMergeHeadsPerCta - 1) / kMergeHeadsPerCta)),
                    dim3(128 * kMergeHeadsPerCta), 0, stream, a);
}

}  // namespace dsa
