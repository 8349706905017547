// Stage 2 of the DSA decode step: top-k selection with the fused page-mapping
// transform ("GLM-52 Runs on RTX 4090", kernel list item 2; glm-5.2-4090 README,
// usage: SGLANG_NSA_FUSE_TOPK=1 fuses the page-mapping transform into top-k).
//
// One CTA per query. Scores are mapped to order-preserving 32-bit keys.
//  1. A threshold is estimated from evenly spaced samples of the row (256, or up to
//     4096 for very long rows), low enough that about 1.25 k / vis of the samples (plus
//     a margin) lie above it.
//  2. One pass over the row gathers every key at or above the threshold into shared
//     memory (per-thread counts, a warp prefix sum and one shared atomic per warp for
//     every 16K keys). Its first batch is loaded before step 1 starts.
//  3. The k-th largest candidate is found exactly by a radix select over the
//     candidates' offsets from the threshold (12-bit digits, shared-memory
//     histograms), and the winners are emitted with their physical slots.
// When the estimate misses (fewer than k candidates, or more than fit), a
// three-digit radix select over the whole row (12 + 12 + 8 bits) decides instead.
// Few very long rows (the 1M-token stream) split step 2 over 16K-key
// chunks, one CTA each, into a per-row candidate buffer in the workspace; a second
// kernel then runs step 3 per row.
// A query that sees no more than top_k tokens takes all of them (the dense path).
#include <cooperative_groups.h>

#include "kernels.cuh"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kHistBins = 4096;
constexpr int kCand = 12288;  // candidates kept in shared memory
constexpr int kTopkChunk = 16384;   // keys per CTA of the long-row gather

struct TopkSmem {
  uint32_t hist[kHistBins];
  uint32_t cand_key[kCand];
  int32_t cand_idx[kCand];
  uint32_t wsum[32];
  uint32_t sel_bin, sel_rem, n_cand, cnt_out, cnt_eq, thr, rmax;
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
  if (warp == 0) {   // suffix sums over the warps: wsum[w] <- sum of warps w+1 .. 31
    const uint32_t x = sm.wsum[lane];
    uint32_t y = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n = __shfl_down_sync(0xffffffffu, y, off);
      if (lane + off < 32) y += n;
    }
    __syncwarp();
    sm.wsum[lane] = y - x;
  }
  __syncthreads();
  uint32_t above = v - mine + sm.wsum[warp];
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

// Per-row context shared by the phases below.
struct TopkRow {
  int q, b, vis, K;
  const float* row;
  int32_t* lo;   // logical out row, or null
  int32_t* po;   // physical out row, or null
};

__device__ __forceinline__ TopkRow topk_row(const TopkArgs& a, int q) {
  TopkRow r;
  r.q = q;
  r.b = q / a.n_q;
  const int L = row_len(a.seq_lens, r.b, a.max_pages);
  r.vis = query_vis(a.q_pos, q, L);
  if (r.vis > a.L_max) r.vis = static_cast<int>(a.L_max);
  r.K = a.top_k;
  r.row = a.scores + static_cast<int64_t>(q) * a.L_max;
  r.lo = a.logical ? a.logical + static_cast<int64_t>(q) * r.K : nullptr;
  r.po = a.physical ? a.physical + static_cast<int64_t>(q) * r.K : nullptr;
  return r;
}

__device__ __forceinline__ void topk_emit(const TopkArgs& a, const TopkRow& r, int pos, int s) {
  if (r.lo) r.lo[pos] = s;
  if (r.po) {
    int slot = -1;
    if (s >= 0) slot = checked_page(a.block_table, r.b, s >> 6, a.max_pages, a.num_pages, a.err) * kPage + (s & 63);
    r.po[pos] = slot;
  }
}

// Dense path: every visible token (vis <= top_k).
__device__ __forceinline__ void topk_dense(const TopkArgs& a, const TopkRow& r) {
  for (int i = threadIdx.x; i < r.K; i += kTopkThreads) topk_emit(a, r, i, i < r.vis ? i : -1);
}

// Threshold estimate (whole CTA): S = min(4096, vis) evenly spaced samples of the row, and
// a key at or below the `need`-th largest sample, need = 1.25 E + 3 sqrt(E) + 4 with
// E = S k / vis the expected number of true top-k keys among the samples. Found by a
// two-digit histogram select (bits 31..20, then 19..8) and rounded down to its 24-bit
// prefix. Deterministic: every CTA that calls it on the same row gets the same value.
// Uses sm.hist and sm.cand_key[0..S).
__device__ uint32_t row_threshold(TopkSmem& sm, const float* row, int vis, int K) {
  constexpr int kMaxSamples = 4096;
  const int tid = threadIdx.x;
  const int S = min(kMaxSamples, vis);
  {
    // all of a thread's samples in flight at once, then stored
    constexpr int kPerT = kMaxSamples / kTopkThreads;
    uint32_t sk[kPerT];
#pragma unroll
    for (int j = 0; j < kPerT; ++j) {
      const int i = tid + j * kTopkThreads;
      sk[j] = i < S ? order_key(__ldg(row + static_cast<int>((static_cast<int64_t>(i) * vis) / S))) : 0u;
    }
#pragma unroll
    for (int j = 0; j < kPerT; ++j)
      if (tid + j * kTopkThreads < S) sm.cand_key[tid + j * kTopkThreads] = sk[j];
  }
  const float expect = static_cast<float>(S) * static_cast<float>(K) / static_cast<float>(vis);
  const uint32_t need = static_cast<uint32_t>(
      fminf(1.25f * expect + 3.0f * sqrtf(expect) + 4.0f, static_cast<float>(S)));
  for (int i = tid; i < kHistBins; i += kTopkThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < S; i += kTopkThreads) atomicAdd(&sm.hist[sm.cand_key[i] >> 20], 1u);
  __syncthreads();
  select_bin(sm, need);
  const uint32_t b1 = sm.sel_bin, r1 = sm.sel_rem;
  for (int i = tid; i < kHistBins; i += kTopkThreads) sm.hist[i] = 0;
  __syncthreads();
  for (int i = tid; i < S; i += kTopkThreads) {
    const uint32_t u = sm.cand_key[i];
    if ((u >> 20) == b1) atomicAdd(&sm.hist[(u >> 8) & 0xFFFu], 1u);
  }
  __syncthreads();
  select_bin(sm, r1);
  const uint32_t thr = (b1 << 20) | (sm.sel_bin << 8);
  __syncthreads();   // sm.cand_key is reused by the caller
  return thr;
}

// Threshold estimate for one CTA per row: 256 evenly spaced samples, each ranked against
// all the others; the largest sample with at least need = 1.25 E + 3 sqrt(E) + 4 samples
// above it (E = 256 k / vis). Cheaper than row_threshold for rows of up to ~64K keys.
__device__ uint32_t row_threshold_small(TopkSmem& sm, const float* row, int vis, int K) {
  constexpr int kSamples = 256;
  const int tid = threadIdx.x;
  uint32_t* samp = sm.hist;
  uint32_t mykey = 0u;
  if (tid < kSamples) {
    mykey = order_key(__ldg(row + static_cast<int>((static_cast<int64_t>(tid) * vis) / kSamples)));
    samp[tid] = mykey;
  }
  if (tid == 0) sm.thr = 0u;
  __syncthreads();
  if (tid < kSamples) {
    uint32_t above = 0;      // samples strictly above this thread's sample
    const uint4* s4 = reinterpret_cast<const uint4*>(samp);
#pragma unroll 8
    for (int i = 0; i < kSamples / 4; ++i) {
      const uint4 v = s4[i];
      above += (v.x > mykey) + (v.y > mykey) + (v.z > mykey) + (v.w > mykey);
    }
    const float expect = static_cast<float>(kSamples) * static_cast<float>(K) / static_cast<float>(vis);
    const uint32_t need = static_cast<uint32_t>(fminf(1.25f * expect + 3.0f * sqrtf(expect) + 4.0f, 1e9f));
    const uint32_t cand = above >= need ? mykey : 0u;
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, cand);
    if ((tid & 31) == 0 && wmax != 0u) atomicMax(&sm.thr, wmax);
  }
  __syncthreads();
  const uint32_t thr = sm.thr;
  __syncthreads();   // sm.hist is reused by the caller
  return thr;
}

constexpr int kGatherU = 16;                               // keys per thread and batch
constexpr int kGatherBatch = kGatherU * kTopkThreads;

// Loads the gather batch of row[base, hi_s) that starts at `base` (a multiple of 4, the
// row 16-byte aligned): thread t gets keys base + 4 (j * 1024 + t) + [0, 4), j < 4, zeros
// past hi_s. A whole batch in range takes plain 16-byte loads (CTA-uniform test).
__device__ __forceinline__ void gather_load(const float* row, int base, int hi_s, float4 (&v)[kGatherU / 4]) {
  const int tid = threadIdx.x;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  if (base + kGatherBatch <= hi_s) {
#pragma unroll
    for (int j = 0; j < kGatherU / 4; ++j) v[j] = __ldg(r4 + (base >> 2) + j * kTopkThreads + tid);
    return;
  }
#pragma unroll
  for (int j = 0; j < kGatherU / 4; ++j) {
    const int s_ = base + 4 * (j * kTopkThreads + tid);
    v[j] = s_ + 3 < hi_s ? __ldg(r4 + (s_ >> 2))
                         : make_float4(s_ < hi_s ? row[s_] : 0.0f, s_ + 1 < hi_s ? row[s_ + 1] : 0.0f,
                                       s_ + 2 < hi_s ? row[s_ + 2] : 0.0f, 0.0f);
  }
}

// Bit 4 j + t set when key t of cur[j] (index base + 4 (j * 1024 + tid) + t) is below
// hi_s (checked unless kWhole) and at least thr. When thr is the key of a non-negative
// float (thr >= 0x80000000), key >= thr holds exactly when the score's bit pattern, read
// as a signed integer, is at least thr's float bit pattern: negative scores (and negative
// NaNs) are negative integers, and non-negative ones (+inf and +NaN included) order like
// their keys. One integer compare per score instead of the key transform.
template <bool kWhole>
__device__ __forceinline__ uint32_t gather_takes(const float4 (&cur)[kGatherU / 4], int base, int hi_s,
                                                 uint32_t thr) {
  uint32_t takes = 0;
  if (thr >= 0x80000000u) {
    const int tb = static_cast<int>(thr & 0x7FFFFFFFu);
#pragma unroll
    for (int j = 0; j < kGatherU / 4; ++j) {
      const int s_ = base + 4 * (j * kTopkThreads + static_cast<int>(threadIdx.x));
      const int e[4] = {__float_as_int(cur[j].x), __float_as_int(cur[j].y), __float_as_int(cur[j].z),
                        __float_as_int(cur[j].w)};
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if ((kWhole || s_ + t < hi_s) && e[t] >= tb) takes |= 1u << (4 * j + t);
    }
    return takes;
  }
#pragma unroll
  for (int j = 0; j < kGatherU / 4; ++j) {
    const int s_ = base + 4 * (j * kTopkThreads + static_cast<int>(threadIdx.x));
    const float e[4] = {cur[j].x, cur[j].y, cur[j].z, cur[j].w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if ((kWhole || s_ + t < hi_s) && order_key(e[t]) >= thr) takes |= 1u << (4 * j + t);
  }
  return takes;
}

// Gathers every key >= thr of row[lo_s, hi_s) (lo_s a multiple of 4, the row 16-byte
// aligned) into out_key / out_idx at slots reserved from *counter (shared or global; one
// atomic per warp per 16K keys; slots >= cap are counted but not stored), and raises
// *rmax_addr to the largest key - thr. `cur` holds the first batch, loaded by
// gather_load(row, lo_s, hi_s, cur) (so that its loads can be in flight while the caller
// derives thr). Whole CTA; the trip count is CTA-uniform.
// kBlock: `counter` and `rmax_addr` are in global memory and shared by many CTAs (the
// long-row chunks), so the CTA reserves its slots with one atomic per batch (a warp-sum
// scan in wsum[0..32]) and publishes its largest offset with one atomicMax; otherwise each
// warp reserves its own (a shared or distributed-shared counter).
template <bool kBlock = false>
__device__ void gather_range(const float* row, int lo_s, int hi_s, uint32_t thr, uint32_t* counter,
                             uint32_t* out_key, int32_t* out_idx, uint32_t cap, uint32_t* rmax_addr,
                             float4 (&cur)[kGatherU / 4], uint32_t* wsum = nullptr) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  uint32_t lmax = 0;
  float4 nxt[kGatherU / 4];
  for (int base = lo_s; base < hi_s; base += kGatherBatch) {
    if (base + kGatherBatch < hi_s) gather_load(row, base + kGatherBatch, hi_s, nxt);
    uint32_t takes = base + kGatherBatch <= hi_s ? gather_takes<true>(cur, base, hi_s, thr)
                                                  : gather_takes<false>(cur, base, hi_s, thr);
    uint32_t c;
    if constexpr (kBlock) {
      const uint32_t n = static_cast<uint32_t>(__popc(takes));
      uint32_t incl = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      if (lane == 31) wsum[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        const uint32_t w = wsum[lane];
        uint32_t wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, wi, off);
          if (lane >= off) wi += t;
        }
        const uint32_t total = __shfl_sync(0xffffffffu, wi, 31);
        uint32_t b0 = 0u;
        if (lane == 0 && total != 0u) b0 = atomicAdd(counter, total);
        b0 = __shfl_sync(0xffffffffu, b0, 0);
        wsum[lane] = b0 + wi - w;   // this warp's first slot
      }
      __syncthreads();
      c = wsum[warp] + incl - n;
      __syncthreads();   // wsum is rewritten by the next batch
    } else {
      c = warp_reserve(counter, static_cast<uint32_t>(__popc(takes)));
    }
    // only the taken keys (a few percent) are visited
    while (takes != 0u) {
      const int bit = __ffs(takes) - 1;
      takes &= takes - 1u;
      const int j = bit >> 2, t = bit & 3;
      float e = cur[0].x;
#pragma unroll
      for (int jj = 0; jj < kGatherU / 4; ++jj)
        if (jj == j) e = t == 0 ? cur[jj].x : (t == 1 ? cur[jj].y : (t == 2 ? cur[jj].z : cur[jj].w));
      const uint32_t u = order_key(e);
      if (c < cap) {
        out_key[c] = u;
        out_idx[c] = base + 4 * (j * kTopkThreads + tid) + t;
      }
      ++c;
      lmax = max(lmax, u - thr);
    }
#pragma unroll
    for (int j = 0; j < kGatherU / 4; ++j) cur[j] = nxt[j];
  }
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, lmax);
  if constexpr (kBlock) {
    if (lane == 0) wsum[warp] = wmax;
    __syncthreads();
    if (warp == 0) {
      const uint32_t bmax = __reduce_max_sync(0xffffffffu, wsum[lane]);
      if (lane == 0 && bmax != 0u) atomicMax(rmax_addr, bmax);
    }
  } else {
    if ((tid & 31) == 0 && wmax != 0u) atomicMax(rmax_addr, wmax);
  }
}

// Exact selection among the n_c shared-memory candidates (all keys >= thr, n_c in
// [K, kCand]): radix select over r = key - thr in 12-bit digits, then emission of the keys
// above the k-th and the needed number equal to it. Whole CTA.
__device__ void select_and_emit(TopkSmem& sm, const TopkArgs& a, const TopkRow& rw, uint32_t n_c, uint32_t thr,
                                uint32_t rmax) {
  const int tid = threadIdx.x;
  const int K = rw.K;
  if (tid == 0) {
    sm.cnt_out = 0;
    sm.cnt_eq = 0;
  }
  int hi = rmax == 0u ? 0 : 32 - __clz(rmax);          // r fits in bits [0, hi)
  uint32_t prefix = 0u, pmask = 0u, remaining = static_cast<uint32_t>(K);
#pragma unroll 1
  while (true) {
    const int lo_bit = hi > 12 ? hi - 12 : 0;
    const uint32_t dm = (1u << (hi - lo_bit)) - 1u;      // hi - lo_bit in [0, 12]
    for (int i = tid; i < kHistBins; i += kTopkThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int c = tid; c < static_cast<int>(n_c); c += kTopkThreads) {
      const uint32_t r = sm.cand_key[c] - thr;
      if ((r & pmask) == prefix) atomicAdd(&sm.hist[(r >> lo_bit) & dm], 1u);
    }
    __syncthreads();
    select_bin(sm, remaining);
    prefix |= sm.sel_bin << lo_bit;
    pmask |= dm << lo_bit;
    remaining = sm.sel_rem;
    if (lo_bit == 0) break;
    hi = lo_bit;
  }
  const uint32_t kth = prefix, take_eq = remaining;
  const uint32_t n_gt = static_cast<uint32_t>(K) - take_eq;
  // each thread takes candidates tid, tid + 1024, ... (at most kCand / 1024)
  constexpr int kPer = kCand / kTopkThreads;
  uint32_t gts = 0, eqs = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int c = j * kTopkThreads + tid;
    if (c < static_cast<int>(n_c)) {
      const uint32_t r = sm.cand_key[c] - thr;
      if (r > kth) gts |= 1u << j;
      else if (r == kth) eqs |= 1u << j;
    }
  }
  uint32_t pg = warp_reserve(&sm.cnt_out, static_cast<uint32_t>(__popc(gts)));
  uint32_t pe = warp_reserve(&sm.cnt_eq, static_cast<uint32_t>(__popc(eqs)));
  // output positions and tokens first, then all block-table lookups, then the stores
  int pos[kPer], tok[kPer], page[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    pos[j] = -1;
    tok[j] = 0;
    const int c = j * kTopkThreads + tid;
    if (gts & (1u << j)) {
      if (pg < n_gt) { pos[j] = static_cast<int>(pg); tok[j] = sm.cand_idx[c]; }
      ++pg;
    } else if (eqs & (1u << j)) {
      if (pe < take_eq) { pos[j] = static_cast<int>(n_gt + pe); tok[j] = sm.cand_idx[c]; }
      ++pe;
    }
  }
  const int32_t* bt_row = a.block_table + static_cast<int64_t>(rw.b) * a.max_pages;
#pragma unroll
  for (int j = 0; j < kPer; ++j) page[j] = (rw.po != nullptr && pos[j] >= 0) ? __ldg(bt_row + (tok[j] >> 6)) : 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (page[j] < 0 || page[j] >= a.num_pages) {
      if (pos[j] >= 0) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(page[j]));
      page[j] = 0;
    }
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (pos[j] < 0) continue;
    if (rw.lo) rw.lo[pos[j]] = tok[j];
    if (rw.po) rw.po[pos[j]] = page[j] * kPage + (tok[j] & 63);
  }
}

// Whole-row exact radix select (12 + 12 + 8 bits); for rows where the sampled path missed
// or the row is not 16-byte aligned. Whole CTA.
__device__ void select_whole_row(TopkSmem& sm, const TopkArgs& a, const TopkRow& rw) {
  const int tid = threadIdx.x;
  const int K = rw.K;
  const int vis = rw.vis;
  const float* row = rw.row;
  auto emit = [&](int pos, int s) { topk_emit(a, rw, pos, s); };
  __syncthreads();
  // digit 1 (key bits 31..20) over the whole row
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

// One CTA per query: threshold, gather into shared memory, exact select.
__global__ void __launch_bounds__(kTopkThreads) topk_pagemap_kernel(const TopkArgs a) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);
  pdl_trigger();
  pdl_wait();   // scores come from the indexer
  const TopkRow rw = topk_row(a, blockIdx.x);
  if (rw.vis <= rw.K) {
    topk_dense(a, rw);
    return;
  }
  // The sampled path needs 16-byte aligned rows (always true for the fused layer, whose
  // row stride is a multiple of 64); other rows take the whole-row radix select.
  if ((reinterpret_cast<uintptr_t>(rw.row) & 15) == 0) {
    float4 first[kGatherU / 4];
    gather_load(rw.row, 0, rw.vis, first);   // in flight while the threshold is derived
    const uint32_t thr = row_threshold_small(sm, rw.row, rw.vis, rw.K);
    if (threadIdx.x == 0) {
      sm.n_cand = 0;
      sm.rmax = 0;
    }
    __syncthreads();
    gather_range(rw.row, 0, rw.vis, thr, &sm.n_cand, sm.cand_key, sm.cand_idx, kCand, &sm.rmax, first);
    __syncthreads();
    const uint32_t n_c = sm.n_cand;
    if (n_c >= static_cast<uint32_t>(rw.K) && n_c <= static_cast<uint32_t>(kCand)) {
      select_and_emit(sm, a, rw, n_c, thr, sm.rmax);
      return;
    }
  }
  select_whole_row(sm, a, rw);
}

// Rows gathered by a cluster of C = 2, 4 or 8 CTAs (query = cluster index): all derive the
// same threshold, each gathers one C-th of the row straight into the first CTA's candidate
// buffer (distributed shared memory, its counters and atomics), and after the cluster
// barrier the first CTA selects and emits. One SM pulls a row at ~16 B/cycle, so C of them
// divide the gather by C. Every branch taken before the barriers depends only on the row,
// the same in every CTA of the cluster.
__global__ void __launch_bounds__(kTopkThreads) topk_pair_kernel(const TopkArgs a) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();
  const int C = static_cast<int>(cluster.num_blocks());
  pdl_trigger();
  pdl_wait();   // scores come from the indexer
  const TopkRow rw = topk_row(a, static_cast<int>(blockIdx.x) / C);
  if (rw.vis <= rw.K) {
    if (rank == 0) topk_dense(a, rw);
    return;
  }
  if ((reinterpret_cast<uintptr_t>(rw.row) & 15) != 0) {
    if (rank == 0) select_whole_row(sm, a, rw);
    return;
  }
  const int part = ((rw.vis + C - 1) / C + 15) & ~15;   // a multiple of 4: 16-byte loads stay aligned
  const int lo = min(rw.vis, static_cast<int>(rank) * part);
  const int hi = min(rw.vis, lo + part);
  float4 first[kGatherU / 4];
  gather_load(rw.row, lo, hi, first);   // in flight while the threshold is derived
  const uint32_t thr = row_threshold_small(sm, rw.row, rw.vis, rw.K);
  if (threadIdx.x == 0) {
    sm.n_cand = 0;
    sm.rmax = 0;
  }
  cluster.sync();   // the first CTA's counters are zero before either half adds to them
  TopkSmem& dst = rank == 0 ? sm : *cluster.map_shared_rank(&sm, 0);
  gather_range(rw.row, lo, hi, thr, &dst.n_cand, dst.cand_key, dst.cand_idx, kCand, &dst.rmax, first);
  cluster.sync();   // every part's candidates are in the first CTA's buffer
  if (rank != 0) return;
  const uint32_t n_c = sm.n_cand;
  if (n_c >= static_cast<uint32_t>(rw.K) && n_c <= static_cast<uint32_t>(kCand)) {
    select_and_emit(sm, a, rw, n_c, thr, sm.rmax);
    return;
  }
  select_whole_row(sm, a, rw);
}

// Long rows, part 1: grid (chunks, queries). Each CTA derives the row's threshold (the same
// in every chunk CTA) and gathers the candidates of its 16K-key chunk into the row's
// global candidate buffer.
__global__ void __launch_bounds__(kTopkThreads) topk_gather_kernel(const TopkArgs a) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);
  pdl_trigger();
  pdl_wait();   // scores come from the indexer
  const TopkRow rw = topk_row(a, blockIdx.y);
  if (rw.vis <= rw.K || (reinterpret_cast<uintptr_t>(rw.row) & 15) != 0) return;   // handled by part 2
  const int lo_s = static_cast<int>(blockIdx.x) * kTopkChunk;
  if (lo_s >= rw.vis) return;
  const int hi_s = min(rw.vis, lo_s + kTopkChunk);
  float4 first[kGatherU / 4];
  gather_load(rw.row, lo_s, hi_s, first);   // in flight while the threshold is derived
  const uint32_t thr = row_threshold(sm, rw.row, rw.vis, rw.K);
  const int64_t q = rw.q;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.g_thr[q] = thr;
  gather_range<true>(rw.row, lo_s, hi_s, thr, a.g_cnt + q, a.g_key + q * a.cand_cap, a.g_idx + q * a.cand_cap,
               static_cast<uint32_t>(a.cand_cap), a.g_rmax + q, first, sm.wsum);
}

// Long rows, part 2: one CTA per query selects exactly among the gathered candidates
// (or the whole row when the estimate missed) and emits logical and physical indices.
__global__ void __launch_bounds__(kTopkThreads) topk_select_kernel(const TopkArgs a) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);
  pdl_trigger();
  pdl_wait();   // candidates come from part 1
  const TopkRow rw = topk_row(a, blockIdx.x);
  if (rw.vis <= rw.K) {
    topk_dense(a, rw);
    return;
  }
  const int64_t q = rw.q;
  const uint32_t n_c = a.g_cnt[q];
  if (n_c >= static_cast<uint32_t>(rw.K) && n_c <= static_cast<uint32_t>(kCand) && n_c <= static_cast<uint32_t>(a.cand_cap)) {
    const uint32_t* gk = a.g_key + q * a.cand_cap;
    const int32_t* gi = a.g_idx + q * a.cand_cap;
    // all of a thread's candidates in flight at once, then stored
    constexpr int kPer = kCand / kTopkThreads;
    uint32_t kk[kPer];
    int32_t ii[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = static_cast<int>(threadIdx.x) + j * kTopkThreads;
      kk[j] = 0u;
      ii[j] = 0;
      if (i < static_cast<int>(n_c)) {
        kk[j] = __ldcg(gk + i);
        ii[j] = __ldcg(gi + i);
      }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = static_cast<int>(threadIdx.x) + j * kTopkThreads;
      if (i < static_cast<int>(n_c)) {
        sm.cand_key[i] = kk[j];
        sm.cand_idx[i] = ii[j];
      }
    }
    __syncthreads();
    select_and_emit(sm, a, rw, n_c, a.g_thr[q], a.g_rmax[q]);
    return;
  }
  select_whole_row(sm, a, rw);
}

// The page-mapping transform alone: physical = table[b, i/64]*64 + i%64, -1 -> -1.
__global__ void pagemap_kernel(int n_q, int top_k, int64_t total, const int32_t* block_table, int max_pages,
                               int num_pages, const int32_t* logical, int32_t* physical, unsigned int* err) {
  pdl_trigger();
  pdl_wait();
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

int topk_chunks(int Bq, int64_t L_max, int sms) {
  // Very long rows (at least 128K keys) and few of them: split the gather over 16K-key
  // chunks, up to two CTAs per SM. Shorter rows are faster with one CTA each.
  if (Bq <= 0 || sms <= 0 || Bq >= sms || L_max < 8 * static_cast<int64_t>(kTopkChunk)) return 1;
  const int64_t want = (L_max + kTopkChunk - 1) / kTopkChunk;
  const int64_t room = (2 * static_cast<int64_t>(sms)) / Bq;
  const int64_t c = want < room ? want : room;
  return c < 2 ? 1 : static_cast<int>(c);
}

int topk_pairs(int Bq, int64_t L_max, int sms) {
  // every cluster resident at once (one 1024-thread CTA per SM), at least 16K keys per
  // CTA for pairs and 8K for larger clusters
  if (Bq <= 0 || sms <= 0) return 0;
  for (int c = 8; c >= 4; c >>= 1)
    if (static_cast<int64_t>(c) * Bq <= sms && L_max >= 8192LL * c) return c;
  return 2LL * Bq <= sms && L_max >= 32768 ? 2 : 0;
}

int topk_candidate_capacity() { return kCand; }

cudaError_t launch_topk(const TopkArgs& a, int Bq, cudaStream_t stream, int* launches) {
  const int smem = static_cast<int>(sizeof(TopkSmem));
  if (a.chunks <= 1 && a.pair > 1) {
    cudaError_t e = set_smem_once<topk_pair_kernel>(smem);
    if (e != cudaSuccess) return e;
    ++*launches;
    return launch_pdl_cluster(topk_pair_kernel, dim3(a.pair * Bq), dim3(kTopkThreads), smem, stream,
                              static_cast<unsigned>(a.pair), a);
  }
  if (a.chunks <= 1) {
    cudaError_t e = set_smem_once<topk_pagemap_kernel>(smem);
    if (e != cudaSuccess) return e;
    ++*launches;
    return launch_pdl(topk_pagemap_kernel, dim3(Bq), dim3(kTopkThreads), smem, stream, a);
  }
  cudaError_t e = set_smem_once<topk_gather_kernel>(smem);
  if (e == cudaSuccess) e = set_smem_once<topk_select_kernel>(smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(topk_gather_kernel, dim3(a.chunks, Bq), dim3(kTopkThreads), smem, stream, a);
  ++*launches;
  if (e != cudaSuccess) return e;
  ++*launches;
  return launch_pdl(topk_select_kernel, dim3(Bq), dim3(kTopkThreads), smem, stream, a);
}

cudaError_t launch_pagemap(int n_q, int top_k, int64_t total, const int32_t* block_table, int max_pages,
                           int num_pages, const int32_t* logical, int32_t* physical, unsigned int* err,
                           cudaStream_t stream, int* launches) {
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  ++*launches;
  return launch_pdl(pagemap_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, n_q, top_k, total,
                    block_table, max_pages, num_pages, logical, physical, err);
}

}  // namespace dsa
