// Stage 1 of the DSA decode step: the lightning indexer ("GLM-52 Runs on RTX 4090",
// kernel list item 1, "Lightning-indexer GEMM"):
//
//   score[q, s] = k_scale[slot(s)] * sum_h (w[q,h] * q_scale[q,h]) * ReLU(<q8[q,h], k8[slot(s)]>)
//
// Design (sm_100a): one persistent CTA per SM walks a contiguous range of tiles of the
// paged key cache: 512 tokens (eight 64-token pages, 64 KB) for fp8 decode, 256 tokens
// otherwise.
//   warp 0     TMA producer: one 64 x 128 B box per page, straight from the block table
//              (fetched a batch ahead), 128-byte swizzled, into a ring of stages (192 KB of
//              keys in flight for fp8 decode); query tiles into their own ring.
//   warp 1     tcgen05 issuer: per 128-token half, D[128 tokens, 64*g heads] =
//              K_half x Q_group^T, fp8 x fp8 (kind::f8f6f4) or bf16 x bf16 (kind::f16),
//              fp32 in a ring of TMEM accumulator units (two halves per unit for decode,
//              so one commit and one wait cover 256 tokens); MMAs come from an elected lane.
//   warps 2-9  epilogue, two groups of four taking alternate units: one thread per token
//              (its TMEM lane) applies ReLU, the head weights and the key scale (loaded two
//              tiles ahead) and writes the fp32 score.
// Every synchronisation step costs a few hundred nanoseconds, so tiles and units are large
// enough to keep that cost per byte low. The work items of a CTA are (row, query group,
// key tile) in that order, query group outer: a group of up to 4 queries (N = 256) and its
// head weights stay in place while the row's key tiles stream past it (from L2 after the
// first group), so decode (one group) and chunked prefill (many) load each query group
// once per row pass.
#include "kernels.cuh"

namespace dsa {

constexpr int kEpiWarps = 8;                 // two groups of four, alternating accumulators
constexpr int kIdxThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kIdxTmemCols = 512;       // accumulators of 64 * min(n_q, 4) columns each
constexpr int kPrefixRows = 1023;            // rows whose work-item prefix a CTA builds itself

// KC: 128-byte K-chunks per row (1 = fp8, 2 = bf16). QG: queries per group (1 for decode,
// 4 for chunked prefill). Decode needs only one query per group, so its query slots and
// head-weight buffers are small and the key ring holds 192 KB: about what page streaming
// needs in flight per SM to approach the copy rate.
template <int KC, int QG>
struct IdxCfg {
  // fp8 decode walks 512-token tiles (eight pages, 64 KB) so that the per-tile barrier work
  // of the tcgen05 issuer is paid per 64 KB; the other forms use 256-token tiles.
  static constexpr int kTileTok = (KC == 1 && QG == 1) ? 512 : 256;
  static constexpr int kPagesPerTile = kTileTok / kPage;
  static constexpr int kBatch = 32 / kPagesPerTile;   // tiles whose block-table entries the producer fetches at once
  static constexpr int kHalves = kTileTok / 128;       // 128-token MMA halves (M = 128) per tile
  // Decode: one accumulator unit per tile, signalled by the stage's own completion barrier
  // (one wait and one commit per tile for the issuer). Prefill: one unit per half and query group.
  static constexpr int kUnitHalves = QG == 1 ? kHalves : 1;
  static constexpr int kChunk = kTileTok * 128;        // one 128-byte K-chunk of a tile
  static constexpr int kStages = KC == 1 ? (QG == 1 ? 3 : 4) : 2;
  static constexpr int kBSlots = (KC == 2 && QG == 4) ? 1 : 2;
  static constexpr int kAStage = KC * kChunk;          // 256 tokens x 128 B per K-chunk
  static constexpr int kQChunk = QG * 8192;            // QG queries x 64 heads x 128 B
  static constexpr int kBSlot = KC * kQChunk;
  static constexpr int kWPer = kHeads * QG;            // head weights of one query group
  static constexpr int kWBytes = kEpiWarps * 2 * kWPer * 4;  // per-warp double-buffered head weights
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kAStage;
  static constexpr int kOffW = kOffB + kBSlots * kBSlot;
  static constexpr int kOffBar = kOffW + kWBytes;
  static constexpr int kMaxAcc = 8;
  static constexpr int kNumBars = 2 * kStages + 2 * kBSlots + 2 * kMaxAcc + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // the work-item prefix when the kernel builds it itself (up to kPrefixRows rows)
  static constexpr int kOffPrefix = kOffMisc + 64;
  static constexpr int kSmem = kOffPrefix + 4 * (kPrefixRows + 1) + 1024;  // + slack to align the base to 1024
};
static_assert(IdxCfg<1, 1>::kHalves / IdxCfg<1, 1>::kUnitHalves == 1 &&
                  IdxCfg<1, 4>::kHalves / IdxCfg<1, 4>::kUnitHalves == 2 &&
                  IdxCfg<2, 1>::kHalves / IdxCfg<2, 1>::kUnitHalves == 1,
              "units per tile");
static_assert(IdxCfg<1, 1>::kSmem <= 232448 && IdxCfg<1, 4>::kSmem <= 232448 && IdxCfg<2, 1>::kSmem <= 232448 &&
                  IdxCfg<2, 4>::kSmem <= 232448,
              "shared memory");

// Walks the CTA's contiguous range of global work items, yielding (row, query group, key
// tile) and the row's clamped length: a row's items are its query groups times its key
// tiles, group-major. Row bounds and lengths live in registers and are reloaded only when
// the walk crosses into the next row.
// The longest visible prefix among query group g of row b (out of line: every role's
// walker calls it once per group).
template <int QG>
__device__ __noinline__ int group_vis(const int32_t* q_pos, int n_q, int b, int g, int len) {
  int v = 0;
  const int q0 = b * n_q + g * QG;
  const int nqg = min(QG, n_q - g * QG);
  for (int j = 0; j < nqg; ++j) v = max(v, query_vis(q_pos, q0 + j, len));
  return v;
}

// kVis: also report whether the item is active (a query of its group sees a token of its
// tile); walkers that only look ahead (key-scale prefetch) take every item as active.
template <int QG, bool kVis = true>
struct TileWalker {
  const int32_t* prefix;
  const int32_t* seq_lens;
  const int32_t* q_pos;
  int max_pages, tile_tok, n_q;
  int b, gt, end, base, bound, len, tiles;
  int vis_b, vis_g, gvis;   // the group whose visible length gvis is cached
  __device__ void init(const IndexerArgs& a, const int32_t* item_prefix, int tile_tokens, int begin, int stop) {
    prefix = item_prefix;
    seq_lens = a.seq_lens;
    q_pos = a.q_pos;
    n_q = a.n_q;
    max_pages = a.max_pages;
    tile_tok = tile_tokens;
    vis_b = vis_g = -1;
    gvis = 0;
    gt = begin;
    end = stop;
    int lo = 0, hi = a.B;  // largest b with prefix[b] <= begin
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= begin) lo = mid; else hi = mid;
    }
    b = lo;
    base = prefix[b];
    bound = prefix[b + 1];
    len = row_len(seq_lens, b, max_pages);
    tiles = (len + tile_tok - 1) / tile_tok;
  }
  // `active`: a query of the group sees a token of the tile (every role skips the others)
  __device__ bool next(int& row, int& group, int& tile, int& L, bool& active) {
    if (gt >= end) return false;
    while (gt >= bound) {
      ++b;
      base = bound;
      bound = prefix[b + 1];
      len = row_len(seq_lens, b, max_pages);
      tiles = (len + tile_tok - 1) / tile_tok;
    }
    row = b;
    const int i = gt - base;   // < groups * tiles, so tiles >= 1 here
    if (QG == 1 || n_q <= QG) {   // one group per row: the item is the tile
      group = 0;
      tile = i;
    } else {
      group = i / tiles;
      tile = i - group * tiles;
    }
    L = len;
    if (kVis) {
      if (b != vis_b || group != vis_g) {
        vis_b = b;
        vis_g = group;
        gvis = group_vis<QG>(q_pos, n_q, b, group, len);
      }
      active = gvis > tile * tile_tok;
    } else {
      active = true;
    }
    ++gt;
    return true;
  }
};

template <int KC, int QG>
__global__ void __launch_bounds__(kIdxThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                   const IndexerArgs a) {
  using C = IdxCfg<KC, QG>;
  constexpr int kTileTok = C::kTileTok;
  constexpr int kPagesPerTile = C::kPagesPerTile;
  constexpr int kBatch = C::kBatch;
  constexpr int UH = C::kUnitHalves;
  constexpr int kUnitsPerTile = C::kHalves / UH;
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
  uint64_t* acc_empty = acc_full + C::kMaxAcc;
  uint64_t* drain = acc_empty + C::kMaxAcc;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // accumulator ring: 64 columns per query of a group; decode (n_q = 1) gets 8 of them
  const int acc_cols = kHeads * min(a.n_q, QG);        // one 128-token half
  const int unit_cols = UH * acc_cols;
  const int n_acc = min(C::kMaxAcc, static_cast<int>(kIdxTmemCols) / unit_cols);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);   // the MMA commit
    }
    for (int i = 0; i < C::kBSlots; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < C::kMaxAcc; ++i) {
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
  pdl_trigger();
  pdl_wait();   // the tile prefix comes from the plan kernel

  // the work-item prefix: from the plan kernel, or built here for up to kPrefixRows rows
  // (each CTA scans the rows' item counts itself; CTA 0 also checks the inputs)
  const int32_t* prefix = a.tile_prefix;
  if (prefix == nullptr) {
    int32_t* sp = reinterpret_cast<int32_t*>(smem + C::kOffPrefix);
    int* wsum = reinterpret_cast<int*>(smem + C::kOffMisc + 16);   // 10 warp totals
    const int groups = QG == 1 ? 1 : (a.n_q + QG - 1) / QG;
    const int tid = threadIdx.x;
    int carry = 0;
    for (int base = 0; base < a.B; base += kIdxThreads) {
      const int b = base + tid;
      int v = 0;
      if (b < a.B) v = groups * ((row_len(a.seq_lens, b, a.max_pages) + kTileTok - 1) / kTileTok);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
      }
      if (lane == 31) wsum[warp] = v;
      __syncthreads();
      int before = carry, tot = 0;
      for (int w = 0; w < kIdxThreads / 32; ++w) {
        if (w < warp) before += wsum[w];
        tot += wsum[w];
      }
      if (b < a.B) sp[b + 1] = before + v;
      carry += tot;
      __syncthreads();
    }
    if (tid == 0) sp[0] = 0;
    if (blockIdx.x == 0) {
      for (int b = tid; b < a.B; b += kIdxThreads) {
        const int raw = a.seq_lens[b];
        if (raw < 0 || raw > a.max_pages * kPage) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(raw));
      }
      if (a.q_pos != nullptr)
        for (int q = tid; q < a.B * a.n_q; q += kIdxThreads) {
          const int L = row_len(a.seq_lens, q / a.n_q, a.max_pages);
          const int p = a.q_pos[q];
          if (p < 0 || p >= L) record_error(a.err, DSA_ERR_DEVICE_BOUNDS, static_cast<unsigned int>(p));
        }
    }
    __syncthreads();
    prefix = sp;
  }
  const int total = prefix[a.B];
  const int per = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  const int t_begin = min(total, static_cast<int>(blockIdx.x) * per);
  const int t_end = min(total, t_begin + per);

  if (t_begin < t_end) {
    TileWalker<QG> walk;
    walk.init(a, prefix, kTileTok, t_begin, t_end);

    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer (whole warp)
      // Lane 4i+p holds page p of batch tile i; the next batch's block-table loads are in
      // flight while this one is issued. Lane 0 issues the page boxes and query tiles.
      if (lane == 0) {
        tma_prefetch_map(&tmap_k);
        tma_prefetch_map(&tmap_q);
      }
      int it = 0, bit = -1, cur_q0 = -1;
      bool ok = true;
      // With one query group per row every key page is read once: it goes to L2 as first to
      // be evicted, so that the streamed keys do not displace the scores, which the top-k
      // reads next. With several groups the row's keys are read again from L2.
      const bool keys_once = a.n_q <= QG;
      const uint64_t evict_first = l2_evict_first_policy();
      // lanes hold the items of a batch; inactive items are marked by my_act = 0
      auto load_batch = [&](int& n, int& my_b, int& my_g, int& my_t, int& my_act, int& my_page) {
        n = 0;
        my_b = my_g = my_t = my_act = 0;
        int my_L = 0;
        for (; n < kBatch; ++n) {
          int b, g, t, L;
          bool act;
          if (!walk.next(b, g, t, L, act)) break;
          if (lane / kPagesPerTile == n) { my_b = b; my_g = g; my_t = t; my_L = L; my_act = act ? 1 : 0; }
        }
        my_page = -1;
        if (lane / kPagesPerTile < n && my_act) {
          const int p = kPagesPerTile * my_t + (lane % kPagesPerTile);
          if (p * kPage < my_L) my_page = checked_page(a.block_table, my_b, p, a.max_pages, a.num_pages, a.err);
        }
      };
      int n, my_b, my_g, my_t, my_act, my_page;
      load_batch(n, my_b, my_g, my_t, my_act, my_page);
      while (ok && n > 0) {
        int n2, nb, ng, nt, nact, npg;
        load_batch(n2, nb, ng, nt, nact, npg);
        for (int i = 0; i < n; ++i) {
          const int src = kPagesPerTile * i;
          if (!__shfl_sync(0xffffffffu, my_act, src)) continue;   // every role skips the item
          const int b = __shfl_sync(0xffffffffu, my_b, src);
          const int g = __shfl_sync(0xffffffffu, my_g, src);
          int pages[kPagesPerTile];
#pragma unroll
          for (int p = 0; p < kPagesPerTile; ++p) pages[p] = __shfl_sync(0xffffffffu, my_page, src + p);
          const int s = it % C::kStages;
          if (!wait_warp(&a_empty[s], ((it / C::kStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
          if (lane == 0) {
            uint32_t npages = 0;
#pragma unroll
            for (int p = 0; p < kPagesPerTile; ++p) npages += pages[p] >= 0 ? 1u : 0u;
            mbar_arrive_expect_tx(&a_full[s], npages * KC * 8192u);
            uint8_t* dst = sA + s * C::kAStage;
#pragma unroll
            for (int p = 0; p < kPagesPerTile; ++p)
              if (pages[p] >= 0)
#pragma unroll
                for (int kc = 0; kc < KC; ++kc) {
                  if (keys_once)
                    tma_load_2d_hint(dst + kc * C::kChunk + p * 8192, &tmap_k, kc * 64, pages[p] * kPage, &a_full[s],
                                     evict_first);
                  else
                    tma_load_2d(dst + kc * C::kChunk + p * 8192, &tmap_k, kc * 64, pages[p] * kPage, &a_full[s]);
                }
          }
          ++it;
          const int q0 = b * a.n_q + g * QG;
          if (q0 != cur_q0) {
            const int nqg = min(QG, a.n_q - g * QG);
            ++bit;
            const int bs = bit % C::kBSlots;
            if (!wait_warp(&b_empty[bs], ((bit / C::kBSlots) & 1) ^ 1, abort_flag)) { ok = false; break; }
            if (lane == 0) {
              mbar_arrive_expect_tx(&b_full[bs], static_cast<uint32_t>(nqg) * KC * 8192u);
              for (int j = 0; j < nqg; ++j)
#pragma unroll
                for (int kc = 0; kc < KC; ++kc)
                  tma_load_2d(sB + bs * C::kBSlot + kc * C::kQChunk + j * 8192, &tmap_q, kc * 64, (q0 + j) * kHeads,
                              &b_full[bs]);
            }
            cur_q0 = q0;
          }
        }
        n = n2; my_b = nb; my_g = ng; my_t = nt; my_act = nact; my_page = npg;
      }
      if (!ok && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 1);
        *abort_flag = 1;
      }
      if (lane == 0) {
        for (int i = max(0, it - C::kStages); i < it; ++i) wait_drain(&a_full[i % C::kStages], (i / C::kStages) & 1);
        for (int i = max(0, bit - C::kBSlots + 1); i <= bit; ++i)
          wait_drain(&b_full[i % C::kBSlots], (i / C::kBSlots) & 1);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------ tcgen05 issuer (whole warp)
      // Descriptors are formed once and advanced by constants (the start address field is
      // address / 16); the MMAs and their commits come from one elected lane.
      const uint32_t fmt = KC == 1 ? 0u : 1u;  // e4m3 (kind::f8f6f4) or bf16 (kind::f16)
      const uint64_t a_desc0 = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      int it = 0, bit = -1, cur_q0 = -1, unit = 0;
      bool ok = true;
      int b, g, t, L;
      bool act;
      while (ok && walk.next(b, g, t, L, act)) {
        if (!act) continue;
        const int s = it % C::kStages;
        if (!wait_warp(&a_full[s], (it / C::kStages) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = a_desc0 + static_cast<uint64_t>((s * C::kAStage) >> 4);
        {
          const int q0 = b * a.n_q + g * QG;
          const int nqg = min(QG, a.n_q - g * QG);
          if (q0 != cur_q0) {
            if (bit >= 0) {
              if (elect_one()) tc_commit(&b_empty[bit % C::kBSlots]);
              __syncwarp();
            }
            ++bit;
            if (!wait_warp(&b_full[bit % C::kBSlots], (bit / C::kBSlots) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            cur_q0 = q0;
          }
          const uint32_t idesc = idesc_make(fmt, fmt, false, false, 128, kHeads * nqg);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(((bit % C::kBSlots) * C::kBSlot) >> 4);
          for (int u = 0; u < kUnitsPerTile; ++u, ++unit) {
            const int ab = unit % n_acc;
            if (!wait_warp(&acc_empty[ab], ((unit / n_acc) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
              for (int hh = 0; hh < UH; ++hh) {
                const int h2 = u * UH + hh;
                const uint32_t d = tmem + static_cast<uint32_t>(ab * unit_cols + hh * acc_cols);
#pragma unroll
                for (int kc = 0; kc < KC; ++kc)
#pragma unroll
                  for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t ao = ad + static_cast<uint64_t>((kc * C::kChunk + h2 * 16384 + ks * 32) >> 4);
                    const uint64_t bo = bd + static_cast<uint64_t>((kc * C::kQChunk + ks * 32) >> 4);
                    if (KC == 1) mma_f8(d, ao, bo, idesc, (kc | ks) != 0);
                    else mma_f16(d, ao, bo, idesc, (kc | ks) != 0);
                  }
              }
              if (QG != 1) tc_commit(&acc_full[ab]);   // decode: the stage commit below signals it
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit(&a_empty[s]);
        __syncwarp();
        ++it;
      }
      if (!ok && lane == 0) {
        record_error(a.err, DSA_ERR_TIMEOUT, 2);
        *abort_flag = 1;
      }
      // every MMA this warp issued has finished before the CTA frees TMEM
      if (elect_one()) {
        tc_commit(drain);
        wait_drain(drain, 0);
      }
      __syncwarp();
    } else {
      // ------------------------------------------------------------ epilogue (warps 2..9)
      // Two groups of four warps take alternate accumulator units (a unit = UH 128-token
      // halves of a tile for one query group); in a group, warp w reads TMEM lanes
      // [32*(w%4), 32*(w%4)+32), one token of every half per thread. Each thread loads the
      // key scales of its tokens of a tile two tiles ahead, from block-table entries
      // loaded four tiles ahead, so neither load stalls the tile it is used in.
      constexpr int H = C::kHalves;
      const int eg = (warp - 2) >> 2;
      const int quarter = warp & 3;
      const int row_in_half = quarter * 32 + lane;
      const int off = row_in_half & 63;
      float* wmine = sW + (warp - 2) * 2 * C::kWPer;   // two buffers of one group's weights per warp
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      int unit = 0, cur_q0 = -1, wb = 1;
      int qvis[QG];   // visible lengths of the current group's queries (clamped to L_max)
#pragma unroll
      for (int j = 0; j < QG; ++j) qvis[j] = 0;
      bool ok = true;
      TileWalker<QG, false> w2, w4;
      w2.init(a, prefix, kTileTok, t_begin, t_end);
      // pages of this thread's tokens in every half of the next tile of walker w (-1 past the end)
      auto tile_pages = [&](TileWalker<QG, false>& w, int (&p)[H]) {
        int bb, gg, tt, LL;
        bool aa;
#pragma unroll
        for (int h = 0; h < H; ++h) p[h] = -1;
        if (!w.next(bb, gg, tt, LL, aa)) return;
        if (a.k_scale == nullptr || !aa) return;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          const int tk = tt * kTileTok + h * 128 + row_in_half;
          if (tk < LL) p[h] = checked_page(a.block_table, bb, tk >> 6, a.max_pages, a.num_pages, a.err);
        }
      };
      auto load_scale = [&](int page) {
        return page >= 0 ? __ldg(a.k_scale + static_cast<int64_t>(page) * kPage + off) : 1.0f;
      };
      int pa[H], pb[H], pc[H], pd[H];
      float ks0[H], ks1[H];
      tile_pages(w2, pa);
      tile_pages(w2, pb);
#pragma unroll
      for (int h = 0; h < H; ++h) {
        ks0[h] = load_scale(pa[h]);   // tile +0
        ks1[h] = load_scale(pb[h]);   // tile +1
      }
      w4 = w2;
      tile_pages(w4, pc);             // tile +2
      tile_pages(w4, pd);             // tile +3
      int b, g, t, L;
      bool act;
      while (ok && walk.next(b, g, t, L, act)) {
        float kscale[H];
#pragma unroll
        for (int h = 0; h < H; ++h) {
          kscale[h] = ks0[h];
          ks0[h] = ks1[h];
          ks1[h] = load_scale(pc[h]);
          pc[h] = pd[h];
        }
        tile_pages(w4, pd);
        const int tok0 = t * kTileTok;
        if (!act) continue;
        {
          const int q0 = b * a.n_q + g * QG;
          const int nqg = min(QG, a.n_q - g * QG);
#pragma unroll 1
          for (int u = 0; u < kUnitsPerTile; ++u, ++unit) {
            if ((unit & 1) != eg) continue;
            if (q0 != cur_q0) {
              wb ^= 1;
              __syncwarp();
              for (int i = lane; i < nqg * kHeads; i += 32) {
                float w = a.head_w[static_cast<int64_t>(q0) * kHeads + i];
                if (a.q_scale != nullptr) w *= a.q_scale[static_cast<int64_t>(q0) * kHeads + i];
                wmine[wb * C::kWPer + i] = w;
              }
#pragma unroll
              for (int j = 0; j < QG; ++j) {
                int v = j < nqg ? query_vis(a.q_pos, q0 + j, L) : 0;
                qvis[j] = v > a.L_max ? static_cast<int>(a.L_max) : v;
              }
              __syncwarp();
              cur_q0 = q0;
            }
            const int ab = unit % n_acc;
            // decode: unit == tile index, and the tile's stage barrier completes with its MMAs
            const bool got = QG == 1 ? wait_warp(&a_empty[unit % C::kStages], (unit / C::kStages) & 1, abort_flag)
                                     : wait_warp(&acc_full[ab], (unit / n_acc) & 1, abort_flag);
            if (!got) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int hh = 0; hh < UH; ++hh) {
              const int h2 = u * UH + hh;
              const int tok = tok0 + h2 * 128 + row_in_half;
#pragma unroll 1
              for (int j = 0; j < nqg; ++j) {
                float acc[64];
                tmem_ld64(lane_addr + static_cast<uint32_t>(ab * unit_cols + hh * acc_cols + j * kHeads), acc);
                const float4* wq = reinterpret_cast<const float4*>(wmine + wb * C::kWPer + j * kHeads);
                // ReLU per head, then head pairs through packed fp32x2 FMAs: eight independent
                // chains (head h feeds chain 4 (h / 4 & 1) + h % 4), as four packed registers
                uint64_t pp[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int h4 = 0; h4 < 16; ++h4) {
                  const float4 w = wq[h4];
                  uint64_t* c = pp + 2 * (h4 & 1);
                  c[0] = fma_f32x2(pack_f32x2(w.x, w.y),
                                   pack_f32x2(fmaxf(acc[4 * h4 + 0], 0.0f), fmaxf(acc[4 * h4 + 1], 0.0f)), c[0]);
                  c[1] = fma_f32x2(pack_f32x2(w.z, w.w),
                                   pack_f32x2(fmaxf(acc[4 * h4 + 2], 0.0f), fmaxf(acc[4 * h4 + 3], 0.0f)), c[1]);
                }
                float part[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float2 f = unpack_f32x2(pp[i]);
                  part[2 * i] = f.x;
                  part[2 * i + 1] = f.y;
                }
                const float sc =
                    ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
                int vis = qvis[0];
#pragma unroll
                for (int jj = 1; jj < QG; ++jj)
                  if (jj == j) vis = qvis[jj];
                if (tok < vis) a.scores[static_cast<int64_t>(q0 + j) * a.L_max + tok] = sc * kscale[h2];
              }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
          }
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

// Work-item prefix over rows (query groups x key tiles per row; single CTA) plus validation
// of lengths and causal positions.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* seq_lens, const int32_t* q_pos, int B, int n_q,
                                                    int max_pages, int tile_tok, int groups, int32_t* tile_prefix,
                                                    unsigned int* err) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();
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
      tiles = groups * ((row_len(seq_lens, b, max_pages) + tile_tok - 1) / tile_tok);
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



int indexer_tile_tokens(bool fp8, int n_q) {
  if (n_q == 1) return fp8 ? IdxCfg<1, 1>::kTileTok : IdxCfg<2, 1>::kTileTok;
  return fp8 ? IdxCfg<1, 4>::kTileTok : IdxCfg<2, 4>::kTileTok;
}

int indexer_prefix_rows() { return kPrefixRows; }

int indexer_query_groups(int n_q) { return n_q == 1 ? 1 : (n_q + 3) / 4; }

cudaError_t launch_plan(const int32_t* seq_lens, const int32_t* q_pos, int B, int n_q, int max_pages, int tile_tok,
                        int32_t* tile_prefix, unsigned int* err, cudaStream_t stream, int* launches) {
  ++*launches;
  return launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, stream, seq_lens, q_pos, B, n_q, max_pages, tile_tok,
                    indexer_query_groups(n_q), tile_prefix, err);
}

template <int KC, int QG>
static cudaError_t launch_indexer_kc(const CUtensorMap& tk, const CUtensorMap& tq, const IndexerArgs& a, int grid,
                                     cudaStream_t stream) {
  constexpr int smem = IdxCfg<KC, QG>::kSmem;
  cudaError_t e = set_smem_once<indexer_kernel<KC, QG>>(smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(indexer_kernel<KC, QG>, dim3(grid), dim3(kIdxThreads), smem, stream, tk, tq, a);
}

cudaError_t launch_indexer(bool fp8, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q, const IndexerArgs& a,
                           int grid, cudaStream_t stream, int* launches) {
  ++*launches;
  if (a.n_q == 1)
    return fp8 ? launch_indexer_kc<1, 1>(tmap_k, tmap_q, a, grid, stream)
               : launch_indexer_kc<2, 1>(tmap_k, tmap_q, a, grid, stream);
  return fp8 ? launch_indexer_kc<1, 4>(tmap_k, tmap_q, a, grid, stream)
             : launch_indexer_kc<2, 4>(tmap_k, tmap_q, a, grid, stream);
}

}  // namespace dsa
