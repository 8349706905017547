"""CUDA path (through the C ABI) against the fp64 oracle, element by element."""
import functools

import numpy as np
import pytest

from dsa_inputs import CaseSpec, generate, spec
import oracle
from tests.compare import (score_magnitude, check_scores, check_topk_exact, check_topk_near_tie,
                           check_attention)

pytestmark = pytest.mark.gpu

SMALL = {
    "ragged_fp8": CaseSpec("ragged_fp8", (37, 64, 200, 1, 129), top_k=64, seed=31),
    "len_eq_topk": CaseSpec("len_eq_topk", (64, 65, 128, 63), top_k=64, seed=32),
    "bf16_small": CaseSpec("bf16_small", (130, 70, 300), top_k=32, idx_dtype="bf16", kv_dtype="bf16",
                           out_dtype="fp32", seed=33),
    "prefill_small": CaseSpec("prefill_small", (300,), top_k=64, n_q=6, q_pos=(0, 63, 64, 150, 298, 299),
                              n_planted=0, seed=34),
    "empty_row": CaseSpec("empty_row", (0, 50, 700), top_k=96, seed=35),
    "many_rows": CaseSpec("many_rows", tuple(range(40, 40 + 37 * 97, 97)), top_k=128, seed=36),
    "wide_table": CaseSpec("wide_table", (500, 1000), top_k=256, max_pages=40, extra_pages=7, seed=37),
    # speculative decode: every row's last n_q positions are queries (causal, so they see
    # L - n_q + 1 .. L tokens); one row is shorter than top_k and takes the dense path
    "mtp_small": CaseSpec("mtp_small", (300, 1000, 70, 2100), top_k=128, n_q=3, q_tail=True, n_planted=0,
                          seed=38),
    # packed 656-byte latent rows (E4M3 codes, four fp32 scales, bf16 rope) on ragged rows
    "packed_fp8": CaseSpec("packed_fp8", (37, 64, 200, 1, 129), top_k=64, kv_dtype="fp8r", seed=40),
    "mtp_bf16": CaseSpec("mtp_bf16", (129, 640), top_k=64, n_q=4, q_tail=True, idx_dtype="bf16", kv_dtype="bf16",
                         out_dtype="fp32", n_planted=0, seed=39),
    # chunked prefill with causal queries spread from the first token to the shortest row's
    # end (nine queries: two full query groups and a partial one; the same positions in
    # every row), so that many (query group, key tile) work items of the indexer see no
    # token, in the longer rows whole runs of tiles, and are skipped by every role
    "prefill_spread": CaseSpec("prefill_spread", (5000, 3000, 1200), top_k=256, n_q=9,
                               q_pos=(0, 100, 255, 256, 511, 700, 900, 1100, 1199), n_planted=0, seed=41),
    # more rows than an indexer CTA builds its work-item prefix for: the plan kernel builds it
    "many_rows_plan": CaseSpec("many_rows_plan", tuple((i * 37) % 97 + 1 for i in range(1100)), top_k=32,
                               seed=46),
    "prefill_spread_bf16": CaseSpec("prefill_spread_bf16", (700, 2100), top_k=128, n_q=5,
                                    q_pos=(3, 255, 256, 511, 699),
                                    idx_dtype="bf16", kv_dtype="bf16", out_dtype="fp32", n_planted=0, seed=42),
}
FULL = ["cfg0", "cfg1"]


@functools.lru_cache(maxsize=None)
def get_case(name):
    if name in SMALL:
        return generate(SMALL[name])
    return generate(spec(name))


@functools.lru_cache(maxsize=None)
def gpu_case(name):
    from tests.gpu_path import GpuCase
    return GpuCase(get_case(name))


@functools.lru_cache(maxsize=None)
def oracle_scores(name):
    return oracle.indexer_scores(get_case(name))


ALL = list(SMALL) + FULL


@pytest.mark.parametrize("name", ALL)
def test_indexer_scores(name):
    case = get_case(name)
    scores, err = gpu_case(name).indexer()
    assert err == 0
    ref = oracle_scores(name)
    check_scores(scores.cpu().numpy(), ref, score_magnitude(case), oracle.visible_lengths(case))


@pytest.mark.parametrize("name", ALL)
def test_topk_exact_on_same_scores(name):
    """Selection on identical fp32 scores (the GPU's own) is exact."""
    case = get_case(name)
    g = gpu_case(name)
    scores, _ = g.indexer()
    lo, ph, err = g.topk(scores)
    assert err == 0
    s32 = scores.cpu().numpy()
    vis = oracle.visible_lengths(case)
    for q in range(case["Bq"]):
        check_topk_exact(lo[q], s32[q], vis[q], case["top_k"])
    assert np.array_equal(ph, oracle.pagemap(case, lo.astype(np.int64)))


@pytest.mark.parametrize("name", ALL)
def test_pagemap_bit_exact(name):
    case = get_case(name)
    rng = np.random.default_rng(7)
    vis = oracle.visible_lengths(case)
    K = case["top_k"]
    logical = np.full((case["Bq"], K), -1, dtype=np.int64)
    for q in range(case["Bq"]):
        n = min(K, int(vis[q]))
        if n:
            logical[q, :n] = rng.choice(int(vis[q]), n, replace=False)
        rng.shuffle(logical[q])
    ph, err = gpu_case(name).pagemap(logical)
    assert err == 0
    assert np.array_equal(ph.astype(np.int64), oracle.pagemap(case, logical))


@pytest.mark.parametrize("name", ALL)
def test_mla_sparse_decode(name):
    """Attention alone, on the oracle's own selection."""
    case = get_case(name)
    ref_sel = oracle.topk_logical(oracle_scores(name), oracle.visible_lengths(case), case["top_k"])
    phys = oracle.pagemap(case, ref_sel)
    out, lse, err = gpu_case(name).mla(phys)
    assert err == 0
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys)
    check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"])


@pytest.mark.parametrize("name", ALL)
def test_decode_layer(name):
    case = get_case(name)
    r = gpu_case(name).layer()
    assert r["err"] == 0
    ref_scores = oracle_scores(name)
    vis = oracle.visible_lengths(case)
    ref_sel = oracle.topk_logical(ref_scores, vis, case["top_k"])
    for q in range(case["Bq"]):
        check_topk_near_tie(r["logical"][q], ref_sel[q], ref_scores[q], vis[q], case["top_k"])
    assert np.array_equal(r["physical"].astype(np.int64), oracle.pagemap(case, r["logical"].astype(np.int64)))
    # attention graded on the GPU's own selection, isolating it from legal near-tie swaps
    ref_out, ref_lse = oracle.mla_sparse_attention(case, r["physical"].astype(np.int64))
    check_attention(r["out"], r["lse"], ref_out, ref_lse, case["kv_dtype"])


def test_split_count_independence():
    """Different split counts (batch sizes) give the same per-query attention."""
    import deepseek_sparse_attention_head_b200 as dsa
    case = get_case("cfg1")
    ref_sel = oracle.topk_logical(oracle_scores("cfg1"), oracle.visible_lengths(case), case["top_k"])
    phys = oracle.pagemap(case, ref_sel)
    g = gpu_case("cfg1")
    full, _, _ = g.mla(phys)                 # 8 queries -> many splits each
    one, _, _ = g.mla(phys[:1])              # 1 query  -> even more splits
    assert dsa.mla_num_splits(1, case["top_k"]) != dsa.mla_num_splits(8, case["top_k"])
    assert np.max(np.abs(full[0] - one[0])) <= 2e-3


def _topk_on_scores(scores_np, vis, top_k, seed=40):
    """Runs dsa_topk_pagemap on caller-chosen fp32 scores (one query per row)."""
    import torch
    import deepseek_sparse_attention_head_b200 as dsa
    from tests.gpu_path import GpuCase
    B, L = scores_np.shape
    case = generate(CaseSpec("topk_custom", tuple(int(v) for v in vis), top_k=top_k, n_planted=0, seed=seed,
                             max_pages=(L + 63) // 64))
    g = GpuCase(case)
    s = torch.from_numpy(np.ascontiguousarray(scores_np.astype(np.float32))).cuda()
    lo, ph, err = g.topk(s, top_k)
    return case, lo, ph, err


def test_topk_ties_and_candidate_overflow():
    """Constant and few-valued rows put every key in one first-digit bin, overflowing the
    shared-memory candidate buffer and taking the global-refinement path."""
    rng = np.random.default_rng(3)
    L = 20032
    rows = [np.full(L, 0.5), rng.choice([0.25, 0.5, 1.0], size=L), rng.standard_normal(L) * 1e-3 + 7.0,
            np.linspace(-3, 3, L)[rng.permutation(L)], -np.abs(rng.standard_normal(L))]
    scores = np.stack(rows)
    vis = np.array([L, L - 5, 19000, L, 12345])
    case, lo, ph, err = _topk_on_scores(scores, vis, 777)
    assert err == 0
    for i in range(len(rows)):
        check_topk_exact(lo[i], scores[i].astype(np.float32), vis[i], 777)
    assert np.array_equal(ph, oracle.pagemap(case, lo.astype(np.int64)))


def test_topk_extreme_values():
    rng = np.random.default_rng(4)
    L = 4096
    base = rng.standard_normal((3, L)).astype(np.float32)
    base[0, ::7] = np.float32(3.0e38)
    base[1, ::5] = -np.float32(3.0e38)
    base[2, :] = np.float32(1e-40) * rng.integers(-5, 5, L)   # subnormals and zeros of both signs
    vis = np.array([L, L, 4000])
    case, lo, ph, err = _topk_on_scores(base, vis, 300)
    assert err == 0
    for i in range(3):
        check_topk_exact(lo[i], base[i], vis[i], 300)


def test_topk_unaligned_rows():
    """A row stride that is not a multiple of 4 floats leaves rows unaligned for 16-byte
    loads; those rows take the whole-row radix path and must select the same sets."""
    rng = np.random.default_rng(5)
    L = 4099
    scores = rng.standard_normal((3, L)).astype(np.float32)
    scores[1, ::97] += 4.0
    vis = np.array([L, L - 3, 3000])
    case, lo, ph, err = _topk_on_scores(scores, vis, 512)
    assert err == 0
    for i in range(3):
        check_topk_exact(lo[i], scores[i], vis[i], 512)
    assert np.array_equal(ph, oracle.pagemap(case, lo.astype(np.int64)))


def test_topk_long_rows_chunked_path():
    """Rows of 200K keys take the chunked gather (one CTA per 16K keys, per-row candidates
    in the workspace). The constant row overflows the candidate buffer and falls back to
    the whole-row select; the random row is selected from its candidates."""
    import deepseek_sparse_attention_head_b200 as dsa
    rng = np.random.default_rng(6)
    L = 200000
    scores = np.stack([np.full(L, 0.75), rng.standard_normal(L)]).astype(np.float32)
    vis = np.array([L, L - 1000])
    case, lo, ph, err = _topk_on_scores(scores, vis, 2048)
    assert err == 0
    for i in range(2):
        check_topk_exact(lo[i], scores[i], vis[i], 2048)
    assert np.array_equal(ph, oracle.pagemap(case, lo.astype(np.int64)))


def test_topk_many_queries_mixed_rows():
    """2400 causal queries over two 4096-token rows (one CTA per query, many waves): rows
    with ties at the k-th, all-negative scores and planted maxima select exactly."""
    import torch
    from tests.gpu_path import GpuCase
    case = generate(CaseSpec("topk_many", (4096, 4096), top_k=512, n_q=1200, q_tail=True, n_planted=0, seed=41))
    Bq, L = case["Bq"], 4096
    rng = np.random.default_rng(42)
    scores = rng.standard_normal((Bq, L)).astype(np.float32)
    scores[1::7] = np.round(scores[1::7] * 2) / 2            # few distinct values: ties at the k-th
    scores[2::7] = -np.abs(scores[2::7])                      # all negative
    scores[3::7, ::61] += 10.0                                # planted maxima
    vis = oracle.visible_lengths(case)
    g = GpuCase(case)
    lo, ph, err = g.topk(torch.from_numpy(scores).cuda(), 512)
    assert err == 0
    for q in range(Bq):
        check_topk_exact(lo[q], scores[q], vis[q], 512)
    assert np.array_equal(ph.astype(np.int64), oracle.pagemap(case, lo.astype(np.int64)))


# rows x keys per row -> CTAs per row's cluster: 40 x 40K -> 2, 6 x 40K -> 4, 3 x 70K -> 8
@pytest.mark.parametrize("n_rows,L,cluster", [(40, 40000, 2), (6, 40000, 4), (3, 70000, 8)])
def test_topk_rows_over_a_cta_cluster(n_rows, L, cluster):
    """Long rows for up to a wave of CTA clusters: each row's gather is split over a cluster
    of 2, 4 or 8 CTAs writing into one candidate buffer. Rows cycle through a constant row
    (the buffer overflows and the first CTA falls back to the whole-row select after the
    cluster barrier), few distinct values (ties at the k-th), a near-constant row,
    all-negative scores, a random row with an odd visible length and a row shorter than
    top_k."""
    rng = np.random.default_rng(7)
    kinds = [lambda: np.full(L, 0.5), lambda: rng.choice([0.25, 0.5, 1.0], size=L),
             lambda: rng.standard_normal(L) * 1e-3 + 7.0, lambda: -np.abs(rng.standard_normal(L)),
             lambda: rng.standard_normal(L), lambda: rng.standard_normal(L)]
    vis_of = [L, L - 5, L - 1000, L, L - 6667, 1500]
    scores = np.stack([kinds[i % 6]() for i in range(n_rows)]).astype(np.float32)
    vis = np.array([vis_of[i % 6] for i in range(n_rows)])
    case, lo, ph, err = _topk_on_scores(scores, vis, 2048)
    assert err == 0
    for i in range(n_rows):
        check_topk_exact(lo[i], scores[i], vis[i], 2048)
    assert np.array_equal(ph, oracle.pagemap(case, lo.astype(np.int64)))


@pytest.mark.parametrize("kv", ["fp8", "bf16"])
def test_mla_two_splits_merged_by_a_cta_pair(kv):
    """64 queries with top_k = 512 take two KV splits, merged inside the decode kernel by
    the cluster of the two split CTAs. Rows shorter than half of top_k leave the second
    split with no valid key (weight zero); a row of one token too."""
    import deepseek_sparse_attention_head_b200 as dsa
    lens = tuple([1, 100, 255, 256, 257, 700] + [300 + 37 * i for i in range(58)])
    sp = CaseSpec(f"pair_{kv}", lens, top_k=512, kv_dtype=kv, idx_dtype=kv, seed=44,
                  out_dtype="fp32" if kv == "bf16" else "bf16")
    case = generate(sp)
    assert dsa.mla_num_splits(case["Bq"], 512) == 2
    vis = oracle.visible_lengths(case)
    rng = np.random.default_rng(45)
    logical = np.full((case["Bq"], 512), -1, dtype=np.int64)
    for q in range(case["Bq"]):
        n = min(512, int(vis[q]))
        logical[q, :n] = rng.choice(int(vis[q]), size=n, replace=False)
    phys = oracle.pagemap(case, logical)
    from tests.gpu_path import GpuCase
    out, lse, err = GpuCase(case).mla(phys)
    assert err == 0
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys)
    check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"])


@pytest.mark.parametrize("rows", [3, 1100])      # prefix built by the indexer / by the plan kernel
def test_indexer_reports_lengths_and_positions_out_of_range(rows):
    """A sequence length past the block table and a causal position past its row's length
    are reported as DSA_ERR_DEVICE_BOUNDS (and clamped), for a prefix built by each indexer
    CTA and for one built by the plan kernel."""
    import deepseek_sparse_attention_head_b200 as dsa
    from tests.gpu_path import GpuCase
    case = generate(CaseSpec(f"bad_len_{rows}", tuple(40 + i % 50 for i in range(rows)), top_k=16, n_q=2,
                             q_pos=(3, 30), n_planted=0, seed=47))
    g = GpuCase(case)
    assert g.indexer()[1] == 0
    g.t["seq_lens"][1] = case["max_pages"] * 64 + 5
    assert g.indexer()[1] == dsa.DSA_ERR_DEVICE_BOUNDS
    g.t["seq_lens"][1] = int(case["seq_lens"][1])
    assert g.indexer()[1] == 0
    g.t["q_pos"][2 * rows - 1] = 10_000
    assert g.indexer()[1] == dsa.DSA_ERR_DEVICE_BOUNDS
