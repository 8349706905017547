"""Pins of the fp64 oracle to facts that do not come from the oracle itself:
exhaustive format decodes against PyTorch's conversions, values fixed by the OCP
FP8 definition, hand-worked examples, closed forms, brute force on tiny inputs,
library routines on special cases, and invariances of the method."""
import itertools
import json
import math
import os

import struct

import numpy as np
import pytest
import torch

import oracle
from dsa_inputs import PAGE, H, DI, DK, DV, CaseSpec, generate
from tests.helpers import blank_case, bf16, slot_of, permute_pages


# ---------------------------------------------------------------- formats

def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.decode_e4m3(codes)
    nan_ref, nan_got = np.isnan(ref), np.isnan(got)
    assert np.array_equal(nan_ref, nan_got)
    assert nan_got.sum() == 2
    assert np.array_equal(got[~nan_got], ref[~nan_ref])
    assert np.array_equal(np.signbit(got[~nan_got]), np.signbit(ref[~nan_ref]))


def test_e4m3_spec_values(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e4m3_spec_values.json")))
    for item in g["values"]:
        v = oracle.decode_e4m3(np.array([int(item["code"], 16)], dtype=np.uint8))[0]
        if item["value"] == "nan":
            assert math.isnan(v), item
        else:
            assert v == item["value"] and math.copysign(1, v) == math.copysign(1, item["value"]), item


def test_bf16_decode_vs_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, size=200000, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]                      # leave out inf/nan patterns
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.decode_bf16(bits), ref)


def _packed_rows(codes, scales, rope):
    """656-byte packed latent rows built byte by byte: codes, the four scales as
    little-endian fp32 (struct), the rope values encoded to bf16 by PyTorch."""
    n = codes.shape[0]
    rows = np.zeros((n, 656), dtype=np.uint8)
    rows[:, :512] = codes
    rows[:, 512:528] = np.frombuffer(struct.pack("<4f", *[float(x) for x in scales]), dtype=np.uint8)
    bits = torch.from_numpy(np.ascontiguousarray(rope, dtype=np.float32)).to(torch.bfloat16).view(torch.int16)
    rows[:, 528:] = bits.numpy().astype("<i2").view(np.uint8).reshape(n, 128)
    return rows


def test_packed_rows_decode_by_their_byte_layout():
    """The packed fp8 latent row (656 bytes, the layout variant with bf16 rope columns):
    E4M3 codes of the 512 latent columns, one fp32 scale per 128-column group at bytes
    512..527, then the 64 rope values in bf16. Codes are decoded by PyTorch, the column
    ranges written out by hand."""
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, size=(64, 512)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                       # no NaN codes
    scales = np.array([0.5, 2.0, 4.0, 8.0], dtype=np.float32)
    rope = rng.standard_normal((64, 64)).astype(np.float32)
    case = dict(kv_cache=_packed_rows(codes, scales, rope), kv_scale=None, kv_dtype="fp8r")
    got = oracle.dequant_latent_rows(case, np.arange(64))
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for g, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 384), (384, 512)]):
        assert np.array_equal(got[:, lo:hi], vals[:, lo:hi] * float(scales[g])), g
    want_rope = torch.from_numpy(rope).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got[:, 512:], want_rope)


def test_packed_rows_agree_with_the_scale_plane_layout():
    """Where the rope values are exact in both formats (E4M3 codes times a power of two),
    a packed row and a row of the five-scale layout hold the same numbers, and attention
    over them is identical."""
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 0x7F, size=(64, DK)).astype(np.uint8)
    scales = np.array([0.25, 0.5, 1.0, 2.0, 0.125], dtype=np.float32)
    plane = blank_case((64,), top_k=64, idx_dtype="fp8", kv_dtype="fp8")
    plane["kv_cache"][:64] = codes
    plane["kv_scale"][:64] = scales
    rope = torch.from_numpy(codes[:, 512:]).view(torch.float8_e4m3fn).to(torch.float64).numpy() * 0.125
    packed = dict(plane, kv_cache=_packed_rows(codes[:, :512], scales[:4], rope), kv_scale=None, kv_dtype="fp8r")
    slots = np.arange(64)
    assert np.array_equal(oracle.dequant_latent_rows(packed, slots), oracle.dequant_latent_rows(plane, slots))
    q = rng.standard_normal((1, H, DK)).astype(np.float32)
    qb = torch.from_numpy(q).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    plane["q_mla"] = qb
    packed["q_mla"] = qb
    phys = slots[None, :].astype(np.int64)
    o1, l1 = oracle.mla_sparse_attention(plane, phys)
    o2, l2 = oracle.mla_sparse_attention(packed, phys)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_scales_apply_to_their_columns():
    """The storage reading for fp8 tensors. Latent rows carry five scales: columns
    [0,128), [128,256), [256,384), [384,512) and the 64 rope columns [512,576). Indexer
    keys carry one scale per token, indexer queries one per (query, head). Codes are
    decoded by PyTorch; the column ranges are written out by hand."""
    rng = np.random.default_rng(3)
    case = blank_case((64,), idx_dtype="fp8", kv_dtype="fp8")
    codes = rng.integers(0, 256, size=(64, DK)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                       # no NaN codes
    case["kv_cache"][:64] = codes
    scales = np.array([0.5, 2.0, 4.0, 8.0, 16.0], dtype=np.float32)
    case["kv_scale"][:64] = scales
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.dequant_latent_rows(case, np.arange(64))
    for g, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 384), (384, 512), (512, 576)]):
        assert np.array_equal(got[:, lo:hi], vals[:, lo:hi] * float(scales[g])), g

    kc = rng.integers(0, 0x7F, size=(64, DI)).astype(np.uint8)
    case["k_cache"][0] = kc
    case["k_scale"][0] = np.arange(1, 65, dtype=np.float32)
    kv = torch.from_numpy(kc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got_k = oracle.dequant_index_keys(case, np.arange(64))
    assert np.array_equal(got_k, kv * np.arange(1, 65, dtype=np.float64)[:, None])

    qc = rng.integers(0, 0x7F, size=(H, DI)).astype(np.uint8)
    case["q_idx"][0] = qc
    case["q_idx_scale"][0] = np.linspace(0.25, 4.0, H).astype(np.float32)
    qv = torch.from_numpy(qc).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got_q = oracle.dequant_index_queries(case)[0]
    assert np.array_equal(got_q, qv * case["q_idx_scale"][0].astype(np.float64)[:, None])


# ---------------------------------------------------------------- indexer

def _worked_indexer_case(golden):
    c = blank_case([3], top_k=golden["top_k"])
    qf = np.zeros((H, DI), dtype=np.float32)
    qf[2:, :] = 1.0
    for h, row in golden["q_rows"].items():
        qf[int(h), :len(row)] = row
    c["q_idx"][0] = bf16(qf)
    for h, wv in golden["w_heads"].items():
        c["head_w"][0, int(h)] = wv
    for s, row in enumerate(golden["k_rows"]):
        kf = np.zeros(DI, dtype=np.float32)
        kf[:len(row)] = row
        c["k_cache"].reshape(-1, DI)[slot_of(c, 0, s)] = bf16(kf)
    return c


def test_indexer_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "indexer_worked_example.json")))
    c = _worked_indexer_case(g)
    sc = oracle.indexer_scores(c)
    assert np.array_equal(sc[0, :3], np.array(g["expected_scores"]))
    assert np.all(np.isneginf(sc[0, 3:]))
    top = oracle.topk_logical(sc, oracle.visible_lengths(c), g["top_k"])
    assert list(top[0]) == g["expected_topk"]


def test_indexer_one_hot_head_reduces_to_single_dot():
    """w = one-hot(h): score = w_h * max(0, q_h . k) - a single dot product (np.dot)."""
    case = generate(CaseSpec("t", (200,), top_k=16, seed=11, n_planted=0))
    h = 17
    case["head_w"][:] = 0.0
    case["head_w"][0, h] = 0.75
    sc = oracle.indexer_scores(case)
    q = oracle.decode_e4m3(case["q_idx"][0, h]) * float(case["q_idx_scale"][0, h])
    for s in (0, 5, 63, 64, 199):
        slot = slot_of(case, 0, s)
        k = oracle.decode_e4m3(case["k_cache"].reshape(-1, DI)[slot]) * float(case["k_scale"].reshape(-1)[slot])
        assert sc[0, s] == pytest.approx(0.75 * max(0.0, float(np.dot(q, k))), rel=1e-14, abs=0)


def test_indexer_all_negative_dots_give_zero():
    """Every key anti-aligned with every head's query: all ReLUs vanish, score = 0."""
    c = blank_case([70])
    qf = np.zeros((H, DI), dtype=np.float32)
    qf[:, 0] = 1.0
    qf[:, 1] = 0.5
    c["q_idx"][0] = bf16(qf)
    c["head_w"][0] = 1.0
    kf = np.zeros((70, DI), dtype=np.float32)
    kf[:, 0] = -np.linspace(0.5, 2.0, 70)
    for s in range(70):
        c["k_cache"].reshape(-1, DI)[slot_of(c, 0, s)] = bf16(kf[s])
    sc = oracle.indexer_scores(c)
    assert np.all(sc[0, :70] == 0.0)


def test_indexer_positive_homogeneity():
    """Doubling every key scale doubles every score exactly (powers of two)."""
    case = generate(CaseSpec("t", (150, 90), top_k=8, seed=12))
    s1 = oracle.indexer_scores(case)
    c2 = dict(case)
    c2["k_scale"] = case["k_scale"] * np.float32(2.0)
    s2 = oracle.indexer_scores(c2)
    fin = np.isfinite(s1)
    assert np.array_equal(s2[fin], 2.0 * s1[fin])


def test_indexer_head_permutation_invariance():
    case = generate(CaseSpec("t", (130,), top_k=8, seed=13))
    perm = np.random.default_rng(0).permutation(H)
    c2 = dict(case)
    c2["q_idx"] = case["q_idx"][:, perm]
    c2["q_idx_scale"] = case["q_idx_scale"][:, perm]
    c2["head_w"] = case["head_w"][:, perm]
    a, b = oracle.indexer_scores(case), oracle.indexer_scores(c2)
    fin = np.isfinite(a)
    assert np.allclose(a[fin], b[fin], rtol=1e-13, atol=0)


def test_indexer_causal_visibility():
    case = generate(CaseSpec("t", (300,), top_k=8, n_q=3, q_pos=(10, 64, 299), n_planted=0, seed=14))
    sc = oracle.indexer_scores(case)
    for i, p in enumerate((10, 64, 299)):
        assert np.all(np.isfinite(sc[i, :p + 1]))
        assert np.all(np.isneginf(sc[i, p + 1:]))


def test_planted_tokens_rank_high():
    """cfg0's hot tokens (+3 sigma along the weighted query) dominate the top-256."""
    case = generate(CaseSpec("t", (4096,), top_k=256, idx_dtype="bf16", kv_dtype="bf16",
                             out_dtype="fp32", n_planted=32, seed=0))
    sc = oracle.indexer_scores(case)
    top = oracle.topk_logical(sc, oracle.visible_lengths(case), 256)
    hit = np.isin(case["planted"][0], top[0]).sum()
    assert hit >= 24, hit


# ---------------------------------------------------------------- top-k

def test_topk_brute_force_subsets():
    """Distinct scores: the selected set is the k-subset with the largest sum."""
    rng = np.random.default_rng(3)
    for L, k in [(7, 3), (9, 4), (8, 1), (6, 5)]:
        s = rng.standard_normal(L)
        best = max(itertools.combinations(range(L), k), key=lambda c: s[list(c)].sum())
        got = oracle.topk_logical(s[None, :], np.array([L]), k)[0]
        assert set(got[:k]) == set(best)
        assert np.all(np.diff(s[got[:k]]) <= 0)      # descending order


def test_topk_ties_lower_index_first():
    s = np.array([[1.0, 2.0, 2.0, 1.0, 2.0, 0.0]])
    got = oracle.topk_logical(s, np.array([6]), 4)[0]
    assert list(got) == [1, 2, 4, 0]


def test_topk_dense_path_and_padding():
    s = np.random.default_rng(0).standard_normal((1, 50))
    got = oracle.topk_logical(s, np.array([30]), 40)[0]
    assert set(got[:30]) == set(range(30))
    assert np.all(got[30:] == -1)
    empty = oracle.topk_logical(s, np.array([0]), 4)[0]
    assert np.all(empty == -1)


def test_topk_never_selects_invisible():
    s = np.arange(100, dtype=np.float64)[None, :]      # the largest scores are past vis
    got = oracle.topk_logical(s, np.array([40]), 8)[0]
    assert set(got) == set(range(32, 40))


# ---------------------------------------------------------------- page map

def test_pagemap_identity_and_hand_example():
    c = blank_case([200])
    logical = np.array([[0, 63, 64, 199, -1]])
    assert np.array_equal(oracle.pagemap(c, logical), logical)
    c["block_table"][0, :4] = [7, 2, 9, 0]
    got = oracle.pagemap(c, logical)[0]
    assert list(got) == [7 * 64, 7 * 64 + 63, 2 * 64, 0 * 64 + 199 - 192, -1]


# ---------------------------------------------------------------- MLA

def test_mla_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "mla_worked_example.json")))
    c = blank_case([2], softmax_scale=math.log(3.0))
    qm = np.zeros((H, DK), dtype=np.float32)
    qm[:, 512] = 1.0
    c["q_mla"][0] = bf16(qm)
    a = np.zeros(DK, dtype=np.float32); a[2] = 4.0
    b = np.zeros(DK, dtype=np.float32); b[512] = 1.0; b[3] = 8.0
    c["kv_cache"][slot_of(c, 0, 0)] = bf16(a)
    c["kv_cache"][slot_of(c, 0, 1)] = bf16(b)
    phys = np.array([[slot_of(c, 0, 0), slot_of(c, 0, 1)]])
    out, lse = oracle.mla_sparse_attention(c, phys)
    s = c["softmax_scale"]                        # ln 3 rounded to fp32
    p1 = math.exp(s) / (1 + math.exp(s))
    assert np.allclose(out[0, :, 2], 4 * (1 - p1), rtol=1e-12)
    assert np.allclose(out[0, :, 3], 8 * p1, rtol=1e-12)
    assert out[0, 0, 2] == pytest.approx(g["expected_out_col2"], rel=1e-7)
    assert out[0, 0, 3] == pytest.approx(g["expected_out_col3"], rel=1e-7)
    assert lse[0, 0] == pytest.approx(g["expected_lse"], rel=1e-7)
    mask = np.ones(DV, dtype=bool); mask[[2, 3]] = False
    assert np.all(out[0][:, mask] == 0)


def _attn_case(L, kv_dtype, seed):
    return generate(CaseSpec("t", (L,), top_k=max(L, 1), idx_dtype="fp8", kv_dtype=kv_dtype,
                             n_planted=0, seed=seed))


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8"])
def test_mla_dense_equals_library_sdpa(kv_dtype):
    """top_k >= L: sparse attention over all selected rows == dense attention
    (torch scaled_dot_product_attention in fp64) over the row's L tokens."""
    L = 150
    case = _attn_case(L, kv_dtype, 21)
    logical = np.arange(L)[None, :]
    phys = oracle.pagemap(case, logical)
    out, lse = oracle.mla_sparse_attention(case, phys)
    qm = torch.from_numpy(oracle.decode_bf16(case["q_mla"][0]))[None]           # [1, 64, 576]
    KV = torch.from_numpy(oracle.dequant_latent_rows(case, phys[0]))             # [L, 576]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qm[:, :, None, :], KV[None, None].expand(1, H, L, DK), KV[None, None, :, :DV].expand(1, H, L, DV),
        scale=case["softmax_scale"])[:, :, 0]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-14)
    z = case["softmax_scale"] * (qm[0] @ KV.T)
    assert np.allclose(lse[0], torch.logsumexp(z, dim=1).numpy(), rtol=1e-13)


def test_mla_dense_then_masked_equals_sparse():
    """Attention over every slot of the row with -inf logits off the selection equals
    attention over the selection only."""
    L = 200
    case = _attn_case(L, "fp8", 22)
    sel_logical = np.array(sorted(np.random.default_rng(1).choice(L, 37, replace=False)))
    phys_sel = oracle.pagemap(case, sel_logical[None, :])
    out, _ = oracle.mla_sparse_attention(case, phys_sel)
    all_phys = oracle.pagemap(case, np.arange(L)[None, :])[0]
    qm = torch.from_numpy(oracle.decode_bf16(case["q_mla"][0]))
    KV = torch.from_numpy(oracle.dequant_latent_rows(case, all_phys))
    mask = torch.zeros(L, dtype=torch.bool)
    mask[sel_logical] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        qm[None, :, None, :], KV[None, None].expand(1, H, L, DK), KV[None, None, :, :DV].expand(1, H, L, DV),
        attn_mask=mask[None, None, None, :], scale=case["softmax_scale"])[0, :, 0]
    assert np.allclose(out[0], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_mla_softmax_rows_sum_to_one():
    """With every value column equal to 1 the output is sum_j p_j = 1 exactly (to 1e-12)."""
    case = _attn_case(100, "bf16", 23)
    case["kv_cache"][:, :DV] = bf16(np.ones(DV, dtype=np.float32))[None, :]
    phys = oracle.pagemap(case, np.arange(100)[None, :])
    out, _ = oracle.mla_sparse_attention(case, phys)
    assert np.all(np.abs(out - 1.0) < 1e-12)


def test_mla_one_dominant_key_and_equal_keys():
    case = _attn_case(64, "bf16", 24)
    phys = oracle.pagemap(case, np.arange(64)[None, :])
    # equal keys -> output equals that row's value
    row = case["kv_cache"][phys[0, 5]].copy()
    c2 = dict(case); c2["kv_cache"] = case["kv_cache"].copy()
    c2["kv_cache"][phys[0]] = row
    out, _ = oracle.mla_sparse_attention(c2, phys)
    assert np.allclose(out[0], oracle.decode_bf16(row[:DV])[None, :], rtol=1e-12, atol=1e-14)
    # one key aligned with a huge query -> its value wins
    c3 = dict(case); c3["q_mla"] = case["q_mla"].copy(); c3["kv_cache"] = case["kv_cache"].copy()
    c3["q_mla"][0] = bf16(np.full((H, DK), 0.0, dtype=np.float32))
    c3["q_mla"][0][:, 512] = bf16(np.float32([1000.0]))[0]
    c3["kv_cache"][phys[0], 512] = bf16(np.float32([0.0]))[0]
    c3["kv_cache"][phys[0, 9], 512] = bf16(np.float32([1.0]))[0]
    out, _ = oracle.mla_sparse_attention(c3, phys)
    v9 = oracle.decode_bf16(c3["kv_cache"][phys[0, 9], :DV])
    assert np.allclose(out[0], v9[None, :], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("S", [1, 2, 3, 7])
def test_split_combine_equals_unsplit(S):
    case = _attn_case(300, "fp8", 25)
    rng = np.random.default_rng(S)
    logical = rng.choice(300, 129, replace=False)[None, :]
    logical = np.concatenate([logical, -np.ones((1, 11), dtype=np.int64)], axis=1)   # padded tail
    phys = oracle.pagemap(case, logical)
    a, la = oracle.mla_sparse_attention(case, phys)
    b, lb = oracle.mla_sparse_attention_split(case, phys, S)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)
    assert np.allclose(la, lb, rtol=1e-12)


def test_empty_selection():
    case = _attn_case(10, "fp8", 26)
    out, lse = oracle.mla_sparse_attention(case, -np.ones((1, 8), dtype=np.int64))
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------- whole step

def test_page_permutation_invariance_whole_step():
    """Moving physical pages (and rewriting the block table) changes no output bit."""
    case = generate(CaseSpec("t", (300, 130), top_k=64, seed=27))
    perm = np.random.default_rng(5).permutation(case["num_pages"])
    a = oracle.decode_layer(case)
    b = oracle.decode_layer(permute_pages(case, perm))
    assert np.array_equal(a["scores"], b["scores"])
    assert np.array_equal(a["logical"], b["logical"])
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["lse"], b["lse"])


def test_topk_ge_len_reduces_to_dense_whole_step():
    case = generate(CaseSpec("t", (100,), top_k=128, seed=28))
    r = oracle.decode_layer(case)
    assert set(r["logical"][0][r["logical"][0] >= 0]) == set(range(100))
    dense_phys = oracle.pagemap(case, np.arange(100)[None, :])
    out, lse = oracle.mla_sparse_attention(case, dense_phys)
    assert np.allclose(r["out"], out, rtol=1e-13, atol=1e-15)


def test_poison_never_reaches_outputs():
    """Tail slots of the last page hold huge poison values; a correct step never reads them."""
    case = generate(CaseSpec("t", (70,), top_k=128, seed=29))
    r = oracle.decode_layer(case)
    assert np.all(np.abs(r["out"]) < 10)


# ---------------------------------------------------------------- token-sharded step

def test_shard_candidates_by_hand():
    row = np.array([5.0, 1.0, 7.0, 7.0, 2.0, 9.0, 3.0])
    sc, tok = oracle.shard_candidates(row, 2, 6, 3)          # slice [7, 7, 2, 9] of tokens 2..5
    assert list(tok) == [5, 2, 3] and list(sc) == [9.0, 7.0, 7.0]
    sc, tok = oracle.shard_candidates(row, 5, 7, 4)          # two tokens: padded
    assert list(tok) == [5, 6, -1, -1] and list(sc[:2]) == [9.0, 3.0] and np.all(np.isneginf(sc[2:]))
    sc, tok = oracle.shard_candidates(row, 3, 3, 2)          # an empty shard
    assert list(tok) == [-1, -1]


def test_shard_global_select_by_hand():
    sc = np.array([4.0, 6.0, -np.inf, 6.0, 1.0, 6.0])
    tok = np.array([10, 31, -1, 7, 2, 40])
    assert list(oracle.shard_global_select(sc, tok, 3)) == [7, 31, 40]
    assert list(oracle.shard_global_select(sc, tok, 2)) == [7, 31]
    assert list(oracle.shard_global_select(sc, tok, 7)) == [7, 31, 40, 10, 2, -1, -1]


_SHARD_LAYOUTS = {
    "one_rank": [[0, 300], [0, 130]],
    "equal_pages": [[0, 128, 256, 300], [0, 64, 128, 130]],
    "empty_ranks": [[0, 0, 192, 300], [0, 130, 130, 130]],
    "shards_shorter_than_top_k": [[0, 64, 128, 192, 256, 300], [0, 64, 64, 128, 128, 130]],
}


@pytest.mark.parametrize("layout", sorted(_SHARD_LAYOUTS))
def test_sharded_step_equals_unsharded(layout):
    """The union of the ranks' local top-k holds a global top-k, and the log-sum-exp merge
    of per-rank softmax states is the softmax over their union: the sharded step gives the
    unsharded step's selection exactly and its attention to rounding."""
    case = generate(CaseSpec("t", (300, 130), top_k=64, seed=31, kv_dtype="fp8"))
    bounds = np.array(_SHARD_LAYOUTS[layout])
    a = oracle.decode_layer(case)
    b = oracle.sharded_decode_layer(case, bounds)
    assert np.array_equal(a["logical"], b["logical"])
    assert np.array_equal(a["physical"], b["physical"])
    assert np.allclose(a["out"], b["out"], rtol=1e-12, atol=1e-14)
    assert np.allclose(a["lse"], b["lse"], rtol=1e-12)
    for i in range(case["Bq"]):
        sel, own = b["logical"][i], b["owner"][i]
        ok = sel >= 0
        assert np.all(bounds[i][own[ok]] <= sel[ok]) and np.all(sel[ok] < bounds[i][own[ok] + 1])


def test_sharded_step_equals_unsharded_with_two_queries_per_row():
    case = generate(CaseSpec("t", (400, 150), top_k=48, n_q=2, n_planted=0, seed=33, kv_dtype="bf16"))
    bounds = np.array([[0, 128, 256, 400], [0, 64, 64, 150]])
    a = oracle.decode_layer(case)
    b = oracle.sharded_decode_layer(case, bounds)
    assert np.array_equal(a["logical"], b["logical"])
    assert np.allclose(a["out"], b["out"], rtol=1e-12, atol=1e-14)
    assert np.allclose(a["lse"], b["lse"], rtol=1e-12)


def test_sharded_step_dense_rows_take_every_token():
    case = generate(CaseSpec("t", (100, 40), top_k=128, seed=32))
    r = oracle.sharded_decode_layer(case, np.array([[0, 64, 100], [0, 0, 40]]))
    assert sorted(r["logical"][0][r["logical"][0] >= 0]) == list(range(100))
    assert sorted(r["logical"][1][r["logical"][1] >= 0]) == list(range(40))


def test_sharded_step_ties_go_to_the_lower_global_token():
    """All scores equal (zero caches): whatever the layout, tokens 0..k-1 are selected."""
    case = blank_case([320], top_k=8)
    for bounds in ([0, 128, 320], [0, 256, 320], [0, 64, 128, 192, 256, 320]):
        r = oracle.sharded_decode_layer(case, np.array([bounds]))
        assert list(r["logical"][0]) == list(range(8))


# ---------------------------------------------------------------- the step before the path

def test_e4m3_encoder_round_trips_ties_to_even_and_saturates():
    """Every finite code's value encodes back to that code; the midpoint of two adjacent
    magnitudes goes to the even code; magnitudes past 448 saturate; random values agree
    with PyTorch's float8_e4m3fn conversion."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.decode_e4m3(codes)
    got = oracle.encode_e4m3(vals)
    zero = vals == 0
    assert np.array_equal(got[~zero], codes[~zero])
    pos = oracle.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    want = np.where(np.arange(1, 0x7F) % 2 == 0, np.arange(1, 0x7F), np.arange(0, 0x7E)).astype(np.uint8)
    assert np.array_equal(oracle.encode_e4m3(mids), want)
    assert oracle.encode_e4m3(np.array([1e6, -500.0])).tolist() == [0x7E, 0xFE]
    x = np.random.default_rng(11).standard_normal(50000) * 60
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(x.astype(np.float32).astype(np.float64)), ref)


def test_bf16_encoder_matches_torch_and_keeps_bf16_values():
    x = np.random.default_rng(12).standard_normal(50000).astype(np.float32) * 7
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.encode_bf16(x.astype(np.float64)), ref)
    exact = oracle.decode_bf16(ref)
    assert np.array_equal(oracle.encode_bf16(exact), ref)


def test_rope_interleaved_by_hand_and_by_its_invariants():
    """pos 0 is the identity; each pair keeps its norm; rotations compose (p1 then p2 is
    p1 + p2); a unit vector in pair 0 turns by pos radians (theta_0 = 1) and one in pair 16
    by pos / 100 (theta_16 = 10000^(-1/2))."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal((5, 64))
    assert np.array_equal(oracle.rope_interleaved(x, np.zeros(5)), x)
    y = oracle.rope_interleaved(x, np.arange(5) * 1000.0 + 3)
    assert np.allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), atol=1e-12)
    two = oracle.rope_interleaved(oracle.rope_interleaved(x, 17.0), 40.0)
    assert np.allclose(two, oracle.rope_interleaved(x, 57.0), atol=1e-12)
    e = np.zeros((2, 64))
    e[0, 0] = 1.0
    e[1, 32] = 1.0
    r = oracle.rope_interleaved(e, np.array([2.5, 300.0]))
    assert np.allclose(r[0, :2], [math.cos(2.5), math.sin(2.5)], atol=1e-15)
    assert np.allclose(r[1, 32:34], [math.cos(3.0), math.sin(3.0)], atol=1e-12)
    assert np.count_nonzero(r[0, 2:]) == 0 and np.count_nonzero(r[1, :32]) == 0


def test_quantize_maps_amax_to_448_and_zero_rows_to_scale_one():
    x = np.array([[0.5, -2.0, 1.0], [0.0, 0.0, 0.0]])
    codes, scale = oracle.quantize_e4m3(x)
    assert scale.dtype == np.float32 and scale.tolist() == [np.float32(2.0 / 448.0), 1.0]
    assert codes[0, 1] == 0xFE and codes[1].tolist() == [0, 0, 0]


def test_rope_quantize_append_slots_and_untouched_columns():
    """The new token of each row goes to table[row, pos // 64] * 64 + pos % 64 (a permuted
    table, written out by hand); the non-rope columns are plain quantisations of the
    inputs; the MLA query keeps its 512 latent columns bit for bit."""
    table = np.array([[3, 0, -1], [1, 2, 4]], dtype=np.int32)
    case = blank_case((70, 150), idx_dtype="fp8", kv_dtype="fp8", max_pages=3, table=table)
    assert oracle.new_token_positions(case).tolist() == [69, 149]
    rng = np.random.default_rng(14)
    new = dict(idx_q=bf16(rng.standard_normal((2, H, DI))), idx_k=bf16(rng.standard_normal((2, DI))),
               latent=bf16(rng.standard_normal((2, DK))), q_mla=bf16(rng.standard_normal((2, H, DK))))
    r = oracle.rope_quantize_append(case, new)
    assert r["slots"].tolist() == [0 * 64 + 5, 4 * 64 + 21]
    k = oracle.decode_bf16(new["idx_k"])
    # the key's columns 64.. are not rotated: their codes are those of x / (the row's scale)
    want = oracle.encode_e4m3(k[:, 64:] / r["k_scale"].astype(np.float64)[:, None])
    assert np.array_equal(r["k_codes"][:, 64:], want)
    assert np.array_equal(r["q_mla"][..., :DV], new["q_mla"][..., :DV])
    lat = oracle.decode_bf16(new["latent"])
    for g in range(4):
        codes, scale = oracle.quantize_e4m3(lat[:, 128 * g:128 * g + 128])
        assert np.array_equal(r["latent_codes"][:, 128 * g:128 * g + 128], codes)
        assert np.array_equal(r["latent_scales"][:, g], scale)
