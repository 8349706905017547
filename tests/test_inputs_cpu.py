"""The seeded input recipe: determinism, the shared shuffled page pool, poisoned tails,
the hot-token placement, the quantisation scales and the algorithmic byte count."""
import math

import numpy as np
import pytest

import dsa_inputs
from dsa_inputs import DI, DK, DV, H, KV_GROUPS, PAGE, CaseSpec, generate

FP8_POISON = 0x7E      # +448, the largest finite E4M3 code
POISON_SCALE = 1.0e4


def _small(**kw):
    base = dict(name="t", seq_lens=(40000, 130, 64), top_k=16, seed=21, extra_pages=3)
    base.update(kw)
    return CaseSpec(**base)


def test_generation_is_deterministic_and_independent_of_threads(monkeypatch):
    s = _small()
    monkeypatch.setattr(dsa_inputs, "_threads", lambda: 1)
    a = generate(s)
    monkeypatch.setattr(dsa_inputs, "_threads", lambda: 4)
    b = generate(s)
    for k in ("block_table", "q_idx", "q_idx_scale", "head_w", "k_cache", "k_scale", "q_mla", "kv_cache", "kv_scale"):
        assert np.array_equal(a[k], b[k]), k
    c = generate(_small(seed=22))
    assert not np.array_equal(a["kv_cache"], c["kv_cache"])


def test_page_pool_is_shuffled_and_rows_share_no_page():
    s = _small()
    case = generate(s)
    lens = np.asarray(s.seq_lens)
    pages_per = (lens + PAGE - 1) // PAGE
    bt = case["block_table"]
    assert case["num_pages"] == pages_per.sum() + s.extra_pages
    used = np.concatenate([bt[b, :pages_per[b]] for b in range(s.B)])
    assert np.unique(used).size == used.size                      # rows share no page
    assert used.min() >= 0 and used.max() < case["num_pages"]
    for b in range(s.B):
        assert np.all(bt[b, pages_per[b]:] == -1)
    assert not np.array_equal(used, np.sort(used))                # shuffled, not in order


@pytest.mark.parametrize("kv_dtype", ["fp8", "bf16"])
def test_tails_and_spare_pages_hold_poison(kv_dtype):
    s = _small(kv_dtype=kv_dtype, idx_dtype=kv_dtype)
    case = generate(s)
    lens = np.asarray(s.seq_lens)
    bt = case["block_table"]
    live = np.zeros(case["num_pages"] * PAGE, dtype=bool)
    for b in range(s.B):
        tok = np.arange(lens[b])
        live[bt[b, tok // PAGE].astype(np.int64) * PAGE + tok % PAGE] = True
    dead = ~live
    assert dead.sum() == (case["num_pages"] * PAGE - lens.sum())
    kflat = case["k_cache"].reshape(-1, DI)
    if kv_dtype == "fp8":
        assert np.all(case["kv_cache"][dead] == FP8_POISON) and np.all(case["kv_scale"][dead] == POISON_SCALE)
        assert np.all(kflat[dead] == FP8_POISON) and np.all(case["k_scale"].reshape(-1)[dead] == POISON_SCALE)
        assert np.all(case["kv_scale"][live] < 1.0)                 # real rows: amax/448 of 0.5 N(0,1)
    else:
        poison_bits = dsa_inputs.to_bf16_bits(np.float32([POISON_SCALE]))[0]
        assert np.all(case["kv_cache"][dead] == poison_bits) and np.all(kflat[dead] == poison_bits)
    poison = FP8_POISON if kv_dtype == "fp8" else dsa_inputs.to_bf16_bits(np.float32([POISON_SCALE]))[0]
    assert not np.all(case["kv_cache"][live] == poison, axis=1).any()   # no live row is all poison


def test_e4m3_quantisation_maps_each_row_amax_to_448():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 128)).astype(np.float32)
    codes, scale = dsa_inputs.quantize_rows_e4m3(x)
    assert np.allclose(scale, np.abs(x).max(axis=1) / 448.0)
    amax_pos = np.abs(x).argmax(axis=1)
    top = codes[np.arange(7), amax_pos] & 0x7F
    assert np.all(top == FP8_POISON)                             # |code| = 448 at the row's amax


def test_planted_positions_uniform_and_loguniform():
    s = CaseSpec("t", (5000,), top_k=8, n_planted=32, seed=3)
    p = dsa_inputs._planted_positions(s, 0, 5000)
    assert p.size == 32 and np.unique(p).size == 32 and p.min() >= 0 and p.max() < 5000
    s2 = CaseSpec("t", (1 << 20,), top_k=8, n_planted=256, planted_mode="loguniform", seed=3)
    q = dsa_inputs._planted_positions(s2, 0, 1 << 20)
    assert q.size == 256 and np.unique(q).size == 256 and q.min() >= 0 and q.max() < (1 << 20)
    # log-uniform: about as many below sqrt(L) as above it
    below = int((q < (1 << 10)).sum())
    assert 80 < below < 176
    # prefill workloads plant nothing
    s3 = CaseSpec("t", (5000,), top_k=8, n_q=2, q_pos=(10, 20), seed=3)
    assert dsa_inputs._planted_positions(s3, 0, 5000).size == 0


def test_planted_keys_point_along_the_weighted_query():
    s = CaseSpec("t", (3000,), top_k=8, idx_dtype="bf16", kv_dtype="bf16", n_planted=32, seed=9)
    case = generate(s)
    import torch
    k = torch.from_numpy(case["k_cache"].reshape(-1, DI).view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    q = torch.from_numpy(case["q_idx"][0].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    u = (case["head_w"][0][:, None].astype(np.float64) * q).sum(axis=0)
    u /= np.linalg.norm(u)
    bt = case["block_table"][0]
    tok = np.arange(3000)
    slots = bt[tok // PAGE].astype(np.int64) * PAGE + tok % PAGE
    proj = k[slots] @ u
    planted = case["planted"][0]
    others = np.setdiff1d(tok, planted)
    # shift 3/sqrt(128) along u against a N(0, 1/128) projection: three standard deviations
    assert proj[planted].mean() - proj[others].mean() == pytest.approx(3.0 / math.sqrt(DI), rel=0.2)


def test_named_workloads():
    c2 = dsa_inputs.spec("cfg2")
    assert c2.B == 64 and min(c2.seq_lens) >= 2048 and max(c2.seq_lens) <= 65536
    assert sum(c2.seq_lens) == 2499586
    c4 = dsa_inputs.spec("cfg4")
    assert c4.q_pos == tuple(range(63488, 65536)) and c4.n_planted == 0 and c4.Bq == 2048
    c3 = dsa_inputs.spec("cfg3")
    assert c3.seq_lens == (1 << 20,) and c3.n_planted == 256 and c3.planted_mode == "loguniform"


def test_algorithmic_bytes_by_hand():
    case = generate(CaseSpec("t", (100, 20), top_k=16, seed=4))
    ab = dsa_inputs.algorithmic_bytes(case)
    assert ab["indexer"] == 120 * (DI + 4) + (2 + 1) * 4
    assert ab["mla"] == (16 + 16) * (DK + 4 * KV_GROUPS)
    per_query = (H * DI + 4 * H) + 4 * H + 2 * H * DK + 2 * H * DV
    assert ab["query_side"] == 2 * per_query
    assert ab["total"] == ab["indexer"] + ab["mla"] + ab["query_side"]
    assert dsa_inputs.indexer_flops(case) == 2 * H * DI * 120


def test_q_tail_places_queries_at_each_rows_last_positions():
    c = dsa_inputs.generate(dsa_inputs.CaseSpec("tail", (5, 9, 3), top_k=4, n_q=3, q_tail=True, n_planted=0, seed=9))
    assert c["q_pos"].tolist() == [2, 3, 4, 6, 7, 8, 0, 1, 2]
    m = dsa_inputs.spec("mtp")
    assert m.n_q == 3 and m.q_tail and m.seq_lens == dsa_inputs.spec("cfg2").seq_lens and m.Bq == 192
    with pytest.raises(ValueError):
        dsa_inputs.generate(dsa_inputs.CaseSpec("short", (5, 2), top_k=4, n_q=3, q_tail=True, n_planted=0))
