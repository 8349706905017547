"""Token-sharded decode on one GPU: the R ranks run in one process, in lockstep, and the
two exchanges become device copies of their buffers (ranks that wait on one another never
run as separate launches on one GPU). Graded against the fp64 oracle: each rank's local
candidates exactly on its own fp32 scores, the global selection exactly on the gathered
candidates (the same precision, the same tie rule) and against the unsharded oracle step
up to near-ties, each rank's slots against the selection, and the merged attention
against the oracle's attention over the selection."""
import functools

import numpy as np
import pytest
import torch

import oracle
from dsa_inputs import CaseSpec, generate, to_torch
from tests.compare import check_attention, check_topk_exact, check_topk_near_tie, fp8_lse_bound

pytestmark = pytest.mark.gpu

CASES = {
    "rows_fp8": CaseSpec("rows_fp8", (3000, 700, 64, 1), top_k=256, seed=51),
    "long_row": CaseSpec("long_row", (40000,), top_k=2048, seed=52),
    "bf16": CaseSpec("bf16", (1500, 129), top_k=128, idx_dtype="bf16", kv_dtype="bf16", out_dtype="fp32", seed=53),
    "packed_two_queries": CaseSpec("packed_two_queries", (2500, 900), top_k=256, kv_dtype="fp8r", n_q=2,
                                   n_planted=0, seed=54),
    # 3 x 8192 candidates per query: the select's shared-memory copy; 4 x 8192: global reads
    "wide_select": CaseSpec("wide_select", (40000,), top_k=8192, seed=55),
    # a top_k that divides nothing, ragged rows
    "odd_topk": CaseSpec("odd_topk", (1000, 333, 77), top_k=100, seed=56),
    # every token's indexer key the same: all scores tie, so the global select takes its
    # second radix pass (lowest global tokens among the candidates)
    "all_ties": CaseSpec("all_ties", (3000, 500), top_k=256, seed=57),
}
TIED = {"all_ties"}
# (case, layout) pairs: every case on every layout except the wide one, which takes the two
# layouts that reach the select's memory paths; 8 x 2048 candidates fill 16 registers a thread
PAIRS = ([(n, l) for n in sorted(CASES) if n not in ("wide_select", "odd_topk", "all_ties")
          for l in ("even1", "even2", "even3", "even4", "uneven")]
         + [("long_row", "even8"), ("wide_select", "even3"), ("wide_select", "even4")]
         + [(n, l) for n in ("odd_topk", "all_ties") for l in ("even1", "even3", "uneven")])


@functools.lru_cache(maxsize=None)
def get_case(name):
    case = generate(CASES[name])
    if name in TIED:
        case["k_cache"][:] = case["k_cache"][0, 0]
        if case["k_scale"] is not None:
            case["k_scale"][:] = case["k_scale"][0, 0]
    return case


@functools.lru_cache(maxsize=None)
def oracle_scores(name):
    return oracle.indexer_scores(get_case(name))


def _bounds(case, layout):
    from deepseek_sparse_attention_head_b200.sharded import shard_bounds
    lens = case["seq_lens"]
    if layout.startswith("even"):
        R = int(layout[4:])
        return np.array([shard_bounds(int(L), R) for L in lens], dtype=np.int64)
    # uneven: random page-aligned cuts, some ranks empty
    rng = np.random.default_rng(7)
    rows = []
    for L in lens:
        pages = (int(L) + 63) // 64
        cuts = np.sort(rng.integers(0, pages + 1, size=3)) * 64
        rows.append([0] + [min(int(L), int(c)) for c in cuts] + [int(L)])
    return np.array(rows, dtype=np.int64)


def run_sharded(case, bounds):
    """Runs every rank's phases in lockstep; returns per-rank results and the gathered candidates."""
    import deepseek_sparse_attention_head_b200 as dsa
    from deepseek_sparse_attention_head_b200.sharded import TokenShardedDecode
    t = to_torch(case, "cuda")
    B, R, K = case["B"], bounds.shape[1] - 1, case["top_k"]
    bt = case["block_table"]
    ranks = []
    for r in range(R):
        lo, hi = bounds[:, r], bounds[:, r + 1]
        lens = (hi - lo).astype(np.int32)
        npg = (lens + 63) // 64
        mp = max(1, int(npg.max()))
        lbt = np.full((B, mp), -1, dtype=np.int32)
        for b in range(B):
            lbt[b, :npg[b]] = bt[b, lo[b] // 64:lo[b] // 64 + npg[b]]
        paging = dsa.Paging(torch.from_numpy(lens).cuda(), torch.from_numpy(lbt).cuda(), case["num_pages"],
                            case["n_q"])
        off = torch.from_numpy(lo.astype(np.int32)).cuda()
        ranks.append(TokenShardedDecode(paging, off, K, case["softmax_scale"], r, R))
    for o in ranks:
        o.local_phase(t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"])
    S = torch.stack([o.cand_score for o in ranks])
    T = torch.stack([o.cand_token for o in ranks])
    logical = []
    for o in ranks:
        o.all_score.copy_(S)
        o.all_token.copy_(T)
        lg = torch.full((case["Bq"], K), -7, dtype=torch.int32, device="cuda")
        o.physical.fill_(-7)
        o.select_phase(logical_out=lg)
        o.attend_phase(t["q_mla"], t["kv_cache"], t["kv_scale"])
        logical.append(lg)
    O = torch.stack([o.state_out for o in ranks])
    L = torch.stack([o.state_lse for o in ranks])
    odt = torch.float32 if case["out_dtype"] == "fp32" else torch.bfloat16
    outs = []
    for o in ranks:
        o.all_out.copy_(O)
        o.all_lse.copy_(L)
        out = torch.full((case["Bq"], 64, 512), float("nan"), dtype=odt, device="cuda")
        lse = torch.full((case["Bq"], 64), float("nan"), dtype=torch.float32, device="cuda")
        o.merge_phase(out, lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    errs = [dsa.dsa_get_error(w) for o in ranks for w in (o.ws_index, o.ws_local, o.ws_select, o.ws_mla)]
    return dict(
        ranks=ranks, errs=errs,
        scores=[o.scores.cpu().numpy() for o in ranks],
        cand_token=T.cpu().numpy(), cand_score=S.cpu().numpy(),
        logical=[x.cpu().numpy().astype(np.int64) for x in logical],
        physical=[o.physical.cpu().numpy().astype(np.int64) for o in ranks],
        out=[x[0].float().cpu().numpy().astype(np.float64) for x in outs],
        out_raw=[x[0].cpu() for x in outs],
        lse=[x[1].cpu().numpy().astype(np.float64) for x in outs],
    )


@pytest.mark.parametrize("name,layout", PAIRS)
def test_sharded_decode(name, layout):
    case = get_case(name)
    bounds = _bounds(case, layout)
    R, K, n_q = bounds.shape[1] - 1, case["top_k"], case["n_q"]
    g = run_sharded(case, bounds)
    assert all(e == 0 for e in g["errs"]), g["errs"]

    for r in range(R):
        # this rank's candidates: an exact top-k of its own fp32 scores, as global tokens
        for q in range(case["Bq"]):
            b = q // n_q
            lo, hi = int(bounds[b, r]), int(bounds[b, r + 1])
            tok = g["cand_token"][r, q]
            local = np.where(tok >= 0, tok - lo, -1)
            check_topk_exact(local, g["scores"][r][q], hi - lo, K)
            ok = tok >= 0
            assert np.array_equal(g["cand_score"][r, q][ok], g["scores"][r][q][local[ok]])
            assert np.all(np.isneginf(g["cand_score"][r, q][~ok]))

    ref_scores = oracle_scores(name)
    vis = oracle.visible_lengths(case)
    ref_sel = oracle.topk_logical(ref_scores, vis, K)
    sel0 = g["logical"][0]
    for q in range(case["Bq"]):
        b = q // n_q
        # the same selection on every rank
        for r in range(1, R):
            assert set(g["logical"][r][q].tolist()) == set(sel0[q].tolist())
        # exact on the gathered fp32 candidates (ties to the lower global token)
        want = oracle.shard_global_select(g["cand_score"][:, q].ravel().astype(np.float64),
                                          g["cand_token"][:, q].ravel(), K)
        assert set(sel0[q][sel0[q] >= 0].tolist()) == set(want[want >= 0].tolist())
        assert np.all(sel0[q][(sel0[q] >= 0).sum():] == -1)
        # against the unsharded oracle step, up to near-ties
        check_topk_near_tie(sel0[q], ref_sel[q], ref_scores[q], vis[q], K)
        # each rank's slots: exactly its share of the selection, first, then -1
        sel = sel0[q][sel0[q] >= 0]
        for r in range(R):
            lo, hi = bounds[b, r], bounds[b, r + 1]
            mine = sel[(sel >= lo) & (sel < hi)]
            ph = g["physical"][r][q]
            n = mine.size
            assert np.all(ph[n:] == -1)
            want_ph = oracle.physical_slots(case["block_table"][b], mine)
            assert sorted(ph[:n].tolist()) == sorted(want_ph.tolist())

    # every rank merges to the same bits; attention against the oracle on the selection
    for r in range(1, R):
        assert torch.equal(g["out_raw"][r], g["out_raw"][0])
        assert np.array_equal(g["lse"][r], g["lse"][0])
    phys = oracle.pagemap(case, sel0)
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys)
    bound = fp8_lse_bound(case, phys) if case["kv_dtype"] != "bf16" else None
    check_attention(g["out"][0], g["lse"][0], ref_out, ref_lse, case["kv_dtype"], lse_bound=bound)


def test_shard_merge_against_the_oracle_combine():
    """The merge alone on random states, with ranks and whole queries that selected nothing."""
    import deepseek_sparse_attention_head_b200 as dsa
    rng = np.random.default_rng(3)
    R, Bq = 5, 3
    all_out = rng.standard_normal((R, Bq, 64, 512)).astype(np.float32)
    all_lse = (rng.standard_normal((R, Bq, 64)) * 30).astype(np.float32)
    all_lse[1] = -np.inf                  # rank 1 holds none of the selection
    all_lse[:, 2, :7] = -np.inf           # query 2, heads 0..6: nothing anywhere
    all_out[:, 2, :7] = 0.0
    for odt in (torch.float32, torch.bfloat16):
        out = torch.full((Bq, 64, 512), float("nan"), dtype=odt, device="cuda")
        lse = torch.full((Bq, 64), float("nan"), dtype=torch.float32, device="cuda")
        dsa.dsa_shard_merge(torch.from_numpy(all_out).cuda(), torch.from_numpy(all_lse).cuda(), out, lse)
        torch.cuda.synchronize()
        for q in range(Bq):
            ref_out, ref_lse = oracle.combine_partials(list(all_lse[:, q].astype(np.float64)),
                                                       [np.ones(64)] * R, list(all_out[:, q].astype(np.float64)))
            got = out[q].float().cpu().numpy()
            tol = 2e-6 if odt == torch.float32 else 8e-3
            assert np.all(np.abs(got - ref_out) <= tol * (1 + np.abs(ref_out)))
            gl = lse[q].cpu().numpy()
            fin = np.isfinite(ref_lse)
            assert np.array_equal(np.isfinite(gl), fin)
            assert np.allclose(gl[fin], ref_lse[fin], rtol=1e-6, atol=1e-5)
            assert np.all(got[~fin] == 0)
