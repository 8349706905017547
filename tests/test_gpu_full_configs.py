"""The serving-size workloads (B=64 serving decode, one 1M-token stream, 2048-query chunked
prefill, and the serving rows with three speculative queries each) through the fused
decode layer, the call bench.py times.

The oracle recomputes sampled query rows element by element (scores, top-k set up to
near-ties, attention on the GPU's own selection). Every row is checked against
properties that hold at any size: the selection count is min(top_k, vis), indices are
distinct and visible, the page map is bit-exact, and the outputs are finite.
"""
import functools

import numpy as np
import pytest

import oracle
from dsa_inputs import generate, spec
from tests.compare import check_attention, check_scores, check_topk_near_tie, score_magnitude

pytestmark = pytest.mark.gpu


def _sample(name, case):
    vis = oracle.visible_lengths(case)
    Bq = case["Bq"]
    if name == "cfg4":
        # chunked prefill: every 16th query plus the last (causal visibility grows along the chunk)
        return sorted(set(range(0, Bq, 16)) | {Bq - 1})
    if Bq == 1:
        return [0]
    picks = {0, Bq - 1, int(np.argmax(vis)), int(np.argmin(vis))}
    if case["n_q"] > 1:
        # every query of the first and of the shortest row (causal visibility differs by one)
        for b in (0, int(np.argmin(case["seq_lens"]))):
            picks |= set(range(b * case["n_q"], (b + 1) * case["n_q"]))
    dense = np.nonzero(vis <= case["top_k"])[0]
    if dense.size:
        picks.add(int(dense[0]))
    return sorted(picks)


@functools.lru_cache(maxsize=1)
def _run(name):
    """GPU scores (dsa_indexer_scores) and one fused dsa_decode_layer call."""
    import torch
    from tests.gpu_path import GpuCase
    case = generate(spec(name))
    g = GpuCase(case)
    scores, serr = g.indexer()
    layer = g.layer()
    q = _sample(name, case)
    sc = scores[torch.as_tensor(q, device=scores.device)].cpu().numpy()
    del scores, g
    torch.cuda.empty_cache()
    return case, q, sc, serr, layer


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4", "mtp"])
def test_full_size_every_row_properties(name):
    case, _, _, serr, r = _run(name)
    assert serr == 0 and r["err"] == 0
    vis = oracle.visible_lengths(case)
    K = case["top_k"]
    lo = r["logical"]
    for q in range(case["Bq"]):
        row = lo[q]
        k = min(K, int(vis[q]))
        sel = row[row >= 0]
        assert sel.size == k, f"query {q}: {sel.size} selected, expected {k}"
        assert np.all(row[row < 0] == -1)
        assert np.unique(sel).size == k and (k == 0 or int(sel.max()) < int(vis[q]))
        if int(vis[q]) <= K:                        # dense path: every visible token
            assert np.array_equal(np.sort(sel), np.arange(int(vis[q])))
    assert np.array_equal(r["physical"].astype(np.int64), oracle.pagemap(case, lo.astype(np.int64)))
    assert np.all(np.isfinite(r["out"]))
    assert np.all(np.isfinite(r["lse"]) == (vis > 0)[:, None])


@pytest.mark.parametrize("name", ["cfg2", "cfg3", "cfg4", "mtp"])
def test_full_size_sampled_rows_against_oracle(name):
    case, q, sc, _, r = _run(name)
    vis = oracle.visible_lengths(case)[q]
    ref = oracle.indexer_scores(case, q)
    check_scores(sc, ref, score_magnitude(case, q), vis)
    ref_sel = oracle.topk_logical(ref, vis, case["top_k"])
    for i, qq in enumerate(q):
        check_topk_near_tie(r["logical"][qq], ref_sel[i], ref[i], vis[i], case["top_k"])
    phys = r["physical"][q].astype(np.int64)
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys, q)
    check_attention(r["out"][q], r["lse"][q], ref_out, ref_lse, case["kv_dtype"])
