"""Parity criteria between the CUDA path and the fp64 oracle.

Tolerances:
  * indexer scores: |gpu - oracle| <= 2e-5 * M + 1e-6 * |oracle|, where
    M = sum_h w[h] * sum_d |q[h,d] * k[s,d]| bounds every term the fp32 sums see. The
    fp8 x fp8 (or bf16 x bf16) products are exact; the 128-term tensor-core accumulation
    and the 64-term fp32 epilogue sum add at most about 2^-24 x 200 = 1.2e-5 of M, and
    the 1e-6 relative term covers the final rounding of the stored fp32 score;
  * top-k on identical fp32 scores: exact (every key above the k-th is selected, the
    right number of keys equal to it, nothing at or past vis);
  * top-k against the fp64 oracle: the selected sets agree except for tokens whose
    oracle score lies within 1e-3 relative of the oracle's k-th score;
  * page map: bit-exact;
  * attention: cosine >= 0.99999 for every (query, head) row, max abs error <= 2e-3
    (bf16 latent cache) or <= 1e-2 (fp8 latent cache), the bounds the problem statement
    sets; lse within 1e-4 (bf16) or 5e-3 (fp8), which bounds the logit error of the
    reduced-precision query operand (bf16 queries against fp8 rows) summed over 576
    columns.
"""
import numpy as np

import oracle


def score_magnitude(case, queries=None):
    """M[q, s] = sum_h |w'[q,h]| sum_d |q[q,h,d] k[s,d]| in fp64 (0 past vis)."""
    queries = np.arange(case["Bq"]) if queries is None else np.asarray(queries)
    L_max = case["max_pages"] * 64
    vis = oracle.visible_lengths(case)
    Q = np.abs(oracle.dequant_index_queries(case))
    w = np.abs(case["head_w"].astype(np.float64))
    M = np.zeros((len(queries), L_max))
    for i, q in enumerate(queries):
        v = int(vis[q])
        for s0 in range(0, v, 65536):
            s1 = min(v, s0 + 65536)
            slots = oracle.physical_slots(case["block_table"][q // case["n_q"]], np.arange(s0, s1))
            K = np.abs(oracle.dequant_index_keys(case, slots))
            M[i, s0:s1] = (w[q][:, None] * (Q[q] @ K.T)).sum(axis=0)
    return M


def check_scores(gpu, ref, M, vis):
    for i in range(ref.shape[0]):
        v = int(vis[i])
        g, r, m = gpu[i, :v].astype(np.float64), ref[i, :v], M[i, :v]
        assert np.all(np.isfinite(g)), f"row {i}: non-finite score"
        err = np.abs(g - r)
        tol = 2e-5 * m + 1e-6 * np.abs(r)
        bad = np.nonzero(err > tol)[0]
        assert bad.size == 0, f"row {i}: {bad.size} scores out of tolerance, first s={bad[0]} gpu={g[bad[0]]} " \
                              f"oracle={r[bad[0]]} tol={tol[bad[0]]}"


def check_topk_exact(sel, scores_f32, vis, K):
    """sel: one row of selected logical indices (-1 padded); scores_f32: the fp32 scores
    the selection was made from. Decision taken in the same precision: exact."""
    v = int(vis)
    k = min(K, v)
    chosen = sel[sel >= 0]
    assert chosen.size == k, f"selected {chosen.size}, expected {k}"
    assert np.all(sel[k:] == -1) or np.sum(sel >= 0) == k
    assert np.unique(chosen).size == k, "duplicate index"
    assert np.all(chosen < v), "index past the visible prefix"
    if k == v:
        assert set(chosen.tolist()) == set(range(v))
        return
    s = scores_f32[:v].astype(np.float32)
    kth = np.sort(s)[::-1][k - 1]
    above = np.nonzero(s > kth)[0]
    assert set(above.tolist()) <= set(chosen.tolist()), "a score above the k-th is missing"
    assert np.all(s[chosen] >= kth), "a score below the k-th was selected"


def check_topk_near_tie(sel, ref_sel, ref_scores, vis, K, rel=1e-3):
    v = int(vis)
    k = min(K, v)
    chosen = set(sel[sel >= 0].tolist())
    assert len(chosen) == k and all(0 <= c < v for c in chosen)
    ref = set(ref_sel[ref_sel >= 0].tolist())
    if k == v:
        assert chosen == set(range(v))
        return 0
    tau = np.sort(ref_scores[:v])[::-1][k - 1]
    diff = chosen ^ ref
    near = [s for s in diff if abs(ref_scores[s] - tau) <= rel * abs(tau)]
    far = sorted(diff - set(near))
    assert not far, f"{len(far)} selection differences outside the near-tie band, e.g. s={far[:4]} " \
                    f"scores={[ref_scores[s] for s in far[:4]]} tau={tau}"
    return len(diff)


def fp8_lse_bound(case, physical):
    """Per (query row, head) bound on the fp8 path's log-sum-exp error, natural-log units.

    The decode kernel folds each row's per-group scale into fp16 key values: the group
    multiplier s_g / 2^E_j and the product code x multiplier are each rounded to fp16 once
    (relative error at most 2^-11 each), so a logit z = sum_g z_g (log2 units, z_g the part
    from scale group g) is off by at most 2^-10 sum_g |z_g|, and the log-sum-exp by at most
    ln 2 times the largest such bound over the selected rows. Built from the inputs with the
    oracle's dequantisation; unused slots (-1) are skipped."""
    import oracle
    log2e = 1.0 / np.log(2.0)
    groups = [slice(128 * g, 128 * g + 128) for g in range(4)] + [slice(512, 576)]
    bq = physical.shape[0]
    bound = np.zeros((bq, 64))
    for q in range(bq):
        sl = physical[q][physical[q] >= 0].astype(np.int64)
        if sl.size == 0:
            continue
        qm = oracle.decode_bf16(case["q_mla"][q])
        kv = oracle.dequant_latent_rows(case, sl)
        mag = sum(np.abs(qm[:, c] @ kv[:, c].T) for c in groups) * case["softmax_scale"] * log2e
        bound[q] = np.log(2.0) * 2.0 ** -10 * mag.max(axis=1)
    return bound


def check_attention(out, lse, ref_out, ref_lse, kv_dtype, lse_bound=None):
    """Element-wise comparison with the oracle. `lse_bound` (fp8 path, see fp8_lse_bound)
    widens the log-sum-exp tolerance where logits are large enough for the fp16 rounding of
    the folded group scales to exceed the fixed one."""
    max_abs = 2e-3 if kv_dtype == "bf16" else 1e-2
    lse_tol = 1e-4 if kv_dtype == "bf16" else 5e-3
    assert np.all(np.isfinite(out)), "non-finite output"
    err = np.abs(out - ref_out)
    assert err.max() <= max_abs, f"max abs error {err.max()} > {max_abs}"
    num = (out * ref_out).sum(-1)
    den = np.linalg.norm(out, axis=-1) * np.linalg.norm(ref_out, axis=-1)
    zero = (np.linalg.norm(ref_out, axis=-1) == 0)
    assert np.all(np.linalg.norm(out, axis=-1)[zero] == 0), "output should be zero for an empty selection"
    cos = np.where(zero, 1.0, num / np.where(den > 0, den, 1.0))
    assert cos.min() >= 0.99999, f"min per-row cosine {cos.min()}"
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse), fin), "lse finiteness differs"
    if fin.any():
        tol = np.full(ref_lse.shape, lse_tol) if lse_bound is None else np.maximum(lse_tol, lse_bound)
        d = np.abs(lse[fin] - ref_lse[fin])
        worst = int(np.argmax(d - tol[fin]))
        assert np.all(d <= tol[fin]), f"lse error {d[worst]} > {tol[fin][worst]}"
    return float(err.max()), float(cos.min())
