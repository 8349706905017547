"""Plausible mistakes planted in the fp64 oracle, on the CPU, to show that its pins catch
them (tests/test_oracle_mutations.py runs the pins once per mistake). Each entry replaces
one oracle function with a copy that carries one error: a wrong constant, a dropped term,
a swapped index, a wrong order or sign. Test infrastructure only."""
import numpy as np

import oracle
from oracle import dsa_oracle as od

PAGE, H, DI, DK, DV = od.PAGE, od.H, od.DI, od.DK, od.DV


def _set(name, fn):
    setattr(od, name, fn)
    if hasattr(oracle, name):
        setattr(oracle, name, fn)


def _e4m3_table(bias=7, subnormal_implicit_one=False):
    c = np.arange(256).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - bias).astype(np.int64))
    sub = np.ldexp((1.0 if subnormal_implicit_one else 0.0) + m / 8.0, -6)
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, v)


def _indexer(relu_after_sum=False, key_scale=True, query_scale=True, vis_extra=0):
    def indexer_scores(case, queries=None):
        queries = np.arange(case["Bq"]) if queries is None else np.asarray(queries)
        L_max = case["max_pages"] * PAGE
        vis = od.visible_lengths(case)
        Q = od._decode(case["q_idx"], case["idx_dtype"])
        if query_scale and case["q_idx_scale"] is not None:
            Q = Q * case["q_idx_scale"].astype(np.float64)[:, :, None]
        w = case["head_w"].astype(np.float64)
        out = np.full((len(queries), L_max), -np.inf)
        for i, q in enumerate(queries):
            v = min(int(vis[q]) + vis_extra, L_max)
            slots = od.physical_slots(case["block_table"][q // case["n_q"]], np.arange(v))
            flat = case["k_cache"].reshape(-1, DI)
            K = od._decode(flat[np.maximum(slots, 0)], case["idx_dtype"])
            if key_scale and case["k_scale"] is not None:
                K = K * case["k_scale"].reshape(-1).astype(np.float64)[np.maximum(slots, 0)][:, None]
            logits = Q[q] @ K.T
            if relu_after_sum:
                out[i, :v] = np.maximum((w[q][:, None] * logits).sum(axis=0), 0.0)
            else:
                out[i, :v] = (w[q][:, None] * np.maximum(logits, 0.0)).sum(axis=0)
        return out
    return indexer_scores


def _topk(ties_high=False, ascending=False):
    def topk_logical(scores, vis, top_k):
        n = scores.shape[0]
        out = np.full((n, top_k), -1, dtype=np.int64)
        for i in range(n):
            v = int(vis[i])
            k = min(top_k, v)
            if k == 0:
                continue
            idx = np.arange(v)
            key = scores[i, :v] if ascending else -scores[i, :v]
            order = np.lexsort((-idx if ties_high else idx, key))
            out[i, :k] = idx[order[:k]]
        return out
    return topk_logical


def _physical_slots_swapped(block_table_row, logical):
    logical = np.asarray(logical, dtype=np.int64)
    out = np.full(logical.shape, -1, dtype=np.int64)
    ok = logical >= 0
    li = logical[ok]
    out[ok] = block_table_row[li % PAGE].astype(np.int64) * PAGE + li // PAGE
    return out


def _latent_rows_rope_scale_from_group3(case, slots):
    kv = od._decode(case["kv_cache"][slots], case["kv_dtype"])
    if case["kv_scale"] is not None:
        sc = case["kv_scale"][slots].astype(np.float64)
        kv = kv * sc[:, np.minimum(np.arange(DK) // 128, 3)]
    return kv


def _packed_rows(scale_shift=0, rope_big_endian=False):
    def dequant(rows):
        rows = np.ascontiguousarray(rows, dtype=np.uint8)
        n = rows.shape[0]
        latent = od.decode_e4m3(rows[:, :DV])
        scales = rows[:, DV:DV + 16].copy().view("<f4").astype(np.float64)
        scales = np.roll(scales, scale_shift, axis=1)
        latent = latent * np.repeat(scales, 128, axis=1)
        rope = od.decode_bf16(rows[:, DV + 16:].copy().view(">u2" if rope_big_endian else "<u2").astype(np.uint16)
                              .reshape(n, DK - DV))
        return np.concatenate([latent, rope], axis=1)
    return dequant


def _mla(scale_on=True, value_cols=slice(0, DV), key_cols=slice(0, DK), lse_with_max=True):
    def attention(case, physical, queries=None):
        queries = np.arange(physical.shape[0]) if queries is None else np.asarray(queries)
        scale = float(case["softmax_scale"]) if scale_on else 1.0
        out = np.zeros((len(queries), H, DV))
        lse = np.full((len(queries), H), -np.inf)
        for i, q in enumerate(queries):
            sel = physical[i][physical[i] >= 0]
            if sel.size == 0:
                continue
            qm = od.decode_bf16(case["q_mla"][q])
            KV = od.dequant_latent_rows(case, sel)
            z = scale * (qm[:, key_cols] @ KV[:, key_cols].T)
            m = z.max(axis=1, keepdims=True)
            e = np.exp(z - m)
            l = e.sum(axis=1, keepdims=True)
            out[i] = (e / l) @ KV[:, value_cols]
            lse[i] = ((m if lse_with_max else 0.0) + np.log(l))[:, 0]
        return out, lse
    return attention


def _combine_wrong_sign(ms, ls, os_):
    ms, ls, os_ = np.stack(ms), np.stack(ls), np.stack(os_)
    M = ms.max(axis=0)
    Msafe = np.where(np.isfinite(M), M, 0.0)
    a = np.where(np.isfinite(ms), np.exp(Msafe[None, :] - ms), 0.0)
    L = (a * ls).sum(axis=0)
    O = (a[:, :, None] * os_).sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(L[:, None] > 0, O / np.where(L > 0, L, 1.0)[:, None], 0.0)
        lse = np.where(L > 0, Msafe + np.log(np.where(L > 0, L, 1.0)), -np.inf)
    return out, lse


def _visible_lengths_causal_off_by_one(case):
    if case.get("q_pos") is not None:
        return case["q_pos"].astype(np.int64)
    return np.repeat(case["seq_lens"].astype(np.int64), case["n_q"])


def _physical_slots_without_page_size(block_table_row, logical):
    logical = np.asarray(logical, dtype=np.int64)
    out = np.full(logical.shape, -1, dtype=np.int64)
    ok = logical >= 0
    li = logical[ok]
    out[ok] = block_table_row[li // PAGE].astype(np.int64) + li % PAGE
    return out


def _mla_softmax_over_heads(case, physical, queries=None):
    queries = np.arange(physical.shape[0]) if queries is None else np.asarray(queries)
    scale = float(case["softmax_scale"])
    out = np.zeros((len(queries), H, DV))
    lse = np.full((len(queries), H), -np.inf)
    for i, q in enumerate(queries):
        sel = physical[i][physical[i] >= 0]
        if sel.size == 0:
            continue
        qm = od.decode_bf16(case["q_mla"][q])
        KV = od.dequant_latent_rows(case, sel)
        z = scale * (qm @ KV.T)                                  # [64 heads, n keys]
        m = z.max(axis=0, keepdims=True)                         # normalised over heads
        e = np.exp(z - m)
        l = e.sum(axis=0, keepdims=True)
        out[i] = (e / l) @ KV[:, :DV]
        lse[i] = np.log(np.exp(z).sum(axis=1))
    return out, lse


def _combine_without_l(ms, ls, os_):
    ms, ls, os_ = np.stack(ms), np.stack(ls), np.stack(os_)
    M = ms.max(axis=0)
    Msafe = np.where(np.isfinite(M), M, 0.0)
    a = np.where(np.isfinite(ms), np.exp(ms - Msafe[None, :]), 0.0)
    L = a.sum(axis=0)                                            # the l_s weights are missing
    O = (a[:, :, None] * os_).sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(L[:, None] > 0, O / np.where(L > 0, L, 1.0)[:, None], 0.0)
        lse = np.where(L > 0, Msafe + np.log(np.where(L > 0, L, 1.0)), -np.inf)
    return out, lse


def _bf16_shift15(bits):
    b = np.asarray(bits).astype(np.uint32) << np.uint32(15)
    return b.view(np.float32).astype(np.float64)


# unmutated copies: the pins must pass with these, which shows that a failure under a
# mutation comes from the planted mistake and not from the copy
CONTROLS = {
    "control_indexer_copy": lambda: _set("indexer_scores", _indexer()),
    "control_topk_copy": lambda: _set("topk_logical", _topk()),
    "control_mla_copy": lambda: _set("mla_sparse_attention", _mla()),
    "control_e4m3_table": lambda: setattr(od, "_E4M3", _e4m3_table()),
    "control_packed_rows_copy": lambda: _set("_dequant_packed_rows", _packed_rows()),
}

MUTATIONS = {
    "e4m3_exponent_bias_8": lambda: setattr(od, "_E4M3", _e4m3_table(bias=8)),
    "e4m3_subnormals_with_implicit_one": lambda: setattr(od, "_E4M3", _e4m3_table(subnormal_implicit_one=True)),
    "bf16_shifted_by_15": lambda: _set("decode_bf16", _bf16_shift15),
    "indexer_relu_after_head_sum": lambda: _set("indexer_scores", _indexer(relu_after_sum=True)),
    "indexer_drops_key_scale": lambda: _set("indexer_scores", _indexer(key_scale=False)),
    "indexer_drops_query_scale": lambda: _set("indexer_scores", _indexer(query_scale=False)),
    "indexer_sees_one_token_too_many": lambda: _set("indexer_scores", _indexer(vis_extra=1)),
    "topk_ties_to_higher_index": lambda: _set("topk_logical", _topk(ties_high=True)),
    "topk_takes_the_smallest": lambda: _set("topk_logical", _topk(ascending=True)),
    "pagemap_page_and_offset_swapped": lambda: _set("physical_slots", _physical_slots_swapped),
    "latent_rope_scaled_by_group_3": lambda: _set("dequant_latent_rows", _latent_rows_rope_scale_from_group3),
    "mla_without_softmax_scale": lambda: _set("mla_sparse_attention", _mla(scale_on=False)),
    "mla_values_are_the_last_512_columns": lambda: _set("mla_sparse_attention", _mla(value_cols=slice(DK - DV, DK))),
    "mla_keys_without_rope_columns": lambda: _set("mla_sparse_attention", _mla(key_cols=slice(0, DV))),
    "mla_lse_without_the_max": lambda: _set("mla_sparse_attention", _mla(lse_with_max=False)),
    "combine_weights_with_wrong_sign": lambda: _set("combine_partials", _combine_wrong_sign),
    "combine_without_the_normalisers": lambda: _set("combine_partials", _combine_without_l),
    "causal_visibility_off_by_one": lambda: _set("visible_lengths", _visible_lengths_causal_off_by_one),
    "pagemap_without_the_page_size": lambda: _set("physical_slots", _physical_slots_without_page_size),
    "mla_softmax_over_heads": lambda: _set("mla_sparse_attention", _mla_softmax_over_heads),
    "packed_rows_scales_one_group_off": lambda: _set("_dequant_packed_rows", _packed_rows(scale_shift=1)),
    "packed_rows_rope_big_endian": lambda: _set("_dequant_packed_rows", _packed_rows(rope_big_endian=True)),
}


def apply(name):
    (MUTATIONS.get(name) or CONTROLS[name])()


def _rope_half_split(x, pos, base=10000.0):
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    theta = base ** (-2.0 * np.arange(n // 2) / n)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :n // 2], x[..., n // 2:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _rope_reversed(x, pos, base=10000.0):
    return _ORIG_ROPE(x, -np.asarray(pos, dtype=np.float64), base)


def _slots_one_page_off(case, rows, pos):
    bt = case["block_table"]
    return bt[rows, np.minimum(pos // PAGE + 1, bt.shape[1] - 1)].astype(np.int64) * PAGE + pos % PAGE


_ORIG_ROPE = od.rope_interleaved
MUTATIONS["rope_rotates_halves_not_pairs"] = lambda: _set("rope_interleaved", _rope_half_split)
MUTATIONS["rope_turns_the_other_way"] = lambda: _set("rope_interleaved", _rope_reversed)
MUTATIONS["append_slot_one_page_off"] = lambda: _set("physical_slots_rows", _slots_one_page_off)


def _shard_select_ties_high(cand_score, cand_token, top_k):
    ok = cand_token >= 0
    sc, tok = cand_score[ok], cand_token[ok]
    order = np.lexsort((-tok, -sc))
    out = np.full(top_k, -1, dtype=np.int64)
    k = min(top_k, tok.size)
    out[:k] = tok[order[:k]]
    return out


def _shard_candidates_local_tokens(scores_row, lo, hi, top_k):
    local = od.topk_logical(scores_row[None, lo:hi], np.array([hi - lo]), top_k)[0]
    ok = local >= 0
    tok = np.where(ok, local, -1)
    sc = np.where(ok, scores_row[np.maximum(local + lo, 0)], -np.inf)
    return sc, tok


def _shard_candidates_one_short(scores_row, lo, hi, top_k):
    sc, tok = _shard_candidates_copy(scores_row, lo, hi, top_k)
    if hi - lo >= top_k:
        sc[-1], tok[-1] = -np.inf, -1
    return sc, tok


def _shard_candidates_copy(scores_row, lo, hi, top_k):
    local = od.topk_logical(scores_row[None, lo:hi], np.array([hi - lo]), top_k)[0]
    ok = local >= 0
    tok = np.where(ok, local + lo, -1)
    sc = np.where(ok, scores_row[np.maximum(tok, 0)], -np.inf)
    return sc, tok


MUTATIONS["shard_select_ties_to_higher_token"] = lambda: _set("shard_global_select", _shard_select_ties_high)
MUTATIONS["shard_candidates_keep_local_tokens"] = lambda: _set("shard_candidates", _shard_candidates_local_tokens)
MUTATIONS["shard_candidates_one_short"] = lambda: _set("shard_candidates", _shard_candidates_one_short)
CONTROLS["control_shard_candidates_copy"] = lambda: _set("shard_candidates", _shard_candidates_copy)
