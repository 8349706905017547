"""fp64 CPU oracle for the DeepSeek-Sparse-Attention (DSA) decode step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
this module: only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline /
reference arm use it. It shares no code with the CUDA library.

What it computes, stage by stage, in the order the pages name the kernels
("GLM-52 Runs on RTX 4090", kernel list: lightning-indexer GEMM, top-k +
page-mapping transforms, MLA sparse decode; glm-5.2-4090 README, "how it works"):

  1. indexer_scores     score[q,s] = sum_h w[q,h] * ReLU(q_idx[q,h] . k_idx[s])  for s < vis(q)
  2. topk_logical       the min(top_k, vis(q)) highest-scoring logical token indices
  3. pagemap            logical token -> physical cache slot through the block table
  4. mla_sparse_attention  64-head softmax attention over only the selected rows of the
                        576-wide latent cache (keys: all 576 columns, values: first 512)
                        ("Show HN: colibri", features: compressed KV of 576 floats per
                        token, 64 heads, no GQA)

Every stored code is decoded exactly to fp64 (own E4M3 and bf16 decoders, from the
OCP 8-bit floating point definition and the bfloat16 bit layout) and multiplied by
its fp32 scale; all arithmetic after that is fp64.

Readings of points the pages leave open (the pages name the kernels but give no formula,
format, page size or tie rule; these are the plainest readings the rest supports):
  * the indexer has no extra 1/sqrt(d) factor, ReLU comes before the head weights;
  * fp8 indexer queries carry one fp32 scale per (query, head); fp8 indexer keys one
    fp32 scale per token; fp8 latent rows five fp32 scales, one per 128-column group of
    the 512 latent columns plus one for the 64 rope columns;
  * ties in top-k go to the lower logical index; output is in descending-score order;
  * with vis(q) <= top_k every visible token is selected (the dense path);
  * an empty selection gives a zero output and lse = -inf.

The token-sharded step (sharded_decode_layer, the long-context extension): each row's
tokens spread over several ranks, a local top-k per rank, an exchange of (score, token)
candidates, a global selection (ties to the lower global token), each rank's attention
state over the selected tokens it holds, and the log-sum-exp merge of those states.

The step before the path (rope_quantize_append, the next step after the hot path): the new
tokens' projected indexer queries and keys and latent rows get partial interleaved RoPE
("Show HN: colibri", features: MLA with partial interleaved RoPE) on their 64 rope columns
(the first 64 of the 128 indexer dims, the last 64 of the 576 latent columns), are
quantised to E4M3 with amax/448 fp32 scales (one per query head, one per key, one per
latent column group), and the keys and latent rows are written into the paged caches at
the token's slot.
"""
from __future__ import annotations

import numpy as np

PAGE = 64
H = 64
DI = 128
DK = 576
DV = 512


# ----------------------------------------------------------------------------------
# storage formats

def _e4m3_value(c: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 ("fn" variant) code -> exact fp64 value.

    1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits. Exponent field 0 is
    subnormal (value = m/8 * 2^-6). There is no infinity; S.1111.111 is NaN, so the
    largest finite magnitude is 1.75 * 2^8 = 448."""
    c = np.asarray(c).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = sign * np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, v)


_E4M3 = _e4m3_value(np.arange(256))   # the definition evaluated once for every code


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes -> exact fp64 values (lookup in the 256-entry table of _e4m3_value)."""
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit pattern -> exact fp64 value (bf16 is the top half of an IEEE fp32)."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def encode_e4m3(x: np.ndarray) -> np.ndarray:
    """E4M3 codes of finite values (OCP 8-bit floating point): the nearest representable
    magnitude, ties to the even code (mantissa LSB 0), saturating at 448; the sign bit
    follows the sign of x (so -0 and small negatives give 0x80)."""
    x = np.asarray(x, dtype=np.float64)
    pos_vals = _E4M3[:0x7F]                       # codes 0x00 .. 0x7E, increasing, 0 .. 448
    m = np.minimum(np.abs(x), pos_vals[-1])
    hi = np.clip(np.searchsorted(pos_vals, m, side="left"), 0, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = m - pos_vals[lo], pos_vals[hi] - m
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(take_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def quantize_e4m3(x: np.ndarray):
    """amax / 448 scaling along the last axis, stored as fp32 (1 for an all-zero row), and
    the E4M3 codes of x / scale (fp64 division by the stored scale) -> (codes, scales)."""
    x = np.asarray(x, dtype=np.float64)
    amax = np.abs(x).max(axis=-1)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
    return encode_e4m3(x / scale.astype(np.float64)[..., None]), scale


def encode_bf16(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of finite fp64 values: round to nearest even on the fp32 value's
    low 16 bits (the fp64 -> fp32 step rounds to nearest too)."""
    u = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def _decode(codes: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return decode_bf16(codes)
    if dtype == "fp8":
        return decode_e4m3(codes)
    raise ValueError(dtype)


def dequant_index_queries(case: dict) -> np.ndarray:
    """q_idx [Bq, 64, 128] as fp64: code value times its per-(query, head) scale."""
    q = _decode(case["q_idx"], case["idx_dtype"])
    if case["q_idx_scale"] is not None:
        q = q * case["q_idx_scale"].astype(np.float64)[:, :, None]
    return q


def dequant_index_keys(case: dict, slots: np.ndarray) -> np.ndarray:
    """Indexer keys of the given physical slots, [n, 128] fp64 (per-token scale applied)."""
    flat = case["k_cache"].reshape(-1, DI)
    k = _decode(flat[slots], case["idx_dtype"])
    if case["k_scale"] is not None:
        k = k * case["k_scale"].reshape(-1).astype(np.float64)[slots][:, None]
    return k


def _dequant_packed_rows(rows: np.ndarray) -> np.ndarray:
    """Packed fp8 latent rows (656 bytes each: the layout variant with bf16 rope columns and
    four fp32 group scales, "Show HN: colibri", features: 576 values per token = 512 latent +
    64 rope) -> [n, 576] fp64. Bytes [0, 512): E4M3 codes of the latent columns, column group
    g = [128g, 128g+128) times the fp32 scale stored little-endian at bytes [512 + 4g,
    516 + 4g); bytes [528, 656): the 64 rope values as bf16."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    latent = decode_e4m3(rows[:, :DV])                                        # [n, 512]
    scales = rows[:, DV:DV + 16].copy().view("<f4").astype(np.float64)        # [n, 4]
    latent = latent * np.repeat(scales, 128, axis=1)
    rope = decode_bf16(rows[:, DV + 16:].copy().view("<u2").reshape(n, DK - DV))
    return np.concatenate([latent, rope], axis=1)


def dequant_latent_rows(case: dict, slots: np.ndarray) -> np.ndarray:
    """Latent KV rows of the given physical slots, [n, 576] fp64.

    fp8 rows: column group g in {0..3} covers columns [128g, 128g+128) and group 4 the
    64 rope columns [512, 576); each group has its own fp32 scale per row."""
    if case["kv_dtype"] == "fp8r":
        return _dequant_packed_rows(case["kv_cache"][slots])
    kv = _decode(case["kv_cache"][slots], case["kv_dtype"])
    if case["kv_scale"] is not None:
        sc = case["kv_scale"][slots].astype(np.float64)
        col_group = np.minimum(np.arange(DK) // 128, 4)
        kv = kv * sc[:, col_group]
    return kv


# ----------------------------------------------------------------------------------
# paging

def visible_lengths(case: dict) -> np.ndarray:
    """vis(q): q_pos[q] + 1 for causal queries, else the sequence length of q's row."""
    if case.get("q_pos") is not None:
        return case["q_pos"].astype(np.int64) + 1
    return np.repeat(case["seq_lens"].astype(np.int64), case["n_q"])


def physical_slots(block_table_row: np.ndarray, logical: np.ndarray) -> np.ndarray:
    """Page-mapping transform of one row: slot = table[i // 64] * 64 + i % 64; -1 stays -1."""
    logical = np.asarray(logical, dtype=np.int64)
    out = np.full(logical.shape, -1, dtype=np.int64)
    ok = logical >= 0
    li = logical[ok]
    out[ok] = block_table_row[li // PAGE].astype(np.int64) * PAGE + li % PAGE
    return out


def pagemap(case: dict, logical: np.ndarray) -> np.ndarray:
    """[Bq, top_k] logical token indices -> physical slots (query q uses row q // n_q)."""
    out = np.empty(logical.shape, dtype=np.int64)
    for q in range(logical.shape[0]):
        out[q] = physical_slots(case["block_table"][q // case["n_q"]], logical[q])
    return out


# ----------------------------------------------------------------------------------
# stage 1: lightning indexer

def indexer_scores(case: dict, queries=None) -> np.ndarray:
    """score[q, s] = sum_h w[q,h] * max(0, <q_idx[q,h], k_idx[s]>) for s < vis(q), else -inf.

    Returns fp64 [len(queries), L_max] with L_max = max_pages * 64. `queries` selects a
    subset of the Bq query rows (default: all)."""
    Bq = case["Bq"]
    queries = np.arange(Bq) if queries is None else np.asarray(queries)
    L_max = case["max_pages"] * PAGE
    vis = visible_lengths(case)
    Q = dequant_index_queries(case)
    w = case["head_w"].astype(np.float64)
    out = np.full((len(queries), L_max), -np.inf)
    chunk = 65536                                            # tokens per step (memory only)
    for i, q in enumerate(queries):
        v = int(vis[q])
        for s0 in range(0, v, chunk):
            s1 = min(v, s0 + chunk)
            slots = physical_slots(case["block_table"][q // case["n_q"]], np.arange(s0, s1))
            K = dequant_index_keys(case, slots)             # [n, 128]
            logits = Q[q] @ K.T                              # [64, n]
            out[i, s0:s1] = (w[q][:, None] * np.maximum(logits, 0.0)).sum(axis=0)
    return out


# ----------------------------------------------------------------------------------
# stage 2: top-k selection

def topk_logical(scores: np.ndarray, vis: np.ndarray, top_k: int) -> np.ndarray:
    """Per query, the min(top_k, vis) largest scores among tokens [0, vis).

    Order: descending score, ties to the lower index (a stable sort). Unused entries -1.
    With vis <= top_k this is every visible token (the dense path)."""
    n = scores.shape[0]
    out = np.full((n, top_k), -1, dtype=np.int64)
    for i in range(n):
        v = int(vis[i])
        k = min(top_k, v)
        if k == 0:
            continue
        idx = np.arange(v)
        order = np.lexsort((idx, -scores[i, :v]))   # primary: -score, secondary: index
        out[i, :k] = idx[order[:k]]
    return out


# ----------------------------------------------------------------------------------
# stage 3: MLA sparse attention (+ the split-KV combine)

def mla_sparse_attention(case: dict, physical: np.ndarray, queries=None):
    """out[q,h,:] = sum_j softmax_j(z[q,h,:]) * V[slot_j], z = scale * <q_mla[q,h], K[slot_j]>.

    K = all 576 columns of the selected latent rows, V = their first 512 columns.
    physical: [n, top_k] slots (-1 = unused). Returns (out fp64 [n, 64, 512],
    lse fp64 [n, 64]) with lse = log sum_j exp(z_j); an empty selection gives 0 and -inf."""
    queries = np.arange(physical.shape[0]) if queries is None else np.asarray(queries)
    scale = float(case["softmax_scale"])
    out = np.zeros((len(queries), H, DV))
    lse = np.full((len(queries), H), -np.inf)
    for i, q in enumerate(queries):
        sel = physical[i][physical[i] >= 0]
        if sel.size == 0:
            continue
        qm = decode_bf16(case["q_mla"][q])                   # [64, 576]
        KV = dequant_latent_rows(case, sel)                  # [n, 576]
        z = scale * (qm @ KV.T)                              # [64, n]
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        l = e.sum(axis=1, keepdims=True)
        out[i] = (e / l) @ KV[:, :DV]
        lse[i] = (m + np.log(l))[:, 0]
    return out, lse


def mla_partials(case: dict, slots: np.ndarray, q: int):
    """Un-normalised attention state of one query over one subset of slots:
    m[h] = max_j z, l[h] = sum_j exp(z - m), o[h] = sum_j exp(z - m) V_j."""
    scale = float(case["softmax_scale"])
    slots = slots[slots >= 0]
    if slots.size == 0:
        return np.full(H, -np.inf), np.zeros(H), np.zeros((H, DV))
    qm = decode_bf16(case["q_mla"][q])
    KV = dequant_latent_rows(case, slots)
    z = scale * (qm @ KV.T)
    m = z.max(axis=1)
    e = np.exp(z - m[:, None])
    return m, e.sum(axis=1), e @ KV[:, :DV]


def combine_partials(ms, ls, os_):
    """Log-sum-exp merge of split states: M = max_s m_s, a_s = exp(m_s - M),
    out = sum_s a_s o_s / sum_s a_s l_s, lse = M + log(sum_s a_s l_s)."""
    ms = np.stack(ms)            # [S, H]
    ls = np.stack(ls)
    os_ = np.stack(os_)          # [S, H, DV]
    M = ms.max(axis=0)
    Msafe = np.where(np.isfinite(M), M, 0.0)
    a = np.where(np.isfinite(ms), np.exp(ms - Msafe[None, :]), 0.0)
    L = (a * ls).sum(axis=0)
    O = (a[:, :, None] * os_).sum(axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        out = np.where(L[:, None] > 0, O / np.where(L > 0, L, 1.0)[:, None], 0.0)
        lse = np.where(L > 0, Msafe + np.log(np.where(L > 0, L, 1.0)), -np.inf)
    return out, lse


def mla_sparse_attention_split(case: dict, physical: np.ndarray, n_splits: int, queries=None):
    """Same result as mla_sparse_attention, computed as n_splits contiguous chunks of the
    index list merged by combine_partials (the split-KV reduction)."""
    queries = np.arange(physical.shape[0]) if queries is None else np.asarray(queries)
    out = np.zeros((len(queries), H, DV))
    lse = np.full((len(queries), H), -np.inf)
    for i, q in enumerate(queries):
        parts = np.array_split(physical[i], n_splits)
        st = [mla_partials(case, p, q) for p in parts]
        out[i], lse[i] = combine_partials([s[0] for s in st], [s[1] for s in st], [s[2] for s in st])
    return out, lse


# ----------------------------------------------------------------------------------
# the whole step

def decode_layer(case: dict, queries=None):
    """Indexer -> top-k -> page map -> MLA sparse attention for the chosen query rows.

    Returns dict(scores, logical, physical, out, lse), all fp64 / int64."""
    queries = np.arange(case["Bq"]) if queries is None else np.asarray(queries)
    scores = indexer_scores(case, queries)
    vis = visible_lengths(case)[queries]
    logical = topk_logical(scores, vis, case["top_k"])
    phys = np.empty_like(logical)
    for i, q in enumerate(queries):
        phys[i] = physical_slots(case["block_table"][q // case["n_q"]], logical[i])
    out, lse = mla_sparse_attention(case, phys, queries)
    return dict(scores=scores, logical=logical, physical=phys, out=out, lse=lse)


# ----------------------------------------------------------------------------------
# the step before the path: partial interleaved RoPE, fp8 quantise-and-append

ROPE_DIMS = 64


def rope_interleaved(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotates consecutive pairs (x[2i], x[2i+1]) of the last axis (n = 64 rope columns) by
    pos * base^(-2i / n): x'[2i] = x[2i] cos - x[2i+1] sin, x'[2i+1] = x[2i] sin + x[2i+1] cos.
    `pos` broadcasts against x's leading axes."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    theta = base ** (-2.0 * np.arange(n // 2) / n)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def new_token_positions(case: dict) -> np.ndarray:
    """Position of each query's new token: q_pos when given, else the row's last token."""
    if case.get("q_pos") is not None:
        return case["q_pos"].astype(np.int64)
    return np.repeat(case["seq_lens"].astype(np.int64) - 1, case["n_q"])


def physical_slots_rows(case: dict, rows: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Slot of token pos[i] of sequence rows[i]: table[row, pos // 64] * 64 + pos % 64."""
    bt = case["block_table"]
    return bt[rows, pos // PAGE].astype(np.int64) * PAGE + pos % PAGE


def rope_quantize_append(case: dict, new: dict, base: float = 10000.0) -> dict:
    """The step before the path for every query's new token. `new` holds the projected,
    pre-RoPE bf16 bit tensors idx_q [Bq, 64, 128], idx_k [Bq, 128], latent [Bq, 576] and
    optionally q_mla [Bq, 64, 576]. Returns
      q_codes [Bq, 64, 128] e4m3, q_scale [Bq, 64] f32   (the indexer queries);
      slots [Bq]                                          (where the new token's rows go);
      k_codes [Bq, 128], k_scale [Bq]                     (the index-cache rows);
      the latent rows in the case's format: latent_codes [Bq, 576] + latent_scales [Bq, 5]
        ("fp8"), latent_packed [Bq, 656] bytes ("fp8r") or latent_bf16 [Bq, 576] ("bf16");
      q_mla [Bq, 64, 576] bf16 bits with its rope columns rotated (when given)."""
    pos = new_token_positions(case)
    b = np.arange(case["Bq"]) // case["n_q"]
    R = ROPE_DIMS
    q = decode_bf16(new["idx_q"])
    q[..., :R] = rope_interleaved(q[..., :R], pos[:, None], base)
    q_codes, q_scale = quantize_e4m3(q)
    k = decode_bf16(new["idx_k"])
    k[..., :R] = rope_interleaved(k[..., :R], pos, base)
    k_codes, k_scale = quantize_e4m3(k)
    lat = decode_bf16(new["latent"])
    lat[..., DV:] = rope_interleaved(lat[..., DV:], pos, base)
    out = dict(q_codes=q_codes, q_scale=q_scale, slots=physical_slots_rows(case, b, pos),
               k_codes=k_codes, k_scale=k_scale)
    kvd = case["kv_dtype"]
    if kvd == "bf16":
        out["latent_bf16"] = encode_bf16(lat)
    else:
        groups = [(128 * g, 128 * g + 128) for g in range(4)] + [(DV, DK)]
        codes = np.zeros(lat.shape, dtype=np.uint8)
        scales = np.zeros((lat.shape[0], 5), dtype=np.float32)
        for g, (lo, hi) in enumerate(groups[:5 if kvd == "fp8" else 4]):
            codes[:, lo:hi], scales[:, g] = quantize_e4m3(lat[:, lo:hi])
        if kvd == "fp8":
            out["latent_codes"], out["latent_scales"] = codes, scales
        else:
            row = np.zeros((lat.shape[0], DV + 16 + 2 * (DK - DV)), dtype=np.uint8)
            row[:, :DV] = codes[:, :DV]
            row[:, DV:DV + 16] = scales[:, :4].astype("<f4").view(np.uint8).reshape(-1, 16)
            row[:, DV + 16:] = encode_bf16(lat[:, DV:]).astype("<u2").view(np.uint8).reshape(-1, 2 * (DK - DV))
            out["latent_packed"] = row
    if new.get("q_mla") is not None:
        qm = decode_bf16(new["q_mla"])
        qm[..., DV:] = rope_interleaved(qm[..., DV:], pos[:, None], base)
        out["q_mla"] = encode_bf16(qm)
    return out


# ----------------------------------------------------------------------------------
# token-sharded decode: one long sequence spread over several ranks, one exchange step
#
# The pages say only that the context reaches 1M tokens (Russian news item on colibri);
# how such a context is spread over GPUs is not on them. The plainest reading that keeps
# the step's result unchanged: each rank holds a contiguous range of every row's tokens,
# scores and ranks only its own tokens, and the ranks exchange their best candidates and
# then their attention states.

def shard_candidates(scores_row: np.ndarray, lo: int, hi: int, top_k: int):
    """One rank's local selection of one query row: the min(top_k, hi - lo) best of its
    tokens [lo, hi) (topk_logical on the slice), as (score, global token) pairs padded
    with (-inf, -1) to top_k entries."""
    local = topk_logical(scores_row[None, lo:hi], np.array([hi - lo]), top_k)[0]
    ok = local >= 0
    tok = np.where(ok, local + lo, -1)
    sc = np.where(ok, scores_row[np.maximum(tok, 0)], -np.inf)
    return sc, tok


def shard_global_select(cand_score: np.ndarray, cand_token: np.ndarray, top_k: int) -> np.ndarray:
    """Global selection from every rank's candidates (flattened): the min(top_k, #valid)
    best, descending score, ties to the lower global token; tokens -1 are padding."""
    ok = cand_token >= 0
    sc, tok = cand_score[ok], cand_token[ok]
    order = np.lexsort((tok, -sc))
    out = np.full(top_k, -1, dtype=np.int64)
    k = min(top_k, tok.size)
    out[:k] = tok[order[:k]]
    return out


def sharded_decode_layer(case: dict, bounds: np.ndarray, queries=None):
    """The decode step with every row's tokens spread over R ranks.

    bounds: int [B, R + 1], nondecreasing from 0 to seq_lens[b]; rank r holds tokens
    [bounds[b, r], bounds[b, r + 1]) of row b. Every query sees its whole row (no q_pos).
    Steps: (1) each rank scores its tokens (a token's score does not depend on where it
    is stored, so the scores are the whole row's, sliced); (2) each rank's local top-k
    as (score, global token) candidates; (3) the exchange: all ranks see all candidates;
    (4) the global selection among them; (5) each rank's attention state over the
    selected tokens it holds (mla_partials); (6) the log-sum-exp merge of the R states
    (combine_partials).
    Returns dict(logical [n, top_k] global tokens in descending-score order, physical,
    owner [n, top_k] rank of each selected token (-1 unused), out, lse)."""
    if case.get("q_pos") is not None:
        raise ValueError("the token-sharded step takes no causal positions")
    queries = np.arange(case["Bq"]) if queries is None else np.asarray(queries)
    bounds = np.asarray(bounds, dtype=np.int64)
    R = bounds.shape[1] - 1
    K = case["top_k"]
    scores = indexer_scores(case, queries)
    n = len(queries)
    logical = np.full((n, K), -1, dtype=np.int64)
    owner = np.full((n, K), -1, dtype=np.int64)
    out = np.zeros((n, H, DV))
    lse = np.full((n, H), -np.inf)
    for i, q in enumerate(queries):
        b = q // case["n_q"]
        cands = [shard_candidates(scores[i], bounds[b, r], bounds[b, r + 1], K) for r in range(R)]
        sel = shard_global_select(np.concatenate([c[0] for c in cands]), np.concatenate([c[1] for c in cands]), K)
        logical[i] = sel
        ok = sel >= 0
        owner[i][ok] = np.searchsorted(bounds[b], sel[ok], side="right") - 1
        states = []
        for r in range(R):
            mine = sel[ok & (owner[i] == r)]
            states.append(mla_partials(case, physical_slots(case["block_table"][b], mine), q))
        out[i], lse[i] = combine_partials([s[0] for s in states], [s[1] for s in states], [s[2] for s in states])
    physical = np.stack([physical_slots(case["block_table"][q // case["n_q"]], logical[i])
                         for i, q in enumerate(queries)])
    return dict(scores=scores, logical=logical, physical=physical, owner=owner, out=out, lse=lse)
