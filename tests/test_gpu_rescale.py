"""MLA sparse decode on selections whose logits rise from tile to tile, against the oracle.

The decode kernel keeps a lazy running maximum per head: it rescales the running sum and
the accumulated output in tensor memory only when a later 64-row tile's maximum logit
exceeds the running one by more than a threshold, and it rescales again when a later
tile's fp8 scale exponents grow past the reference it normalised earlier tiles with.
Seeded generator data almost never triggers either. These cases do, on purpose: row h of
tile t is aimed at head h's query with a strength growing with t
(dsa_inputs.rising_selection), so every head's maximum climbs by a fixed number of log2
units per tile while the rows keep the generator's magnitudes, and the fp8 scales grow
with the rows. A CPU check on the oracle's fp64 logits asserts the rise for every head,
so each case is known to cross the threshold before the GPU result is compared element
by element with the oracle (MLA sparse decode: "GLM-52 Runs on RTX 4090", kernel list
item 3).
"""
import functools
import math

import numpy as np
import pytest

import oracle
from dsa_inputs import CaseSpec, generate, rising_selection
from tests.compare import check_attention, fp8_lse_bound

TILE = 64
LOG2E = 1.0 / math.log(2.0)

# (name, kv dtype, queries, tiles per query, designed climb per tile, minimum climb asserted
# for every head, both in log2 units)
CASES = [
    # 150 queries: one KV split each, so a whole 4-tile list goes through one CTA
    ("fp8_unsplit_steep", "fp8", 150, 4, 12.0, 8.5),
    ("bf16_unsplit_steep", "bf16", 150, 4, 12.0, 8.5),
    # 40 queries: two splits of two tiles, each split rescales once
    ("fp8_split_steep", "fp8", 40, 4, 12.0, 8.5),
    ("bf16_split_steep", "bf16", 40, 4, 12.0, 8.5),
    # a gentler climb (a few log2 units per tile) over more tiles
    ("fp8_unsplit_gentle", "fp8", 150, 6, 6.0, 3.2),
    ("fp8_split_gentle", "fp8", 50, 6, 6.0, 3.2),
    # packed 656-byte rows: the scales grow with the rows, the rope stays bf16
    ("fp8r_split_steep", "fp8r", 40, 4, 12.0, 8.5),
]


@functools.lru_cache(maxsize=None)
def _case(name):
    _, kv, nq, tiles, climb, _ = next(c for c in CASES if c[0] == name)
    spec = CaseSpec(f"rise_{name}", (tiles * TILE + 37,) * nq, top_k=tiles * TILE,
                    idx_dtype="bf16" if kv == "bf16" else "fp8", kv_dtype=kv,
                    out_dtype="fp32" if kv == "bf16" else "bf16", n_planted=0, seed=61)
    case, phys = rising_selection(generate(spec), tiles, climb, seed=7, noise_std=0.15)
    return case, phys


def _tile_maxima(case, phys, q):
    """fp64 logits of query q in log2 units, reduced to the per-head maximum of every tile."""
    qm = oracle.decode_bf16(case["q_mla"][q])
    kv = oracle.dequant_latent_rows(case, phys[q].astype(np.int64))
    z = case["softmax_scale"] * (qm @ kv.T) * LOG2E          # [64, n]
    return z.reshape(64, -1, TILE).max(axis=2)               # [64, tiles]


@pytest.mark.parametrize("name", [c[0] for c in CASES])
def test_rising_logits_cross_the_rescale_threshold(name):
    """CPU side: every head's tile maximum climbs past the previous tiles' by the stated
    margin, and (fp8) later tiles carry larger scale exponents than the first."""
    _, kv, nq, tiles, _, rise = next(c for c in CASES if c[0] == name)
    case, phys = _case(name)
    for q in range(case["Bq"]):
        tm = _tile_maxima(case, phys, q)
        prev = np.maximum.accumulate(tm, axis=1)
        climb = tm[:, 1:] - prev[:, :-1]
        assert climb.min() >= rise, f"query {q}: smallest climb {climb.min():.2f} < {rise}"
        if kv == "fp8":
            e = np.floor(np.log2(case["kv_scale"][phys[q].astype(np.int64)]))   # [n, 5]
            per_tile = e.reshape(tiles, TILE, 5).max(axis=(1, 2))
            assert per_tile[-1] > per_tile[0]


@pytest.mark.gpu
@pytest.mark.parametrize("name", [c[0] for c in CASES])
def test_mla_matches_oracle_on_rising_logits(name):
    import deepseek_sparse_attention_head_b200 as dsa
    from tests.gpu_path import GpuCase
    case, phys = _case(name)
    splits = dsa.mla_num_splits(case["Bq"], case["top_k"])
    assert (splits == 1) == ("unsplit" in name), "the case should exercise the intended split layout"
    out, lse, err = GpuCase(case).mla(phys)
    assert err == 0
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys.astype(np.int64))
    bound = fp8_lse_bound(case, phys) if case["kv_dtype"] != "bf16" else None
    check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"], lse_bound=bound)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["fp8_split_gentle", "bf16_split_steep"])
def test_mla_matches_oracle_on_falling_logits(name):
    """The same lists in reverse: the first tile holds the maximum, nothing rescales, and
    later tiles' weights underflow towards zero."""
    from tests.gpu_path import GpuCase
    case, phys = _case(name)
    rev = np.ascontiguousarray(phys[:, ::-1])
    out, lse, err = GpuCase(case).mla(rev)
    assert err == 0
    ref_out, ref_lse = oracle.mla_sparse_attention(case, rev.astype(np.int64))
    bound = fp8_lse_bound(case, rev) if case["kv_dtype"] != "bf16" else None
    check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"], lse_bound=bound)
