"""mla_sparse_decode_noalloc against mla_sparse_decode and the fp64 oracle, through the C ABI.

The no-allocation entry point serves callers that cannot allocate device memory (a
plugin inside an engine that owns all of the GPU's memory, or a loop that must not call
cudaMalloc/cudaFree): its split partials live in an array the library defines in device
memory, shared by every call on a device. These tests run two different calls in a row,
so the second one starts on the scratch contents the first left behind, and compare each
with the workspace entry point on the same inputs and with the oracle's attention on the
same selection. This file sorts last so that a stop-at-first-failure run has finished
every other test before it.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_inputs import CaseSpec, DV, H, generate
from tests.compare import check_attention

pytestmark = pytest.mark.gpu

CASES = [
    # fp8 latent cache, few queries: many KV splits, so the partials are in use
    CaseSpec("noalloc_fp8", (900, 3000, 61), top_k=256, seed=51),
    # bf16 cache, fp32 output, more queries (four splits of two tiles): another split layout
    CaseSpec("noalloc_bf16", tuple(range(50, 50 + 29 * 71, 71)), top_k=512, idx_dtype="bf16", kv_dtype="bf16",
             out_dtype="fp32", seed=52),
]


def _selection(case, seed):
    """A seeded random selection of visible tokens per query (padded with -1), as slots."""
    rng = np.random.default_rng(seed)
    vis = oracle.visible_lengths(case)
    K = case["top_k"]
    logical = np.full((case["Bq"], K), -1, dtype=np.int64)
    for q in range(case["Bq"]):
        n = min(K, int(vis[q]))
        logical[q, :n] = rng.choice(int(vis[q]), size=n, replace=False)
    return oracle.pagemap(case, logical).astype(np.int32)


def _run(dsa, t, case, physical, noalloc):
    Bq = case["Bq"]
    out_dtype = torch.float32 if case["out_dtype"] == "fp32" else torch.bfloat16
    out = torch.full((Bq, H, DV), float("nan"), dtype=out_dtype, device="cuda")
    lse = torch.full((Bq, H), float("nan"), dtype=torch.float32, device="cuda")
    if noalloc:
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        dsa.mla_sparse_decode_noalloc(t["q_mla"], t["kv_cache"], t["kv_scale"], physical, case["softmax_scale"], out,
                                      lse, status=status)
        err = dsa.dsa_get_error(status)
    else:
        ws = dsa.alloc_workspace(dsa.mla_workspace_size(Bq, physical.shape[1]))
        dsa.mla_sparse_decode(t["q_mla"], t["kv_cache"], t["kv_scale"], physical, case["softmax_scale"], out, lse,
                              ws)
        err = dsa.dsa_get_error(ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), err


def test_noalloc_matches_workspace_entry_on_consecutive_calls():
    import deepseek_sparse_attention_head_b200 as dsa
    from dsa_inputs import to_torch

    prepared = []
    for i, spec in enumerate(CASES):
        case = generate(spec)
        t = to_torch(case, "cuda")
        physical = torch.from_numpy(_selection(case, 100 + i)).cuda()
        assert dsa.mla_num_splits(case["Bq"], case["top_k"]) > 1, "the case should exercise the partials"
        prepared.append((case, t, physical))

    # two different calls in a row, then the first again on what the second left behind
    for case, t, physical in prepared + prepared[:1]:
        out, lse, err = _run(dsa, t, case, physical, noalloc=True)
        assert err == dsa.DSA_OK, dsa.dsa_status_string(err)
        ref_out, ref_lse, ref_err = _run(dsa, t, case, physical, noalloc=False)
        assert ref_err == dsa.DSA_OK
        check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"])
        o_out, o_lse = oracle.mla_sparse_attention(case, physical.cpu().numpy().astype(np.int64))
        check_attention(out, lse, o_out, o_lse, case["kv_dtype"])


def test_noalloc_reports_device_errors_through_status():
    """A slot past the cache is skipped and reported, as by the workspace entry point."""
    import deepseek_sparse_attention_head_b200 as dsa
    from dsa_inputs import to_torch

    case = generate(CASES[0])
    t = to_torch(case, "cuda")
    sel = _selection(case, 7)
    sel[0, 3] = case["kv_cache"].shape[0] + 5          # one slot beyond the cache
    physical = torch.from_numpy(sel).cuda()
    out, lse, err = _run(dsa, t, case, physical, noalloc=True)
    assert err == dsa.DSA_ERR_DEVICE_BOUNDS
    ref_out, ref_lse, ref_err = _run(dsa, t, case, physical, noalloc=False)
    assert ref_err == dsa.DSA_ERR_DEVICE_BOUNDS
    check_attention(out, lse, ref_out, ref_lse, case["kv_dtype"])
    # the next call starts with clear error words
    out, lse, err = _run(dsa, t, case, torch.from_numpy(_selection(case, 8)).cuda(), noalloc=True)
    assert err == dsa.DSA_OK
