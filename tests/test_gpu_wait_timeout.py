"""Bounded waits of the fp8-cache MLA decode kernel, made to run out on purpose.

Every wait inside the kernels is bounded; when one runs out, the kernel raises a shared
abort flag so the other warp roles stop waiting, drains its own copies and tensor-core
operations, frees its tensor memory, leaves empty split partials and records
DSA_ERR_TIMEOUT. The test hook dsa_test_set_wait_hooks makes the softmax warps wait on a
barrier nothing arrives on, with a bound of about a millisecond, so that whole unwind
runs without any fault: the call must return, report the timeout through the workspace,
and leave the context and the workspace usable for the next, normal call, whose result
is checked against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from dsa_inputs import CaseSpec, DV, H, generate, to_torch
from tests.compare import check_attention

pytestmark = pytest.mark.gpu

SHORT = 2_000_000    # SM cycles: about a millisecond


def _selection(case, seed):
    rng = np.random.default_rng(seed)
    vis = oracle.visible_lengths(case)
    K = case["top_k"]
    logical = np.full((case["Bq"], K), -1, dtype=np.int64)
    for q in range(case["Bq"]):
        n = min(K, int(vis[q]))
        logical[q, :n] = rng.choice(int(vis[q]), size=n, replace=False)
    return oracle.pagemap(case, logical).astype(np.int32)


# several KV splits per query merged by the combine kernel / two splits merged inside the
# kernel by a CTA pair / one split each
@pytest.mark.parametrize("nq,splits", [(3, "many"), (64, "pair"), (160, "one")])
def test_stalled_wait_times_out_and_the_next_call_is_correct(nq, splits):
    import deepseek_sparse_attention_head_b200 as dsa
    case = generate(CaseSpec(f"timeout_{nq}", (700,) * nq, top_k=512, n_planted=0, seed=71))
    t = to_torch(case, "cuda")
    phys = torch.from_numpy(_selection(case, 3)).cuda()
    Bq = case["Bq"]
    n = dsa.mla_num_splits(Bq, case["top_k"])
    assert {"many": n > 2, "pair": n == 2, "one": n == 1}[splits]
    ws = dsa.alloc_workspace(dsa.mla_workspace_size(Bq, case["top_k"]))
    out = torch.full((Bq, H, DV), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((Bq, H), float("nan"), dtype=torch.float32, device="cuda")

    def call():
        dsa.mla_sparse_decode(t["q_mla"], t["kv_cache"], t["kv_scale"], phys, case["softmax_scale"], out, lse, ws)

    try:
        dsa.dsa_test_set_wait_hooks(SHORT, stall=True)
        call()
    finally:
        dsa.dsa_test_set_wait_hooks(0, stall=False)
    assert dsa.dsa_get_error(ws) == dsa.DSA_ERR_TIMEOUT
    # the context is intact and the same workspace serves the next call
    call()
    assert dsa.dsa_get_error(ws) == dsa.DSA_OK
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys.cpu().numpy().astype(np.int64))
    check_attention(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ref_out,
                    ref_lse, case["kv_dtype"])


def test_short_bound_alone_does_not_break_a_normal_call():
    """A bound far above the kernel's real waits (tens of milliseconds) changes nothing."""
    import deepseek_sparse_attention_head_b200 as dsa
    case = generate(CaseSpec("timeout_long", (900,) * 5, top_k=256, n_planted=0, seed=72))
    t = to_torch(case, "cuda")
    phys = torch.from_numpy(_selection(case, 4)).cuda()
    ws = dsa.alloc_workspace(dsa.mla_workspace_size(case["Bq"], case["top_k"]))
    out = torch.full((case["Bq"], H, DV), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((case["Bq"], H), float("nan"), dtype=torch.float32, device="cuda")
    try:
        dsa.dsa_test_set_wait_hooks(100_000_000, stall=False)
        dsa.mla_sparse_decode(t["q_mla"], t["kv_cache"], t["kv_scale"], phys, case["softmax_scale"], out, lse, ws)
    finally:
        dsa.dsa_test_set_wait_hooks(0, stall=False)
    assert dsa.dsa_get_error(ws) == dsa.DSA_OK
    ref_out, ref_lse = oracle.mla_sparse_attention(case, phys.cpu().numpy().astype(np.int64))
    check_attention(out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), ref_out,
                    ref_lse, case["kv_dtype"])
