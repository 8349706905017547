"""The token-sharded step's host logic on CPU: two or three gloo ranks run TokenShardedDecode.step
with its real exchanges (all-gathers over the process group) while the library calls it
makes are replaced, in the child processes of this test only, by fp64 oracle stand-ins of
each stage. The merged output must be the oracle's sharded (and unsharded) step on every
rank: the buffers are exchanged in rank order, each rank passes its own rank, offsets and
slots, and the phases run in the right order."""
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_stages(case, bounds, rank):
    """Stand-ins of the library calls TokenShardedDecode makes, for rank `rank`."""
    import oracle
    full_scores = oracle.indexer_scores(case)
    n_q, K = case["n_q"], case["top_k"]

    def indexer(paging, q_idx, q_scale, head_w, k_cache, k_scale, scores, ws, stream=None):
        for q in range(case["Bq"]):
            b = q // n_q
            lo, hi = bounds[b, rank], bounds[b, rank + 1]
            scores[q, :hi - lo] = torch.from_numpy(full_scores[q, lo:hi])

    def local_topk(paging, scores, top_k, token_offset, cand_score, cand_token, ws, stream=None):
        for q in range(case["Bq"]):
            b = q // n_q
            n = int(bounds[b, rank + 1] - bounds[b, rank])
            sc, tok = oracle.shard_candidates(scores[q].double().numpy(), 0, n, top_k)
            cand_score[q] = torch.from_numpy(sc)
            cand_token[q] = torch.from_numpy(np.where(tok >= 0, tok + int(token_offset[b]), -1))

    def select(paging, n_ranks, rk, all_score, all_token, top_k, token_offset, physical, ws, logical_out=None,
               stream=None):
        assert rk == rank and n_ranks == bounds.shape[1] - 1
        for q in range(case["Bq"]):
            b = q // n_q
            sel = oracle.shard_global_select(all_score[:, q].double().numpy().ravel(),
                                             all_token[:, q].numpy().ravel().astype(np.int64), top_k)
            mine = sel[np.isin(sel, all_token[rk, q].numpy()) & (sel >= 0)]
            ph = np.full(top_k, -1, dtype=np.int64)
            ph[:mine.size] = oracle.physical_slots(case["block_table"][b], mine)
            physical[q] = torch.from_numpy(ph)
            if logical_out is not None:
                logical_out[q] = torch.from_numpy(sel)

    def mla(q_mla, kv_cache, kv_scale, physical, softmax_scale, out, lse, ws, stream=None):
        for q in range(case["Bq"]):
            m, l, o = oracle.mla_partials(case, physical[q].numpy().astype(np.int64), q)
            ok = l > 0
            out[q] = torch.from_numpy(np.where(ok[:, None], o / np.where(ok, l, 1.0)[:, None], 0.0))
            lse[q] = torch.from_numpy(np.where(ok, m + np.log(np.where(ok, l, 1.0)), -np.inf))

    def merge(all_out, all_lse, out, lse=None, stream=None):
        R = all_out.shape[0]
        for q in range(all_out.shape[1]):
            o, ls = oracle.combine_partials(list(all_lse[:, q].double().numpy()), [np.ones(64)] * R,
                                            list(all_out[:, q].double().numpy()))
            out[q] = torch.from_numpy(o)
            if lse is not None:
                lse[q] = torch.from_numpy(ls)

    return dict(dsa_indexer_scores=indexer, dsa_shard_local_topk=local_topk, dsa_shard_select=select,
                mla_sparse_decode=mla, dsa_shard_merge=merge)


def _rank(rank, world, port, bounds, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from dsa_inputs import CaseSpec, generate
    from deepseek_sparse_attention_head_b200 import sharded
    case = generate(CaseSpec("gloo", (300, 130), top_k=64, seed=61, kv_dtype="fp8"))
    for name, fn in _oracle_stages(case, bounds, rank).items():
        setattr(sharded, name, fn)
    sharded.dsa_workspace_size = lambda *a: 256
    sharded.mla_workspace_size = lambda *a: 256
    sharded.alloc_workspace = lambda n, dev=None: torch.zeros(n, dtype=torch.uint8)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    lens = bounds[:, rank + 1] - bounds[:, rank]
    paging = SimpleNamespace(q_pos=None, Bq=case["Bq"], L_layer=int(max(64, ((lens.max() + 63) // 64) * 64)))
    offset = torch.from_numpy(bounds[:, rank].astype(np.int32))
    dec = sharded.TokenShardedDecode(paging, offset, case["top_k"], case["softmax_scale"], rank, world,
                                     device="cpu")
    res = torch.empty(case["Bq"], 64, 512)
    lse = torch.empty(case["Bq"], 64)
    logical = torch.full((case["Bq"], case["top_k"]), -7, dtype=torch.int32)
    none = torch.empty(0)
    dec.step(none, none, none, none, none, none, none, none, res, lse, logical_out=logical)
    out[rank] = (res.numpy().copy(), lse.numpy().copy(), logical.numpy().copy())
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [
    [[0, 192, 300], [0, 0, 130]],                  # two ranks; row 1 lives on rank 1 only
    [[0, 64, 256, 300], [0, 128, 128, 130]],       # three ranks; rank 1 holds none of row 1
], ids=["two_ranks", "three_ranks"])
def test_gloo_ranks_merge_to_the_unsharded_step(bounds):
    import oracle
    from dsa_inputs import CaseSpec, generate
    bounds = np.array(bounds, dtype=np.int64)
    world = bounds.shape[1] - 1
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, _free_port(), bounds, out), nprocs=world, join=True)
        res = dict(out)
    case = generate(CaseSpec("gloo", (300, 130), top_k=64, seed=61, kv_dtype="fp8"))
    ref = oracle.sharded_decode_layer(case, bounds)
    unsharded = oracle.decode_layer(case)
    assert np.array_equal(ref["logical"], unsharded["logical"])
    for r in range(world):
        o, lse, logical = res[r]
        assert np.array_equal(logical.astype(np.int64), ref["logical"])
        assert np.allclose(o, ref["out"], rtol=1e-5, atol=1e-6)
        assert np.allclose(lse, ref["lse"], rtol=1e-6)
    for r in range(1, world):
        assert np.array_equal(res[r][0], res[0][0])
