"""Token-sharded decode of long sequences over torch.distributed ranks (one GPU each).

Every row's tokens are spread over the R ranks of a process group in contiguous,
page-aligned ranges; each rank holds its range in its own paged caches. One decode step
runs the library's stages on every rank with two exchanges between them (include/dsa.h,
"Token-sharded decode"):

    indexer scores -> local top-k as (score, global token) candidates
    -> all-gather of the candidates -> global selection, this rank's winners as slots
    -> MLA sparse decode over them (fp32 state) -> all-gather of the states
    -> log-sum-exp merge

The exchanges are NCCL all-gathers of a few KB (candidates) and Bq x 128 KB (states);
every step of the arithmetic runs in the library's kernels. The result is the unsharded
step's, whatever the split.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch

from . import (DIM_V, HEADS, PAGE_SIZE, DSA_OP_INDEXER, DSA_OP_SHARD_LOCAL, DSA_OP_SHARD_SELECT, Paging,
               alloc_workspace, dsa_indexer_scores, dsa_shard_local_topk, dsa_shard_merge, dsa_shard_select,
               dsa_workspace_size, mla_sparse_decode, mla_workspace_size)


def shard_bounds(seq_len: int, n_ranks: int, page: int = PAGE_SIZE) -> List[int]:
    """Token boundaries [b_0 = 0, ..., b_R = seq_len] of one row over n_ranks ranks: each
    rank takes the same whole number of pages (the last ones may hold fewer tokens or none)."""
    if n_ranks < 1 or seq_len < 0:
        raise ValueError("n_ranks >= 1 and seq_len >= 0 required")
    pages = (seq_len + page - 1) // page
    per = (pages + n_ranks - 1) // n_ranks
    return [min(seq_len, r * per * page) for r in range(n_ranks + 1)]


def _all_gather(dst: torch.Tensor, src: torch.Tensor, group) -> None:
    # dst [R, *src.shape] seen as the rank-major concatenation [R * src.shape[0], ...]
    torch.distributed.all_gather_into_tensor(dst.view(-1, *src.shape[1:]), src, group=group)


class TokenShardedDecode:
    """One rank's share of the token-sharded decode step.

    paging        this rank's local paging (its seq_lens are its local lengths; q_pos None)
    token_offset  device int32 [B]: global token index of each row's first local token
    The buffers for both exchanges are allocated once; `step` runs one decode step.
    `gather(dst, src)` fills dst [R, ...] with every rank's src in rank order (default: an
    all-gather over `group`)."""

    def __init__(self, paging: Paging, token_offset: torch.Tensor, top_k: int, softmax_scale: float,
                 rank: int, n_ranks: int, group=None, gather: Optional[Callable] = None, device=None):
        if paging.q_pos is not None:
            raise ValueError("the token-sharded step takes no causal positions (q_pos must be None)")
        self.paging, self.token_offset = paging, token_offset
        self.top_k, self.softmax_scale = int(top_k), float(softmax_scale)
        self.rank, self.n_ranks = int(rank), int(n_ranks)
        self.group = group
        self._gather = gather or (lambda dst, src: _all_gather(dst, src, group))
        dev = device or token_offset.device
        Bq, K, R = paging.Bq, self.top_k, self.n_ranks
        self.L_max = paging.L_layer
        self.scores = torch.empty(Bq, self.L_max, dtype=torch.float32, device=dev)
        self.cand_score = torch.empty(Bq, K, dtype=torch.float32, device=dev)
        self.cand_token = torch.empty(Bq, K, dtype=torch.int32, device=dev)
        self.all_score = torch.empty(R, Bq, K, dtype=torch.float32, device=dev)
        self.all_token = torch.empty(R, Bq, K, dtype=torch.int32, device=dev)
        self.physical = torch.empty(Bq, K, dtype=torch.int32, device=dev)
        self.state_out = torch.empty(Bq, HEADS, DIM_V, dtype=torch.float32, device=dev)
        self.state_lse = torch.empty(Bq, HEADS, dtype=torch.float32, device=dev)
        self.all_out = torch.empty(R, Bq, HEADS, DIM_V, dtype=torch.float32, device=dev)
        self.all_lse = torch.empty(R, Bq, HEADS, dtype=torch.float32, device=dev)
        self.ws_index = alloc_workspace(dsa_workspace_size(paging, self.L_max, 0, DSA_OP_INDEXER), dev)
        self.ws_local = alloc_workspace(dsa_workspace_size(paging, self.L_max, K, DSA_OP_SHARD_LOCAL), dev)
        self.ws_select = alloc_workspace(dsa_workspace_size(paging, 0, K, DSA_OP_SHARD_SELECT), dev)
        self.ws_mla = alloc_workspace(mla_workspace_size(Bq, K), dev)

    # the phases of one step, in order (each rank runs the same sequence)
    def local_phase(self, q_idx, q_scale, head_w, k_cache, k_scale, stream=None):
        dsa_indexer_scores(self.paging, q_idx, q_scale, head_w, k_cache, k_scale, self.scores, self.ws_index,
                           stream=stream)
        dsa_shard_local_topk(self.paging, self.scores, self.top_k, self.token_offset, self.cand_score,
                             self.cand_token, self.ws_local, stream=stream)

    def exchange_candidates(self):
        self._gather(self.all_score, self.cand_score)
        self._gather(self.all_token, self.cand_token)

    def select_phase(self, logical_out=None, stream=None):
        dsa_shard_select(self.paging, self.n_ranks, self.rank, self.all_score, self.all_token, self.top_k,
                         self.token_offset, self.physical, self.ws_select, logical_out=logical_out, stream=stream)

    def attend_phase(self, q_mla, kv_cache, kv_scale, stream=None):
        mla_sparse_decode(q_mla, kv_cache, kv_scale, self.physical, self.softmax_scale, self.state_out,
                          self.state_lse, self.ws_mla, stream=stream)

    def exchange_states(self):
        self._gather(self.all_out, self.state_out)
        self._gather(self.all_lse, self.state_lse)

    def merge_phase(self, out, lse=None, stream=None):
        dsa_shard_merge(self.all_out, self.all_lse, out, lse, stream=stream)

    def step(self, q_idx, q_scale, head_w, k_cache, k_scale, q_mla, kv_cache, kv_scale, out, lse=None,
             logical_out=None):
        """One decode step on the current stream: out [Bq, 64, 512] (bf16 or fp32) and
        lse [Bq, 64] are the unsharded step's; logical_out [Bq, top_k] int32 (optional)
        receives the global selection as global tokens."""
        self.local_phase(q_idx, q_scale, head_w, k_cache, k_scale)
        self.exchange_candidates()
        self.select_phase(logical_out)
        self.attend_phase(q_mla, kv_cache, kv_scale)
        self.exchange_states()
        self.merge_phase(out, lse)
        return out
