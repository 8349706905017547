"""Runs the CUDA path (through the C ABI binding) on a generated case; GPU tests only."""
import numpy as np
import torch

import deepseek_sparse_attention_head_b200 as dsa
from dsa_inputs import to_torch, DV, H


class GpuCase:
    def __init__(self, case, device="cuda"):
        self.case = case
        self.t = to_torch(case, device)
        self.device = device
        self.paging = dsa.Paging(self.t["seq_lens"], self.t["block_table"], case["num_pages"], case["n_q"],
                                 self.t["q_pos"])
        self.Bq = case["Bq"]
        self.top_k = case["top_k"]

    def _ws(self, nbytes):
        return dsa.alloc_workspace(nbytes, self.device)

    def out_dtype(self):
        return torch.float32 if self.case["out_dtype"] == "fp32" else torch.bfloat16

    def indexer(self, L_max=None):
        L_max = L_max or self.paging.L_layer
        scores = torch.full((self.Bq, L_max), float("nan"), dtype=torch.float32, device=self.device)
        ws = self._ws(dsa.dsa_workspace_size(self.paging, L_max, 0, dsa.DSA_OP_INDEXER))
        t = self.t
        dsa.dsa_indexer_scores(self.paging, t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"],
                               scores, ws)
        err = dsa.dsa_get_error(ws)
        return scores, err

    def topk(self, scores: torch.Tensor, top_k=None):
        K = top_k or self.top_k
        lo = torch.full((self.Bq, K), -7, dtype=torch.int32, device=self.device)
        ph = torch.full((self.Bq, K), -7, dtype=torch.int32, device=self.device)
        ws = self._ws(dsa.dsa_workspace_size(self.paging, scores.shape[1], K, dsa.DSA_OP_TOPK))
        dsa.dsa_topk_pagemap(self.paging, scores, K, lo, ph, ws)
        err = dsa.dsa_get_error(ws)
        return lo.cpu().numpy(), ph.cpu().numpy(), err

    def pagemap(self, logical: np.ndarray):
        lo = torch.from_numpy(np.ascontiguousarray(logical.astype(np.int32))).to(self.device)
        ph = torch.full_like(lo, -7)
        ws = self._ws(dsa.dsa_workspace_size(self.paging, 0, lo.shape[1], dsa.DSA_OP_PAGEMAP))
        dsa.dsa_pagemap(self.paging, lo, ph, ws)
        err = dsa.dsa_get_error(ws)
        return ph.cpu().numpy(), err

    def mla(self, physical: np.ndarray):
        ph = torch.from_numpy(np.ascontiguousarray(physical.astype(np.int32))).to(self.device)
        Bq = ph.shape[0]
        out = torch.full((Bq, H, DV), float("nan"), dtype=self.out_dtype(), device=self.device)
        lse = torch.full((Bq, H), float("nan"), dtype=torch.float32, device=self.device)
        ws = self._ws(dsa.mla_workspace_size(Bq, ph.shape[1]))
        t = self.t
        dsa.mla_sparse_decode(t["q_mla"][:Bq].contiguous(), t["kv_cache"], t["kv_scale"], ph,
                              self.case["softmax_scale"], out, lse, ws)
        err = dsa.dsa_get_error(ws)
        return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64), err

    def layer(self, stream=None):
        t = self.t
        out = torch.full((self.Bq, H, DV), float("nan"), dtype=self.out_dtype(), device=self.device)
        lse = torch.full((self.Bq, H), float("nan"), dtype=torch.float32, device=self.device)
        lo = torch.full((self.Bq, self.top_k), -7, dtype=torch.int32, device=self.device)
        ph = torch.full((self.Bq, self.top_k), -7, dtype=torch.int32, device=self.device)
        ws = self._ws(dsa.dsa_workspace_size(self.paging, 0, self.top_k, dsa.DSA_OP_LAYER))
        dsa.dsa_decode_layer(self.paging, t["q_idx"], t["q_idx_scale"], t["head_w"], t["k_cache"], t["k_scale"],
                             t["q_mla"], t["kv_cache"], t["kv_scale"], self.top_k, self.case["softmax_scale"], out,
                             ws, lse=lse, logical_out=lo, physical_out=ph, stream=stream)
        err = dsa.dsa_get_error(ws)
        return dict(out=out.float().cpu().numpy().astype(np.float64), lse=lse.cpu().numpy().astype(np.float64),
                    logical=lo.cpu().numpy(), physical=ph.cpu().numpy(), err=err)
