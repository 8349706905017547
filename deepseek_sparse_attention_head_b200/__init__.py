"""B200 (sm_100a) DeepSeek-Sparse-Attention decode step.

Thin ctypes binding of libdsa_b200.so (C ABI in include/dsa.h): every function here
only checks and marshals torch tensors into pointers and sizes; every step of the
computation runs in the library's CUDA kernels. Importing this package fails when
the library has not been built (python -m deepseek_sparse_attention_head_b200.build).

The three stages ("GLM-52 Runs on RTX 4090", kernel list; glm-5.2-4090 README, how it
works): dsa_indexer_scores (lightning indexer), dsa_topk_pagemap (top-k + fused page
mapping), mla_sparse_decode (MLA sparse decode with split-KV combine), and the fused
dsa_decode_layer.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa_b200.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA, DSA_ERR_WORKSPACE, \
    DSA_ERR_DEVICE_BOUNDS, DSA_ERR_TIMEOUT = range(7)
DSA_BF16, DSA_FP8_E4M3, DSA_FP32, DSA_FP8_E4M3_ROPE_BF16 = range(4)
DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_PAGEMAP, DSA_OP_LAYER, DSA_OP_SHARD_LOCAL, DSA_OP_SHARD_SELECT = range(6)

PAGE_SIZE = 64
HEADS = 64
DIM_INDEX = 128
DIM_K = 576
DIM_V = 512


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dsa_status_string(status)} (status {status})")


class _Paging(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32),
        ("n_q", ctypes.c_int32),
        ("seq_lens", ctypes.c_void_p),
        ("q_pos", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("max_pages_per_seq", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
    ]


_vp, _i32, _i64, _sz, _f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_PP = ctypes.POINTER(_Paging)

_SIGNATURES = {
    "dsa_indexer_scores": (_i32, [_PP, _vp, _i32, _vp, _vp, _vp, _i32, _vp, _vp, _i64, _vp, _sz, _vp]),
    "dsa_topk_pagemap": (_i32, [_PP, _vp, _i64, _i32, _vp, _vp, _vp, _sz, _vp]),
    "dsa_pagemap": (_i32, [_PP, _vp, _i32, _vp, _vp, _sz, _vp]),
    "mla_sparse_decode": (_i32, [_i32, _vp, _vp, _i32, _vp, _i64, _vp, _i32, _f32, _vp, _i32, _vp, _vp, _sz, _vp]),
    "mla_sparse_decode_noalloc": (_i32, [_i32, _vp, _vp, _i32, _vp, _i64, _vp, _i32, _f32, _vp, _i32, _vp, _vp,
                                         _vp]),
    "dsa_decode_layer": (_i32, [_PP, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _f32, _vp, _i32,
                                _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_rope_quantize_append": (_i32, [_PP, _vp, _vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp,
                                        _vp]),
    "dsa_shard_local_topk": (_i32, [_PP, _vp, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_shard_select": (_i32, [_PP, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dsa_shard_merge": (_i32, [_i32, _i32, _vp, _vp, _vp, _i32, _vp, _vp]),
    "dsa_workspace_size": (_sz, [_PP, _i64, _i32, _i32]),
    "mla_workspace_size": (_sz, [_i32, _i32]),
    "mla_num_splits": (_i32, [_i32, _i32]),
    "dsa_get_error": (_i32, [_vp, _vp]),
    "dsa_status_string": (ctypes.c_char_p, [_i32]),
    "dsa_last_launch_count": (_i32, []),
    "dsa_test_set_wait_hooks": (_i32, [_i64, _i32]),
}


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python deepseek_sparse_attention_head_b200/build.py` (needs nvcc)")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
LIBRARY_PATH = _LIB_PATH


def exported_symbols():
    return sorted(_SIGNATURES)


# ---------------------------------------------------------------------- helpers

def _kv_code(t: torch.Tensor) -> int:
    """Latent-cache layout code: uint8 rows 656 bytes wide are the packed layout (E4M3 codes,
    four fp32 scales, bf16 rope); other caches follow their element type."""
    if t.dtype == torch.uint8 and t.dim() >= 1 and t.shape[-1] == 656:
        return DSA_FP8_E4M3_ROPE_BF16
    return _dtype_code(t)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DSA_BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return DSA_FP8_E4M3
    if t.dtype == torch.float32:
        return DSA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to the DSA library must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the DSA library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != DSA_OK:
        raise DsaError(status, where)


def dsa_status_string(status: int) -> str:
    return _lib.dsa_status_string(status).decode()


def dsa_last_launch_count() -> int:
    return int(_lib.dsa_last_launch_count())


def dsa_test_set_wait_hooks(wait_limit_cycles: int = 0, stall: bool = False):
    """Test hook of the fp8-cache MLA kernel's bounded waits (this host thread's later
    calls): a shorter wait bound, and optionally a wait that nothing satisfies."""
    _check(_lib.dsa_test_set_wait_hooks(int(wait_limit_cycles), 1 if stall else 0), "dsa_test_set_wait_hooks")


class Paging:
    """Paged-cache description (dsa_paging): device int32 tensors seq_lens [B],
    block_table [B, max_pages], optional q_pos [B*n_q], plus the physical page count."""

    def __init__(self, seq_lens: torch.Tensor, block_table: torch.Tensor, num_pages: int, n_q: int = 1,
                 q_pos: Optional[torch.Tensor] = None, page_size: int = PAGE_SIZE):
        for name, t in (("seq_lens", seq_lens), ("block_table", block_table), ("q_pos", q_pos)):
            if t is not None and t.dtype != torch.int32:
                raise TypeError(f"{name} must be int32")
        self.seq_lens, self.block_table, self.q_pos = seq_lens, block_table, q_pos
        self.B = int(seq_lens.shape[0])
        self.n_q = int(n_q)
        self.max_pages = int(block_table.shape[1])
        self.num_pages = int(num_pages)
        self.page_size = int(page_size)
        self._s = _Paging(self.B, self.n_q, _ptr(seq_lens), _ptr(q_pos), _ptr(block_table),
                          self.max_pages, self.page_size, self.num_pages)

    @property
    def Bq(self) -> int:
        return self.B * self.n_q

    @property
    def L_layer(self) -> int:
        return self.max_pages * PAGE_SIZE

    def ref(self):
        return ctypes.byref(self._s)


def dsa_workspace_size(paging: Paging, L_max: int, top_k: int, op: int) -> int:
    return int(_lib.dsa_workspace_size(paging.ref(), int(L_max), int(top_k), int(op)))


def mla_workspace_size(Bq: int, top_k: int) -> int:
    return int(_lib.mla_workspace_size(int(Bq), int(top_k)))


def mla_num_splits(Bq: int, top_k: int) -> int:
    return int(_lib.mla_num_splits(int(Bq), int(top_k)))


def alloc_workspace(nbytes: int, device=None) -> torch.Tensor:
    """Zero-filled uint8 device buffer (torch allocations are at least 256-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def dsa_get_error(workspace: torch.Tensor, stream=None) -> int:
    return int(_lib.dsa_get_error(_ptr(workspace), _stream(stream)))


# ---------------------------------------------------------------------- stages

def dsa_indexer_scores(paging: Paging, q_idx, q_scale, head_w, k_cache, k_scale, scores: torch.Tensor,
                       workspace: torch.Tensor, stream=None):
    """scores[q, s] = sum_h w[q,h] * ReLU(q_idx[q,h] . k_idx[slot(s)]) for s < vis(q)."""
    L_max = int(scores.shape[-1])
    st = _lib.dsa_indexer_scores(paging.ref(), _ptr(q_idx), _dtype_code(q_idx), _ptr(q_scale), _ptr(head_w),
                                 _ptr(k_cache), _dtype_code(k_cache), _ptr(k_scale), _ptr(scores), L_max,
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "dsa_indexer_scores")
    return scores


def dsa_topk_pagemap(paging: Paging, scores: torch.Tensor, top_k: int, logical_out, physical_out,
                     workspace: torch.Tensor, stream=None):
    st = _lib.dsa_topk_pagemap(paging.ref(), _ptr(scores), int(scores.shape[-1]), int(top_k), _ptr(logical_out),
                               _ptr(physical_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "dsa_topk_pagemap")
    return logical_out, physical_out


def dsa_pagemap(paging: Paging, logical: torch.Tensor, physical: torch.Tensor, workspace: torch.Tensor,
                stream=None):
    st = _lib.dsa_pagemap(paging.ref(), _ptr(logical), int(logical.shape[-1]), _ptr(physical), _ptr(workspace),
                          workspace.numel(), _stream(stream))
    _check(st, "dsa_pagemap")
    return physical


def dsa_rope_quantize_append(paging: Paging, idx_q: torch.Tensor, idx_k: torch.Tensor, latent: torch.Tensor,
                             q_mla, q_idx_out: torch.Tensor, q_scale_out: torch.Tensor, k_cache: torch.Tensor,
                             k_scale: torch.Tensor, kv_cache: torch.Tensor, kv_scale, rope_base: float = 10000.0,
                             status=None, stream=None):
    """The step before the path for every query's new token (see include/dsa.h): RoPE on
    the rope columns, E4M3 quantisation, and the key and latent rows written at the
    token's cache slot. Returns (q_idx_out, q_scale_out)."""
    st = _lib.dsa_rope_quantize_append(paging.ref(), _ptr(idx_q), _ptr(idx_k), _ptr(latent), _ptr(q_mla),
                                       float(rope_base), _ptr(q_idx_out), _ptr(q_scale_out), _ptr(k_cache),
                                       _ptr(k_scale), _ptr(kv_cache), _kv_code(kv_cache), _ptr(kv_scale),
                                       _ptr(status), _stream(stream))
    _check(st, "dsa_rope_quantize_append")
    return q_idx_out, q_scale_out


def mla_sparse_decode(q: torch.Tensor, kv_cache: torch.Tensor, kv_scale, physical: torch.Tensor,
                      softmax_scale: float, out: torch.Tensor, lse, workspace: torch.Tensor, stream=None):
    Bq = int(q.shape[0])
    st = _lib.mla_sparse_decode(Bq, _ptr(q), _ptr(kv_cache), _kv_code(kv_cache), _ptr(kv_scale),
                                int(kv_cache.shape[0]), _ptr(physical), int(physical.shape[-1]),
                                float(softmax_scale), _ptr(out), _dtype_code(out), _ptr(lse), _ptr(workspace),
                                workspace.numel(), _stream(stream))
    _check(st, "mla_sparse_decode")
    return out


def mla_sparse_decode_noalloc(q: torch.Tensor, kv_cache: torch.Tensor, kv_scale, physical: torch.Tensor,
                              softmax_scale: float, out: torch.Tensor, lse=None, status=None, stream=None):
    """mla_sparse_decode with its scratch in the library's own device array (no workspace).

    For callers that cannot allocate device memory. `status`, if given, is a device int32
    tensor of 2 elements that receives the call's device-side error words."""
    Bq = int(q.shape[0])
    st = _lib.mla_sparse_decode_noalloc(Bq, _ptr(q), _ptr(kv_cache), _kv_code(kv_cache), _ptr(kv_scale),
                                        int(kv_cache.shape[0]), _ptr(physical), int(physical.shape[-1]),
                                        float(softmax_scale), _ptr(out), _dtype_code(out), _ptr(lse),
                                        _ptr(status), _stream(stream))
    _check(st, "mla_sparse_decode_noalloc")
    return out


def dsa_decode_layer(paging: Paging, q_idx, q_scale, head_w, k_cache, k_scale, q_mla, kv_cache, kv_scale,
                     top_k: int, softmax_scale: float, out: torch.Tensor, workspace: torch.Tensor, lse=None,
                     logical_out=None, physical_out=None, stream=None):
    """Indexer -> top-k + page map -> MLA sparse decode, one call on one stream."""
    st = _lib.dsa_decode_layer(paging.ref(), _ptr(q_idx), _dtype_code(q_idx), _ptr(q_scale), _ptr(head_w),
                               _ptr(k_cache), _ptr(k_scale), _ptr(q_mla), _ptr(kv_cache), _kv_code(kv_cache),
                               _ptr(kv_scale), int(top_k), float(softmax_scale), _ptr(out), _dtype_code(out),
                               _ptr(lse), _ptr(logical_out), _ptr(physical_out), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(st, "dsa_decode_layer")
    return out


# ---------------------------------------------------------------------- token-sharded decode

def dsa_shard_local_topk(paging: Paging, scores: torch.Tensor, top_k: int, token_offset: torch.Tensor,
                         cand_score: torch.Tensor, cand_token: torch.Tensor, workspace: torch.Tensor, stream=None):
    """This rank's top-k as exchange candidates: (score, global token) pairs [Bq, top_k]."""
    st = _lib.dsa_shard_local_topk(paging.ref(), _ptr(scores), int(scores.shape[-1]), int(top_k),
                                   _ptr(token_offset), _ptr(cand_score), _ptr(cand_token), _ptr(workspace),
                                   workspace.numel(), _stream(stream))
    _check(st, "dsa_shard_local_topk")
    return cand_score, cand_token


def dsa_shard_select(paging: Paging, n_ranks: int, rank: int, all_score: torch.Tensor, all_token: torch.Tensor,
                     top_k: int, token_offset: torch.Tensor, physical_out: torch.Tensor, workspace: torch.Tensor,
                     logical_out=None, stream=None):
    """Global selection among every rank's candidates [n_ranks, Bq, top_k]; this rank's
    winners as slots of its own caches (first, then -1)."""
    st = _lib.dsa_shard_select(paging.ref(), int(n_ranks), int(rank), _ptr(all_score), _ptr(all_token), int(top_k),
                               _ptr(token_offset), _ptr(physical_out), _ptr(logical_out), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _check(st, "dsa_shard_select")
    return physical_out


def dsa_shard_merge(all_out: torch.Tensor, all_lse: torch.Tensor, out: torch.Tensor, lse=None, stream=None):
    """Log-sum-exp merge of every rank's (out fp32 [Bq, 64, 512], lse [Bq, 64]) state."""
    n_ranks, Bq = int(all_out.shape[0]), int(all_out.shape[1])
    st = _lib.dsa_shard_merge(Bq, n_ranks, _ptr(all_out), _ptr(all_lse), _ptr(out), _dtype_code(out), _ptr(lse),
                              _stream(stream))
    _check(st, "dsa_shard_merge")
    return out

