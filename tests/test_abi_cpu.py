"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol include/dsa.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import deepseek_sparse_attention_head_b200 as dsa
from deepseek_sparse_attention_head_b200 import _lib, _Paging

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(0x100000)      # never dereferenced: every call below fails validation first


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)) - {"if"})


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "dsa_decode_layer" in names and len(names) >= 10
    for n in names:
        assert hasattr(_lib, n), n
    assert sorted(names) == dsa.exported_symbols()


def paging(B=2, n_q=1, page_size=64, max_pages=4, num_pages=8, seq=FAKE, table=FAKE):
    return _Paging(B, n_q, seq, None, table, max_pages, page_size, num_pages)


def ws_ok(pg, op=dsa.DSA_OP_INDEXER, L=256, top_k=16):
    return _lib.dsa_workspace_size(ctypes.byref(pg), L, top_k, op)


def call_indexer(pg, qd=dsa.DSA_FP8_E4M3, kd=dsa.DSA_FP8_E4M3, qs=FAKE, ks=FAKE, ws_bytes=None, ws=FAKE, L=256):
    if ws_bytes is None:
        ws_bytes = ws_ok(pg) if pg is not None else 1 << 20
    return _lib.dsa_indexer_scores(ctypes.byref(pg) if pg is not None else None, FAKE, qd, qs, FAKE, FAKE, kd, ks,
                                   FAKE, L, ws, ws_bytes, None)


def test_indexer_argument_errors():
    pg = paging()
    assert call_indexer(None) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(paging(B=0)) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(paging(page_size=32)) == dsa.DSA_ERR_UNSUPPORTED
    assert call_indexer(paging(seq=None)) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(pg, qd=dsa.DSA_BF16) == dsa.DSA_ERR_INVALID_ARG            # dtype mismatch
    assert call_indexer(pg, qs=None) == dsa.DSA_ERR_INVALID_ARG                      # fp8 needs scales
    assert call_indexer(pg, qd=dsa.DSA_BF16, kd=dsa.DSA_BF16) == dsa.DSA_ERR_INVALID_ARG  # bf16 takes none
    assert call_indexer(pg, qd=dsa.DSA_FP32, kd=dsa.DSA_FP32) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(pg, qd=dsa.DSA_FP8_E4M3_ROPE_BF16, kd=dsa.DSA_FP8_E4M3_ROPE_BF16) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(pg, L=0) == dsa.DSA_ERR_INVALID_ARG
    assert call_indexer(pg, ws_bytes=16) == dsa.DSA_ERR_WORKSPACE
    assert call_indexer(pg, ws=None) == dsa.DSA_ERR_WORKSPACE
    assert call_indexer(pg, ws=ctypes.c_void_p(0x100010)) == dsa.DSA_ERR_WORKSPACE   # misaligned


def test_topk_and_pagemap_argument_errors():
    pg = paging()
    ws = ws_ok(pg, dsa.DSA_OP_TOPK)
    assert _lib.dsa_topk_pagemap(ctypes.byref(pg), FAKE, 256, 0, FAKE, FAKE, FAKE, ws, None) == dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_topk_pagemap(ctypes.byref(pg), FAKE, 256, 16, None, None, FAKE, ws, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_topk_pagemap(ctypes.byref(pg), None, 256, 16, FAKE, FAKE, FAKE, ws, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_pagemap(ctypes.byref(pg), None, 16, FAKE, FAKE, 4096, None) == dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_pagemap(ctypes.byref(pg), FAKE, 0, FAKE, FAKE, 4096, None) == dsa.DSA_ERR_INVALID_ARG


def test_mla_argument_errors():
    def call(Bq=2, kvd=dsa.DSA_FP8_E4M3, kvs=FAKE, top_k=64, scale=0.07, outd=dsa.DSA_BF16, q=FAKE):
        return _lib.mla_sparse_decode(Bq, q, FAKE, kvd, kvs, 1024, FAKE, top_k, scale, FAKE, outd, None, FAKE,
                                      1 << 30, None)
    assert call(Bq=0) == dsa.DSA_ERR_INVALID_ARG
    assert call(q=None) == dsa.DSA_ERR_INVALID_ARG
    assert call(top_k=0) == dsa.DSA_ERR_INVALID_ARG
    assert call(top_k=16385) == dsa.DSA_ERR_INVALID_ARG
    assert call(scale=-1.0) == dsa.DSA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == dsa.DSA_ERR_INVALID_ARG
    assert call(kvs=None) == dsa.DSA_ERR_INVALID_ARG
    assert call(kvd=dsa.DSA_BF16) == dsa.DSA_ERR_INVALID_ARG
    assert call(outd=dsa.DSA_FP8_E4M3) == dsa.DSA_ERR_INVALID_ARG
    assert call(q=ctypes.c_void_p(0x100008)) == dsa.DSA_ERR_INVALID_ARG   # TMA needs 16-byte alignment
    # packed 656-byte rows carry their scales: a scale plane is an error
    assert call(kvd=dsa.DSA_FP8_E4M3_ROPE_BF16) == dsa.DSA_ERR_INVALID_ARG
    assert call(outd=dsa.DSA_FP8_E4M3_ROPE_BF16) == dsa.DSA_ERR_INVALID_ARG


def test_workspace_sizes_are_consistent():
    pg = paging(B=3, n_q=2, max_pages=10)
    a = ws_ok(pg, dsa.DSA_OP_INDEXER, 640, 0)
    assert a >= 256 + 4 * 4 and a % 256 == 0
    layer = _lib.dsa_workspace_size(ctypes.byref(pg), 0, 64, dsa.DSA_OP_LAYER)
    # scores [6, 640] fp32 + two [6, 64] int32 lists at least
    assert layer >= 256 + 6 * 640 * 4 + 2 * 6 * 64 * 4
    assert _lib.dsa_workspace_size(ctypes.byref(pg), 0, 0, dsa.DSA_OP_LAYER) == 0     # invalid top_k
    assert _lib.dsa_workspace_size(None, 0, 64, dsa.DSA_OP_LAYER) == 0
    assert _lib.mla_workspace_size(0, 64) == 0
    assert _lib.mla_workspace_size(4, 64) >= 256


def test_status_strings():
    for s in range(7):
        assert dsa.dsa_status_string(s)
    assert dsa.dsa_status_string(99) == "unknown status"


def test_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError):
        dsa._ptr(torch.zeros(4))
    # the token-sharded entry points marshal through the same checks: no host tensor reaches
    # the library, and nothing falls back to a CPU computation
    with pytest.raises(ValueError):
        dsa.dsa_shard_merge(torch.zeros(2, 1, 64, 512), torch.zeros(2, 1, 64), torch.zeros(1, 64, 512))


def test_noalloc_argument_errors():
    def call(Bq=2, top_k=64, q=FAKE, scale=0.07, status=None):
        return _lib.mla_sparse_decode_noalloc(Bq, q, FAKE, dsa.DSA_FP8_E4M3, FAKE, 1024, FAKE, top_k, scale, FAKE,
                                              dsa.DSA_BF16, None, status, None)
    assert call(Bq=0) == dsa.DSA_ERR_INVALID_ARG
    assert call(q=None) == dsa.DSA_ERR_INVALID_ARG
    assert call(top_k=16385) == dsa.DSA_ERR_INVALID_ARG
    assert call(scale=0.0) == dsa.DSA_ERR_INVALID_ARG
    assert call(status=ctypes.c_void_p(0x100004)) == dsa.DSA_ERR_INVALID_ARG   # status words need 8-byte alignment


def test_wait_hook_argument_errors():
    assert _lib.dsa_test_set_wait_hooks(-1, 0) == dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_test_set_wait_hooks(0, 2) == dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_test_set_wait_hooks(1000, 1) == dsa.DSA_OK
    assert _lib.dsa_test_set_wait_hooks(0, 0) == dsa.DSA_OK


def test_append_argument_errors():
    pg = paging(B=2, n_q=1, max_pages=4)

    def call(idx_q=FAKE, kvd=dsa.DSA_FP8_E4M3, kvs=FAKE, base=10000.0, status=None, q_mla=None):
        return _lib.dsa_rope_quantize_append(ctypes.byref(pg), idx_q, FAKE, FAKE, q_mla, base, FAKE, FAKE, FAKE,
                                             FAKE, FAKE, kvd, kvs, status, None)
    assert call(idx_q=None) == dsa.DSA_ERR_INVALID_ARG
    assert call(kvs=None) == dsa.DSA_ERR_INVALID_ARG                               # fp8 needs its scale plane
    assert call(kvd=dsa.DSA_FP8_E4M3_ROPE_BF16) == dsa.DSA_ERR_INVALID_ARG          # packed rows take none
    assert call(kvd=dsa.DSA_BF16) == dsa.DSA_ERR_INVALID_ARG
    assert call(kvd=dsa.DSA_FP32) == dsa.DSA_ERR_INVALID_ARG
    assert call(base=1.0) == dsa.DSA_ERR_INVALID_ARG
    assert call(base=float("inf")) == dsa.DSA_ERR_INVALID_ARG
    assert call(idx_q=ctypes.c_void_p(0x100008)) == dsa.DSA_ERR_INVALID_ARG         # 16-byte alignment
    assert call(q_mla=ctypes.c_void_p(0x100008)) == dsa.DSA_ERR_INVALID_ARG
    assert call(status=ctypes.c_void_p(0x100004)) == dsa.DSA_ERR_INVALID_ARG
    assert _lib.dsa_rope_quantize_append(None, FAKE, FAKE, FAKE, None, 10000.0, FAKE, FAKE, FAKE, FAKE, FAKE,
                                         dsa.DSA_FP8_E4M3, FAKE, None, None) == dsa.DSA_ERR_INVALID_ARG


def test_shard_argument_errors():
    pg = paging(B=2, max_pages=4)
    ws_l = _lib.dsa_workspace_size(ctypes.byref(pg), 256, 16, dsa.DSA_OP_SHARD_LOCAL)
    assert ws_l >= 256 + 2 * 16 * 4 and ws_l % 256 == 0
    assert _lib.dsa_workspace_size(ctypes.byref(pg), 256, 0, dsa.DSA_OP_SHARD_LOCAL) == 0
    assert _lib.dsa_workspace_size(ctypes.byref(pg), 256, 16, 6) == 0
    ws_s = _lib.dsa_workspace_size(ctypes.byref(pg), 0, 16, dsa.DSA_OP_SHARD_SELECT)
    assert ws_s >= 256

    def local(p=pg, top_k=16, offset=FAKE, ws_bytes=ws_l):
        return _lib.dsa_shard_local_topk(ctypes.byref(p), FAKE, 256, top_k, offset, FAKE, FAKE, FAKE, ws_bytes, None)

    assert local(offset=None) == dsa.DSA_ERR_INVALID_ARG
    assert local(top_k=0) == dsa.DSA_ERR_INVALID_ARG
    assert local(top_k=16385) == dsa.DSA_ERR_INVALID_ARG
    assert local(ws_bytes=ws_l - 1) == dsa.DSA_ERR_WORKSPACE
    causal = _Paging(2, 1, FAKE, FAKE, FAKE, 4, 64, 8)
    assert local(p=causal) == dsa.DSA_ERR_UNSUPPORTED

    def select(p=pg, n_ranks=2, rank=0, top_k=16, physical=FAKE, ws_bytes=ws_s):
        return _lib.dsa_shard_select(ctypes.byref(p), n_ranks, rank, FAKE, FAKE, top_k, FAKE, physical, None, FAKE,
                                     ws_bytes, None)

    assert select(rank=2) == dsa.DSA_ERR_INVALID_ARG
    assert select(rank=-1) == dsa.DSA_ERR_INVALID_ARG
    assert select(n_ranks=0) == dsa.DSA_ERR_INVALID_ARG
    assert select(physical=None) == dsa.DSA_ERR_INVALID_ARG
    assert select(n_ranks=1 << 17, top_k=8192) == dsa.DSA_ERR_UNSUPPORTED
    assert select(ws_bytes=0) == dsa.DSA_ERR_WORKSPACE
    assert select(p=causal) == dsa.DSA_ERR_UNSUPPORTED

    def merge(Bq=1, n_ranks=2, all_out=FAKE, out=FAKE, dt=dsa.DSA_FP32):
        return _lib.dsa_shard_merge(Bq, n_ranks, all_out, FAKE, out, dt, None, None)

    assert merge(Bq=0) == dsa.DSA_ERR_INVALID_ARG
    assert merge(n_ranks=0) == dsa.DSA_ERR_INVALID_ARG
    assert merge(dt=dsa.DSA_FP8_E4M3) == dsa.DSA_ERR_INVALID_ARG
    assert merge(all_out=ctypes.c_void_p(0x100004)) == dsa.DSA_ERR_INVALID_ARG
    assert merge(out=ctypes.c_void_p(0x100008)) == dsa.DSA_ERR_INVALID_ARG        # fp32 out needs 16 bytes
    assert merge(out=None) == dsa.DSA_ERR_INVALID_ARG


def test_shard_bounds_are_page_aligned_and_cover_the_row():
    from deepseek_sparse_attention_head_b200.sharded import shard_bounds
    assert shard_bounds(1000, 1) == [0, 1000]
    assert shard_bounds(1000, 2) == [0, 512, 1000]
    assert shard_bounds(1000, 3) == [0, 384, 768, 1000]
    assert shard_bounds(100, 4) == [0, 64, 100, 100, 100]
    assert shard_bounds(0, 3) == [0, 0, 0, 0]
    for L in (1, 63, 64, 65, 4095, 1 << 20):
        for R in (1, 2, 3, 8):
            b = shard_bounds(L, R)
            assert b[0] == 0 and b[-1] == L and all(x <= y for x, y in zip(b, b[1:]))
            assert all(x % 64 == 0 or x == L for x in b)   # every shard starts on a page
    with pytest.raises(ValueError):
        shard_bounds(10, 0)


def test_token_sharded_decode_rejects_causal_positions():
    from types import SimpleNamespace
    import torch
    from deepseek_sparse_attention_head_b200.sharded import TokenShardedDecode
    paging = SimpleNamespace(q_pos=torch.zeros(1, dtype=torch.int32), Bq=1, L_layer=64)
    with pytest.raises(ValueError):
        TokenShardedDecode(paging, torch.zeros(1, dtype=torch.int32), 8, 0.1, 0, 2)

