"""Hand-built cases for the oracle pins (numpy only, no method arithmetic)."""
import math

import numpy as np

from dsa_inputs import PAGE, H, DI, DK, to_bf16_bits


def blank_case(seq_lens, n_q=1, top_k=4, idx_dtype="bf16", kv_dtype="bf16", max_pages=None,
               q_pos=None, softmax_scale=1.0 / math.sqrt(192.0), table=None):
    """A case dict with zero-filled caches and an identity-or-given block table."""
    lens = np.asarray(seq_lens, dtype=np.int32)
    B = len(lens)
    pages = (lens.astype(np.int64) + PAGE - 1) // PAGE
    mp = int(max_pages or max(1, int(pages.max(initial=1))))
    P = int(pages.sum())
    if table is None:
        bt = np.full((B, mp), -1, dtype=np.int32)
        off = 0
        for b in range(B):
            bt[b, :pages[b]] = np.arange(off, off + pages[b])
            off += pages[b]
    else:
        bt = np.asarray(table, dtype=np.int32)
        P = max(P, int(bt.max()) + 1)
    Bq = B * n_q
    idt = np.uint16 if idx_dtype == "bf16" else np.uint8
    kdt = np.uint16 if kv_dtype == "bf16" else np.uint8
    return dict(
        B=B, n_q=n_q, Bq=Bq, page_size=PAGE, num_pages=P, max_pages=mp,
        seq_lens=lens, q_pos=None if q_pos is None else np.asarray(q_pos, dtype=np.int32),
        block_table=bt,
        q_idx=np.zeros((Bq, H, DI), dtype=idt),
        q_idx_scale=None if idx_dtype == "bf16" else np.ones((Bq, H), dtype=np.float32),
        head_w=np.zeros((Bq, H), dtype=np.float32),
        k_cache=np.zeros((P, PAGE, DI), dtype=idt),
        k_scale=None if idx_dtype == "bf16" else np.ones((P, PAGE), dtype=np.float32),
        q_mla=np.zeros((Bq, H, DK), dtype=np.uint16),
        kv_cache=np.zeros((P * PAGE, DK), dtype=kdt),
        kv_scale=None if kv_dtype == "bf16" else np.ones((P * PAGE, 5), dtype=np.float32),
        top_k=top_k, softmax_scale=float(np.float32(softmax_scale)),
        idx_dtype=idx_dtype, kv_dtype=kv_dtype, out_dtype="fp32", planted=[],
    )


def bf16(x):
    return to_bf16_bits(np.asarray(x, dtype=np.float32))


def slot_of(case, b, token):
    return int(case["block_table"][b, token // PAGE]) * PAGE + token % PAGE


def permute_pages(case, perm):
    """Move every physical page p to position perm[p] and rewrite the block table to
    match: the logical content of every sequence is unchanged."""
    c = dict(case)
    P = case["num_pages"]
    perm = np.asarray(perm)
    inv_target = np.empty(P, dtype=np.int64)
    inv_target[perm] = np.arange(P)
    c["k_cache"] = case["k_cache"][inv_target]
    if case["k_scale"] is not None:
        c["k_scale"] = case["k_scale"][inv_target]
    kv = case["kv_cache"].reshape(P, PAGE, DK)[inv_target].reshape(P * PAGE, DK)
    c["kv_cache"] = kv
    if case["kv_scale"] is not None:
        c["kv_scale"] = case["kv_scale"].reshape(P, PAGE, 5)[inv_target].reshape(P * PAGE, 5)
    bt = case["block_table"].copy()
    m = bt >= 0
    bt[m] = perm[bt[m]]
    c["block_table"] = bt
    return c
