"""The step before the path (dsa_rope_quantize_append) against the fp64 oracle: partial
interleaved RoPE on the rope columns, E4M3 quantisation with amax/448 scales, and the new
token's key and latent rows written at its cache slot ("Show HN: colibri", features: MLA
with partial interleaved RoPE; the per-token caches of the GLM-52 kernel list).

Comparisons: fp32 scales within 1e-6 relative; E4M3 codes exactly, except where the
oracle's value lies within 1e-5 relative of a rounding midpoint (fp32 against fp64
arithmetic), where either neighbour is accepted; bf16 outputs within one unit in the last
place; every cache row that is not an appended slot unchanged, bit for bit."""
import numpy as np
import pytest

import oracle
from dsa_inputs import CaseSpec, generate, new_token_inputs, to_torch

pytestmark = pytest.mark.gpu

CASES = {
    "fp8_decode": CaseSpec("app_fp8", (70, 150, 1, 300), top_k=32, kv_dtype="fp8", seed=81),
    "packed_decode": CaseSpec("app_fp8r", (70, 150, 1, 300), top_k=32, kv_dtype="fp8r", seed=82),
    "bf16_latent": CaseSpec("app_bf16", (64, 65, 129), top_k=32, kv_dtype="bf16", seed=83),
    # speculative decode: three new tokens per row, at the row's last positions
    "fp8_mtp": CaseSpec("app_mtp", (70, 1000, 3), top_k=32, n_q=3, q_tail=True, n_planted=0, seed=84),
    # positions in the millions: the angles are reduced in fp64 on the GPU
    "long_positions": CaseSpec("app_long", (1 << 20,), top_k=32, n_q=2, q_pos=(999_999, 1_048_575),
                               n_planted=0, seed=85),
}


def _codes_ok(got, values):
    """E4M3 codes `got` against the oracle's unquantised values (x / scale, fp64)."""
    lo = oracle.encode_e4m3(values * (1 - 1e-5))
    hi = oracle.encode_e4m3(values * (1 + 1e-5))
    exact = oracle.encode_e4m3(values)
    ok = (got == exact) | (got == lo) | (got == hi)
    return bool(ok.all()), int((got != exact).sum())


def _bf16_close(got_bits, want_bits):
    g = oracle.decode_bf16(got_bits)
    w = oracle.decode_bf16(want_bits)
    return bool(np.all(np.abs(g - w) <= np.abs(w) * 2.0 ** -7 + 1e-30))


def _run(name):
    import torch
    import deepseek_sparse_attention_head_b200 as dsa
    case = generate(CASES[name])
    new = new_token_inputs(case, seed=7)
    t = to_torch(case, "cuda")
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16).cuda()
    idx_q, idx_k, lat, q_mla = bf(new["idx_q"]), bf(new["idx_k"]), bf(new["latent"]), bf(new["q_mla"])
    Bq = case["Bq"]
    q_out = torch.empty(Bq, 64, 128, dtype=torch.uint8, device="cuda")
    q_sc = torch.empty(Bq, 64, dtype=torch.float32, device="cuda")
    k_cache = t["k_cache"].view(torch.uint8).clone()
    k_scale = t["k_scale"].clone()
    kv_cache = t["kv_cache"].clone()
    kv_scale = None if t["kv_scale"] is None else t["kv_scale"].clone()
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    paging = dsa.Paging(t["seq_lens"], t["block_table"], case["num_pages"], case["n_q"], t["q_pos"])
    dsa.dsa_rope_quantize_append(paging, idx_q, idx_k, lat, q_mla, q_out, q_sc, k_cache, k_scale, kv_cache,
                                 kv_scale, status=status)
    torch.cuda.synchronize()
    as_np = lambda x: None if x is None else (x.view(torch.uint8) if x.dtype == torch.float8_e4m3fn else x).cpu().numpy()
    gpu = dict(q_codes=as_np(q_out), q_scale=as_np(q_sc), k_cache=as_np(k_cache), k_scale=as_np(k_scale),
               kv_cache=as_np(kv_cache.view(torch.int16) if kv_cache.dtype == torch.bfloat16 else kv_cache),
               kv_scale=as_np(kv_scale), q_mla=as_np(q_mla.view(torch.int16)).view(np.uint16),
               status=status.cpu().numpy())
    return case, new, gpu


@pytest.mark.parametrize("name", list(CASES))
def test_append_matches_oracle(name):
    case, new, gpu = _run(name)
    assert gpu["status"][0] == 0
    ref = oracle.rope_quantize_append(case, new)
    # indexer queries: scales, then codes against x / scale
    assert np.allclose(gpu["q_scale"], ref["q_scale"], rtol=1e-6, atol=0)
    q = oracle.decode_bf16(new["idx_q"])
    pos = oracle.new_token_positions(case)
    q[..., :64] = oracle.rope_interleaved(q[..., :64], pos[:, None])
    ok, n = _codes_ok(gpu["q_codes"], q / ref["q_scale"].astype(np.float64)[..., None])
    assert ok, f"{n} query codes off by more than a rounding near-tie"
    # the new keys at their slots; every other key row untouched
    slots = ref["slots"]
    kflat = gpu["k_cache"].reshape(-1, 128)
    assert np.allclose(gpu["k_scale"].reshape(-1)[slots], ref["k_scale"], rtol=1e-6, atol=0)
    k = oracle.decode_bf16(new["idx_k"])
    k[..., :64] = oracle.rope_interleaved(k[..., :64], pos)
    ok, n = _codes_ok(kflat[slots], k / ref["k_scale"].astype(np.float64)[:, None])
    assert ok, f"{n} key codes off"
    other = np.setdiff1d(np.arange(kflat.shape[0]), slots)
    assert np.array_equal(kflat[other], case["k_cache"].reshape(-1, 128)[other])
    assert np.array_equal(gpu["k_scale"].reshape(-1)[other], case["k_scale"].reshape(-1)[other])
    # the latent rows at their slots, in the cache's format; every other row untouched
    lat = oracle.decode_bf16(new["latent"])
    lat[..., 512:] = oracle.rope_interleaved(lat[..., 512:], pos)
    kv = gpu["kv_cache"]
    rows_other = np.setdiff1d(np.arange(kv.shape[0]), slots)
    kv0 = case["kv_cache"].view(np.int16) if case["kv_dtype"] == "bf16" else case["kv_cache"]
    assert np.array_equal(kv[rows_other], kv0[rows_other])
    if case["kv_dtype"] == "fp8":
        sc = gpu["kv_scale"][slots]
        assert np.allclose(sc, ref["latent_scales"], rtol=1e-6, atol=0)
        bounds = [(0, 128), (128, 256), (256, 384), (384, 512), (512, 576)]
        for g, (lo, hi) in enumerate(bounds):
            ok, n = _codes_ok(kv[slots, lo:hi], lat[:, lo:hi] / ref["latent_scales"][:, g:g + 1].astype(np.float64))
            assert ok, f"group {g}: {n} latent codes off"
        assert np.array_equal(gpu["kv_scale"][rows_other], case["kv_scale"][rows_other])
    elif case["kv_dtype"] == "fp8r":
        row = kv[slots]
        sc = row[:, 512:528].copy().view("<f4")
        assert np.allclose(sc, ref["latent_packed"][:, 512:528].copy().view("<f4"), rtol=1e-6, atol=0)
        for g in range(4):
            ok, n = _codes_ok(row[:, 128 * g:128 * g + 128],
                              lat[:, 128 * g:128 * g + 128] / sc[:, g:g + 1].astype(np.float64))
            assert ok, f"group {g}: {n} latent codes off"
        assert _bf16_close(row[:, 528:].copy().view("<u2"), ref["latent_packed"][:, 528:].copy().view("<u2"))
    else:
        assert _bf16_close(kv[slots].view(np.uint16), ref["latent_bf16"])
    # the MLA query: latent columns bit for bit, rope columns within one bf16 unit
    assert np.array_equal(gpu["q_mla"][..., :512], new["q_mla"][..., :512])
    assert _bf16_close(gpu["q_mla"][..., 512:], ref["q_mla"][..., 512:])


def test_position_outside_the_table_reports_and_writes_nothing():
    """A query whose position lies past its row's block table: DSA_ERR_DEVICE_BOUNDS, and
    no cache row changes for it (the other queries still append)."""
    import torch
    import deepseek_sparse_attention_head_b200 as dsa
    case = generate(CaseSpec("app_oob", (100, 100), top_k=32, n_q=1, n_planted=0, seed=86))
    new = new_token_inputs(case, seed=8, with_q_mla=False)
    t = to_torch(case, "cuda")
    q_pos = torch.tensor([99, 64 * case["max_pages"] + 5], dtype=torch.int32, device="cuda")   # second is past the table
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16).cuda()
    k_cache = t["k_cache"].view(torch.uint8).clone()
    k_scale = t["k_scale"].clone()
    kv_cache = t["kv_cache"].view(torch.uint8).clone()
    kv_scale = t["kv_scale"].clone()
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    paging = dsa.Paging(t["seq_lens"], t["block_table"], case["num_pages"], 1, q_pos)
    q_out = torch.empty(2, 64, 128, dtype=torch.uint8, device="cuda")
    q_sc = torch.empty(2, 64, dtype=torch.float32, device="cuda")
    dsa.dsa_rope_quantize_append(paging, bf(new["idx_q"]), bf(new["idx_k"]), bf(new["latent"]), None, q_out, q_sc,
                                 k_cache, k_scale, kv_cache, kv_scale, status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == dsa.DSA_ERR_DEVICE_BOUNDS
    slot0 = int(case["block_table"][0, 1]) * 64 + 35
    changed = np.nonzero((k_cache.cpu().numpy().reshape(-1, 128) != case["k_cache"].reshape(-1, 128)).any(axis=1))[0]
    assert set(changed.tolist()) <= {slot0}
    changed_kv = np.nonzero((kv_cache.cpu().numpy() != case["kv_cache"]).any(axis=1))[0]
    assert set(changed_kv.tolist()) <= {slot0} and slot0 in changed_kv.tolist()


def test_decode_right_after_append_sees_the_rotated_queries():
    """mla_sparse_decode replayed from one CUDA graph directly behind dsa_rope_quantize_append
    (programmatic dependent launch lets the second kernel start while the first runs) reads
    the queries only after the append has rotated them: its output equals that of the same
    two calls separated by a device synchronisation, bit for bit."""
    import torch
    import deepseek_sparse_attention_head_b200 as dsa
    case = generate(CaseSpec("app_then_mla", (3000, 1500, 4100, 2222) * 16, top_k=512, kv_dtype="fp8", seed=87))
    new = new_token_inputs(case, seed=9)
    t = to_torch(case, "cuda")
    Bq = case["Bq"]
    vis = oracle.visible_lengths(case)
    logical = np.full((Bq, 512), -1, dtype=np.int64)
    for q in range(Bq):
        n = min(512, int(vis[q]))
        logical[q, :n] = np.arange(int(vis[q]) - n, int(vis[q]))    # the newest tokens, the new one included
    phys = torch.from_numpy(oracle.pagemap(case, logical).astype(np.int32)).cuda()
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.int16).view(torch.bfloat16).cuda()
    paging = dsa.Paging(t["seq_lens"], t["block_table"], case["num_pages"], case["n_q"], t["q_pos"])
    q0, iq, ik, lat = bf(new["q_mla"]), bf(new["idx_q"]), bf(new["idx_k"]), bf(new["latent"])
    q_mla = q0.clone()
    k_cache, k_scale = t["k_cache"].view(torch.uint8).clone(), t["k_scale"].clone()
    kv_cache, kv_scale = t["kv_cache"].clone(), t["kv_scale"].clone()
    q_out = torch.empty(Bq, 64, 128, dtype=torch.uint8, device="cuda")
    q_sc = torch.empty(Bq, 64, dtype=torch.float32, device="cuda")
    out = torch.empty((Bq, 64, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(Bq, 64, dtype=torch.float32, device="cuda")
    ws = dsa.alloc_workspace(dsa.mla_workspace_size(Bq, 512))

    def reset():
        q_mla.copy_(q0)
        k_cache.copy_(t["k_cache"].view(torch.uint8))
        k_scale.copy_(t["k_scale"])
        kv_cache.copy_(t["kv_cache"])
        kv_scale.copy_(t["kv_scale"])
        out.fill_(float("nan"))
        torch.cuda.synchronize()

    def append():
        dsa.dsa_rope_quantize_append(paging, iq, ik, lat, q_mla, q_out, q_sc, k_cache, k_scale, kv_cache, kv_scale)

    def decode():
        dsa.mla_sparse_decode(q_mla, kv_cache, kv_scale, phys, case["softmax_scale"], out, lse, ws)

    reset()
    append()
    torch.cuda.synchronize()
    decode()
    torch.cuda.synchronize()
    assert dsa.dsa_get_error(ws) == 0
    want = (out.view(torch.int16).cpu().numpy(), lse.cpu().numpy())
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            append()
            decode()
    for _ in range(5):
        reset()
        graph.replay()
        torch.cuda.synchronize()
        assert dsa.dsa_get_error(ws) == 0
        assert np.array_equal(out.view(torch.int16).cpu().numpy(), want[0])
        assert np.array_equal(lse.cpu().numpy(), want[1])
