"""Paged cache through the fused multi-block kernel: retrieval with a
workspace and the paged decode step, at lengths past what the one-block
paged kernel handles.  Index sets and distances must equal the oracle's on
the cache read back in token order; attention must agree with the oracle
within ATOL, and bit for bit with the contiguous-layout call on the gathered
copy (the same kernel with only the addressing changed)."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL, margin_inputs, u32
from tests.test_gpu_paged import RETRIEVE_CASES, _scatter

pytestmark = pytest.mark.gpu
DEV = "cuda"

MULTIBLOCK_CASES = RETRIEVE_CASES + [
    # B, Hq, Hkv, bits, N, page_size, sink, local, top_k
    (1, 28, 4, 128, 200003, 256, 4, 128, 1024),  # many blocks per KV head, ragged last page
    (2, 8, 2, 64, 100001, 100, 4, 64, 500),      # 64-bit codes, page size not a power of two
]


@pytest.mark.parametrize("case", MULTIBLOCK_CASES)
def test_paged_retrieval_with_workspace(case):
    B, Hq, Hkv, bits, N, P, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(171 + N, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(172 + N, B * Hq, W).view(B, Hq, W)
    pool, table = _scatter(kc, P, 173 + N)
    ws = hkv.workspace(B, Hq, Hkv, N, bits, k, s, l)
    st = hkv.status_word()
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    dist = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    hkv.hkv_retrieve_topk_paged(qc.to(DEV), pool.to(DEV), table.to(DEV), N, s, l, k, idx, dist, status=st, ws=ws)
    assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    gathered = oracle.gather_pages(u32(pool), table.numpy(), P, N)
    want_i, want_d = oracle.retrieve(u32(qc), gathered, N, s, l, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_i)
    np.testing.assert_array_equal(dist.cpu().numpy(), want_d)


def test_paged_retrieval_with_workspace_reports_a_page_outside_the_pool():
    B, Hq, Hkv, W, N, P = 1, 4, 1, 4, 40000, 64
    kc = synth.random_codes(190, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(191, B * Hq, W).view(B, Hq, W)
    pool, table = _scatter(kc, P, 192)
    table[0, 3] = pool.shape[0]  # tokens 192..255 point past the pool
    ws = hkv.workspace(B, Hq, Hkv, N, 128, 10, 0, 0)
    st = hkv.status_word()
    idx = torch.full((B, Hkv, 10), -7, dtype=torch.int32, device=DEV)
    hkv.hkv_retrieve_topk_paged(qc.to(DEV), pool.to(DEV), table.to(DEV), N, 0, 0, 10, idx, status=st, ws=ws)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
    assert not np.isin(idx.cpu().numpy(), np.arange(192, 256)).any()


DECODE_CASES = [
    # workload, overrides, page size
    ("qwen7b_512k", dict(N=9001, layers=1), 256),
    ("qwen7b_512k", dict(N=120001, layers=1), 128),   # many blocks per KV head: speculative tile
    ("hashevict_lsh", dict(B=2, N=5003), 48),          # page size not a power of two
    ("signvq", dict(B=2, N=4099), 64),
    ("tiny_lsh", dict(), 64),                          # fp32
]


def _hash(w, inp):
    if w.hash == "lsh":
        return hkv.HashParams.lsh(inp["R"].to(DEV)), inp["R"], inp["R"]
    return hkv.HashParams.sign(hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32), None, None


def _decode_paged_vs_contiguous(w, inp, P):
    B, Hq, Hkv, N, W, k = w.B, w.Hq, w.Hkv, w.N, w.words, w.top_k
    K, V, q = inp["K"][:, :, :N].contiguous(), inp["V"][:, :, :N].contiguous(), inp["q"]
    h, qparams, kparams = _hash(w, inp)
    codes = torch.zeros(B, Hkv, N, W, dtype=torch.int32, device=DEV)
    norms = torch.zeros(B, Hkv, N, dtype=torch.float16, device=DEV) if w.hash == "sign" else None
    hkv.hkv_encode_keys(h, K.to(DEV).reshape(-1, 128), codes.view(-1, W), None if norms is None else norms.view(-1))
    cpool, table = _scatter(codes.cpu(), P, 195)
    kpool, _ = _scatter(K, P, 195)
    vpool, _ = _scatter(V, P, 195)
    ws = hkv.workspace(B, Hq, Hkv, N, w.bits, k, w.n_sink, w.n_local)
    st = hkv.status_word()
    res = {}
    for mode in ("paged", "contiguous"):
        out = torch.full((B, Hq, 128), float("nan"), device=DEV)
        lse = torch.full((B, Hq), float("nan"), device=DEV)
        idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
        qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
        if mode == "paged":
            hkv.hkv_decode_step_paged(h, q.to(DEV), cpool.to(DEV), kpool.to(DEV), vpool.to(DEV), table.to(DEV), N,
                                      w.n_sink, w.n_local, k, out, lse=lse, q_codes=qc, idx=idx, ws=ws, status=st)
        else:
            hkv.hkv_decode_step(h, q.to(DEV), codes, K.to(DEV), V.to(DEV), N, w.n_sink, w.n_local, k, out, lse=lse,
                                q_codes=qc, idx=idx, ws=ws, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
        res[mode] = (out.cpu(), lse.cpu(), idx.cpu(), qc.cpu())
    return res, codes, qparams, kparams


@pytest.mark.parametrize("name,over,P", DECODE_CASES)
def test_paged_decode_step(name, over, P):
    w = synth.WORKLOADS[name].with_(**over)
    inp = margin_inputs(w, cap=w.N)
    res, codes, qparams, kparams = _decode_paged_vs_contiguous(w, inp, P)
    (out, lse, idx, qc), (out_c, lse_c, idx_c, qc_c) = res["paged"], res["contiguous"]
    assert torch.equal(idx, idx_c) and torch.equal(qc, qc_c)
    assert torch.equal(out, out_c) and torch.equal(lse, lse_c)
    N = w.N
    kcodes = oracle.encode(w.hash, inp["K"][:, :, :N], kparams)
    kcodes = kcodes[0] if w.hash == "sign" else kcodes
    np.testing.assert_array_equal(u32(codes), kcodes)
    ref = oracle.decode_step(inp["q"], inp["K"][:, :, :N], inp["V"][:, :, :N], kcodes, N, w.n_sink, w.n_local,
                             w.top_k, w.hash, qparams)
    np.testing.assert_array_equal(u32(qc), ref["q_codes"])
    np.testing.assert_array_equal(idx.numpy(), ref["idx"])
    assert np.abs(out.numpy() - ref["out"]).max() < ATOL
    assert np.abs(lse.numpy() - ref["lse"]).max() < ATOL


@pytest.mark.slow
def test_paged_decode_step_512k():
    """The 512K-token layer of the Qwen2.5-7B-shaped workload in 256-token pages."""
    test_paged_decode_step("qwen7b_512k", dict(layers=1), 256)


def test_paged_decode_step_skips_a_page_outside_the_pool():
    B, Hq, Hkv, N, P, k = 1, 4, 1, 3000, 64, 16
    g = torch.Generator().manual_seed(15)
    K = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16)
    R = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    h = hkv.HashParams.lsh(R.to(DEV))
    codes = torch.zeros(B, Hkv, N, 4, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, K.to(DEV).reshape(-1, 128), codes.view(-1, 4))
    cpool, table = _scatter(codes.cpu(), P, 17)
    kpool, _ = _scatter(K, P, 17)
    vpool, _ = _scatter(V, P, 17)
    table[0, 3] = cpool.shape[0] + 2  # tokens 192..255 point past the pool
    ws = hkv.workspace(B, Hq, Hkv, N, 128, k, 4, 8)
    st = hkv.status_word()
    out = torch.zeros(B, Hq, 128, device=DEV)
    lse = torch.zeros(B, Hq, device=DEV)
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    hkv.hkv_decode_step_paged(h, q.to(DEV), cpool.to(DEV), kpool.to(DEV), vpool.to(DEV), table.to(DEV), N, 4, 8, k,
                              out, lse=lse, idx=idx, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
    got = idx.cpu().numpy()[0, 0]
    assert not np.isin(got, np.arange(192, 256)).any()
    # the attention is over exactly the selected, sink and local rows
    rows = np.concatenate([np.arange(0, 4), got[got >= 0], np.arange(N - 8, N)])
    o, l = oracle.attend(q[0], K[0, 0], V[0, 0], rows, 1.0 / np.sqrt(128))
    assert np.abs(out.cpu().numpy()[0] - o).max() < ATOL
    assert np.abs(lse.cpu().numpy()[0] - l).max() < ATOL
