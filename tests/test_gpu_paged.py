"""Paged cache on the GPU: retrieval and attention read through a page table
must give what the oracle gives on the same tokens read back in order
(index sets and distances exactly; attention within ATOL, and bit for bit
the same as the contiguous-layout call on the gathered copy)."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL, margin_inputs, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _scatter(x, P, seed, spare=3):
    """x [B, Hkv, N, ...] -> (pool [num_pages, Hkv, P, ...], table [B, max_pages]) with the
    pages of all sequences shuffled through the pool and `spare` unused pages."""
    B, Hkv, N = x.shape[:3]
    pages = -(-N // P)
    rng = np.random.default_rng(seed)
    perm = rng.permutation(B * pages + spare)
    table = perm[: B * pages].reshape(B, pages).astype(np.int32)
    pool = torch.zeros((B * pages + spare, Hkv, P) + tuple(x.shape[3:]), dtype=x.dtype)
    for b in range(B):
        for j in range(pages):
            n = min(P, N - j * P)
            pool[int(table[b, j]), :, :n] = x[b, :, j * P:j * P + n]
    return pool, torch.from_numpy(table)


RETRIEVE_CASES = [
    # B, Hq, Hkv, bits, N, page_size, sink, local, top_k
    (2, 8, 2, 128, 5000, 64, 4, 64, 100),
    (1, 28, 4, 128, 20001, 256, 4, 128, 1024),
    (3, 32, 8, 64, 3001, 100, 0, 0, 77),         # page size not a power of two
    (1, 16, 1, 64, 777, 1, 4, 64, 1),            # one token per page
    (2, 4, 2, 128, 300, 16, 8, 8, 400),          # top_k above the candidates
    (2, 4, 2, 128, 50, 16, 40, 30, 8),           # no candidates
    (1, 8, 8, 128, 65536, 512, 0, 0, 512),       # 65536 candidates
]


def _retrieve(qc, pool, table, N, s, l, k):
    B, Hq, W = qc.shape
    Hkv = pool.shape[1]
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    dist = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    st = hkv.status_word()
    hkv.hkv_retrieve_topk_paged(qc.to(DEV), pool.to(DEV), table.to(DEV), N, s, l, k, idx, dist, status=st)
    return idx.cpu().numpy(), dist.cpu().numpy(), hkv.hkv_check(st)


@pytest.mark.parametrize("case", RETRIEVE_CASES)
def test_paged_retrieval(case):
    B, Hq, Hkv, bits, N, P, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(71 + N, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(72 + N, B * Hq, W).view(B, Hq, W)
    pool, table = _scatter(kc, P, 73 + N)
    got_i, got_d, rc = _retrieve(qc, pool, table, N, s, l, k)
    assert rc == hkv.HKV_OK
    gathered = oracle.gather_pages(u32(pool), table.numpy(), P, N)
    want_i, want_d = oracle.retrieve(u32(qc), gathered, N, s, l, k)
    np.testing.assert_array_equal(got_i, want_i)
    np.testing.assert_array_equal(got_d, want_d)


def test_paged_retrieval_ties():
    """Few distinct codes: long runs of equal distances across warps and pages."""
    B, Hq, Hkv, W, N, P = 2, 8, 2, 4, 9000, 32
    codes = synth.random_codes(80, 5, W)
    rng = np.random.default_rng(81)
    kc = codes[torch.from_numpy(rng.integers(0, 5, size=B * Hkv * N))].view(B, Hkv, N, W)
    qc = synth.random_codes(82, B * Hq, W).view(B, Hq, W)
    pool, table = _scatter(kc, P, 83)
    gathered = oracle.gather_pages(u32(pool), table.numpy(), P, N)
    for k in (1, 333, 4000, 8990):
        got_i, got_d, rc = _retrieve(qc, pool, table, N, 4, 4, k)
        assert rc == hkv.HKV_OK
        want_i, want_d = oracle.retrieve(u32(qc), gathered, N, 4, 4, k)
        np.testing.assert_array_equal(got_i, want_i)
        np.testing.assert_array_equal(got_d, want_d)


def test_paged_retrieval_reports_a_page_outside_the_pool():
    B, Hq, Hkv, W, N, P = 1, 4, 1, 4, 1000, 64
    kc = synth.random_codes(90, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(91, B * Hq, W).view(B, Hq, W)
    pool, table = _scatter(kc, P, 92)
    table[0, 3] = pool.shape[0]  # tokens 192..255 point past the pool
    got_i, _, rc = _retrieve(qc, pool, table, N, 0, 0, 10)
    assert rc == hkv.HKV_ERR_DEVICE_RANGE
    assert not np.isin(got_i, np.arange(192, 256)).any()


ATTEND_CASES = [
    # workload overrides, page size
    ("qwen7b_512k", dict(N=9001, layers=1), 256),
    ("hashevict_lsh", dict(B=2, N=5003), 48),
    ("tiny_lsh", dict(), 64),  # fp32
]


@pytest.mark.parametrize("name,over,P", ATTEND_CASES)
def test_paged_decode_composition(name, over, P):
    """Query encode, paged retrieval and paged attention against the oracle's
    decode step on the gathered cache, and bit for bit against the
    contiguous-layout attention on that cache."""
    w = synth.WORKLOADS[name].with_(**over)
    inp = margin_inputs(w, cap=w.N)
    B, Hq, Hkv, N, W, k = w.B, w.Hq, w.Hkv, w.N, w.words, w.top_k
    K, V, q = inp["K"][:, :, :N], inp["V"][:, :, :N], inp["q"]
    h = hkv.HashParams.lsh(inp["R"].to(DEV))
    codes = torch.zeros(B, Hkv, N, W, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, K.to(DEV).reshape(-1, 128), codes.view(-1, W))
    qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, q.to(DEV).reshape(-1, 128), qc.view(-1, W))
    cpool, table = _scatter(codes.cpu(), P, 95)
    kpool, _ = _scatter(K, P, 95)
    vpool, _ = _scatter(V, P, 95)
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    st = hkv.status_word()
    hkv.hkv_retrieve_topk_paged(qc, cpool.to(DEV), table.to(DEV), N, w.n_sink, w.n_local, k, idx, status=st)
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, N, w.bits, k, w.n_sink, w.n_local)
    hkv.hkv_sparse_attend_paged(q.to(DEV), kpool.to(DEV), vpool.to(DEV), table.to(DEV), N, idx, w.n_sink, w.n_local,
                                out, lse, ws=ws, status=st)
    # the same attention on the contiguous copy
    out_c = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse_c = torch.full((B, Hq), float("nan"), device=DEV)
    hkv.hkv_sparse_attend(q.to(DEV), K.to(DEV).contiguous(), V.to(DEV).contiguous(), N, idx, w.n_sink, w.n_local,
                          out_c, lse_c, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_OK
    kcodes = oracle.encode("lsh", K, inp["R"])
    np.testing.assert_array_equal(u32(codes), kcodes)
    ref = oracle.decode_step(inp["q"], inp["K"], inp["V"], kcodes, N, w.n_sink, w.n_local, k, "lsh", inp["R"])
    np.testing.assert_array_equal(u32(qc), ref["q_codes"])
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() < ATOL
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() < ATOL
    assert torch.equal(out, out_c) and torch.equal(lse, lse_c)


def test_paged_attention_skips_a_page_outside_the_pool():
    B, Hq, Hkv, N, P, k = 1, 4, 1, 300, 32, 16
    g = torch.Generator().manual_seed(5)
    K = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, 128, generator=g).to(torch.bfloat16)
    kpool, table = _scatter(K, P, 7)
    vpool, _ = _scatter(V, P, 7)
    idx = torch.arange(100, 100 + k, dtype=torch.int32).view(1, 1, k)  # tokens 100..115: page 3
    table[0, 3] = kpool.shape[0] + 5
    out = torch.zeros(B, Hq, 128, device=DEV)
    lse = torch.zeros(B, Hq, device=DEV)
    st = hkv.status_word()
    ws = hkv.workspace(B, Hq, Hkv, N, 128, k, 4, 8)
    hkv.hkv_sparse_attend_paged(q.to(DEV), kpool.to(DEV), vpool.to(DEV), table.to(DEV), N, idx.to(DEV), 4, 8, out,
                                lse, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
    # what remains is attention over the sink and local rows only
    rows = np.concatenate([np.arange(0, 4), np.arange(N - 8, N)])
    o, l = oracle.attend(q[0], K[0, 0], V[0, 0], rows, 1.0 / np.sqrt(128))
    assert np.abs(out.cpu().numpy()[0] - o).max() < ATOL
    assert np.abs(lse.cpu().numpy()[0] - l).max() < ATOL
