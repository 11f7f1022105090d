"""Norm-weighted sign-VQ retrieval on the GPU against the fp64 oracle
(Self-Indexing KVCache, "Abstract": the sign code with the key's norm is a
1-bit vector quantisation; the score is norm * (g * bits - 2 D), largest
first, ties to the lowest index).  Index sets and scores are compared
exactly: the fp32 score of an fp16 norm times a small integer is exact."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _norms(seed, B, Hkv, cap, pool=None):
    rng = np.random.default_rng(seed)
    if pool is None:
        n = rng.uniform(2.0, 5.0, size=(B, Hkv, cap))
    else:
        n = np.asarray(pool)[rng.integers(0, len(pool), size=(B, Hkv, cap))]
    return n.astype(np.float16)


def _run(qc, kc, norms, N, s, l, k, segmented=False):
    B, Hq, W = qc.shape
    Hkv = kc.shape[1]
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    score = torch.full((B, Hkv, k), 7.0, dtype=torch.float32, device=DEV)
    ws = None
    if segmented:
        ws = hkv.normw_workspace(B, Hkv, N, s, l, k)
        if ws is not None:
            ws.fill_(0x5A)  # the call needs no zero fill: every entry it reads is written first
    hkv.hkv_retrieve_topk_normw(qc.to(DEV), kc.to(DEV), torch.from_numpy(norms).to(DEV), N, s, l, k, idx, score,
                                ws=ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), score.cpu().numpy()


def _check(qc, kc, norms, N, s, l, k, segmented=False):
    got_i, got_s = _run(qc, kc, norms, N, s, l, k, segmented)
    want_i, want_s = oracle.retrieve_normw(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), norms, N, s, l, k)
    np.testing.assert_array_equal(got_i, want_i)
    np.testing.assert_array_equal(got_s, want_s.astype(np.float32))


CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local, top_k
    (2, 8, 2, 128, 5000, 5000, 4, 64, 100),      # g 4, ragged tail, unaligned sink (scalar norm loads)
    (1, 28, 4, 128, 20001, 20008, 8, 128, 1024),  # g 7, aligned window (vector norm loads)
    (3, 32, 8, 64, 3001, 3100, 0, 0, 77),
    (1, 16, 1, 64, 777, 800, 4, 64, 1),           # g 16, top-1
    (2, 4, 2, 128, 300, 304, 8, 8, 400),          # top_k above the candidates
    (2, 4, 2, 128, 50, 64, 40, 30, 8),            # no candidates
    (4, 8, 8, 128, 65536, 65536, 0, 0, 512),      # g 1, 65536 candidates
]


@pytest.mark.parametrize("case", CASES)
def test_normw_parity(case):
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(51 + N, B * Hkv * cap, W).view(B, Hkv, cap, W)
    qc = synth.random_codes(52 + N, B * Hq, W).view(B, Hq, W)
    _check(qc, kc, _norms(53 + N, B, Hkv, cap), N, s, l, k)


@pytest.mark.parametrize("pool", [[1.5], [0.0, 1.0, 2.5], [0.0]])
def test_normw_ties(pool):
    """Few distinct codes and norms: long runs of equal scores spread over
    every warp's range, so the tie quota crosses warps and chunks."""
    B, Hq, Hkv, W, N = 2, 8, 2, 4, 9000
    codes = synth.random_codes(60, 6, W)
    rng = np.random.default_rng(61)
    kc = codes[torch.from_numpy(rng.integers(0, 6, size=B * Hkv * N))].view(B, Hkv, N, W)
    qc = synth.random_codes(62, B * Hq, W).view(B, Hq, W)
    norms = _norms(63, B, Hkv, N, pool)
    for k in (1, 333, 4000, 8990):
        _check(qc, kc, norms, N, 4, 4, k)


def test_normw_signvq_workload():
    """Two KV heads of the sign-VQ workload (groups of 4 query heads, 65536
    tokens, top 512; its other (batch, KV head) pairs are independent pairs
    of the same shape) with the sign codes and fp16 norms of two-cone keys."""
    w = synth.WORKLOADS["signvq"]
    g = w.Hq // w.Hkv
    B, Hq, Hkv, N, k = 1, 2 * g, 2, w.N, w.top_k
    W = w.bits // 32
    seed = synth.layer_seed(w, 0)
    mu_k, mu_q, _ = synth.cone_means(seed, 0, w.d)
    keys = synth.cone_rows(seed, 0, 1, mu_k, B * Hkv * N, "bf16")
    qs = synth.cone_rows(seed, 0, 0, mu_q, B * Hq, "bf16")
    kcodes, norms = oracle.encode("sign", keys)
    qcodes, _ = oracle.encode("sign", qs)
    kc = torch.from_numpy(kcodes.view(np.int32)).view(B, Hkv, N, W)
    qc = torch.from_numpy(qcodes.view(np.int32)).view(B, Hq, W)
    _check(qc, kc, norms.reshape(B, Hkv, N), N, w.n_sink, w.n_local, k)


def test_normw_too_many_candidates():
    qc = torch.zeros(1, 2, 4, dtype=torch.int32, device=DEV)
    kc = torch.zeros(1, 1, 70000, 4, dtype=torch.int32, device=DEV)
    norms = torch.zeros(1, 1, 70000, dtype=torch.float16, device=DEV)
    idx = torch.empty(1, 1, 8, dtype=torch.int32, device=DEV)
    with pytest.raises(hkv.HkvError) as e:
        hkv.hkv_retrieve_topk_normw(qc, kc, norms, 70000, 0, 0, 8, idx)
    assert e.value.code == hkv.HKV_ERR_UNSUPPORTED


SEGMENTED_CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local, top_k
    (1, 8, 2, 128, 200003, 200008, 4, 64, 1024),  # past 65536: many segments per pair, ragged last one
    (2, 4, 2, 64, 70001, 70001, 0, 0, 100),       # 64-bit codes, g 2
    (1, 28, 4, 128, 20001, 20008, 8, 128, 1024),  # few pairs: segments fill the GPU
    (1, 4, 1, 128, 30000, 30000, 0, 0, 5000),     # top_k above a segment: each keeps all of its tokens
    (1, 16, 1, 64, 777, 800, 4, 64, 1),           # one segment: no workspace
    (2, 8, 2, 128, 65536, 65536, 0, 0, 512),      # a full one-block window cut into segments
    # 75..148 pairs: one block per pair even with a workspace
    (16, 32, 8, 128, 65536, 65536, 0, 0, 512),    # the sign-VQ layer shape
    (32, 12, 4, 64, 50001, 50008, 4, 64, 300),    # g 3, 64-bit codes
    (20, 28, 4, 128, 40000, 40000, 4, 128, 1024),  # g 7
]


@pytest.mark.parametrize("case", SEGMENTED_CASES)
def test_normw_segmented_parity(case):
    """With a workspace: segments of at most 65536 candidates, each
    segment's top-k kept, then the top-k of those lists."""
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(81 + N, B * Hkv * cap, W).view(B, Hkv, cap, W)
    qc = synth.random_codes(82 + N, B * Hq, W).view(B, Hq, W)
    _check(qc, kc, _norms(83 + N, B, Hkv, cap), N, s, l, k, segmented=True)


@pytest.mark.parametrize("pool", [[1.5], [0.0, 1.0, 2.5]])
def test_normw_segmented_ties(pool):
    """Equal scores on both sides of every segment boundary: the merge must
    take the tied tokens of earlier segments first."""
    B, Hq, Hkv, W, N = 1, 8, 2, 4, 40000
    codes = synth.random_codes(90, 5, W)
    rng = np.random.default_rng(91)
    kc = codes[torch.from_numpy(rng.integers(0, 5, size=B * Hkv * N))].view(B, Hkv, N, W)
    qc = synth.random_codes(92, B * Hq, W).view(B, Hq, W)
    norms = _norms(93, B, Hkv, N, pool)
    assert hkv.hkv_normw_workspace_bytes(B, Hkv, N, 4, 4, 1) > 0
    for k in (1, 777, 6000, 39990):
        _check(qc, kc, norms, N, 4, 4, k, segmented=True)


def test_normw_segmented_workspace_too_small():
    qc = torch.zeros(1, 2, 4, dtype=torch.int32, device=DEV)
    kc = torch.zeros(1, 1, 70000, 4, dtype=torch.int32, device=DEV)
    norms = torch.zeros(1, 1, 70000, dtype=torch.float16, device=DEV)
    idx = torch.empty(1, 1, 8, dtype=torch.int32, device=DEV)
    need = hkv.hkv_normw_workspace_bytes(1, 1, 70000, 0, 0, 8)
    assert need > 0
    ws = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(hkv.HkvError) as e:
        hkv.hkv_retrieve_topk_normw(qc, kc, norms, 70000, 0, 0, 8, idx, ws=ws)
    assert e.value.code == hkv.HKV_ERR_CAPACITY


@pytest.mark.parametrize("segmented", [False, True])
def test_normw_best_tokens_in_one_warp_range(segmented):
    """Every high score sits in the first 3000 tokens: the tokens at or
    above the threshold bin crowd one warp's share of the block, so the
    select falls back from its per-warp lists to full passes."""
    B, Hq, Hkv, W, N, k = 2, 8, 2, 4, 65536, 1000
    kc = synth.random_codes(95, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(96, B * Hq, W).view(B, Hq, W)
    norms = _norms(97, B, Hkv, N)
    norms[:, :, 3000:] = (norms[:, :, 3000:] / 8).astype(np.float16)
    _check(qc, kc, norms, N, 0, 0, k, segmented)


@pytest.mark.slow
def test_normw_segmented_512k():
    """One 524288-token layer of the Qwen2.5-7B-shaped cache (28 query and
    4 KV heads, top 1024) scored norm-weighted through the workspace path."""
    B, Hq, Hkv, W, N, s, l, k = 1, 28, 4, 4, 524288, 4, 128, 1024
    kc = synth.random_codes(98, B * Hkv * N, W).view(B, Hkv, N, W)
    qc = synth.random_codes(99, B * Hq, W).view(B, Hq, W)
    _check(qc, kc, _norms(100, B, Hkv, N), N, s, l, k, segmented=True)


# --------------------------------------------------- norm-weighted decode step

def _sign_inputs(seed, B, Hq, Hkv, cap, dtype):
    g = torch.Generator().manual_seed(seed)
    def draw(*shape):
        x = torch.randn(*shape, generator=g)
        x = torch.where(x.abs() < 1e-2, torch.full_like(x, 0.5), x)  # no value at or near zero
        return x.to(torch.bfloat16) if dtype == "bf16" else x
    return draw(B, Hq, 128), draw(B, Hkv, cap, 128), draw(B, Hkv, cap, 128)


def _check_decode_normw(B, Hq, Hkv, N, cap, s, l, k, dtype="bf16", workspace=False):
    q, K, V = _sign_inputs(1000 + N + k, B, Hq, Hkv, cap, dtype)
    kc, norms = oracle.encode("sign", K)
    qc, _ = oracle.encode("sign", q)
    kcodes = torch.from_numpy(kc.view(np.int32)).view(B, Hkv, cap, 4)
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device=DEV)
    score = torch.full((B, Hkv, k), 7.0, device=DEV)
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    q_codes = torch.zeros(B, Hq, 4, dtype=torch.int32, device=DEV)
    ws = hkv.normw_decode_workspace(B, Hq, Hkv, N, 128, k, s, l) if workspace else None
    st = hkv.status_word()
    hkv.hkv_decode_step_normw(q.to(DEV), kcodes.to(DEV), torch.from_numpy(norms.reshape(B, Hkv, cap)).to(DEV),
                              K.to(DEV), V.to(DEV), N, s, l, k, idx, out, lse=lse, score=score, q_codes=q_codes,
                              ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    np.testing.assert_array_equal(q_codes.cpu().numpy().view(np.uint32), qc.reshape(B, Hq, 4))
    want_i, want_s = oracle.retrieve_normw(qc.reshape(B, Hq, 4), kc.reshape(B, Hkv, cap, 4), norms.reshape(B, Hkv, cap),
                                           N, s, l, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_i)
    np.testing.assert_array_equal(score.cpu().numpy(), want_s.astype(np.float32))
    g = Hq // Hkv
    o, ls = out.cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for j in range(Hkv):
            rows = oracle.attention_rows(N, s, l, want_i[b, j])
            wo, wl = oracle.attend(q[b, j * g:(j + 1) * g], K[b, j], V[b, j], rows, 1.0 / np.sqrt(128))
            assert np.abs(o[b, j * g:(j + 1) * g] - wo).max() < ATOL
            assert np.abs(ls[b, j * g:(j + 1) * g] - wl).max() < ATOL


DECODE_CASES = [
    # B, Hq, Hkv, N, cap, sink, local, top_k
    (2, 8, 2, 5000, 5000, 4, 64, 100),        # one launch, g 4, unaligned sink (scalar norm loads)
    (1, 28, 4, 20001, 20008, 8, 128, 1024),   # g 7, aligned window
    (1, 16, 1, 777, 800, 4, 64, 1),           # g 16, top-1
    (2, 4, 2, 300, 304, 8, 8, 400),           # top_k above the candidates
    (2, 4, 2, 50, 64, 40, 30, 8),             # no candidates: the sink and local rows only
]


@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_step_normw_one_launch(case):
    _check_decode_normw(*case)


@pytest.mark.parametrize("case,dtype", [
    ((1, 8, 2, 70001, 70001, 4, 64, 300), "bf16"),   # past 65536: segmented retrieval, then the attention
    ((1, 28, 4, 20001, 20008, 8, 128, 1024), "bf16"),  # few pairs with a workspace: segments
    ((2, 8, 2, 5000, 5000, 4, 64, 100), "f32"),       # fp32: query encode + retrieval + SIMT attention
])
def test_decode_step_normw_multi_launch(case, dtype):
    _check_decode_normw(*case, dtype=dtype, workspace=True)


def test_decode_step_normw_signvq_workload():
    """Two KV heads of the sign-VQ workload's shape (65536 tokens, top 512,
    groups of 4) through the one-launch step."""
    _check_decode_normw(1, 8, 2, 65536, 65536, 0, 0, 512)
