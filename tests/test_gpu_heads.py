"""One index set per query head (RetrievalAttention, "Key points") on the GPU
against the fp64 oracle: indices and distances exact, outputs within 2e-3."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL, margin_inputs, oracle_params, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local, top_k
    (1, 28, 4, 128, 20011, 20011, 4, 128, 1024),
    (2, 8, 2, 64, 5000, 5004, 4, 64, 300),
    (3, 32, 8, 128, 3001, 3100, 0, 0, 512),
    (2, 12, 4, 128, 900, 900, 4, 64, 5000),   # top_k > candidates
    (2, 4, 2, 128, 50, 64, 40, 30, 8),        # no candidates
]


@pytest.mark.parametrize("case", CASES)
def test_retrieve_topk_heads(case):
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(51 + N, B * Hkv * cap, W).view(B, Hkv, cap, W)
    qc = synth.random_codes(52 + N, B * Hq, W).view(B, Hq, W)
    idx = torch.full((B, Hq, k), -9, dtype=torch.int32, device=DEV)
    dist = torch.full((B, Hq, k), -9, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hq, N, bits, k, s, l)
    st = hkv.status_word()
    for _ in range(2):
        hkv.hkv_retrieve_topk_heads(qc.to(DEV), kc.to(DEV), N, s, l, k, idx, dist, ws=ws, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    wi, wd = oracle.retrieve_heads(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, s, l, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), wi)
    np.testing.assert_array_equal(dist.cpu().numpy(), wd)


SMALL = {
    "hashevict_lsh": dict(B=2, N=5003),
    "spotlight_mlp": dict(N=6007),
    "signvq": dict(B=2, N=5001),
    "qwen7b_512k": dict(N=9001, layers=1),
    "tiny_lsh": dict(),
}


def _hash(w, inp, side):
    code = hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32
    if w.hash == "lsh":
        return hkv.HashParams.lsh(inp["R"].to(DEV))
    if w.hash == "mlp":
        return hkv.HashParams.mlp(*(t.to(DEV) for t in inp[side + "_mlp"]), dtype=code)
    return hkv.HashParams.sign(code)


@pytest.mark.parametrize("name", list(SMALL))
def test_decode_step_heads(name):
    w = synth.WORKLOADS[name].with_(**SMALL[name])
    inp = margin_inputs(w, cap=w.N + 5)
    B, Hq, Hkv, N, W = w.B, w.Hq, w.Hkv, w.N, w.words
    K, V, q = inp["K"].to(DEV), inp["V"].to(DEV), inp["q"].to(DEV)
    kh, qh = _hash(w, inp, "k"), _hash(w, inp, "q")
    codes = torch.full((B, Hkv, N + 5, W), -1, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(kh, K.view(-1, 128), codes.view(-1, W))
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    idx = torch.full((B, Hq, w.top_k), -9, dtype=torch.int32, device=DEV)
    qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hq, N, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()
    hkv.hkv_decode_step_heads(qh, q, codes, K, V, N, w.n_sink, w.n_local, w.top_k, out, lse, q_codes=qc, idx=idx,
                              ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    kcodes = oracle.encode(w.hash, inp["K"][:, :, :N], oracle_params(w, inp, "k"))
    if w.hash == "sign":
        kcodes = kcodes[0]
    np.testing.assert_array_equal(u32(codes)[:, :, :N], kcodes)
    ref = oracle.decode_step_heads(inp["q"], inp["K"], inp["V"], kcodes, N, w.n_sink, w.n_local, w.top_k, w.hash,
                                   oracle_params(w, inp, "q"))
    np.testing.assert_array_equal(u32(qc), ref["q_codes"])
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() < ATOL
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() < ATOL
