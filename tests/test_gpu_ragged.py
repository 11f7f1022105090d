"""Ragged batches (sequences of different lengths in one decode step) on the
GPU against the fp64 oracle: indices exact, outputs within 2e-3."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL, margin_inputs, oracle_params, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _hash(w, inp, side):
    code = hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32
    if w.hash == "lsh":
        return hkv.HashParams.lsh(inp["R"].to(DEV))
    if w.hash == "mlp":
        return hkv.HashParams.mlp(*(t.to(DEV) for t in inp[side + "_mlp"]), dtype=code)
    return hkv.HashParams.sign(code)


CASES = {
    # name, overrides, lengths (the first is the longest)
    "qwen": ("qwen7b_512k", dict(B=3, N=9001, layers=1), [9001, 4097, 132]),      # last: no candidates
    "hashevict": ("hashevict_lsh", dict(B=4, N=5003), [5003, 5002, 1000, 69]),   # last: one candidate
    "signvq": ("signvq", dict(B=3, N=5001), [3000, 5001, 1]),
    "spotlight": ("spotlight_mlp", dict(B=2, N=6007), [6007, 2500]),
}


@pytest.mark.parametrize("case", list(CASES))
def test_decode_step_ragged(case):
    name, over, lens = CASES[case]
    w = synth.WORKLOADS[name].with_(**over)
    inp = margin_inputs(w, cap=w.N + 3)
    B, Hq, Hkv, N, W = w.B, w.Hq, w.Hkv, w.N, w.words
    nmax = max(lens)
    K, V, q = inp["K"].to(DEV), inp["V"].to(DEV), inp["q"].to(DEV)
    kh, qh = _hash(w, inp, "k"), _hash(w, inp, "q")
    codes = torch.full((B, Hkv, N + 3, W), -1, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(kh, K.view(-1, 128), codes.view(-1, W))
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    idx = torch.full((B, Hkv, w.top_k), -9, dtype=torch.int32, device=DEV)
    qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
    nb = torch.tensor(lens, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, nmax, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()
    for _ in range(2):
        hkv.hkv_decode_step_ragged(qh, q, codes, K, V, nb, nmax, w.n_sink, w.n_local, w.top_k, out, lse, q_codes=qc,
                                   idx=idx, ws=ws, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    kcodes = oracle.encode(w.hash, inp["K"], oracle_params(w, inp, "k"))
    if w.hash == "sign":
        kcodes = kcodes[0]
    ref = oracle.decode_step_ragged(inp["q"], inp["K"], inp["V"], kcodes, lens, w.n_sink, w.n_local, w.top_k, w.hash,
                                    oracle_params(w, inp, "q"))
    np.testing.assert_array_equal(u32(qc), ref["q_codes"])
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    assert np.abs(out.cpu().numpy() - ref["out"]).max() < ATOL
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() < ATOL


def test_ragged_length_out_of_range_is_reported():
    w = synth.WORKLOADS["qwen7b_512k"].with_(B=2, N=3001, layers=1)
    B, Hq, Hkv, W = w.B, w.Hq, w.Hkv, w.words
    K = torch.zeros(B, Hkv, 3001, 128, dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros(B, Hkv, 3001, W, dtype=torch.int32, device=DEV)
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros(B, Hq, 128, device=DEV)
    qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
    nb = torch.tensor([3001, 5000], dtype=torch.int32, device=DEV)  # 5000 > n_tokens_max
    ws = hkv.workspace(B, Hq, Hkv, 3001, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()
    hkv.hkv_decode_step_ragged(hkv.HashParams.given(hkv.HKV_BF16, 128), q, codes, K, K, nb, 3001, w.n_sink,
                               w.n_local, w.top_k, out, q_codes=qc, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
