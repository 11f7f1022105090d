"""HashEvict eviction on the GPU against the fp64 oracle (HashEvict,
"Abstract": at every decoding step the new token replaces the cached token
whose code is farthest from the query's).  Victims and their distances are
compared exactly; a three-step eviction loop compares the whole cache."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import margin_inputs, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local
    (2, 8, 2, 128, 5000, 5004, 4, 64),
    (1, 28, 4, 128, 70001, 70001, 4, 128),
    (3, 32, 8, 64, 3001, 3100, 0, 0),
    (1, 16, 1, 64, 777, 800, 4, 64),
    (2, 4, 2, 128, 50, 64, 40, 30),   # sink + local cover everything: no victim
    (64, 64, 8, 128, 300, 300, 4, 16),
]


def _evict(qc, kc, N, s, l):
    B, Hq, W = qc.shape
    Hkv = kc.shape[1]
    victim = torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV)
    vdist = torch.full((B, Hkv), -9, dtype=torch.int32, device=DEV)
    ws = torch.zeros(8 * B * Hkv, dtype=torch.uint8, device=DEV)
    for _ in range(2):  # twice: the workspace must come back to zero
        hkv.hkv_evict_select(qc.to(DEV), kc.to(DEV), N, s, l, victim, vdist, ws=ws)
    torch.cuda.synchronize()
    assert int(ws.sum()) == 0
    return victim.cpu().numpy(), vdist.cpu().numpy()


@pytest.mark.parametrize("case", CASES)
def test_evict_select(case):
    B, Hq, Hkv, bits, N, cap, s, l = case
    W = bits // 32
    kc = synth.random_codes(41 + N, B * Hkv * cap, W).view(B, Hkv, cap, W)
    qc = synth.random_codes(42 + N, B * Hq, W).view(B, Hq, W)
    v, d = _evict(qc, kc, N, s, l)
    wv, wd = oracle.evict_victim(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, s, l)
    np.testing.assert_array_equal(v, wv)
    np.testing.assert_array_equal(d, wd)


def test_evict_select_ties_across_blocks():
    """Keys from three codes: the largest distance is shared by a third of the
    tokens, spread over many blocks; the lowest index must win."""
    B, Hq, Hkv, N = 1, 8, 2, 200003
    base = synth.random_codes(15, 3, 4).numpy()
    pick = np.random.default_rng(16).integers(0, 3, B * Hkv * N)
    kc = torch.from_numpy(base[pick].copy()).view(B, Hkv, N, 4)
    qc = synth.random_codes(17, B * Hq, 4).view(B, Hq, 4)
    v, d = _evict(qc, kc, N, 4, 64)
    wv, wd = oracle.evict_victim(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, 4, 64)
    np.testing.assert_array_equal(v, wv)
    np.testing.assert_array_equal(d, wd)


def test_write_slots():
    B, Hkv, cap, W = 3, 2, 40, 4
    g = torch.Generator().manual_seed(3)
    K = torch.randn(B, Hkv, cap, 128, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, cap, 128, generator=g).to(torch.bfloat16)
    codes = torch.randint(-2**31, 2**31 - 1, (B, Hkv, cap, W), generator=g, dtype=torch.int32)
    kn = torch.randn(B, Hkv, 128, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, 128, generator=g).to(torch.bfloat16)
    cn = torch.randint(-2**31, 2**31 - 1, (B, Hkv, W), generator=g, dtype=torch.int32)
    slot = torch.tensor([[5, -1], [39, 0], [17, 17]], dtype=torch.int32)
    Kg, Vg, cg = K.to(DEV), V.to(DEV), codes.to(DEV)
    st = hkv.status_word()
    hkv.hkv_write_slots(kn.to(DEV), vn.to(DEV), cn.to(DEV), Kg, Vg, cg, slot.to(DEV), status=st)
    assert hkv.hkv_check(st) == hkv.HKV_OK
    for b in range(B):
        for j in range(Hkv):
            t = int(slot[b, j])
            if t >= 0:
                K[b, j, t], V[b, j, t], codes[b, j, t] = kn[b, j], vn[b, j], cn[b, j]
    assert torch.equal(Kg.cpu(), K) and torch.equal(Vg.cpu(), V) and torch.equal(cg.cpu(), codes)


def test_write_slots_out_of_range_is_reported():
    B, Hkv, cap = 1, 1, 8
    K = torch.zeros(B, Hkv, cap, 128, dtype=torch.bfloat16, device=DEV)
    V = torch.zeros_like(K)
    codes = torch.zeros(B, Hkv, cap, 4, dtype=torch.int32, device=DEV)
    kn = torch.ones(B, Hkv, 128, dtype=torch.bfloat16, device=DEV)
    cn = torch.ones(B, Hkv, 4, dtype=torch.int32, device=DEV)
    st = hkv.status_word()
    hkv.hkv_write_slots(kn, kn, cn, K, V, codes, torch.tensor([[8]], dtype=torch.int32, device=DEV), status=st)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
    assert int(K.abs().sum()) == 0 and int(codes.abs().sum()) == 0


def test_hashevict_decode_loop():
    """Three decode steps of a full cache: attend, pick the victim from the
    step's query codes, encode the new key and write it over the victim.  The
    cache after each step equals the oracle's."""
    w = synth.WORKLOADS["hashevict_lsh"].with_(B=2, N=3001)
    inp = margin_inputs(w, cap=w.N)
    R = inp["R"]
    K, V = inp["K"].clone(), inp["V"].clone()
    h = hkv.HashParams.lsh(R.to(DEV))
    W = w.words
    Kg, Vg = K.to(DEV), V.to(DEV)
    codes = torch.zeros(w.B, w.Hkv, w.N, W, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, Kg.view(-1, 128), codes.view(-1, W))
    ref_codes = oracle.encode("lsh", K, R)
    ws = hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()
    for step in range(3):
        q = torch.roll(inp["q"], shifts=step, dims=1).contiguous()  # other query rows, still inside the margin
        kn = K[:, :, step + 10].clone()  # new keys: copies of cached keys (inside the margin)
        vn = V[:, :, step + 20].clone()
        out = torch.zeros(w.B, w.Hq, 128, device=DEV)
        qc = torch.zeros(w.B, w.Hq, W, dtype=torch.int32, device=DEV)
        hkv.hkv_decode_step(h, q.to(DEV), codes, Kg, Vg, w.N, w.n_sink, w.n_local, w.top_k, out, q_codes=qc, ws=ws,
                            status=st)
        victim = torch.zeros(w.B, w.Hkv, dtype=torch.int32, device=DEV)
        hkv.hkv_evict_select(qc, codes, w.N, w.n_sink, w.n_local, victim, ws=ws)
        cn = torch.zeros(w.B, w.Hkv, W, dtype=torch.int32, device=DEV)
        hkv.hkv_encode_keys(h, kn.to(DEV).view(-1, 128), cn.view(-1, W))
        hkv.hkv_write_slots(kn.to(DEV), vn.to(DEV), cn, Kg, Vg, codes, victim, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_OK
        qcodes_ref = oracle.encode("lsh", q, R)
        np.testing.assert_array_equal(u32(qc), qcodes_ref)
        wv, _ = oracle.evict_victim(qcodes_ref, ref_codes, w.N, w.n_sink, w.n_local)
        np.testing.assert_array_equal(victim.cpu().numpy(), wv)
        new_codes = oracle.encode("lsh", kn, R)
        for b in range(w.B):
            for j in range(w.Hkv):
                t = int(wv[b, j])
                K[b, j, t], V[b, j, t] = kn[b, j], vn[b, j]
                ref_codes[b, j, t] = new_codes[b, j]
        np.testing.assert_array_equal(u32(codes), ref_codes)
        assert torch.equal(Kg.cpu(), K) and torch.equal(Vg.cpu(), V)
