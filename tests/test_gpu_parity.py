"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Codes, distances and selected index sets must match bit for bit; attention
outputs within ATOL (max abs) of the oracle.  Inputs are seeded and synthetic,
with every pre-sign value at least MARGIN from zero."""
import math

import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import ATOL, hash_params, margin_inputs, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dt(dtype: str):
    return (torch.bfloat16, hkv.HKV_BF16) if dtype == "bf16" else (torch.float32, hkv.HKV_F32)


def _rows(seed, n, d, dtype, bad=None, tensor=2):
    mu = synth.cone_means(seed, 0, d)[0]
    return synth.cone_rows(seed, 0, tensor, mu, n, dtype, bad)


def _gpu_hash(w, inp, side):
    tdt, code = _dt(w.dtype)
    if w.hash == "lsh":
        return hkv.HashParams.lsh(inp["R"].to(DEV))
    if w.hash == "mlp":
        return hkv.HashParams.mlp(*(t.to(DEV) for t in inp[side + "_mlp"]), dtype=code)
    return hkv.HashParams.sign(code)


def _oracle_params(w, inp, side):
    if w.hash == "lsh":
        return inp["R"]
    if w.hash == "mlp":
        return inp[side + "_mlp"]
    return None


def _check(status):
    assert hkv.hkv_check(status) == hkv.HKV_OK, hkv.hkv_last_error()


# ------------------------------------------------------------------ encoders

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bits", [64, 128])
def test_encode_lsh(dtype, bits):
    tdt, code = _dt(dtype)
    R = synth.gaussian_projection(21, 0, bits, 128, dtype)
    from tests.helpers import lsh_bad
    x = _rows(21, 1037, 128, dtype, lsh_bad(R))
    wide = torch.zeros(1037, 192, dtype=tdt)
    wide[:, :128] = x
    xg = wide.to(DEV)[:, :128]  # row stride 192
    codes = torch.full((1037, bits // 32 + 3), -7, dtype=torch.int32, device=DEV)
    h = hkv.HashParams.lsh(R.to(DEV))
    hkv.hkv_encode_keys(h, xg, codes)
    torch.cuda.synchronize()
    want = oracle.encode("lsh", x, R)
    np.testing.assert_array_equal(u32(codes[:, : bits // 32]), want)
    assert (codes[:, bits // 32:] == -7).all()


@pytest.mark.parametrize("bits,rows,x_pitch,code_pitch", [
    (128, 70001, 192, 8),    # tensor-core path, ragged last tile, padded rows and codes
    (128, 4096, 128, 4),     # tensor-core path, whole tiles only
    (64, 4097, 136, 2),      # tensor-core path, 64-bit codes
    (128, 5000, 128, 7),     # code pitch not a multiple of the code width: SIMT path
])
def test_encode_lsh_large_batches(bits, rows, x_pitch, code_pitch):
    """Large bf16 batches (the prefill of a cache) against the fp64 oracle, bit-exact."""
    R = synth.gaussian_projection(24, 1, bits, 128, "bf16")
    from tests.helpers import lsh_bad
    x = _rows(24, rows, 128, "bf16", lsh_bad(R))
    wide = torch.zeros(rows, x_pitch, dtype=torch.bfloat16)
    wide[:, :128] = x
    xg = wide.to(DEV)[:, :128]
    W = bits // 32
    codes = torch.full((rows, code_pitch), -7, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    h = hkv.HashParams.lsh(R.to(DEV))
    for _ in range(2):
        hkv.hkv_encode_keys(h, xg, codes[:, :W], status=status)
    assert hkv.hkv_check(status) == hkv.HKV_OK
    np.testing.assert_array_equal(u32(codes[:, :W]), oracle.encode("lsh", x, R))
    assert (codes[:, W:] == -7).all()


@pytest.mark.parametrize("bits,hidden,rows,x_pitch,code_pitch", [
    (128, 512, 40000, 128, 4),   # tensor-core path; 313 tiles, so some CTAs run three
    (64, 200, 4097, 136, 2),     # hidden width padded to 256 inside the packed weights
])
def test_encode_mlp_large_batches(bits, hidden, rows, x_pitch, code_pitch):
    """Large bf16 batches through the packed-weight tensor-core MLP encoder,
    bit-exact against the fp64 oracle; the unpacked hash gives the same codes."""
    params = synth.mlp_params(25, 0, "k", 128, hidden, bits)
    from tests.helpers import mlp_bad
    x = _rows(25, rows, 128, "bf16", mlp_bad(params))
    wide = torch.zeros(rows, x_pitch, dtype=torch.bfloat16)
    wide[:, :128] = x
    xg = wide.to(DEV)[:, :128]
    W = bits // 32
    want = oracle.encode("mlp", x, params)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for pack in (True, False):
        h = hkv.HashParams.mlp(*(t.to(DEV) for t in params), dtype=hkv.HKV_BF16, pack=pack)
        codes = torch.full((rows, code_pitch), -7, dtype=torch.int32, device=DEV)
        for _ in range(2):
            hkv.hkv_encode_keys(h, xg, codes[:, :W], status=status)
        assert hkv.hkv_check(status) == hkv.HKV_OK
        np.testing.assert_array_equal(u32(codes[:, :W]), want)
        assert (codes[:, W:] == -7).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("bits,hidden", [(128, 512), (64, 200)])
def test_encode_mlp(dtype, bits, hidden):
    tdt, code = _dt(dtype)
    params = synth.mlp_params(22, 0, "k", 128, hidden, bits)
    from tests.helpers import mlp_bad
    x = _rows(22, 301, 128, dtype, mlp_bad(params))
    codes = torch.zeros(301, bits // 32, dtype=torch.int32, device=DEV)
    h = hkv.HashParams.mlp(*(t.to(DEV) for t in params), dtype=code)
    hkv.hkv_encode_keys(h, x.to(DEV), codes)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(u32(codes), oracle.encode("mlp", x, params))


@pytest.mark.parametrize("dtype,rows,code_pitch", [("f32", 2049, 4), ("bf16", 2049, 4), ("bf16", 70001, 4),
                                                   ("bf16", 3001, 5)])
def test_encode_sign_and_norms(dtype, rows, code_pitch):
    """Sign codes and fp16 norms, bit-exact; a code pitch of 5 words takes
    the scalar-store path."""
    tdt, code = _dt(dtype)
    from tests.helpers import sign_bad
    x = _rows(23, rows, 128, dtype, sign_bad())
    codes = torch.full((rows, code_pitch), -7, dtype=torch.int32, device=DEV)
    norms = torch.zeros(rows, dtype=torch.float16, device=DEV)
    hkv.hkv_encode_keys(hkv.HashParams.sign(code), x.to(DEV), codes[:, :4], norms)
    torch.cuda.synchronize()
    wc, wn = oracle.encode("sign", x)
    np.testing.assert_array_equal(u32(codes[:, :4]), wc)
    assert (codes[:, 4:] == -7).all()
    np.testing.assert_array_equal(norms.cpu().numpy().view(np.uint16), wn.view(np.uint16))


# ----------------------------------------------------------------- retrieval

RETRIEVE_CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local, top_k
    (1, 1, 1, 128, 4096, 4096, 0, 0, 64),
    (2, 8, 2, 64, 5000, 5004, 4, 64, 300),
    (1, 28, 4, 128, 20011, 20011, 4, 128, 1024),
    (3, 32, 8, 128, 3001, 3100, 0, 0, 512),
    (1, 16, 1, 64, 777, 800, 4, 64, 100),
    (2, 12, 4, 128, 900, 900, 4, 64, 5000),   # top_k > candidates
    (2, 4, 2, 128, 50, 64, 40, 30, 8),        # sink + local cover everything
    (1, 4, 4, 128, 0, 16, 4, 64, 8),          # empty sequence
    (64, 64, 8, 128, 300, 300, 4, 16, 32),    # blocks span several (batch, head) pairs
    (1, 3, 1, 128, 70001, 70001, 0, 0, 7000),  # group of 3 (two bit planes)
]


def _retrieve(q_codes, k_codes, N, s, l, k):
    B, Hq, W = q_codes.shape
    Hkv = k_codes.shape[1]
    qg, kg = q_codes.to(DEV), k_codes.to(DEV)
    idx = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
    dist = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, N, W * 32, k, s, l)
    st = hkv.status_word()
    for _ in range(2):  # the second call relies on the first leaving its counters at zero
        idx.fill_(-9)
        dist.fill_(-9)
        hkv.hkv_retrieve_topk(qg, kg, N, s, l, k, idx, dist, ws=ws, status=st)
        _check(st)
    return idx.cpu().numpy(), dist.cpu().numpy(), (qg, kg, idx, dist, ws, st)


@pytest.mark.parametrize("case", RETRIEVE_CASES)
def test_retrieve_topk(case):
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(31 + N, B * Hkv * cap, W).view(B, Hkv, cap, W)
    qc = synth.random_codes(32 + N, B * Hq, W).view(B, Hq, W)
    idx, dist, _ = _retrieve(qc, kc, N, s, l, k)
    wi, wd = oracle.retrieve(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, s, l, k)
    np.testing.assert_array_equal(idx, wi)
    np.testing.assert_array_equal(dist, wd)


def test_retrieve_heavy_ties_across_blocks():
    """Keys drawn from three codes: the threshold bin holds tens of thousands
    of tokens spread over many blocks; ties must go to the lowest indices."""
    B, Hq, Hkv, N, k = 1, 8, 2, 200003, 40000
    base = synth.random_codes(5, 3, 4).numpy()
    pick = np.random.default_rng(7).integers(0, 3, B * Hkv * N)
    kc = torch.from_numpy(base[pick].copy()).view(B, Hkv, N, 4)
    qc = synth.random_codes(6, B * Hq, 4).view(B, Hq, 4)
    for _ in range(2):  # twice: the second call checks the workspace was left clean
        idx, dist, _ = _retrieve(qc, kc, N, 4, 64, k)
        wi, wd = oracle.retrieve(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, 4, 64, k)
        np.testing.assert_array_equal(idx, wi)
        np.testing.assert_array_equal(dist, wd)


def test_retrieve_one_block_per_pair_over_32k_candidates():
    """148 (batch, KV head) pairs of 40001 tokens: one block per pair holds all
    of its distances (more than 32768) in shared memory.  Keys from three
    codes put tens of thousands of ties on both sides of the threshold."""
    B, Hq, Hkv, N, k = 37, 8, 4, 40001, 30000
    base = synth.random_codes(12, 3, 2).numpy()
    pick = np.random.default_rng(13).integers(0, 3, B * Hkv * N)
    kc = torch.from_numpy(base[pick].copy()).view(B, Hkv, N, 2)
    qc = synth.random_codes(14, B * Hq, 2).view(B, Hq, 2)
    for _ in range(2):
        idx, dist, _ = _retrieve(qc, kc, N, 4, 64, k)
        wi, wd = oracle.retrieve(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, 4, 64, k)
        np.testing.assert_array_equal(idx, wi)
        np.testing.assert_array_equal(dist, wd)


def test_retrieve_in_pair_batches():
    """More candidates than one launch keeps in shared memory: several launches."""
    B, Hq, Hkv, N, k = 16, 32, 8, 100000, 512
    kc = synth.random_codes(8, B * Hkv * N, 4).view(B, Hkv, N, 4)
    qc = synth.random_codes(9, B * Hq, 4).view(B, Hq, 4)
    idx, dist, _ = _retrieve(qc, kc, N, 0, 0, k)
    wi, wd = oracle.retrieve(qc.numpy().view(np.uint32), kc.numpy().view(np.uint32), N, 0, 0, k)
    np.testing.assert_array_equal(idx, wi)
    np.testing.assert_array_equal(dist, wd)


def test_retrieve_wait_times_out_and_recovers():
    """One block withholds its arrival: the bounded wait expires, the status
    word reports HKV_ERR_TIMEOUT, the context stays usable and the workspace
    is clean for the next call."""
    B, Hq, Hkv, N, k = 1, 28, 4, 300000, 1024
    kc = synth.random_codes(10, B * Hkv * N, 4).view(B, Hkv, N, 4).to(DEV)
    qc = synth.random_codes(11, B * Hq, 4).view(B, Hq, 4).to(DEV)
    idx = torch.zeros(B, Hkv, k, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, N, 128, k, 4, 128)
    st = hkv.status_word()
    hkv.hkv_debug_set(1, 20_000_000)
    try:
        hkv.hkv_retrieve_topk(qc, kc, N, 4, 128, k, idx, ws=ws, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_ERR_TIMEOUT
    finally:
        hkv.hkv_debug_set(0, 0)
    hkv.hkv_retrieve_topk(qc, kc, N, 4, 128, k, idx, ws=ws, status=st)
    _check(st)
    wi, _ = oracle.retrieve(u32(qc), u32(kc), N, 4, 128, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), wi)


# ----------------------------------------------------------------- attention

ATTEND_CASES = [
    # dtype, B, Hq, Hkv, N, cap, sink, local, top_k
    ("f32", 1, 1, 1, 4096, 4096, 0, 0, 64),
    ("bf16", 2, 32, 8, 3000, 3010, 4, 64, 1024),
    ("bf16", 1, 28, 4, 9000, 9000, 4, 128, 1024),
    ("bf16", 2, 32, 8, 6000, 6000, 0, 0, 512),
    ("bf16", 1, 16, 1, 500, 512, 4, 64, 2000),
    ("bf16", 20, 32, 8, 2000, 2000, 4, 64, 300),   # more pairs than SMs: one block per pair, several waves
    ("bf16", 20, 8, 8, 6000, 6000, 4, 64, 5000),   # rows past the block's shared token list
]


def _random_selection(rng, N, s, l, k):
    lo, hi = oracle.candidate_range(N, s, l)
    C = hi - lo
    take = min(k, C)
    sel = np.sort(rng.choice(np.arange(lo, hi), size=take, replace=False)) if take else np.zeros(0, np.int64)
    out = np.full(k, -1, dtype=np.int64)
    out[:take] = sel
    return out


@pytest.mark.parametrize("case", ATTEND_CASES)
def test_sparse_attend(case):
    dtype, B, Hq, Hkv, N, cap, s, l, k = case
    tdt, code = _dt(dtype)
    w = synth.WORKLOADS["hashevict_lsh"].with_(B=B, Hq=Hq, Hkv=Hkv, N=N, dtype=dtype)
    inp = synth.layer_inputs(w, cap=cap)
    rng = np.random.default_rng(N)
    idx = np.stack([[_random_selection(rng, N, s, l, k) for _ in range(Hkv)] for _ in range(B)])
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, N, 128, k, s, l)
    st = hkv.status_word()
    hkv.hkv_sparse_attend(inp["q"].to(DEV), inp["K"].to(DEV), inp["V"].to(DEV), N,
                          torch.from_numpy(idx.astype(np.int32)).to(DEV), s, l, out, lse, ws=ws, status=st)
    _check(st)
    g = Hq // Hkv
    o = out.cpu().numpy()
    ls = lse.cpu().numpy()
    for b in range(B):
        for kh in range(Hkv):
            rows = oracle.attention_rows(N, s, l, idx[b, kh])
            wo, wl = oracle.attend(inp["q"][b, kh * g:(kh + 1) * g], inp["K"][b, kh], inp["V"][b, kh], rows,
                                   1 / math.sqrt(128))
            assert np.abs(o[b, kh * g:(kh + 1) * g] - wo).max() < ATOL
            assert np.abs(ls[b, kh * g:(kh + 1) * g] - wl).max() < ATOL


def test_sparse_attend_empty_and_out_of_range():
    w = synth.WORKLOADS["hashevict_lsh"].with_(B=1, Hq=4, Hkv=2, N=100)
    inp = synth.layer_inputs(w)
    q, K, V = inp["q"].to(DEV), inp["K"].to(DEV), inp["V"].to(DEV)
    out = torch.zeros(1, 4, 128, device=DEV)
    lse = torch.zeros(1, 4, device=DEV)
    ws = hkv.workspace(1, 4, 2, 100, 128, 8, 0, 0)
    st = hkv.status_word()
    idx = torch.full((1, 2, 8), -1, dtype=torch.int32, device=DEV)
    hkv.hkv_sparse_attend(q, K, V, 100, idx, 0, 0, out, lse, ws=ws, status=st)
    _check(st)
    assert (out == 0).all() and torch.isneginf(lse).all()
    idx[0, 0, 0] = 7
    idx[0, 0, 1] = 100  # out of range: skipped and reported
    hkv.hkv_sparse_attend(q, K, V, 100, idx, 0, 0, out, lse, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_ERR_DEVICE_RANGE
    wo, _ = oracle.attend(inp["q"][0, :2], inp["K"][0, 0], inp["V"][0, 0], [7], 1 / math.sqrt(128))
    assert np.abs(out[0, :2].cpu().numpy() - wo).max() < ATOL


def test_lse_merge_matches_oracle():
    rng = np.random.default_rng(3)
    rows, d = 333, 128
    o1, o2 = rng.standard_normal((rows, d)), rng.standard_normal((rows, d))
    l1, l2 = rng.standard_normal(rows) * 5, rng.standard_normal(rows) * 5
    l1[:3] = -np.inf
    l2[1:5] = -np.inf
    T = lambda a: torch.tensor(a, dtype=torch.float32, device=DEV)
    out = torch.zeros(rows, d, device=DEV)
    lo = torch.zeros(rows, device=DEV)
    hkv.hkv_lse_merge(T(o1), T(l1), T(o2), T(l2), out, lo)
    torch.cuda.synchronize()
    wo, wl = oracle.lse_merge(o1.astype(np.float32), l1.astype(np.float32), o2.astype(np.float32), l2.astype(np.float32))
    np.testing.assert_allclose(out.cpu().numpy(), wo, atol=1e-5)
    np.testing.assert_allclose(lo.cpu().numpy(), wl, atol=1e-5)


# -------------------------------------------------------------------- append

@pytest.mark.parametrize("kind", ["lsh", "sign", "mlp"])
def test_append(kind):
    name = {"lsh": "qwen7b_512k", "sign": "signvq", "mlp": "spotlight_mlp"}[kind]
    w = synth.WORKLOADS[name].with_(B=2, N=64, layers=1)
    inp = margin_inputs(w, cap=80)
    params, _, kbad = hash_params(w)
    B, Hkv, cap = w.B, w.Hkv, 80
    h = _gpu_hash(w, inp, "k")
    K = torch.zeros(B, Hkv, cap, 128, dtype=torch.bfloat16, device=DEV)
    V = torch.zeros_like(K)
    codes = torch.zeros(B, Hkv, cap, 4, dtype=torch.int32, device=DEV)
    norms = torch.zeros(B, Hkv, cap, dtype=torch.float16, device=DEV)
    kn = inp["K"][:, :, 10:13].contiguous()
    vn = inp["V"][:, :, 10:13].contiguous()
    hkv.hkv_append(h, kn.to(DEV), vn.to(DEV), K, V, codes, 50, norms=norms if kind == "sign" else None)
    torch.cuda.synchronize()
    assert torch.equal(K[:, :, 50:53].cpu(), kn) and torch.equal(V[:, :, 50:53].cpu(), vn)
    assert (K[:, :, :50] == 0).all() and (K[:, :, 53:] == 0).all() and (codes[:, :, 53:] == 0).all()
    want = oracle.encode(kind, kn, _oracle_params(w, inp, "k"))
    if kind == "sign":
        want, wn = want
        np.testing.assert_array_equal(norms[:, :, 50:53].cpu().numpy().view(np.uint16), wn.view(np.uint16))
    np.testing.assert_array_equal(u32(codes[:, :, 50:53]), want)
    with pytest.raises(hkv.HkvError):
        hkv.hkv_append(h, kn.to(DEV), vn.to(DEV), K, V, codes, 78)


# --------------------------------------------------------------- decode step

def run_decode(w, inp, layer_codes=None, next_k_codes=False):
    """GPU: encode keys, then one decode step; returns host results.  With
    next_k_codes, the step also gets a same-shape buffer as its L2 prefetch hint."""
    tdt, code = _dt(w.dtype)
    B, Hq, Hkv, N, cap, W = w.B, w.Hq, w.Hkv, w.N, inp["cap"], w.words
    K, V, q = inp["K"].to(DEV), inp["V"].to(DEV), inp["q"].to(DEV)
    kh, qh = _gpu_hash(w, inp, "k"), _gpu_hash(w, inp, "q")
    codes = torch.full((B, Hkv, cap, W), -1, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(kh, K.view(-1, 128), codes.view(-1, W))
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    idx = torch.full((B, Hkv, w.top_k), -9, dtype=torch.int32, device=DEV)
    qc = torch.zeros(B, Hq, W, dtype=torch.int32, device=DEV)
    ws = hkv.workspace(B, Hq, Hkv, N, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()
    nxt = torch.randint(-2**31, 2**31 - 1, codes.shape, dtype=torch.int32, device=DEV) if next_k_codes else None
    hkv.hkv_decode_step(qh, q, codes, K, V, N, w.n_sink, w.n_local, w.top_k, out, lse, q_codes=qc, idx=idx,
                        ws=ws, status=st, next_k_codes=nxt)
    _check(st)
    return {"codes": u32(codes), "q_codes": u32(qc), "idx": idx.cpu().numpy(), "out": out.cpu().numpy(),
            "lse": lse.cpu().numpy()}


def compare_decode(w, inp, got):
    N = w.N
    kcodes = oracle.encode(w.hash, inp["K"][:, :, :N], _oracle_params(w, inp, "k"))
    if w.hash == "sign":
        kcodes = kcodes[0]
    np.testing.assert_array_equal(got["codes"][:, :, :N], kcodes)
    ref = oracle.decode_step(inp["q"], inp["K"], inp["V"], kcodes, N, w.n_sink, w.n_local, w.top_k, w.hash,
                             _oracle_params(w, inp, "q"))
    np.testing.assert_array_equal(got["q_codes"], ref["q_codes"])
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    assert np.abs(got["out"] - ref["out"]).max() < ATOL
    assert np.abs(got["lse"] - ref["lse"]).max() < ATOL


SMALL = {
    "tiny_lsh": dict(),
    "hashevict_lsh": dict(B=2, N=5003),
    "spotlight_mlp": dict(N=6007),
    "signvq": dict(B=2, N=5001),
    "qwen7b_512k": dict(N=9001, layers=1),
}


@pytest.mark.parametrize("hint", [False, True])
@pytest.mark.parametrize("name", list(SMALL))
def test_decode_step_small(name, hint):
    """Every workload at a small size; with `hint` the step also prefetches
    another code buffer (the next layer's), which must not change anything."""
    w = synth.WORKLOADS[name].with_(**SMALL[name])
    inp = margin_inputs(w, cap=w.N + 5)
    compare_decode(w, inp, run_decode(w, inp, next_k_codes=hint))
