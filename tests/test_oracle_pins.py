"""Pins for the oracle: each test ties it to something other than itself --
hand-worked fixtures, closed forms, invariants of the method, brute force on
tiny inputs, or a library routine that the case reduces to."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.conftest import golden


def _hex(vals):
    return np.array([int(v, 16) for v in vals], dtype=np.uint32)


# ------------------------------------------------------------- packing -----

def test_pack_bits_fixture():
    fx = golden("pack_bits_64.txt")
    y = -np.ones((1, 64))
    for j in fx["positive"]:
        y[0, int(j)] = 1.0
    np.testing.assert_array_equal(oracle.pack_bits(y)[0], _hex(fx["words"]))


def test_pack_bits_zero_is_zero_bit():
    y = np.zeros((1, 32))
    y[0, 3] = 1e-300
    assert oracle.pack_bits(y)[0, 0] == 8


# ------------------------------------------------------------- encoders ----

def test_lsh_fixture_nonsquare():
    fx = golden("lsh_signed_selector.txt")
    R = np.zeros((32, 4))
    for j in range(32):
        R[j, j % 4] = 1.0 if (j // 4) % 2 == 0 else -1.0
    x = np.array([[float(v) for v in fx["x"]]])
    np.testing.assert_array_equal(oracle.encode("lsh", x, R)[0], _hex(fx["words"]))


def test_lsh_identity_projection_is_sign_code():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((50, 128))
    lsh = oracle.encode("lsh", x, np.eye(128))
    sign, _ = oracle.encode("sign", x)
    np.testing.assert_array_equal(lsh, sign)


def test_lsh_charikar_angle_law():
    """Random-hyperplane LSH: P[bit differs] = angle / pi (Charikar)."""
    rng = np.random.default_rng(11)
    d, bits, pairs = 64, 128, 400
    theta = 1.1
    u = rng.standard_normal((pairs, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    w = rng.standard_normal((pairs, d))
    w -= (w * u).sum(1, keepdims=True) * u
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    v = math.cos(theta) * u + math.sin(theta) * w
    total = 0
    for i in range(pairs):
        R = rng.standard_normal((bits, d))
        cu = oracle.encode("lsh", u[i:i + 1], R)
        cv = oracle.encode("lsh", v[i:i + 1], R)
        total += int(oracle.hamming(cu, cv)[0])
    n = pairs * bits
    p = theta / math.pi
    assert abs(total / n - p) < 5 * math.sqrt(p * (1 - p) / n)


@pytest.mark.parametrize("kind", ["lsh", "sign"])
def test_negated_input_flips_every_bit(kind):
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 128))
    R = rng.standard_normal((64, 128))
    params = R if kind == "lsh" else None
    c1 = oracle.encode(kind, x, params)
    c2 = oracle.encode(kind, -x, params)
    if kind == "sign":
        c1, c2 = c1[0], c2[0]
    bits = c1.shape[1] * 32
    for i in range(20):
        assert oracle.hamming(c1[i:i + 1], c2[i:i + 1])[0] == bits


def _mlp_fixture_params():
    W1 = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, -1.0]])
    b1 = np.array([0.0, -1.0, 0.0])
    W2 = np.zeros((32, 3))
    b2 = -np.ones(32)
    W2[0, 0], b2[0] = 1.0, -0.8
    W2[1, 0], b2[1] = 1.0, -0.85
    W2[2, 1], b2[2] = 1.0, 0.01
    W2[3, 1], b2[3] = -1.0, 0.01
    W2[4, 2], b2[4] = 1.0, -0.05
    W2[5, 2], b2[5] = 1.0, -0.052
    b2[6] = 0.5
    b2[7] = -0.5
    W2[8, 0], W2[8, 2], b2[8] = 1.0, -1.0, -0.77
    return W1, b1, W2, b2


def test_mlp_fixture():
    fx = golden("mlp_hash_worked.txt")
    x = np.array([[math.log(3.0), 1.0]])
    params = _mlp_fixture_params()
    y = oracle.presign_mlp(x, *params)
    h0 = 0.75 * math.log(3.0)
    h2 = (math.log(3.0) - 1.0) / (1.0 + math.e / 3.0)
    assert abs(h0 - float(fx["h0"][0])) < 1e-13
    assert abs(h2 - float(fx["h2"][0])) < 1e-7
    assert abs(y[0, 0] - (h0 - 0.8)) < 1e-13
    assert abs(y[0, 4] - (h2 - 0.05)) < 1e-13
    assert abs(y[0, 8] - (h0 - h2 - 0.77)) < 1e-13
    np.testing.assert_array_equal(oracle.encode("mlp", x, params)[0], _hex(fx["words"]))


def test_mlp_zero_first_layer_gives_constant_code():
    rng = np.random.default_rng(8)
    d, hidden, bits = 16, 24, 64
    W1 = np.zeros((hidden, d))
    b1 = rng.uniform(-1, 1, hidden)
    W2 = rng.uniform(-1, 1, (bits, hidden))
    b2 = rng.uniform(-1, 1, bits)
    x = rng.standard_normal((30, d))
    y = oracle.presign_mlp(x, W1, b1, W2, b2)
    expect = W2 @ (b1 / (1 + np.exp(-b1))) + b2
    np.testing.assert_allclose(y, np.broadcast_to(expect, y.shape), rtol=0, atol=1e-14)


def test_mlp_matches_torch_library_layers():
    rng = np.random.default_rng(9)
    d, hidden, bits = 128, 512, 128
    W1 = rng.uniform(-0.09, 0.09, (hidden, d))
    b1 = rng.uniform(-0.09, 0.09, hidden)
    W2 = rng.uniform(-0.04, 0.04, (bits, hidden))
    b2 = rng.uniform(-0.04, 0.04, bits)
    x = rng.standard_normal((64, d))
    T = lambda a: torch.from_numpy(a)
    ref = torch.nn.functional.linear(torch.nn.functional.silu(torch.nn.functional.linear(T(x), T(W1), T(b1))), T(W2), T(b2))
    np.testing.assert_allclose(oracle.presign_mlp(x, W1, b1, W2, b2), ref.numpy(), rtol=0, atol=1e-13)


def test_sign_norms_fp16():
    x = np.zeros((3, 128))
    x[0, :2] = [3.0, 4.0]
    x[1, :] = 1.0
    x[2, 7] = -2.5
    n = oracle.sign_norms(x)
    assert n.dtype == np.float16
    assert float(n[0]) == 5.0
    assert float(n[1]) == 11.3125  # sqrt(128) = 11.3137 -> nearest fp16 (spacing 2^-7)
    assert float(n[2]) == 2.5


# ------------------------------------------------------------- hamming -----

def test_hamming_fixture():
    fx = golden("hamming_group.txt")
    q = np.stack([_hex(fx["cq0"]), _hex(fx["cq1"])])
    k = _hex(fx["ck"])[None, :]
    assert oracle.hamming(q, k)[0] == int(fx["D"][0])


def test_hamming_counts_differing_signs():
    """Brute force from the pre-sign values, with no packing involved."""
    rng = np.random.default_rng(1)
    g, n, bits = 3, 40, 64
    yq = rng.standard_normal((g, bits))
    yk = rng.standard_normal((n, bits))
    D = oracle.hamming(oracle.pack_bits(yq), oracle.pack_bits(yk))
    for t in range(n):
        brute = sum(int((yq[h, j] > 0) != (yk[t, j] > 0)) for h in range(g) for j in range(bits))
        assert D[t] == brute


# ------------------------------------------------------------- top-k -------

def test_topk_fixture():
    fx = golden("topk_ties.txt")
    D = np.array([int(v) for v in fx["D"]])
    lo, hi = oracle.candidate_range(len(D), int(fx["sink"][0]), int(fx["local"][0]))
    got = oracle.select_topk(D, lo, hi, int(fx["k"][0]))
    np.testing.assert_array_equal(got, [int(v) for v in fx["idx"]])


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_rank(seed):
    """Selected iff fewer than k candidates precede it in (D, t) order."""
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 90))
    s, l = int(rng.integers(0, 6)), int(rng.integers(0, 6))
    k = int(rng.integers(0, 100))
    D = rng.integers(0, 6, N)
    lo, hi = oracle.candidate_range(N, s, l)
    got = oracle.select_topk(D, lo, hi, k)
    want = [t for t in range(lo, hi)
            if sum(1 for u in range(lo, hi) if (D[u], u) < (D[t], t)) < k]
    np.testing.assert_array_equal(got, want)


def test_topk_degenerate_cases():
    D = np.full(50, 7)
    np.testing.assert_array_equal(oracle.select_topk(D, 4, 40, 5), [4, 5, 6, 7, 8])
    np.testing.assert_array_equal(oracle.select_topk(D, 4, 40, 1000), np.arange(4, 40))
    assert oracle.select_topk(D, 4, 40, 0).size == 0
    assert oracle.select_topk(D, 10, 10, 5).size == 0


def test_candidate_range_short_sequence():
    assert oracle.candidate_range(100, 4, 64) == (4, 36)
    assert oracle.candidate_range(50, 4, 64) == (4, 4)
    assert oracle.candidate_range(3, 4, 64) == (3, 3)
    assert oracle.candidate_range(0, 0, 0) == (0, 0)


# ------------------------------------------------------------- attention ---

def test_attention_fixture_and_merge():
    fx = golden("attention_worked.txt")
    q = np.array([[math.log(3.0), 0.0]])
    K = np.array([[0.0, 5.0], [1.0, 7.0], [2.0, 0.0]])
    V = np.array([[4.0, 0.0], [0.0, 8.0], [9.0, 9.0]])
    o, lse = oracle.attend(q, K, V, [0, 1], 1.0)
    np.testing.assert_allclose(o[0], [float(v) for v in fx["out"]], atol=1e-14)
    assert abs(lse[0] - math.log(float(fx["lse_is_ln"][0]))) < 1e-14
    o0, l0 = oracle.attend(q, K, V, [0], 1.0)
    o1, l1 = oracle.attend(q, K, V, [1], 1.0)
    om, lm = oracle.lse_merge(o0, l0, o1, l1)
    np.testing.assert_allclose(om, o, atol=1e-14)
    np.testing.assert_allclose(lm, lse, atol=1e-14)


def test_attention_all_rows_is_library_sdpa():
    rng = np.random.default_rng(4)
    g, N, d = 4, 300, 128
    q = rng.standard_normal((g, d))
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    o, lse = oracle.attend(q, K, V, np.arange(N), 1 / math.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0]
    np.testing.assert_allclose(o, ref.numpy(), atol=1e-12)
    z = (q @ K.T) / math.sqrt(d)
    np.testing.assert_allclose(lse, np.log(np.exp(z).sum(1)), atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((20, 8))
    V = rng.standard_normal((20, 8))
    q = rng.standard_normal((2, 8))
    o, _ = oracle.attend(q, K, V, [13], 0.3)
    np.testing.assert_allclose(o, np.stack([V[13], V[13]]), atol=1e-15)
    o, lse = oracle.attend(np.zeros((1, 8)), K, V, [1, 4, 9], 0.3)
    np.testing.assert_allclose(o[0], V[[1, 4, 9]].mean(0), atol=1e-15)
    assert abs(lse[0] - math.log(3)) < 1e-15
    o, lse = oracle.attend(q, K, V, [], 0.3)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("seed", range(4))
def test_lse_merge_any_partition(seed):
    rng = np.random.default_rng(seed)
    g, N, d = 3, 64, 16
    q = rng.standard_normal((g, d)) * 2
    K = rng.standard_normal((N, d))
    V = rng.standard_normal((N, d))
    rows = rng.permutation(N)[:40]
    o, lse = oracle.attend(q, K, V, rows, 0.5)
    parts = np.array_split(rng.permutation(rows), int(rng.integers(2, 6)))
    parts.insert(int(rng.integers(0, len(parts))), np.array([], dtype=np.int64))
    acc_o, acc_l = oracle.attend(q, K, V, parts[0], 0.5)
    for p in parts[1:]:
        po, pl = oracle.attend(q, K, V, p, 0.5)
        acc_o, acc_l = oracle.lse_merge(acc_o, acc_l, po, pl)
    np.testing.assert_allclose(acc_o, o, atol=1e-12)
    np.testing.assert_allclose(acc_l, lse, atol=1e-12)


def test_lse_merge_two_empty_parts():
    o, lse = oracle.lse_merge(np.zeros((2, 4)), np.full(2, -np.inf), np.zeros((2, 4)), np.full(2, -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# ------------------------------------------------------------- composite ---

def test_decode_step_full_budget_is_dense_attention():
    """k >= candidates: the step attends every token, i.e. dense attention."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, N, d = 2, 4, 2, 50, 128
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    R = rng.standard_normal((64, d))
    codes = oracle.encode("lsh", K, R)
    res = oracle.decode_step(q, K, V, codes, N, 3, 5, 1000, "lsh", R)
    g = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, h])[None, None], torch.from_numpy(K[b, h // g])[None],
                torch.from_numpy(V[b, h // g])[None])[0, 0]
            np.testing.assert_allclose(res["out"][b, h], ref.numpy(), atol=1e-12)


def test_decode_step_uses_group_sum():
    """KV head j's selection depends only on query heads j*g .. j*g+g-1, and
    equals the brute-force top-k of their summed distances."""
    rng = np.random.default_rng(13)
    B, Hq, Hkv, N, d = 1, 6, 3, 200, 128
    g = Hq // Hkv
    q = rng.standard_normal((B, Hq, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    codes, _ = oracle.encode("sign", K)
    r1 = oracle.decode_step(q, K, V, codes, N, 0, 0, 10, "sign")
    q2 = q.copy()
    q2[0, 2 * g:] = rng.standard_normal((g, d))
    r2 = oracle.decode_step(q2, K, V, codes, N, 0, 0, 10, "sign")
    np.testing.assert_array_equal(r1["idx"][0, :2], r2["idx"][0, :2])
    qc, _ = oracle.encode("sign", q)
    for j in range(Hkv):
        D = [sum(int(np.bitwise_count(qc[0, h] ^ codes[0, j, t]).sum()) for h in range(j * g, (j + 1) * g))
             for t in range(N)]
        want = sorted(sorted(range(N), key=lambda t: (D[t], t))[:10])
        np.testing.assert_array_equal(r1["idx"][0, j], want)


# --------------------------------------------------------------- eviction

def test_evict_fixture():
    gl = golden("evict_dissimilar.txt")
    q = np.array([[[int(gl["q"][0], 16)]]], dtype=np.uint32)
    keys = np.array([int(v, 16) for v in gl["keys"]], dtype=np.uint32).reshape(1, 1, -1, 1)
    s, l = (int(v) for v in gl["sink_local"])
    victim, vdist = oracle.evict_victim(q, keys, keys.shape[2], s, l)
    assert victim[0, 0] == int(gl["victim"][0]) and vdist[0, 0] == int(gl["vdist"][0])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_evict_brute_force(seed):
    """Bit strings and a plain maximum scan, independent of the oracle's
    vectorised popcount and argmax."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, W, N, s, l = 2, 6, 2, 2, 23, 2, 3
    # few distinct codes, so the maximum is often tied
    pool = rng.integers(0, 2**32, size=(4, W), dtype=np.uint64).astype(np.uint32)
    k = pool[rng.integers(0, 4, size=(B, Hkv, N))]
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    victim, vdist = oracle.evict_victim(q, k, N, s, l)
    g = Hq // Hkv
    for b in range(B):
        for j in range(Hkv):
            best, arg = -1, -1
            for t in range(s, N - l):
                d = sum(bin(int(q[b, j * g + h, w]) ^ int(k[b, j, t, w])).count("1") for h in range(g) for w in range(W))
                if d > best:
                    best, arg = d, t
            assert victim[b, j] == arg and vdist[b, j] == best


def test_evict_complemented_query_is_top1_retrieval():
    """With every query bit flipped D becomes g * bits - D, so the eviction
    victim is the top-1 retrieved token (both take the lowest index on ties)."""
    rng = np.random.default_rng(5)
    B, Hq, Hkv, W, N, s, l = 1, 4, 2, 4, 300, 4, 16
    pool = rng.integers(0, 2**32, size=(16, W), dtype=np.uint64).astype(np.uint32)
    k = pool[rng.integers(0, 16, size=(B, Hkv, N))]
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    victim, _ = oracle.evict_victim(~q, k, N, s, l)
    idx, _ = oracle.retrieve(q, k, N, s, l, 1)
    np.testing.assert_array_equal(victim, idx[..., 0])


def test_evict_without_candidates():
    q = np.zeros((1, 2, 4), dtype=np.uint32)
    k = np.zeros((1, 1, 10, 4), dtype=np.uint32)
    victim, vdist = oracle.evict_victim(q, k, 10, 6, 6)
    assert victim[0, 0] == -1 and vdist[0, 0] == -1


# ------------------------------------------------- one index set per query head

def test_heads_equal_group_selection_when_groups_are_single_heads():
    """With g = 1 every query head has its own KV head: both readings agree."""
    rng = np.random.default_rng(8)
    q = rng.integers(0, 2**32, size=(2, 3, 4), dtype=np.uint64).astype(np.uint32)
    k = rng.integers(0, 2**32, size=(2, 3, 50, 4), dtype=np.uint64).astype(np.uint32)
    a = oracle.retrieve_heads(q, k, 50, 2, 5, 7)
    b = oracle.retrieve(q, k, 50, 2, 5, 7)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_heads_with_identical_queries_match_the_group():
    """If all g heads of a group share one code, the group distance is g times
    the head distance: the same order, so the same index sets."""
    rng = np.random.default_rng(9)
    one = rng.integers(0, 2**32, size=(1, 2, 1, 4), dtype=np.uint64).astype(np.uint32)
    q = np.repeat(one, 3, axis=2).reshape(1, 6, 4)  # heads 0-2 share a code, heads 3-5 another
    pool = rng.integers(0, 2**32, size=(5, 4), dtype=np.uint64).astype(np.uint32)
    k = pool[rng.integers(0, 5, size=(1, 2, 80))]
    ih, dh = oracle.retrieve_heads(q, k, 80, 3, 4, 9)
    ig, dg = oracle.retrieve(q, k, 80, 3, 4, 9)
    for h in range(6):
        np.testing.assert_array_equal(ih[0, h], ig[0, h // 3])
        np.testing.assert_array_equal(dh[0, h] * 3, np.where(dg[0, h // 3] >= 0, dg[0, h // 3], -3))


def test_heads_brute_force():
    rng = np.random.default_rng(10)
    B, Hq, Hkv, W, N, s, l, kk = 1, 4, 2, 2, 30, 2, 3, 5
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    k = rng.integers(0, 2**32, size=(B, Hkv, N, W), dtype=np.uint64).astype(np.uint32)
    idx, _ = oracle.retrieve_heads(q, k, N, s, l, kk)
    for h in range(Hq):
        d = [sum(bin(int(q[0, h, w]) ^ int(k[0, h // 2, t, w])).count("1") for w in range(W)) for t in range(N)]
        order = sorted(range(s, N - l), key=lambda t: (d[t], t))[:kk]
        assert list(idx[0, h]) == sorted(order)


def test_decode_step_heads_single_head_groups_equal_decode_step():
    rng = np.random.default_rng(11)
    B, H, N, d = 1, 2, 40, 128
    q = rng.normal(size=(B, H, d))
    K = rng.normal(size=(B, H, N, d))
    V = rng.normal(size=(B, H, N, d))
    kc = oracle.encode("sign", K)[0]
    a = oracle.decode_step_heads(q, K, V, kc, N, 2, 3, 6, "sign")
    b = oracle.decode_step(q, K, V, kc, N, 2, 3, 6, "sign")
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=1e-14)


# ------------------------------------------------------- ragged batches

def test_ragged_with_equal_lengths_is_the_uniform_step():
    rng = np.random.default_rng(12)
    B, H, N, d = 3, 2, 60, 128
    q = rng.normal(size=(B, H, d))
    K = rng.normal(size=(B, H, N, d))
    V = rng.normal(size=(B, H, N, d))
    kc = oracle.encode("sign", K)[0]
    a = oracle.decode_step_ragged(q, K, V, kc, [N] * B, 2, 5, 7, "sign")
    b = oracle.decode_step(q, K, V, kc, N, 2, 5, 7, "sign")
    for key in ("q_codes", "idx", "dist"):
        np.testing.assert_array_equal(a[key], b[key])
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=1e-14)


def test_ragged_ignores_tokens_past_each_length():
    """Garbage beyond a sequence's length changes nothing for that sequence."""
    rng = np.random.default_rng(13)
    B, H, N, d = 2, 1, 50, 128
    q = rng.normal(size=(B, H, d))
    K = rng.normal(size=(B, H, N, d))
    V = rng.normal(size=(B, H, N, d))
    kc = oracle.encode("sign", K)[0]
    lens = [50, 31]
    a = oracle.decode_step_ragged(q, K, V, kc, lens, 2, 4, 6, "sign")
    K2, V2, kc2 = K.copy(), V.copy(), kc.copy()
    K2[1, :, 31:] = 1e6
    V2[1, :, 31:] = -1e6
    kc2[1, :, 31:] = 0
    b = oracle.decode_step_ragged(q, K2, V2, kc2, lens, 2, 4, 6, "sign")
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=1e-12)


# ------------------------------------------- norm-weighted sign-VQ retrieval

def _normw_golden():
    gl = golden("normw_worked.txt")
    q = _hex(gl["q"]).reshape(1, 1, 1)
    keys = _hex(gl["keys"]).reshape(1, 1, -1, 1)
    norms = np.array([float(v) for v in gl["norms"]], dtype=np.float16).reshape(1, 1, -1)
    return gl, q, keys, norms


@pytest.mark.parametrize("case", "abcd")
def test_normw_fixture(case):
    gl, q, keys, norms = _normw_golden()
    s, l, k = (int(v) for v in gl[f"case_{case}"])
    idx, score = oracle.retrieve_normw(q, keys, norms, keys.shape[2], s, l, k)
    np.testing.assert_array_equal(idx[0, 0], [int(v) for v in gl[f"idx_{case}"]])
    np.testing.assert_array_equal(score[0, 0], [float(v) for v in gl[f"score_{case}"]])


def _pm1_codes(signs):
    """Codes of +-1 vectors (any leading shape): bit i set where the entry is +1."""
    signs = np.asarray(signs, dtype=np.float64)
    return oracle.pack_bits(signs.reshape(-1, signs.shape[-1])).reshape(*signs.shape[:-1], -1)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_normw_score_is_norm_times_sign_inner_product(seed):
    """S(t) equals norm_t * sum_h sign(q_h) . sign(k_t), the inner product of
    the +-1 vectors themselves (no popcount), for every candidate."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, bits, N = 2, 6, 2, 64, 37
    g = Hq // Hkv
    qs = rng.choice([-1.0, 1.0], size=(B, Hq, bits))
    ks = rng.choice([-1.0, 1.0], size=(B, Hkv, N, bits))
    norms = rng.uniform(0.5, 4.0, size=(B, Hkv, N)).astype(np.float16)
    idx, score = oracle.retrieve_normw(_pm1_codes(qs), _pm1_codes(ks), norms, N, 0, 0, N)
    for b in range(B):
        for j in range(Hkv):
            np.testing.assert_array_equal(idx[b, j], np.arange(N))
            dots = (qs[b, j * g:(j + 1) * g] @ ks[b, j].T).sum(axis=0)
            np.testing.assert_array_equal(score[b, j], norms[b, j].astype(np.float64) * dots)


@pytest.mark.parametrize("seed", [3, 4])
def test_normw_brute_force(seed):
    """Few distinct codes and norms (many exact ties); the ranking is a plain
    sort of (-S, t) with S from the +-1 inner products."""
    rng = np.random.default_rng(seed)
    B, Hq, Hkv, bits, N, s, l, k = 2, 4, 2, 32, 41, 3, 5, 9
    g = Hq // Hkv
    pool = rng.choice([-1.0, 1.0], size=(5, bits))
    ks = pool[rng.integers(0, 5, size=(B, Hkv, N))]
    qs = rng.choice([-1.0, 1.0], size=(B, Hq, bits))
    norms = np.array([0.0, 1.0, 2.5], dtype=np.float16)[rng.integers(0, 3, size=(B, Hkv, N))]
    idx, _ = oracle.retrieve_normw(_pm1_codes(qs), _pm1_codes(ks), norms, N, s, l, k)
    for b in range(B):
        for j in range(Hkv):
            S = {t: float(norms[b, j, t]) * sum(float(qs[b, j * g + h] @ ks[b, j, t]) for h in range(g))
                 for t in range(s, N - l)}
            want = sorted(sorted(S, key=lambda t: (-S[t], t))[:k])
            np.testing.assert_array_equal(idx[b, j], want)


def test_normw_equal_norms_is_hamming_retrieval():
    """With one norm for every key S decreases with D, so the selection is the
    pinned smallest-distance retrieval."""
    rng = np.random.default_rng(6)
    B, Hq, Hkv, W, N = 2, 8, 2, 4, 500
    pool = rng.integers(0, 2**32, size=(12, W), dtype=np.uint64).astype(np.uint32)
    k = pool[rng.integers(0, 12, size=(B, Hkv, N))]
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    norms = np.full((B, Hkv, N), 3.25, dtype=np.float16)
    for top_k in (1, 17, 300):
        idx, _ = oracle.retrieve_normw(q, k, norms, N, 4, 16, top_k)
        want, _ = oracle.retrieve(q, k, N, 4, 16, top_k)
        np.testing.assert_array_equal(idx, want)


def test_normw_norm_scaling_and_zero_norms():
    """Doubling every norm (exact in fp16) doubles S and keeps the selection;
    a zero norm scores 0, between every positive and every negative score."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, W, N = 1, 2, 1, 2, 200
    k = rng.integers(0, 2**32, size=(B, Hkv, N, W), dtype=np.uint64).astype(np.uint32)
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    norms = rng.uniform(0.5, 3.0, size=(B, Hkv, N)).astype(np.float16)
    i1, s1 = oracle.retrieve_normw(q, k, norms, N, 0, 0, 50)
    i2, s2 = oracle.retrieve_normw(q, k, (norms * 2).astype(np.float16), N, 0, 0, 50)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_array_equal(s2, 2 * s1)
    z = norms.copy()
    z[0, 0, 10] = 0.0
    _, S = oracle.retrieve_normw(q, k, z, N, 0, 0, N)
    D = oracle.hamming(q[0], k[0, 0])
    m = 2 * 64 - 2 * D
    assert S[0, 0, 10] == 0.0
    other = np.arange(N) != 10
    assert (S[0, 0][(m > 0) & other] > 0).all() and (S[0, 0][(m < 0) & other] < 0).all()


# ------------------------------------------------------------ paged layout

def test_gather_pages_identity_table_is_a_reshape():
    """Pages laid out in order, one sequence per run of pages: gathering is
    the plain reshape of the pool (numpy), for every N up to the capacity."""
    rng = np.random.default_rng(8)
    B, Hkv, P, pages, W = 2, 3, 4, 5, 2
    pool = rng.integers(0, 2**31, size=(B * pages, Hkv, P, W))
    table = np.arange(B * pages).reshape(B, pages)
    whole = pool.reshape(B, pages, Hkv, P, W).transpose(0, 2, 1, 3, 4).reshape(B, Hkv, pages * P, W)
    for N in (1, 7, 20):
        np.testing.assert_array_equal(oracle.gather_pages(pool, table, P, N), whole[:, :, :N])


def test_gather_pages_permuted_table():
    """Hand-built: page size 2, two sequences sharing a pool of four pages in
    scrambled order; every token's value names its (sequence, token)."""
    P, Hkv = 2, 1
    table = np.array([[3, 0], [1, 2]])
    pool = np.zeros((4, Hkv, P), dtype=np.int64)
    for b in range(2):
        for t in range(4):
            pool[table[b, t // P], 0, t % P] = 100 * b + t
    got = oracle.gather_pages(pool, table, P, 3)
    np.testing.assert_array_equal(got[:, 0], [[0, 1, 2], [100, 101, 102]])


def test_paged_retrieval_equals_contiguous_retrieval():
    """Retrieval over a gathered paged cache is the retrieval of the same
    tokens stored contiguously (pages scattered at random in the pool)."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, W, P, N = 2, 4, 2, 4, 16, 100
    pages = -(-N // P)
    k = rng.integers(0, 2**32, size=(B, Hkv, pages * P, W), dtype=np.uint64).astype(np.uint32)
    q = rng.integers(0, 2**32, size=(B, Hq, W), dtype=np.uint64).astype(np.uint32)
    perm = rng.permutation(B * pages + 3)[: B * pages]
    table = perm.reshape(B, pages)
    pool = np.zeros((B * pages + 3, Hkv, P, W), dtype=np.uint32)
    for b in range(B):
        for j in range(pages):
            pool[table[b, j]] = k[b, :, j * P:(j + 1) * P]
    gathered = oracle.gather_pages(pool, table, P, N)
    np.testing.assert_array_equal(gathered, k[:, :, :N])
    i1, d1 = oracle.retrieve(q, gathered, N, 4, 16, 20)
    i2, d2 = oracle.retrieve(q, k, N, 4, 16, 20)
    np.testing.assert_array_equal(i1, i2)
    np.testing.assert_array_equal(d1, d2)
