"""Oracle for hash-code KV retrieval and sparse decode attention.

TEST INFRASTRUCTURE.  This is a plain, slow, fp64 CPU statement of what the
decode-time retrieval path computes, written to be checked by eye against the
pages it cites.  It is used only by the tests, by the package's smoke check and
by the benchmark's CPU-baseline leg.  The library never imports it, and it
shares no code with the CUDA path.

Pages cited (title, section):
  [SA]  Spotlight Attention: Towards Efficient LLM Generation via Non-linear
        Hashing-based KV Cache Retrieval -- "Approach", "Key results"
  [SIK] Self-Indexing KVCache: Predicting Sparse Attention from Compressed Keys
        -- "Abstract"
  [RA]  RetrievalAttention: Accelerating Long-Context LLM Inference via Vector
        Retrieval -- "Summary", "Approach"
  [HE]  HashEvict: A Pre-Attention KV Cache Eviction Strategy using
        Locality-Sensitive Hashing -- "Abstract"

Readings taken where the pages are silent (each is listed with its reason in
the design notes): bit j of a code is 1 iff the pre-sign value is > 0; bits are
packed least-significant first into uint32 words (bit j -> word j // 32, bit
j % 32); a KV head's score is the sum of the Hamming distances of its query
heads; ties in the score go to the lowest token index; sink tokens [0, s) and
the local window [N - l, N) are always attended and are not candidates; the
softmax scale is 1/sqrt(d).

Pinned by tests/test_oracle_pins.py and the fixtures in tests/golden/.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "as_f64", "presign_lsh", "presign_mlp", "presign_sign", "pack_bits", "encode",
    "sign_norms", "hamming", "candidate_range", "select_topk", "attention_rows",
    "attend", "lse_merge", "retrieve", "retrieve_normw", "decode_step", "gather_pages", "ROW_CHUNK",
]

ROW_CHUNK = 1 << 15


def as_f64(x) -> np.ndarray:
    """Exact widening of stored values (fp32, bf16 or fp16) to fp64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------- encoders --

def presign_lsh(x, R) -> np.ndarray:
    """[HE] "binarized Gaussian projections": y = R x for each row x.
    x [rows, d], R [bits, d] -> y [rows, bits]."""
    x, R = as_f64(x), as_f64(R)
    return x @ R.T


def presign_mlp(x, W1, b1, W2, b2) -> np.ndarray:
    """[SA] "Approach": the hash is the sign of a two-layer MLP output,
    y = W2 SiLU(W1 x + b1) + b2, SiLU(z) = z / (1 + exp(-z)).
    x [rows, d], W1 [hidden, d], W2 [bits, hidden] -> y [rows, bits]."""
    x = as_f64(x)
    W1, b1, W2, b2 = (as_f64(a) for a in (W1, b1, W2, b2))
    out = np.empty((x.shape[0], W2.shape[0]))
    for r0 in range(0, x.shape[0], ROW_CHUNK):
        z = x[r0:r0 + ROW_CHUNK] @ W1.T + b1
        h = z / (1.0 + np.exp(-z))
        out[r0:r0 + ROW_CHUNK] = h @ W2.T + b2
    return out


def presign_sign(x) -> np.ndarray:
    """[SIK] "sign-based 1-bit vector quantization": the code of x is sign(x)."""
    return as_f64(x)


def pack_bits(y: np.ndarray) -> np.ndarray:
    """Codes from pre-sign values: bit j = [y_j > 0], packed LSB first into
    uint32 words.  y [rows, bits] -> [rows, bits // 32] uint32."""
    rows, bits = y.shape
    assert bits % 32 == 0
    b = (y > 0).astype(np.uint64).reshape(rows, bits // 32, 32)
    weights = np.left_shift(np.uint64(1), np.arange(32, dtype=np.uint64))
    return (b * weights).sum(axis=2).astype(np.uint32)


def sign_norms(x) -> np.ndarray:
    """Per-row L2 norm kept beside the sign-VQ code, rounded to fp16."""
    x = as_f64(x)
    return np.sqrt(np.sum(x * x, axis=-1)).astype(np.float16)


def encode(kind: str, x, params=None):
    """Codes of the rows of x (any leading shape, last dim d).
    kind "lsh": params = R; "mlp": params = (W1, b1, W2, b2); "sign": none.
    Returns uint32 codes [..., bits // 32] (and fp16 norms for "sign").
    Rows are processed in chunks of ROW_CHUNK to bound memory."""
    lead = tuple(x.shape[:-1])
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    n = flat.shape[0]
    codes, norms = None, None
    for r0 in range(0, max(n, 1), ROW_CHUNK):
        xs = as_f64(flat[r0:r0 + ROW_CHUNK])
        if kind == "lsh":
            y = presign_lsh(xs, params)
        elif kind == "mlp":
            y = presign_mlp(xs, *params)
        elif kind == "sign":
            y = presign_sign(xs)
        else:
            raise ValueError(kind)
        c = pack_bits(y)
        if codes is None:
            codes = np.empty((n, c.shape[1]), dtype=np.uint32)
            norms = np.empty(n, dtype=np.float16) if kind == "sign" else None
        codes[r0:r0 + ROW_CHUNK] = c
        if kind == "sign":
            norms[r0:r0 + ROW_CHUNK] = sign_norms(xs)
    codes = codes.reshape(*lead, -1)
    if kind == "sign":
        return codes, norms.reshape(lead)
    return codes


# --------------------------------------------------------------- retrieval --

def hamming(q_codes: np.ndarray, k_codes: np.ndarray) -> np.ndarray:
    """[HE] Hamming distance between the query's code and each key's code,
    summed over the query heads that share the key head:
    D(t) = sum_h popcount(cq_h XOR ck_t).
    q_codes [g, W], k_codes [N, W] (uint32) -> D [N] int64."""
    q = np.asarray(q_codes, dtype=np.uint32)
    k = np.asarray(k_codes, dtype=np.uint32)
    D = np.zeros(k.shape[0], dtype=np.int64)
    for h in range(q.shape[0]):
        D += np.bitwise_count(k ^ q[h][None, :]).sum(axis=1, dtype=np.int64)
    return D


def candidate_range(N: int, n_sink: int, n_local: int):
    """Sink rows [0, sink_end), candidates [sink_end, local_start), local rows
    [local_start, N).  [SA] keeps sink and local-window tokens; [RA] keeps a
    fixed sink/window pattern resident beside the retrieved tokens."""
    sink_end = min(n_sink, N)
    local_start = max(sink_end, N - n_local)
    return sink_end, local_start


def select_topk(D: np.ndarray, lo: int, hi: int, k: int) -> np.ndarray:
    """[SA] top-k retrieval by code similarity: the k candidates in [lo, hi)
    with the smallest D, ties to the lowest index, returned in ascending
    token order."""
    if hi <= lo or k <= 0:
        return np.zeros(0, dtype=np.int64)
    cand = np.arange(lo, hi, dtype=np.int64)
    order = np.argsort(D[lo:hi], kind="stable")
    return np.sort(cand[order[: min(k, hi - lo)]])


def attention_rows(N: int, n_sink: int, n_local: int, idx) -> np.ndarray:
    """The attended rows of one KV head: sink, selected, local window."""
    sink_end, local_start = candidate_range(N, n_sink, n_local)
    sel = np.asarray(idx, dtype=np.int64)
    sel = sel[sel >= 0]
    return np.concatenate([np.arange(0, sink_end), sel, np.arange(local_start, N)]).astype(np.int64)


def _take(x, rows: np.ndarray):
    if hasattr(x, "detach"):
        import torch
        return x[torch.from_numpy(rows)]
    return np.asarray(x)[rows]


def attend(q, K, V, rows, scale: float):
    """[SA] exact attention over only the retrieved rows:
    o_h = sum_t softmax_t(scale * q_h . K_t) V_t,  lse_h = log sum_t exp(scale * q_h . K_t).
    q [g, d]; K, V [N, d]; rows [R] -> (o [g, d], lse [g]).  No rows gives
    o = 0 and lse = -inf."""
    q = as_f64(q)
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        return np.zeros_like(q), np.full(q.shape[0], -np.inf)
    Kr = as_f64(_take(K, rows))
    Vr = as_f64(_take(V, rows))
    z = (q @ Kr.T) * scale  # [g, R]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    l = p.sum(axis=1, keepdims=True)
    return (p @ Vr) / l, (m + np.log(l))[:, 0]


def lse_merge(o1, lse1, o2, lse2):
    """[RA] "Approach": partial attention results are combined by exact
    log-sum-exp rescaling.  With m = max(lse1, lse2) and w_i = exp(lse_i - m):
    o = (w1 o1 + w2 o2) / (w1 + w2),  lse = m + log(w1 + w2).
    An empty part has lse = -inf and weight 0; two empty parts give o = 0,
    lse = -inf."""
    o1, o2 = as_f64(o1), as_f64(o2)
    lse1, lse2 = as_f64(lse1), as_f64(lse2)
    m = np.maximum(lse1, lse2)
    empty = np.isneginf(m)
    m_safe = np.where(empty, 0.0, m)
    w1 = np.exp(lse1 - m_safe)
    w2 = np.exp(lse2 - m_safe)
    s = np.where(empty, 1.0, w1 + w2)
    o = (w1[..., None] * o1 + w2[..., None] * o2) / s[..., None]
    lse = np.where(empty, -np.inf, m_safe + np.log(s))
    return o, lse


def retrieve(q_codes, k_codes, N: int, n_sink: int, n_local: int, top_k: int):
    """Top-k per KV head.  q_codes [B, Hq, W]; k_codes [B, Hkv, cap, W].
    Returns idx [B, Hkv, top_k] int64 (ascending, -1 past k_eff) and the
    selected distances [B, Hkv, top_k] (-1 past k_eff)."""
    q_codes = np.asarray(q_codes, dtype=np.uint32)
    k_codes = np.asarray(k_codes, dtype=np.uint32)
    B, Hq, _ = q_codes.shape
    Hkv = k_codes.shape[1]
    g = Hq // Hkv
    lo, hi = candidate_range(N, n_sink, n_local)
    idx = np.full((B, Hkv, top_k), -1, dtype=np.int64)
    dist = np.full((B, Hkv, top_k), -1, dtype=np.int64)
    for b in range(B):
        for kh in range(Hkv):
            D = hamming(q_codes[b, kh * g:(kh + 1) * g], k_codes[b, kh, :N])
            sel = select_topk(D, lo, hi, top_k)
            idx[b, kh, : sel.size] = sel
            dist[b, kh, : sel.size] = D[sel]
    return idx, dist


def retrieve_normw(q_codes, k_codes, norms, N: int, n_sink: int, n_local: int, top_k: int):
    """[SIK] "Abstract": a key's sign code together with its norm is its 1-bit
    vector quantisation.  Reading (the page gives no scoring formula): the pair
    stands for the key |k| sign(k) / sqrt(b), query head h for sign(q_h) / sqrt(b);
    their inner product is |k| (b - 2 popcount(cq_h XOR ck)) / b.  Summed over
    the g query heads of a KV head, with the constant 1/b dropped:
        S(t) = norm_t * (g * b - 2 * D(t)).
    The top_k candidates with the LARGEST S are kept, ties to the lowest index,
    in ascending token order.  q_codes [B, Hq, W]; k_codes [B, Hkv, cap, W];
    norms [B, Hkv, cap] fp16.  Returns idx [B, Hkv, top_k] (-1 past k_eff) and
    S of the selected tokens (-inf past k_eff)."""
    q_codes = np.asarray(q_codes, dtype=np.uint32)
    k_codes = np.asarray(k_codes, dtype=np.uint32)
    norms = np.asarray(norms, dtype=np.float16)
    B, Hq, W = q_codes.shape
    Hkv = k_codes.shape[1]
    g = Hq // Hkv
    bits = 32 * W
    lo, hi = candidate_range(N, n_sink, n_local)
    idx = np.full((B, Hkv, top_k), -1, dtype=np.int64)
    score = np.full((B, Hkv, top_k), -np.inf)
    for b in range(B):
        for kh in range(Hkv):
            D = hamming(q_codes[b, kh * g:(kh + 1) * g], k_codes[b, kh, :N])
            S = as_f64(norms[b, kh, :N]) * (g * bits - 2 * D)
            sel = select_topk(-S, lo, hi, top_k)
            idx[b, kh, : sel.size] = sel
            score[b, kh, : sel.size] = S[sel]
    return idx, score


def evict_victim(q_codes, k_codes, N: int, n_sink: int, n_local: int):
    """[HE] eviction: at each decoding step the token expected to receive the
    lowest attention -- the cached key whose code is least similar to the
    current query's, i.e. the largest D(t) -- is replaced by the new token.
    Candidates are [sink_end, local_start) (sink and local rows stay); ties go
    to the lowest index.  q_codes [B, Hq, W]; k_codes [B, Hkv, cap, W].
    Returns victim [B, Hkv] int64 (-1 without candidates) and its D (-1)."""
    q_codes = np.asarray(q_codes, dtype=np.uint32)
    k_codes = np.asarray(k_codes, dtype=np.uint32)
    B, Hq, _ = q_codes.shape
    Hkv = k_codes.shape[1]
    g = Hq // Hkv
    lo, hi = candidate_range(N, n_sink, n_local)
    victim = np.full((B, Hkv), -1, dtype=np.int64)
    vdist = np.full((B, Hkv), -1, dtype=np.int64)
    if hi <= lo:
        return victim, vdist
    for b in range(B):
        for kh in range(Hkv):
            D = hamming(q_codes[b, kh * g:(kh + 1) * g], k_codes[b, kh, lo:hi])
            best = int(D.max())
            victim[b, kh] = lo + int(np.flatnonzero(D == best)[0])
            vdist[b, kh] = best
    return victim, vdist


def decode_step(q, K, V, k_codes, N: int, n_sink: int, n_local: int, top_k: int,
                kind: str, q_params=None, scale: float | None = None):
    """One decode step: encode the query heads, retrieve the top-k keys of each
    KV head, attend over sink + selected + local rows.
    q [B, Hq, d]; K, V [B, Hkv, cap, d]; k_codes [B, Hkv, cap, W].
    Returns dict(q_codes, idx, dist, out [B, Hq, d], lse [B, Hq])."""
    qa = as_f64(q)
    B, Hq, d = qa.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qc = encode(kind, qa, q_params)
    if kind == "sign":
        qc = qc[0]
    idx, dist = retrieve(qc, k_codes, N, n_sink, n_local, top_k)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for kh in range(Hkv):
            rows = attention_rows(N, n_sink, n_local, idx[b, kh])
            o, l = attend(qa[b, kh * g:(kh + 1) * g], K[b, kh], V[b, kh], rows, scale)
            out[b, kh * g:(kh + 1) * g] = o
            lse[b, kh * g:(kh + 1) * g] = l
    return {"q_codes": qc, "idx": idx, "dist": dist, "out": out, "lse": lse}


def retrieve_heads(q_codes, k_codes, N: int, n_sink: int, n_local: int, top_k: int):
    """[RA] one index set per query head: head h of batch b scores the keys of
    its KV head j = h // g by its own Hamming distance
    D_h(t) = popcount(cq_h XOR ck_t) and keeps its k smallest (ties to the
    lowest index).  q_codes [B, Hq, W]; k_codes [B, Hkv, cap, W].
    Returns idx, dist [B, Hq, top_k] (ascending, -1 past k_eff)."""
    q_codes = np.asarray(q_codes, dtype=np.uint32)
    k_codes = np.asarray(k_codes, dtype=np.uint32)
    B, Hq, _ = q_codes.shape
    g = Hq // k_codes.shape[1]
    lo, hi = candidate_range(N, n_sink, n_local)
    idx = np.full((B, Hq, top_k), -1, dtype=np.int64)
    dist = np.full((B, Hq, top_k), -1, dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            D = hamming(q_codes[b, h:h + 1], k_codes[b, h // g, :N])
            sel = select_topk(D, lo, hi, top_k)
            idx[b, h, : sel.size] = sel
            dist[b, h, : sel.size] = D[sel]
    return idx, dist


def decode_step_heads(q, K, V, k_codes, N: int, n_sink: int, n_local: int, top_k: int,
                      kind: str, q_params=None, scale: float | None = None):
    """decode_step with one index set per query head ([RA]): head h attends
    over sink + its own selected rows + local rows of its KV head."""
    qa = as_f64(q)
    B, Hq, d = qa.shape
    g = Hq // K.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    qc = encode(kind, qa, q_params)
    if kind == "sign":
        qc = qc[0]
    idx, dist = retrieve_heads(qc, k_codes, N, n_sink, n_local, top_k)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            rows = attention_rows(N, n_sink, n_local, idx[b, h])
            o, l = attend(qa[b, h:h + 1], K[b, h // g], V[b, h // g], rows, scale)
            out[b, h], lse[b, h] = o[0], l[0]
    return {"q_codes": qc, "idx": idx, "dist": dist, "out": out, "lse": lse}


def decode_step_ragged(q, K, V, k_codes, n_tokens_b, n_sink: int, n_local: int, top_k: int,
                       kind: str, q_params=None, scale: float | None = None):
    """decode_step for a batch whose sequence b holds n_tokens_b[b] tokens:
    each sequence has its own sink, local window and candidates.  Returns the
    per-sequence results stacked along the batch."""
    parts = [decode_step(q[b:b + 1], K[b:b + 1], V[b:b + 1], k_codes[b:b + 1], int(n_tokens_b[b]), n_sink,
                         n_local, top_k, kind, q_params, scale) for b in range(len(n_tokens_b))]
    return {key: np.concatenate([r[key] for r in parts], axis=0) for key in ("q_codes", "idx", "dist", "out", "lse")}


def gather_pages(pool, page_table, page_size: int, N: int):
    """A paged cache read back in token order (the paged layout is this
    library's storage choice; the pages say nothing about it).  pool
    [num_pages, Hkv, page_size, ...] holds page j of sequence b at
    pool[page_table[b, j]]; token t of sequence b is slot t % page_size of
    page t // page_size.  Returns [B, Hkv, N, ...], one explicit copy per
    token, so that every other oracle function applies unchanged."""
    table = np.asarray(page_table, dtype=np.int64)
    B = table.shape[0]
    is_torch = hasattr(pool, "detach")
    if is_torch:
        import torch
        out = torch.empty((B, pool.shape[1], N) + tuple(pool.shape[3:]), dtype=pool.dtype)
    else:
        pool = np.asarray(pool)
        out = np.empty((B, pool.shape[1], N) + pool.shape[3:], dtype=pool.dtype)
    for b in range(B):
        for t in range(N):
            out[b, :, t] = pool[int(table[b, t // page_size]), :, t % page_size]
    return out
