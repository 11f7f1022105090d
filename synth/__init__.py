"""Seeded synthetic workloads for hash-code KV retrieval.

This module only draws random numbers and lays them out.  It holds none of the
retrieval method's arithmetic: no projection, no hash, no distance, no softmax.
Where a workload needs every pre-sign value to keep a margin from zero, the
caller passes a predicate (``bad_rows``) that flags rows to redraw; the
predicate is computed elsewhere.

Distributions (two narrow cones, as the Spotlight Attention page's "Problem"
paragraph describes queries and keys; RetrievalAttention's summary reports the
same query/key distribution gap):
  mu_k = normalize(g1);  mu_q = normalize(g2 - (g2 . mu_k) mu_k)  (unit, mu_q _|_ mu_k)
  k = mu_k + 0.3 z,  q = mu_q + 0.3 z,  v = mu_v + 0.3 z  (z ~ N(0, I), fresh per row)
One (mu_k, mu_q, mu_v) triple per layer.  Values are rounded to bfloat16 for the
bf16 workloads (round to nearest even), and kept fp32 otherwise.

Hash parameters are inputs to the method, drawn here:
  LSH: R[bits, d] ~ N(0, 1)  (HashEvict's "binarized Gaussian projections"),
       rounded to bf16 for bf16 workloads so tensor-core products are exact.
  MLP: W1[hidden, d], b1[hidden], W2[bits, hidden], b2[bits] ~ U(-1/sqrt(fan_in),
       +1/sqrt(fan_in)) (the default init of a linear layer), rounded to
       bf16-representable values and stored fp32.  One MLP for queries and a
       separate one for keys (Spotlight Attention, "Approach").

Every draw comes from a Philox stream keyed by (seed, layer, tensor, chunk,
attempt), so any slice regenerates independently of the others.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Optional

import numpy as np
import torch

# Tensor identifiers used in the Philox keys.
_T_MU, _T_Q, _T_K, _T_V, _T_R, _T_MLPQ, _T_MLPK, _T_CODES, _T_JUNK = range(1, 10)
_CHUNK_ROWS = 1 << 16
_REDRAW_BASE = 1 << 20


@dataclasses.dataclass(frozen=True)
class Workload:
    """One decode-step workload: shapes, hash family, budgets and seed."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    dtype: str  # "f32" or "bf16": dtype of q, K and V
    hash: str  # "lsh", "mlp" or "sign"
    bits: int
    hidden: int
    top_k: int
    n_sink: int
    n_local: int
    layers: int
    seed: int

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def words(self) -> int:
        return self.bits // 32

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def candidates(self) -> int:
        sink_end = min(self.n_sink, self.N)
        local_start = max(sink_end, self.N - self.n_local)
        return local_start - sink_end

    def algorithmic_bytes(self) -> int:
        """Bytes one decode step must move per layer: candidate codes scanned,
        sink/local/selected K and V rows gathered, q read and fp32 out written."""
        elt = 4 if self.dtype == "f32" else 2
        C = self.candidates()
        k_eff = min(self.top_k, C)
        rows = k_eff + (self.N - C)
        pairs = self.B * self.Hkv
        codes = pairs * C * self.bits // 8
        kv = pairs * rows * self.d * 2 * elt
        q = self.B * self.Hq * self.d * elt
        out = self.B * self.Hq * self.d * 4
        return codes + kv + q + out


# The five workloads.  Seeds: 0 for the tiny case; 1..4 for the others
# (layer L of the 28-layer case uses seed 4000 + L).
WORKLOADS = {
    "tiny_lsh": Workload("tiny_lsh", 1, 1, 1, 128, 4096, "f32", "lsh", 128, 0, 64, 0, 0, 1, 0),
    "hashevict_lsh": Workload("hashevict_lsh", 8, 32, 8, 128, 32768, "bf16", "lsh", 64, 0, 1024, 4, 64, 1, 1),
    "spotlight_mlp": Workload("spotlight_mlp", 1, 32, 8, 128, 131072, "bf16", "mlp", 128, 512, 2621, 4, 64, 1, 2),
    "signvq": Workload("signvq", 16, 32, 8, 128, 65536, "bf16", "sign", 128, 0, 512, 0, 0, 1, 3),
    "qwen7b_512k": Workload("qwen7b_512k", 1, 28, 4, 128, 524288, "bf16", "lsh", 128, 0, 1024, 4, 128, 28, 4),
}


def layer_seed(w: Workload, layer: int) -> int:
    return w.seed * 1000 + layer if w.layers > 1 else w.seed


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([int(k) for k in key])))


def _store(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _normal_rows(seed: int, layer: int, tensor: int, n_rows: int, d: int) -> np.ndarray:
    out = np.empty((n_rows, d), dtype=np.float32)
    for c0 in range(0, n_rows, _CHUNK_ROWS):
        c1 = min(n_rows, c0 + _CHUNK_ROWS)
        out[c0:c1] = _rng(seed, layer, tensor, c0 // _CHUNK_ROWS, 0).standard_normal((c1 - c0, d), dtype=np.float32)
    return out


def cone_means(seed: int, layer: int, d: int):
    """Unit means (mu_k, mu_q, mu_v) with mu_q orthogonal to mu_k."""
    g = _rng(seed, layer, _T_MU, 0, 0).standard_normal((3, d))
    mu_k = g[0] / np.linalg.norm(g[0])
    gq = g[1] - np.dot(g[1], mu_k) * mu_k
    mu_q = gq / np.linalg.norm(gq)
    mu_v = g[2] / np.linalg.norm(g[2])
    return mu_k, mu_q, mu_v


BadRows = Callable[[torch.Tensor], np.ndarray]


def cone_rows(seed: int, layer: int, tensor: int, mu: np.ndarray, n_rows: int, dtype: str,
              bad_rows: Optional[BadRows] = None, max_attempts: int = 200) -> torch.Tensor:
    """n_rows vectors mu + 0.3 z in the storage dtype.  Rows flagged by
    ``bad_rows`` (called on the stored values) are redrawn from a fresh stream
    until none is flagged."""
    d = mu.shape[0]
    x = _normal_rows(seed, layer, tensor, n_rows, d)
    x *= np.float32(0.3)
    x += mu.astype(np.float32)
    t = _store(x, dtype)
    if bad_rows is None:
        return t
    bad = np.flatnonzero(bad_rows(t))
    for attempt in range(1, max_attempts + 1):
        if bad.size == 0:
            return t
        z = _rng(seed, layer, tensor, _REDRAW_BASE + attempt, 0).standard_normal((bad.size, d), dtype=np.float32)
        rows = torch.from_numpy(bad)
        t[rows] = _store(mu.astype(np.float32) + np.float32(0.3) * z, dtype)
        bad = bad[np.asarray(bad_rows(t[rows]), dtype=bool)]
    raise RuntimeError(f"margin redraw did not converge for tensor {tensor}")


def gaussian_projection(seed: int, layer: int, bits: int, d: int, dtype: str) -> torch.Tensor:
    """R[bits, d] ~ N(0, 1), stored in the workload dtype."""
    r = _rng(seed, layer, _T_R, 0, 0).standard_normal((bits, d), dtype=np.float32)
    return _store(r, dtype)


def _bf16_exact_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32)


def mlp_params(seed: int, layer: int, side: str, d: int, hidden: int, bits: int):
    """(W1, b1, W2, b2) for the q-side (side="q") or k-side (side="k") hash MLP."""
    g = _rng(seed, layer, _T_MLPQ if side == "q" else _T_MLPK, 0, 0)
    a1, a2 = 1.0 / math.sqrt(d), 1.0 / math.sqrt(hidden)
    W1 = g.uniform(-a1, a1, (hidden, d))
    b1 = g.uniform(-a1, a1, (hidden,))
    W2 = g.uniform(-a2, a2, (bits, hidden))
    b2 = g.uniform(-a2, a2, (bits,))
    return tuple(_bf16_exact_f32(a) for a in (W1, b1, W2, b2))


def random_codes(seed: int, n_rows: int, words: int) -> torch.Tensor:
    """Uniform random packed codes, uint32 words stored in an int32 tensor."""
    g = _rng(seed, 0, _T_CODES, 0, 0)
    return torch.from_numpy(g.integers(0, 1 << 32, (n_rows, words), dtype=np.uint64).astype(np.uint32).view(np.int32))


def junk_fill(t: torch.Tensor, seed: int) -> None:
    """Fill a tensor with canary values: NaN for floats, random bits for ints."""
    if t.dtype.is_floating_point:
        t.fill_(float("nan"))
    else:
        g = _rng(seed, 0, _T_JUNK, 0, 0)
        t.copy_(torch.from_numpy(g.integers(-(1 << 31), 1 << 31, t.numel(), dtype=np.int64).astype(np.int32)).view(t.shape).to(t.dtype))


def layer_inputs(w: Workload, layer: int = 0, cap: Optional[int] = None,
                 key_bad_rows: Optional[BadRows] = None, query_bad_rows: Optional[BadRows] = None,
                 pad_junk: bool = True) -> dict:
    """All host tensors of one layer of a workload.

    Returns q [B,Hq,d], K and V [B,Hkv,cap,d] (rows >= N hold canaries), and the
    hash parameters: R [bits,d] for LSH; q_mlp and k_mlp tuples for MLP.
    ``key_bad_rows`` / ``query_bad_rows`` flag rows whose pre-sign values lie
    too close to zero; those rows are redrawn.
    """
    cap = w.N if cap is None else cap
    seed = layer_seed(w, layer)
    mu_k, mu_q, mu_v = cone_means(seed, layer, w.d)
    pairs = w.B * w.Hkv
    out = {"workload": w, "layer": layer, "cap": cap}
    if w.hash == "lsh":
        out["R"] = gaussian_projection(seed, layer, w.bits, w.d, w.dtype)
    elif w.hash == "mlp":
        out["q_mlp"] = mlp_params(seed, layer, "q", w.d, w.hidden, w.bits)
        out["k_mlp"] = mlp_params(seed, layer, "k", w.d, w.hidden, w.bits)
    q = cone_rows(seed, layer, _T_Q, mu_q, w.B * w.Hq, w.dtype, query_bad_rows)
    out["q"] = q.view(w.B, w.Hq, w.d)
    k = cone_rows(seed, layer, _T_K, mu_k, pairs * w.N, w.dtype, key_bad_rows)
    v = cone_rows(seed, layer, _T_V, mu_v, pairs * w.N, w.dtype, None)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    K = torch.empty(pairs, cap, w.d, dtype=tdt)
    V = torch.empty(pairs, cap, w.d, dtype=tdt)
    K[:, : w.N] = k.view(pairs, w.N, w.d)
    V[:, : w.N] = v.view(pairs, w.N, w.d)
    if cap > w.N:
        if pad_junk:
            K[:, w.N:] = float("nan")
            V[:, w.N:] = float("nan")
        else:
            K[:, w.N:] = 0
            V[:, w.N:] = 0
    out["K"] = K.view(w.B, w.Hkv, cap, w.d)
    out["V"] = V.view(w.B, w.Hkv, cap, w.d)
    return out


def device_layer_inputs(w: Workload, layer: int, device, cap: Optional[int] = None) -> dict:
    """Bench-scale inputs drawn directly on the device with torch's Philox
    generator (same distributions, no margin redraw; used for timing only)."""
    cap = w.N if cap is None else cap
    seed = layer_seed(w, layer)
    mu_k, mu_q, mu_v = (torch.from_numpy(m).to(device=device, dtype=torch.float32) for m in cone_means(seed, layer, w.d))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 7919 + 17)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    pairs = w.B * w.Hkv

    def cone(mu, n):
        out = torch.empty(n, w.d, dtype=tdt, device=device)
        step = 1 << 22
        for r0 in range(0, n, step):
            r1 = min(n, r0 + step)
            z = torch.randn(r1 - r0, w.d, generator=gen, device=device, dtype=torch.float32)
            out[r0:r1] = (mu + 0.3 * z).to(tdt)
        return out

    out = {"workload": w, "layer": layer, "cap": cap}
    if w.hash == "lsh":
        out["R"] = gaussian_projection(seed, layer, w.bits, w.d, w.dtype).to(device)
    elif w.hash == "mlp":
        out["q_mlp"] = tuple(t.to(device) for t in mlp_params(seed, layer, "q", w.d, w.hidden, w.bits))
        out["k_mlp"] = tuple(t.to(device) for t in mlp_params(seed, layer, "k", w.d, w.hidden, w.bits))
    out["q"] = cone(mu_q, w.B * w.Hq).view(w.B, w.Hq, w.d)
    K = torch.zeros(pairs, cap, w.d, dtype=tdt, device=device)
    V = torch.zeros(pairs, cap, w.d, dtype=tdt, device=device)
    K[:, : w.N] = cone(mu_k, pairs * w.N).view(pairs, w.N, w.d)
    V[:, : w.N] = cone(mu_v, pairs * w.N).view(pairs, w.N, w.d)
    out["K"] = K.view(w.B, w.Hkv, cap, w.d)
    out["V"] = V.view(w.B, w.Hkv, cap, w.d)
    return out
