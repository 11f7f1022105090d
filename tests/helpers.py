"""Shared helpers for the parity tests: oracle-based margin predicates and
input construction.  Only tests use this module."""
import numpy as np
import torch

import oracle
import synth

MARGIN = 1e-3  # no pre-sign value within this distance of zero
ATOL = 2e-3    # max abs error of attention outputs against the fp64 oracle
_CHUNK = 1 << 17


def _chunked(fn):
    def bad(x):
        x = x.reshape(-1, x.shape[-1])
        out = np.zeros(x.shape[0], dtype=bool)
        for r0 in range(0, x.shape[0], _CHUNK):
            out[r0:r0 + _CHUNK] = (np.abs(fn(x[r0:r0 + _CHUNK])) < MARGIN).any(axis=1)
        return out
    return bad


def lsh_bad(R):
    return _chunked(lambda x: oracle.presign_lsh(x, R))


def mlp_bad(params):
    return _chunked(lambda x: oracle.presign_mlp(x, *params))


def sign_bad():
    return _chunked(oracle.presign_sign)


def hash_params(w: synth.Workload, layer: int = 0):
    seed = synth.layer_seed(w, layer)
    if w.hash == "lsh":
        R = synth.gaussian_projection(seed, layer, w.bits, w.d, w.dtype)
        return {"R": R}, lsh_bad(R), lsh_bad(R)
    if w.hash == "mlp":
        qp = synth.mlp_params(seed, layer, "q", w.d, w.hidden, w.bits)
        kp = synth.mlp_params(seed, layer, "k", w.d, w.hidden, w.bits)
        return {"q_mlp": qp, "k_mlp": kp}, mlp_bad(qp), mlp_bad(kp)
    return {}, sign_bad(), sign_bad()


def margin_inputs(w: synth.Workload, layer: int = 0, cap=None) -> dict:
    """Host inputs of one layer with every pre-sign value at least MARGIN from zero."""
    _, qbad, kbad = hash_params(w, layer)
    return synth.layer_inputs(w, layer, cap, key_bad_rows=kbad, query_bad_rows=qbad)


def oracle_params(w: synth.Workload, inp: dict, side: str):
    if w.hash == "lsh":
        return inp["R"]
    if w.hash == "mlp":
        return inp["q_mlp" if side == "q" else "k_mlp"]
    return None


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)
