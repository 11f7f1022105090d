"""Informational check of the method on the synthetic inputs (not a parity
gate): the hashed top-k overlaps the exact top-k by group-summed inner
product (the pages' IoU measure, Spotlight Attention "Key results") well
above the overlap of a random choice.  The hashes are random, not trained,
so the overlap stays far below the pages' trained figures; what this guards
against is a retrieval that no longer tracks q . k at all (a sign slip in an
encoder, a reversed selection order)."""
import numpy as np
import pytest

import oracle
import synth


def _iou(a, b):
    a, b = set(a[a >= 0].tolist()), set(b[b >= 0].tolist())
    return len(a & b) / max(1, len(a | b))


@pytest.mark.parametrize("name,N", [("qwen7b_512k", 8192), ("signvq", 4096)])
def test_hashed_topk_tracks_the_exact_topk(name, N):
    w = synth.WORKLOADS[name].with_(N=N, B=1, layers=1)
    inp = synth.layer_inputs(w, 0, pad_junk=False)
    q, K = inp["q"], inp["K"]
    g = w.Hq // w.Hkv
    qf, Kf = oracle.as_f64(q), oracle.as_f64(K)
    lo, hi = oracle.candidate_range(N, w.n_sink, w.n_local)
    if w.hash == "lsh":
        kc, qc = oracle.encode("lsh", K, inp["R"]), oracle.encode("lsh", q, inp["R"])
        picks = [oracle.retrieve(qc, kc, N, w.n_sink, w.n_local, w.top_k)[0]]
    else:
        (kc, kn), (qc, _) = oracle.encode("sign", K), oracle.encode("sign", q)
        picks = [oracle.retrieve(qc, kc, N, w.n_sink, w.n_local, w.top_k)[0],
                 oracle.retrieve_normw(qc, kc, kn, N, w.n_sink, w.n_local, w.top_k)[0]]
    chance = w.top_k / (2 * (hi - lo) - w.top_k)  # expected IoU of two independent random k-subsets
    for idx in picks:
        ious = []
        for j in range(w.Hkv):
            s = (qf[0, j * g:(j + 1) * g] @ Kf[0, j].T).sum(axis=0)
            ious.append(_iou(idx[0, j], oracle.select_topk(-s, lo, hi, w.top_k)))
        assert np.mean(ious) > 2 * chance, (name, np.mean(ious), chance)
