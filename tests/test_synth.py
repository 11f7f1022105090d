"""The seeded generators: determinism, slice independence, margin redraw."""
import numpy as np
import torch

import oracle
import synth


def test_cone_means_orthonormal():
    mu_k, mu_q, mu_v = synth.cone_means(4, 0, 128)
    for m in (mu_k, mu_q, mu_v):
        assert abs(np.linalg.norm(m) - 1) < 1e-12
    assert abs(np.dot(mu_k, mu_q)) < 1e-12


def test_layer_inputs_deterministic_and_shaped():
    w = synth.WORKLOADS["hashevict_lsh"].with_(B=2, N=300)
    a = synth.layer_inputs(w, cap=320)
    b = synth.layer_inputs(w, cap=320)
    assert a["q"].shape == (2, 32, 128) and a["K"].shape == (2, 8, 320, 128)
    assert a["K"].dtype == torch.bfloat16 and a["R"].shape == (64, 128)
    assert torch.equal(a["q"], b["q"]) and torch.equal(a["K"][:, :, :300], b["K"][:, :, :300])
    assert torch.isnan(a["K"][:, :, 300:].float()).all()


def test_margin_redraw_removes_small_presign_values():
    w = synth.WORKLOADS["tiny_lsh"].with_(N=2000)

    def bad(R):
        return lambda x: (np.abs(oracle.presign_lsh(x.reshape(-1, x.shape[-1]), R)) < 1e-3).any(axis=1)

    R = synth.gaussian_projection(synth.layer_seed(w, 0), 0, w.bits, w.d, w.dtype)
    inp = synth.layer_inputs(w, key_bad_rows=bad(R), query_bad_rows=bad(R))
    y = oracle.presign_lsh(inp["K"].reshape(-1, 128), inp["R"])
    assert np.abs(y).min() >= 1e-3
    plain = synth.layer_inputs(w)
    changed = (plain["K"] != inp["K"]).any(dim=-1).sum().item()
    assert 0 < changed < 0.1 * w.N  # a few percent of rows need a redraw


def test_algorithmic_bytes_of_long_context_case():
    w = synth.WORKLOADS["qwen7b_512k"]
    C = w.N - 4 - 128
    assert w.candidates() == C
    expect = 4 * C * 16 + 4 * (1024 + 132) * 128 * 2 * 2 + 28 * 128 * 2 + 28 * 128 * 4
    assert w.algorithmic_bytes() == expect
