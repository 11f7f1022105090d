"""Token-split decode on the GPU against the fp64 oracle.

G ranks are emulated one after another on one GPU: each holds a copy of its
own token range, and the two exchanges are copies of every rank's buffers.
No kernel waits on another.  The union of the ranks' selections must be the
oracle's index set for the whole sequence, bit for bit, and the merged
attention must match the oracle's decode step within ATOL."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from hash_sparse_kv_b200 import split
from tests.helpers import ATOL, margin_inputs, u32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _emulated_step(w, inp, G):
    B, Hq, Hkv, N, W, k = w.B, w.Hq, w.Hkv, w.N, w.words, w.top_k
    K, V, q = inp["K"][:, :, :N].to(DEV), inp["V"][:, :, :N].to(DEV), inp["q"].to(DEV)
    h = hkv.HashParams.lsh(inp["R"].to(DEV))
    codes = torch.zeros(B, Hkv, N, W, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, K.reshape(-1, 128), codes.view(-1, W))
    ops = split.LibraryOps()
    states, parts = [], []
    for r in range(G):
        r0, r1 = split.token_range(N, G, r)
        st = split.SplitState.make(G, r, B, Hq, Hkv, w.bits, k, N, w.n_sink, w.n_local, DEV)
        parts.append((codes[:, :, r0:r1].contiguous(), K[:, :, r0:r1].contiguous(), V[:, :, r0:r1].contiguous()))
        split.phase_candidates(ops, st, h, q, parts[r][0], N, w.n_sink, w.n_local)
        states.append(st)
    cand_idx = torch.stack([st.own_idx for st in states])
    cand_dist = torch.stack([st.own_dist for st in states])
    for st, (_, Kr, Vr) in zip(states, parts):
        st.cand_idx.copy_(cand_idx)
        st.cand_dist.copy_(cand_dist)
        split.phase_attend(ops, st, q, Kr, Vr, N, w.n_sink, w.n_local, w.bits, 1.0 / np.sqrt(128))
    all_out = torch.stack([st.part_out.view(B * Hq, 128) for st in states])
    all_lse = torch.stack([st.part_lse.view(B * Hq) for st in states])
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    states[0].all_out.copy_(all_out)
    states[0].all_lse.copy_(all_lse)
    split.phase_merge(ops, states[0], out, lse)
    torch.cuda.synchronize()
    for st in states:
        assert int(st.status.item()) == 0
    # the ranks' selections in global indices
    sel = []
    for r, st in enumerate(states):
        r0, _ = split.token_range(N, G, r)
        s = st.sel_idx.cpu().numpy().astype(np.int64)
        sel.append(np.where(s >= 0, s + r0, -1))
    union = np.full((B, Hkv, k), -1, dtype=np.int64)
    for b in range(B):
        for j in range(Hkv):
            u = np.sort(np.concatenate([s[b, j][s[b, j] >= 0] for s in sel]))
            union[b, j, : u.size] = u
    return {"codes": u32(codes), "q_codes": u32(states[0].q_codes), "idx": union, "out": out.cpu().numpy(),
            "lse": lse.cpu().numpy()}


CASES = [
    # workload overrides, G
    (dict(N=20011, layers=1), 2),
    (dict(N=20011, layers=1), 3),
    (dict(N=9001, layers=1), 8),
    (dict(N=700, layers=1, top_k=300), 4),               # short ranges; the top-k takes half the candidates
    (dict(N=5003, layers=1, n_sink=2000, n_local=2500), 3),  # ranks 0 and 2 hold only sink / local rows
]


@pytest.mark.parametrize("over,G", CASES)
def test_token_split_decode(over, G):
    w = synth.WORKLOADS["qwen7b_512k"].with_(**over)
    inp = margin_inputs(w, cap=w.N)
    got = _emulated_step(w, inp, G)
    kcodes = oracle.encode("lsh", inp["K"][:, :, :w.N], inp["R"])
    np.testing.assert_array_equal(got["codes"], kcodes)
    ref = oracle.decode_step(inp["q"], inp["K"], inp["V"], kcodes, w.N, w.n_sink, w.n_local, w.top_k, "lsh",
                             inp["R"])
    np.testing.assert_array_equal(got["q_codes"], ref["q_codes"])
    np.testing.assert_array_equal(got["idx"], ref["idx"])
    assert np.abs(got["out"] - ref["out"]).max() < ATOL
    assert np.abs(got["lse"] - ref["lse"]).max() < ATOL


def test_split_select_ties_across_ranks():
    """Hand-made candidate lists: the threshold distance is shared by tokens
    of three ranks, and the quota of ties goes to the lowest global index."""
    G, k = 3, 4
    # per rank: (local index, distance), ascending index, -1 past its k_eff
    ranks = [
        [(0, 5), (3, 7), (4, 7), (9, 2)],
        [(1, 7), (2, 1), (-1, 0), (-1, 0)],
        [(0, 7), (5, 7), (6, 3), (8, 7)],
    ]
    cand_idx = torch.tensor([[[[i for i, _ in r]]] for r in ranks], dtype=torch.int32, device=DEV)
    cand_dist = torch.tensor([[[[d for _, d in r]]] for r in ranks], dtype=torch.int32, device=DEV)
    # sequence order: rank 0 tokens, then rank 1, then rank 2 (global = (rank, local))
    flat = [(d, g, i) for g, r in enumerate(ranks) for i, d in r if i >= 0]
    best = sorted(flat)[:k]  # distances 1, 2, 3, then the first tie at 5
    for me in range(G):
        idx = torch.full((1, 1, k), -9, dtype=torch.int32, device=DEV)
        hkv.hkv_split_select(me, 1, 64, cand_idx, cand_dist, idx)
        want = sorted(i for _, g, i in best if g == me)
        np.testing.assert_array_equal(idx.cpu().numpy()[0, 0], want + [-1] * (k - len(want)))
    # with k = 6 the quota is two of the five tokens at distance 7: rank 0's t = 3, 4
    k6 = 6
    ci = torch.full((G, 1, 1, k6), -1, dtype=torch.int32, device=DEV)
    cd = torch.zeros((G, 1, 1, k6), dtype=torch.int32, device=DEV)
    ci[..., :k] = cand_idx
    cd[..., :k] = cand_dist
    best6 = sorted(flat)[:k6]
    for me in range(G):
        idx = torch.full((1, 1, k6), -9, dtype=torch.int32, device=DEV)
        hkv.hkv_split_select(me, 1, 64, ci, cd, idx)
        want = sorted(i for _, g, i in best6 if g == me)
        np.testing.assert_array_equal(idx.cpu().numpy()[0, 0], want + [-1] * (k6 - len(want)))


@pytest.mark.parametrize("G", [1, 3, 8])
def test_lse_merge_n(G):
    rng = np.random.default_rng(G)
    rows = 37
    o = rng.standard_normal((G, rows, 128)).astype(np.float32)
    lse = rng.uniform(-3, 3, size=(G, rows)).astype(np.float32)
    lse[:, 0] = -np.inf           # a row with only empty parts
    lse[0, 1:5] = -np.inf         # some empty parts
    out = torch.full((rows, 128), float("nan"), device=DEV)
    lse_out = torch.full((rows,), float("nan"), device=DEV)
    hkv.hkv_lse_merge_n(torch.from_numpy(o).to(DEV), torch.from_numpy(lse).to(DEV), out, lse_out)
    want_o, want_l = o[0].astype(np.float64), lse[0].astype(np.float64)
    for g in range(1, G):
        want_o, want_l = oracle.lse_merge(want_o, want_l, o[g], lse[g])
    if G == 1:
        want_o = np.where(np.isneginf(want_l)[:, None], 0.0, want_o)
    got_o, got_l = out.cpu().numpy(), lse_out.cpu().numpy()
    assert np.abs(got_o - want_o).max() < 1e-5
    fin = np.isfinite(want_l)
    assert np.abs(got_l[fin] - want_l[fin]).max() < 1e-5
    assert np.isneginf(got_l[~fin]).all()
