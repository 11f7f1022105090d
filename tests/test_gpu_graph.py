"""The decode step inside a CUDA graph: replays give the results of eager
calls (the workspace returns its counters and histograms to zero each call,
so one capture can be replayed any number of times)."""
import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import synth
from tests.helpers import margin_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("name,over", [("qwen7b_512k", dict(N=20011, layers=1)), ("hashevict_lsh", dict(B=2, N=5003)),
                                       ("signvq", dict(B=2, N=5001))])
def test_graph_replays_match_eager_calls(name, over):
    w = synth.WORKLOADS[name].with_(**over)
    inp = margin_inputs(w)
    B, Hq, Hkv, N, W = w.B, w.Hq, w.Hkv, w.N, w.words
    K, V, q = inp["K"].to(DEV), inp["V"].to(DEV), inp["q"].to(DEV)
    if w.hash == "lsh":
        h = hkv.HashParams.lsh(inp["R"].to(DEV))
    else:
        h = hkv.HashParams.sign(hkv.HKV_BF16)
    codes = torch.zeros(B, Hkv, N, W, dtype=torch.int32, device=DEV)
    hkv.hkv_encode_keys(h, K.view(-1, 128), codes.view(-1, W))
    ws = hkv.workspace(B, Hq, Hkv, N, w.bits, w.top_k, w.n_sink, w.n_local)
    st = hkv.status_word()

    def run(out, idx):
        hkv.hkv_decode_step(h, q, codes, K, V, N, w.n_sink, w.n_local, w.top_k, out, idx=idx, ws=ws, status=st)

    out_e = torch.zeros(B, Hq, 128, device=DEV)
    idx_e = torch.zeros(B, Hkv, w.top_k, dtype=torch.int32, device=DEV)
    run(out_e, idx_e)
    torch.cuda.synchronize()
    out_g = torch.zeros_like(out_e)
    idx_g = torch.zeros_like(idx_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(out_g, idx_g)  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(out_g, idx_g)
    for _ in range(3):
        out_g.zero_()
        idx_g.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
        np.testing.assert_array_equal(idx_g.cpu().numpy(), idx_e.cpu().numpy())
        assert torch.equal(out_g, out_e)
