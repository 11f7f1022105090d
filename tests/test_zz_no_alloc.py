"""The allocation-free retrieval entry point (hkv_retrieve_topk_static).

Some callers cannot allocate device memory -- their runtime's allocator owns
the GPU, or they are plugins handed buffers they may not add to -- so they
cannot pass a workspace.  hkv_retrieve_topk_static takes its scratch from a
fixed array inside the library instead.  These checks call it through the C
ABI and compare it with hkv_retrieve_topk (workspace version) on the same
inputs, twice in a row, since every call shares the array and relies on the
previous call having left its counters clean.  This file is collected last.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import hash_sparse_kv_b200 as hkv
import oracle
import synth
from tests.helpers import u32

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    # B, Hq, Hkv, bits, N, cap, sink, local, top_k
    (1, 28, 4, 128, 60001, 60001, 4, 128, 1024),   # several blocks per (batch, KV head): cross-block counters
    (2, 8, 2, 64, 5000, 5004, 4, 64, 300),
    (64, 64, 8, 128, 300, 300, 4, 16, 32),          # one block per (batch, KV head)
]


def _inputs(case):
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    W = bits // 32
    kc = synth.random_codes(91 + N, B * Hkv * cap, W).view(B, Hkv, cap, W).to(DEV)
    qc = synth.random_codes(92 + N, B * Hq, W).view(B, Hq, W).to(DEV)
    return qc, kc


@pytest.mark.parametrize("case", CASES)
def test_static_scratch_matches_workspace_version(case):
    B, Hq, Hkv, bits, N, cap, s, l, k = case
    qc, kc = _inputs(case)
    st = hkv.status_word()
    ws = hkv.workspace(B, Hq, Hkv, N, bits, k, s, l)
    ref_idx = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
    ref_dist = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
    hkv.hkv_retrieve_topk(qc, kc, N, s, l, k, ref_idx, ref_dist, ws=ws, status=st)
    assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
    # the workspace version itself against the oracle
    want_i, want_d = oracle.retrieve(u32(qc), u32(kc), N, s, l, k)
    np.testing.assert_array_equal(ref_idx.cpu().numpy(), want_i)
    np.testing.assert_array_equal(ref_dist.cpu().numpy(), want_d)
    for _ in range(2):
        idx = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
        dist = torch.full((B, Hkv, k), -9, dtype=torch.int32, device=DEV)
        hkv.hkv_retrieve_topk_static(qc, kc, N, s, l, k, idx, dist, status=st)
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx.cpu().numpy())
        np.testing.assert_array_equal(dist.cpu().numpy(), ref_dist.cpu().numpy())


def test_static_scratch_rejects_shapes_over_the_limit():
    # 4096 (batch, KV head) pairs with groups of 8: about 17 MB of scratch.  The
    # buffers have their full size, so nothing is out of bounds either way.
    B, Hq, Hkv, N, k = 512, 64, 8, 16384, 64
    qc = torch.zeros(B, Hq, 4, dtype=torch.int32, device=DEV)
    kc = torch.empty(B, Hkv, N, 4, dtype=torch.int32, device=DEV)
    idx = torch.zeros(B, Hkv, k, dtype=torch.int32, device=DEV)
    with pytest.raises(hkv.HkvError) as e:
        hkv.hkv_retrieve_topk_static(qc, kc, N, 0, 0, k, idx)
    assert e.value.code == hkv.HKV_ERR_CAPACITY and "static scratch" in str(e.value)
    del kc


# Run in a fresh process, so that the first call of the allocation-free entry
# point in that process is made on a non-blocking side stream (the case a
# set-up step on another stream would race with), then alternate a shape with
# several blocks per (batch, KV head) and one with a single block on two side
# streams, each checked against the workspace version.
_SIDE_STREAM = textwrap.dedent("""
    import sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    import hash_sparse_kv_b200 as hkv
    import synth

    cases = {cases!r}
    inputs, refs = [], []
    for (B, Hq, Hkv, bits, N, cap, s, l, k) in cases:
        W = bits // 32
        kc = synth.random_codes(91 + N, B * Hkv * cap, W).view(B, Hkv, cap, W).cuda()
        qc = synth.random_codes(92 + N, B * Hq, W).view(B, Hq, W).cuda()
        ws = hkv.workspace(B, Hq, Hkv, N, bits, k, s, l)
        ridx = torch.full((B, Hkv, k), -9, dtype=torch.int32, device="cuda")
        rdist = torch.full((B, Hkv, k), -9, dtype=torch.int32, device="cuda")
        hkv.hkv_retrieve_topk(qc, kc, N, s, l, k, ridx, rdist, ws=ws)
        inputs.append((qc, kc))
        refs.append((ridx.cpu().numpy(), rdist.cpu().numpy()))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    st = hkv.status_word()
    for it in range(4):
        j = it % len(cases)
        B, Hq, Hkv, bits, N, cap, s, l, k = cases[j]
        qc, kc = inputs[j]
        side = streams[it % 2]
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            idx = torch.full((B, Hkv, k), -9, dtype=torch.int32, device="cuda")
            dist = torch.full((B, Hkv, k), -9, dtype=torch.int32, device="cuda")
            hkv.hkv_retrieve_topk_static(qc, kc, N, s, l, k, idx, dist, status=st, stream=side)
        side.synchronize()
        assert hkv.hkv_check(st) == hkv.HKV_OK, hkv.hkv_last_error()
        np.testing.assert_array_equal(idx.cpu().numpy(), refs[j][0])
        np.testing.assert_array_equal(dist.cpu().numpy(), refs[j][1])
        # the next call runs on the other stream: order it after this one
        torch.cuda.current_stream().wait_stream(side)
    print("side streams ok")
""")


def test_static_scratch_first_call_on_a_side_stream():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = _SIDE_STREAM.format(root=root, cases=[CASES[0], CASES[2]])
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "side streams ok" in res.stdout
