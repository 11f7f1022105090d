"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
the step time is the maximum over ranks and the job value counts every
rank's work (weak scaling, one replica per rank)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms_local = [2.0, 3.5][rank]
        value, ms = bench.job_throughput(1000.0, ms_local, world, torch.device("cpu"))
        bench.barrier(world)
        q.put((rank, value, ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms in results:
        assert ms == pytest.approx(3.5)
        assert value == pytest.approx(1000.0 * 2 / 3.5e-3)


def test_single_rank_needs_no_process_group():
    import bench
    value, ms = bench.job_throughput(500.0, 4.0, 1, torch.device("cpu"))
    assert ms == 4.0 and value == pytest.approx(500.0 / 4e-3)


# ------------------------------------------------------- token-split protocol

class _OracleOps:
    """The five steps of a token-split rank written with the oracle on CPU
    tensors, so that the exchange protocol (ranges, windows, gathers, merge)
    runs under gloo without a GPU."""

    def __init__(self, R):
        self.R = R

    @staticmethod
    def _u32(t):
        import numpy as np
        return t.numpy().view(np.uint32)

    def encode_queries(self, h, q, q_codes):
        import numpy as np
        import oracle
        q_codes.copy_(torch.from_numpy(oracle.encode("lsh", q, self.R).view(np.int32)))

    def retrieve(self, q_codes, k_codes, n, sink, local, idx, dist_, ws, status):
        import oracle
        i, d = oracle.retrieve(self._u32(q_codes), self._u32(k_codes), n, sink, local, idx.shape[-1])
        idx.copy_(torch.from_numpy(i).to(torch.int32))
        dist_.copy_(torch.from_numpy(d).to(torch.int32))

    def select(self, rank, Hq, code_bits, cand_idx, cand_dist, idx, status):
        # the sequence's top-k: smallest distance, then rank, then position
        G, B, Hkv, k = cand_idx.shape
        idx.fill_(-1)
        for b in range(B):
            for j in range(Hkv):
                c = [(int(cand_dist[g, b, j, p]), g, p, int(cand_idx[g, b, j, p]))
                     for g in range(G) for p in range(k) if cand_idx[g, b, j, p] >= 0]
                mine = sorted(i for _, g, _, i in sorted(c)[:k] if g == rank)
                idx[b, j, : len(mine)] = torch.tensor(mine, dtype=torch.int32)

    def attend(self, q, K, V, n, idx, sink, local, out, lse, scale, ws, status):
        import oracle
        B, Hq, _ = q.shape
        Hkv = K.shape[1]
        g = Hq // Hkv
        for b in range(B):
            for j in range(Hkv):
                rows = oracle.attention_rows(n, sink, local, idx[b, j].numpy())
                o, l = oracle.attend(q[b, j * g:(j + 1) * g], K[b, j], V[b, j], rows, scale)
                out[b, j * g:(j + 1) * g] = torch.from_numpy(o)
                lse[b, j * g:(j + 1) * g] = torch.from_numpy(l)

    def merge(self, o, lse, out, lse_out):
        import oracle
        mo, ml = o[0].double().numpy(), lse[0].double().numpy()
        for g in range(1, o.shape[0]):
            mo, ml = oracle.lse_merge(mo, ml, o[g].numpy(), lse[g].numpy())
        out.copy_(torch.from_numpy(mo))
        if lse_out is not None:
            lse_out.copy_(torch.from_numpy(ml))


# B, Hq, Hkv, bits, N, sink, local, top_k
_SPLITS = {
    "short_window": (1, 4, 2, 64, 97, 3, 10, 20),
    "window_covers_ranks": (2, 4, 1, 64, 90, 30, 40, 8),  # the first and last ranges hold no candidates
}


def _split_inputs(shape):
    g = torch.Generator().manual_seed(11)
    B, Hq, Hkv, bits, N, _, _, _ = shape
    q = torch.randn(B, Hq, 128, generator=g, dtype=torch.float64)
    K = torch.randn(B, Hkv, N, 128, generator=g, dtype=torch.float64)
    V = torch.randn(B, Hkv, N, 128, generator=g, dtype=torch.float64)
    R = torch.randn(bits, 128, generator=g, dtype=torch.float64)
    return q, K, V, R


def _split_worker(rank, world, port, q_out, shape):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import oracle
        from hash_sparse_kv_b200 import split
        B, Hq, Hkv, bits, N, s, l, k = shape
        q, K, V, R = _split_inputs(shape)
        kc = torch.from_numpy(oracle.encode("lsh", K, R).view(np.int32))
        r0, r1 = split.token_range(N, world, rank)
        st = split.SplitState.make(world, rank, B, Hq, Hkv, bits, k, N, s, l, "cpu", workspaces=False)
        out = torch.zeros(B, Hq, 128)
        lse = torch.zeros(B, Hq)
        split.decode_step_split(st, None, q, kc[:, :, r0:r1].contiguous(), K[:, :, r0:r1], V[:, :, r0:r1], N, s, l,
                                bits, out, lse, ops=_OracleOps(R))
        sel = st.sel_idx.numpy().astype(np.int64)
        q_out.put((rank, np.where(sel >= 0, sel + r0, -1), out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, "short_window"), (3, "short_window"), (3, "window_covers_ranks"),
                                         (4, "window_covers_ranks")])
def test_token_split_protocol_equals_the_whole_sequence_step(world, shape):
    shape = _SPLITS[shape]
    import numpy as np
    import oracle
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q_out, shape)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q_out.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, Hq, Hkv, bits, N, s, l, k = shape
    q, K, V, R = _split_inputs(shape)
    ref = oracle.decode_step(q, K, V, oracle.encode("lsh", K, R), N, s, l, k, "lsh", R)
    for b in range(B):
        for j in range(Hkv):
            union = np.sort(np.concatenate([r[1][b, j][r[1][b, j] >= 0] for r in results]))
            want = ref["idx"][b, j]
            np.testing.assert_array_equal(union, want[want >= 0])
    for _, _, out, lse in results:  # every rank holds the merged result
        assert np.abs(out - ref["out"]).max() < 1e-5
        assert np.abs(lse - ref["lse"]).max() < 1e-5


def test_local_windows_partition_the_sequence():
    """For many splits the ranks' sink, candidate and local rows, shifted by
    their offsets, are exactly the sequence's sink, candidates and local rows."""
    import oracle
    from hash_sparse_kv_b200 import split
    for N in (1, 7, 100, 1001):
        for world in (1, 2, 3, 8):
            if world > N:
                continue
            for s, l in ((0, 0), (4, 16), (50, 60), (N, 0), (0, N), (N, N)):
                se, ls = oracle.candidate_range(N, s, l)
                got = {"sink": [], "cand": [], "local": []}
                for r in range(world):
                    r0, r1 = split.token_range(N, world, r)
                    ss, ll = split.local_window(N, s, l, r0, r1)
                    lse_, lls = oracle.candidate_range(r1 - r0, ss, ll)
                    got["sink"] += [r0 + t for t in range(0, lse_)]
                    got["cand"] += [r0 + t for t in range(lse_, lls)]
                    got["local"] += [r0 + t for t in range(lls, r1 - r0)]
                assert got["sink"] == list(range(0, se))
                assert got["cand"] == list(range(se, ls))
                assert got["local"] == list(range(ls, N))


def test_split_step_rejects_a_short_range():
    """A rank handed fewer tokens than its range fails before any exchange."""
    from hash_sparse_kv_b200 import split
    st = split.SplitState.make(2, 1, 1, 4, 2, 64, 8, 100, 0, 0, "cpu", workspaces=False)
    kc = torch.zeros(1, 2, 49, 2, dtype=torch.int32)  # rank 1 of 2 owns tokens [50, 100)
    K = torch.zeros(1, 2, 50, 128)
    with pytest.raises(ValueError, match="k_codes holds 49 tokens"):
        split.decode_step_split(st, None, torch.zeros(1, 4, 128), kc, K, K, 100, 0, 0, 64, torch.zeros(1, 4, 128))
