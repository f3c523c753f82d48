"""The multi-GPU split of the hot path (sparse_gemm_wanda_b200/sharded.py) on
CPU ranks: gloo process groups of 2 and 3 ranks.

The ranks run the module's own host logic (token and row splits, the two
all-gathers in rank order, the block-wide selection over the gathered tile
losses); the per-call arithmetic the CUDA library does on a GPU is done here
by the oracle on the CPU (a stand-in with the binding's call names).  Each
rank's column sums, codes, map slice and the gathered Y must be bit-identical
to the one-rank result of the same oracle on the whole problem.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_gemm_wanda_b200 import sharded

CHUNK = 128


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


class _Packed:
    def __init__(self, weff):
        self.weff = weff

    def close(self):
        pass


class OracleOps:
    """The binding's call names, computed by the CPU oracle (test stand-in)."""

    def __init__(self, oracle):
        self.o = oracle

    def patch_colsq_partials(self, xcal):
        b = _bits(xcal)
        parts = [self.o.colsq(np.ascontiguousarray(b[c:c + CHUNK])) for c in range(0, b.shape[0], CHUNK)]
        return torch.from_numpy(np.stack(parts))

    def patch_colsq_fold(self, partials):
        s = np.zeros(partials.shape[1])
        for p in partials.numpy():  # chunk order
            s = s + p
        return torch.from_numpy(s)

    def patch_score_mask(self, w, xcal, tile_n, tile_k, fraction, colsq_in, want_loss):
        ref = self.o.score_mask(_bits(w), None, tile_n, tile_k, fraction=fraction,
                                colsq_in=colsq_in.numpy())
        return {"meta": torch.from_numpy(ref["meta"].view(np.int32)),
                "map": torch.from_numpy(ref["map"].view(np.int32)),
                "loss": torch.from_numpy(ref["loss"])}

    def patch_select_maps_global(self, losses, fraction):
        maps = self.o.select_maps_global([l.numpy() for l in losses], fraction)
        return [torch.from_numpy(m.view(np.int32)) for m in maps]

    def patch_pack(self, w, meta, tmap, tile_n, tile_k):
        return _Packed(self.o.weff(_bits(w), meta.numpy().view(np.uint32),
                                   tmap.numpy().view(np.uint32), tile_n, tile_k))

    def patch_hybrid_gemm(self, pk, x):
        return torch.from_numpy(self.o.gemm(_bits(x), pk.weff))


def _problem(N, K, T, M):
    from sparse_gemm_wanda_b200 import inputs
    o = inputs.outlier_channels(K, 77, 3)
    w = inputs.weight(N, K, 77)
    xc = inputs.activations(T, K, 77, o, role=0)
    x = inputs.activations(M, K, 77, o, role=1)
    return w, xc, x


def _worker(rank, world, port, case, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        N, K, T, M, tn, tk, f = case
        w, xc, x = _problem(N, K, T, M)
        t0, t1 = sharded.token_ranges(T, world)[rank]
        n0, n1 = sharded.row_ranges(N, world)[rank]
        res = sharded.linear_sharded(OracleOps(oracle), w[n0:n1].contiguous(), N,
                                     xc[t0:t1].contiguous(), T, x, f, tn, tk)
        out[rank] = {k: v.numpy().copy() for k, v in res.items()}
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (512, 256, 300, 5, 64, 64, 0.4)),    # 3 chunks: 2 + 1; 4 bands: 2 + 2
    (3, (512, 384, 1000, 3, 128, 128, 0.5)), # 8 chunks: 3 + 3 + 2; 4 bands: 2 + 1 + 1
    (2, (256, 256, 100, 4, 64, 128, 0.75)),  # 1 chunk: rank 1 holds no tokens
])
def test_sharded_path_equals_one_rank(oracle_mod, world, case):
    N, K, T, M, tn, tk, f = case
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, case, out), nprocs=world, join=True,
                       start_method="spawn")
    w, xc, x = _problem(N, K, T, M)
    full = oracle_mod.score_mask(_bits(w), _bits(xc), tn, tk, fraction=f)
    weff = oracle_mod.weff(_bits(w), full["meta"], full["map"], tn, tk)
    y_full = oracle_mod.gemm(_bits(x), weff)
    tiles_k = K // tk
    for rank, (n0, n1) in enumerate(sharded.row_ranges(N, world)):
        r = out[rank]
        assert np.array_equal(r["colsq"], full["colsq"]), rank
        assert np.array_equal(r["meta"].view(np.uint32), full["meta"][n0:n1]), rank
        # the rank's map slice: its t-th tile is global tile n0/tn*tiles_k + t
        g0 = n0 // tn * tiles_k
        nt = (n1 - n0) // tn * tiles_k
        mine = r["map"].view(np.uint32)
        for t in range(nt):
            g = g0 + t
            assert ((int(mine[t // 32]) >> (t % 32)) & 1) == ((int(full["map"][g // 32]) >> (g % 32)) & 1)
        assert np.array_equal(r["y"], y_full), rank


def test_token_and_row_ranges():
    for T in (1, 127, 128, 129, 1000, 262144):
        for world in (1, 2, 3, 8):
            rs = sharded.token_ranges(T, world)
            assert rs[0][0] == 0 and rs[-1][1] == T
            for (a0, a1), (b0, b1) in zip(rs, rs[1:]):
                assert a1 == b0
            for t0, t1 in rs[:-1]:
                assert (t0 % CHUNK == 0 or t0 == T) and (t1 % CHUNK == 0 or t1 == T)
            chunks = [(t1 - t0 + CHUNK - 1) // CHUNK for t0, t1 in rs]
            assert max(chunks) - min(chunks) <= 1 and sum(chunks) == (T + CHUNK - 1) // CHUNK
    for N in (128, 512, 4096, 11008):
        for world in (1, 2, 3, 8):
            rs = sharded.row_ranges(N, world)
            assert rs[0][0] == 0 and rs[-1][1] == N
            assert all(a % 128 == 0 and b % 128 == 0 for a, b in rs)
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 128
    with pytest.raises(ValueError):
        sharded.row_ranges(100, 2)
