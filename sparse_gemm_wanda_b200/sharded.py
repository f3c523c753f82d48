"""Multi-GPU split of the hot path: one process per GPU, ``torch.distributed``.

One weight matrix W[N, K] and its calibration set Xcal[T, K] are split over
the ranks of a process group, and every rank ends up with exactly what one GPU
computes for its part:

* Column sums of squares.  The calibration tokens are split into consecutive
  pieces at multiples of 128 tokens (``token_ranges``).  Each rank computes the
  128-token chunk partials of its piece (``patch_colsq_partials``); the
  partials are all-gathered in rank order, which is token order, and every
  rank adds them in chunk order (``patch_colsq_fold``).  This is the fixed
  order of the one-GPU sums, so ``s`` is bit-identical.  An all-reduce would
  add the ranks' sums in an unspecified order and is therefore not used.
* Tile map.  The weight rows are split into consecutive runs of whole
  128-row bands (``row_ranges``); a rank's tiles are then a consecutive run of
  the row-major tile indices.  Each rank scores its rows
  (``patch_score_mask`` with the shared ``s``: codes and tile losses depend
  only on a tile's own rows and columns), the tile losses are all-gathered,
  and the floor(f * all tiles) tiles of least loss are chosen over all of them
  with ``patch_select_maps_global``, one "matrix" per rank in rank order.  Its
  ties go to the earlier matrix and then the lower tile, i.e. to the lower
  global tile index: each rank receives its own slice of the one-GPU map.
* Pack and GEMM need no exchange: each rank packs its rows and computes
  Y[:, its rows] = X * W_eff[its rows]^T.  ``gather_columns`` all-gathers the
  pieces along N when the consumer needs the whole Y (column-parallel layers
  can keep it split).

The two exchanges move 8 * K * ceil(T/128) bytes (1/32 of the calibration
bytes) and 8 bytes per tile; both are NCCL all-gathers over NVLink in a
multi-GPU job.  Source of the split: the path is data-parallel (rows of W are
independent outputs, "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs",
section 2, core mechanism: tiles chosen independently; the Wanda activation
term is a sum over calibration tokens, "SparseGPT vs Wanda", section on
Wanda).

``P`` is the binding module ``sparse_gemm_wanda_b200.patch`` (the CUDA
library); any object with the same call names works, which is how the CPU
tests drive this host logic with gloo ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

CHUNK = 128  # calibration tokens per chunk partial
BAND = 128   # weight rows per band of the packed format


def token_ranges(T: int, world: int) -> list:
    """Consecutive token pieces [t0, t1), one per rank, cut at multiples of 128.

    The chunks are dealt as evenly as possible (the first ranks take one more
    when they do not divide); the last piece may end in a partial chunk.  A
    rank may receive an empty piece when there are fewer chunks than ranks."""
    chunks = (T + CHUNK - 1) // CHUNK
    out = []
    c0 = 0
    for r in range(world):
        n = chunks // world + (1 if r < chunks % world else 0)
        t0, t1 = min(T, c0 * CHUNK), min(T, (c0 + n) * CHUNK)
        out.append((t0, t1))
        c0 += n
    return out


def row_ranges(N: int, world: int) -> list:
    """Consecutive row pieces [n0, n1), one per rank, each a run of whole
    128-row bands (N must be a multiple of 128)."""
    if N % BAND:
        raise ValueError("N must be a multiple of 128 to split in whole bands")
    bands = N // BAND
    out = []
    b0 = 0
    for r in range(world):
        n = bands // world + (1 if r < bands % world else 0)
        out.append((b0 * BAND, (b0 + n) * BAND))
        b0 += n
    return out


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def gather_rows(t: torch.Tensor, sizes: list, group=None) -> torch.Tensor:
    """All-gather along dim 0 in rank order; rank r holds sizes[r] rows.

    Pieces are padded to the largest size for the collective and trimmed after,
    so unequal pieces need no size exchange (every rank knows `sizes`)."""
    world, rank = _world(group)
    if t.shape[0] != sizes[rank]:
        raise ValueError(f"rank {rank} holds {t.shape[0]} rows, the split says {sizes[rank]}")
    big = max(sizes)
    pad = torch.zeros((big,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[: t.shape[0]] = t
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad, group=group)
    return torch.cat([b[:n] for b, n in zip(bufs, sizes)], dim=0)


def gather_columns(y: torch.Tensor, sizes: list, group=None) -> torch.Tensor:
    """All-gather Y[M, N_r] pieces along N (rank order) into Y[M, N]."""
    return gather_rows(y.t().contiguous(), sizes, group).t().contiguous()


def colsq_sharded(P, xcal_piece: torch.Tensor, T: int, group=None) -> torch.Tensor:
    """Column sums of squares of a calibration set split by token_ranges(T).

    `xcal_piece` is this rank's piece (rows t0..t1 of the set; it may be empty).
    Returns s[K] fp64 on every rank, bit-identical to patch_colsq on the whole
    set."""
    world, rank = _world(group)
    ranges = token_ranges(T, world)
    chunks = [(t1 - t0 + CHUNK - 1) // CHUNK for t0, t1 in ranges]
    K = xcal_piece.shape[1]
    if xcal_piece.shape[0] != ranges[rank][1] - ranges[rank][0]:
        raise ValueError("calibration piece does not match token_ranges")
    if chunks[rank]:
        part = P.patch_colsq_partials(xcal_piece)
    else:
        part = torch.zeros((0, K), dtype=torch.float64, device=xcal_piece.device)
    allp = gather_rows(part, chunks, group)
    return P.patch_colsq_fold(allp)


def mask_sharded(P, w_rows: torch.Tensor, N: int, colsq: torch.Tensor, fraction: float,
                 tile_n: int = 128, tile_k: int = 128, group=None) -> dict:
    """Codes and this rank's slice of the least-loss tile map of W[N, K], the
    rows split by row_ranges(N).

    Returns {"meta": codes of this rank's rows, "map": the map of this rank's
    tiles (bit t for its t-th tile), "loss": its tile losses}, each equal to
    the matching part of the one-GPU result."""
    world, rank = _world(group)
    ranges = row_ranges(N, world)
    n0, n1 = ranges[rank]
    if w_rows.shape[0] != n1 - n0:
        raise ValueError("weight rows do not match row_ranges")
    K = w_rows.shape[1]
    tiles_k = K // tile_k
    counts = [(b - a) // tile_n * tiles_k for a, b in ranges]
    r = P.patch_score_mask(w_rows, None, tile_n=tile_n, tile_k=tile_k, fraction=fraction,
                           colsq_in=colsq, want_loss=True)
    losses = gather_rows(r["loss"], counts, group)
    pieces, off = [], 0
    for c in counts:
        pieces.append(losses[off:off + c])
        off += c
    maps = P.patch_select_maps_global(pieces, fraction)
    return {"meta": r["meta"], "map": maps[rank], "loss": r["loss"]}


def linear_sharded(P, w_rows: torch.Tensor, N: int, xcal_piece: torch.Tensor, T: int,
                   x: torch.Tensor, fraction: float, tile_n: int = 128, tile_k: int = 128,
                   gather_y: bool = True, group=None) -> dict:
    """The whole path for one matrix over the ranks of `group`: column sums
    (token split), codes and map (row split), pack and GEMM of this rank's
    rows, and optionally the full Y.  Returns {"colsq", "meta", "map", "y"}."""
    world, rank = _world(group)
    s = colsq_sharded(P, xcal_piece, T, group)
    m = mask_sharded(P, w_rows, N, s, fraction, tile_n, tile_k, group)
    pk = P.patch_pack(w_rows, m["meta"], m["map"], tile_n=tile_n, tile_k=tile_k)
    y = P.patch_hybrid_gemm(pk, x)
    if gather_y:
        y = gather_columns(y, [b - a for a, b in row_ranges(N, world)], group)
    pk.close()
    return {"colsq": s, "meta": m["meta"], "map": m["map"], "y": y}
