"""CPU oracle for the tile-hybrid (dense / 2:4) Wanda-masked linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``sparse_gemm_wanda_b200``) never imports it and the
two share no code.

Every function here is a thin ``ctypes`` call into ``patch_oracle.c`` (plain C,
fp64, built with ``-ffp-contract=off``), whose header comment cites the pages
each step follows.  Arrays are numpy; bf16 tensors travel as their ``uint16``
bit patterns.

Pins (tests/test_oracle.py) tie each function to closed forms, brute force and
invariants; see the header of that file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "patch_oracle.c")
_LIB = os.path.join(_HERE, "libpatch_oracle.so")
_lib = None

COLSQ_CHUNK = 128  # tokens per fixed-order chunk of the column sum of squares


def build(force: bool = False) -> str:
    """Compile patch_oracle.c into libpatch_oracle.so (gcc, OpenMP, no FMA)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared",
               "-fPIC", "-std=c11", _SRC, "-o", _LIB, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        sig = {
            "oracle_colsq": [p, i64, i64, i64, p],
            "oracle_wanda_scores": [p, p, i64, i64, p],
            "oracle_select_2of4": [p, i64, i64, p],
            "oracle_tile_loss": [p, p, i64, i64, i64, i64, p],
            "oracle_n_sparse": [ctypes.c_double, i64],
            "oracle_select_map": [p, i64, i64, p],
            "oracle_select_maps_global": [p, p, i64, i64, p, p],
            "oracle_weff": [p, p, p, i64, i64, i64, i64, p],
            "oracle_pack_bytes": [p, i64, i64, i64, i64],
            "oracle_pack": [p, p, p, i64, i64, i64, i64, p, p],
            "oracle_unpack": [p, p, i64, i64, p],
            "oracle_gemm": [p, p, i64, i64, i64, p],
            "oracle_gemm_at": [p, p, i64, p, p, i64, p],
            "oracle_select_4of8": [p, i64, i64, p],
            "oracle_tile_loss_4of8": [p, p, i64, i64, i64, i64, p],
            "oracle_weff_4of8": [p, p, p, i64, i64, i64, i64, p],
            "oracle_pack_bytes_4of8": [p, i64, i64, i64, i64],
            "oracle_pack_4of8": [p, p, p, i64, i64, i64, i64, p, p],
            "oracle_unpack_4of8": [p, p, i64, i64, p],
            "oracle_e4m3_encode_array": [p, i64, p],
            "oracle_fp8_row_scales": [p, i64, i64, p],
            "oracle_fp8_quantize": [p, p, i64, i64, p],
            "oracle_gemm_fp8": [p, p, p, p, i64, i64, i64, p],
            "oracle_gemm_fp8_at": [p, p, p, p, i64, p, p, i64, p],
            "oracle_pack_bytes_fp8": [p, i64, i64, i64, i64],
            "oracle_pack_fp8": [p, p, p, i64, i64, i64, i64, p, p],
            "oracle_unpack_fp8": [p, p, i64, i64, p],
        }
        for name, args in sig.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = None
        _lib.oracle_n_sparse.restype = i64
        _lib.oracle_pack_bytes.restype = i64
        _lib.oracle_pack_bytes_4of8.restype = i64
        _lib.oracle_pack_bytes_fp8.restype = i64
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_ubyte]
        _lib.oracle_e4m3_decode.restype = ctypes.c_float
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, f"bf16 data must be passed as uint16 bits, got {a.dtype}"
    return a


def colsq(xcal_bits: np.ndarray, chunk: int = COLSQ_CHUNK) -> np.ndarray:
    """s[j] = sum_t x[t,j]^2 in the fixed chunked order (fp64)."""
    x = _u16(xcal_bits)
    T, K = x.shape
    s = np.empty(K, dtype=np.float64)
    _load().oracle_colsq(_ptr(x), T, K, chunk, _ptr(s))
    return s


def wanda_scores(w_bits: np.ndarray, s: np.ndarray) -> np.ndarray:
    """score[i,j] = |W[i,j]| * sqrt(s[j]) (fp64)."""
    w = _u16(w_bits)
    N, K = w.shape
    s = np.ascontiguousarray(s, dtype=np.float64)
    out = np.empty((N, K), dtype=np.float64)
    _load().oracle_wanda_scores(_ptr(w), _ptr(s), N, K, _ptr(out))
    return out


def select_2of4(score: np.ndarray) -> np.ndarray:
    """Top-2-of-4 codes, idx0 | idx1 << 2 per group, 8 groups per uint32 word."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    N, K = score.shape
    meta = np.empty((N, K // 32), dtype=np.uint32)
    _load().oracle_select_2of4(_ptr(score), N, K, _ptr(meta))
    return meta


def tile_loss(score: np.ndarray, meta: np.ndarray, tn: int, tk: int) -> np.ndarray:
    """Pruned Wanda score per tile: inside each 32-column word of a row left to
    right, the row's words left to right, then the tile's row sums as a balanced
    pairwise tree ((0,1), (2,3), ..., then pairs of those)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    N, K = score.shape
    out = np.empty((N // tn) * (K // tk), dtype=np.float64)
    _load().oracle_tile_loss(_ptr(score), _ptr(meta), N, K, tn, tk, _ptr(out))
    return out


def n_sparse(f: float, n_tiles: int) -> int:
    """floor(f * n_tiles)."""
    return int(_load().oracle_n_sparse(float(f), int(n_tiles)))


def select_map(loss: np.ndarray, n_sp: int) -> np.ndarray:
    """Bitmap of the n_sp tiles first in (loss asc, index asc) order."""
    loss = np.ascontiguousarray(loss, dtype=np.float64)
    n = loss.shape[0]
    out = np.zeros((n + 31) // 32, dtype=np.uint32)
    _load().oracle_select_map(_ptr(loss), n, int(n_sp), _ptr(out))
    return out


def select_maps_global(losses, fraction: float) -> list:
    """Per-matrix bitmaps of the floor(fraction * all tiles) tiles of least
    loss over ALL the matrices (ties: lower matrix, then lower tile)."""
    losses = [np.ascontiguousarray(l, dtype=np.float64) for l in losses]
    n = np.array([l.shape[0] for l in losses], dtype=np.int64)
    words = (n + 31) // 32
    woff = np.concatenate([[0], np.cumsum(words)[:-1]]).astype(np.int64)
    cat = np.ascontiguousarray(np.concatenate(losses)) if losses else np.zeros(0)
    out = np.zeros(int(words.sum()) + 1, dtype=np.uint32)
    n_sp = n_sparse(fraction, int(n.sum()))
    _load().oracle_select_maps_global(_ptr(cat), _ptr(n), len(losses), int(n_sp), _ptr(out), _ptr(woff))
    return [out[woff[m]:woff[m] + words[m]].copy() for m in range(len(losses))]


def weff(w_bits, meta, tile_map, tn: int, tk: int) -> np.ndarray:
    """Effective weight (bf16 bits): W on dense tiles, kept entries on 2:4 tiles."""
    w = _u16(w_bits)
    N, K = w.shape
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    out = np.empty_like(w)
    _load().oracle_weff(_ptr(w), _ptr(meta), _ptr(tile_map), N, K, tn, tk, _ptr(out))
    return out


def pack_bytes(tile_map, N: int, K: int, tn: int, tk: int) -> int:
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    return int(_load().oracle_pack_bytes(_ptr(tile_map), N, K, tn, tk))


def pack(w_bits, meta, tile_map, tn: int, tk: int):
    """Packed bytes (uint8) and k-step table (uint64) of the library's format."""
    w = _u16(w_bits)
    N, K = w.shape
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    nbytes = pack_bytes(tile_map, N, K, tn, tk)
    out = np.zeros(nbytes, dtype=np.uint8)
    table = np.zeros((N // 128) * (K // 64), dtype=np.uint64)
    _load().oracle_pack(_ptr(w), _ptr(meta), _ptr(tile_map), N, K, tn, tk, _ptr(out), _ptr(table))
    return out, table


def unpack(packed: np.ndarray, table: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    table = np.ascontiguousarray(table, dtype=np.uint64)
    out = np.zeros((N, K), dtype=np.uint16)
    _load().oracle_unpack(_ptr(packed), _ptr(table), N, K, _ptr(out))
    return out


def gemm(x_bits, weff_bits) -> np.ndarray:
    """y = X @ W_eff^T, naive triple loop, fp64 accumulation."""
    x = _u16(x_bits)
    w = _u16(weff_bits)
    M, K = x.shape
    N = w.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _load().oracle_gemm(_ptr(x), _ptr(w), M, N, K, _ptr(y))
    return y


def gemm_at(x_bits, weff_bits, ms, ns) -> np.ndarray:
    """The same sums at the listed (m, n) output positions only."""
    x = _u16(x_bits)
    w = _u16(weff_bits)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.empty(ms.shape[0], dtype=np.float64)
    _load().oracle_gemm_at(_ptr(x), _ptr(w), x.shape[1], _ptr(ms), _ptr(ns), ms.shape[0], _ptr(y))
    return y


def score_mask(w_bits, xcal_bits=None, tn: int = 128, tk: int = 128, fraction: float = 0.0,
               tile_map=None, colsq_in=None):
    """Steps 1-5 chained: returns dict(colsq, score, meta, loss, map)."""
    s = colsq(xcal_bits) if colsq_in is None else np.ascontiguousarray(colsq_in, dtype=np.float64)
    sc = wanda_scores(w_bits, s)
    meta = select_2of4(sc)
    loss = tile_loss(sc, meta, tn, tk)
    if tile_map is None:
        tile_map = select_map(loss, n_sparse(fraction, loss.shape[0]))
    return {"colsq": s, "score": sc, "meta": meta, "loss": loss,
            "map": np.ascontiguousarray(tile_map, dtype=np.uint32)}


# ---------------------------------------------------------------- 4:8 pattern

def select_4of8(score: np.ndarray) -> np.ndarray:
    """Top-4-of-8 keep masks (bit q = position q kept), 4 groups per uint32 word."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    N, K = score.shape
    meta = np.empty((N, K // 32), dtype=np.uint32)
    _load().oracle_select_4of8(_ptr(score), N, K, _ptr(meta))
    return meta


def tile_loss_4of8(score: np.ndarray, meta: np.ndarray, tn: int, tk: int) -> np.ndarray:
    """Pruned Wanda score per tile with the 4:8 kept set (same order as tile_loss)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    N, K = score.shape
    out = np.empty((N // tn) * (K // tk), dtype=np.float64)
    _load().oracle_tile_loss_4of8(_ptr(score), _ptr(meta), N, K, tn, tk, _ptr(out))
    return out


def weff_4of8(w_bits, meta, tile_map, tn: int, tk: int) -> np.ndarray:
    w = _u16(w_bits)
    N, K = w.shape
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    out = np.empty_like(w)
    _load().oracle_weff_4of8(_ptr(w), _ptr(meta), _ptr(tile_map), N, K, tn, tk, _ptr(out))
    return out


def pack_bytes_4of8(tile_map, N: int, K: int, tn: int, tk: int) -> int:
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    return int(_load().oracle_pack_bytes_4of8(_ptr(tile_map), N, K, tn, tk))


def pack_4of8(w_bits, meta, tile_map, tn: int, tk: int):
    """Packed bytes (uint8) and k-step table (uint64) of a 4:8 handle."""
    w = _u16(w_bits)
    N, K = w.shape
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    out = np.zeros(pack_bytes_4of8(tile_map, N, K, tn, tk), dtype=np.uint8)
    table = np.zeros((N // 128) * (K // 64), dtype=np.uint64)
    _load().oracle_pack_4of8(_ptr(w), _ptr(meta), _ptr(tile_map), N, K, tn, tk, _ptr(out), _ptr(table))
    return out, table


def unpack_4of8(packed: np.ndarray, table: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    table = np.ascontiguousarray(table, dtype=np.uint64)
    out = np.zeros((N, K), dtype=np.uint16)
    _load().oracle_unpack_4of8(_ptr(packed), _ptr(table), N, K, _ptr(out))
    return out


def score_mask_4of8(w_bits, xcal_bits=None, tn: int = 128, tk: int = 128, fraction: float = 0.0,
                    tile_map=None, colsq_in=None):
    """Steps 1-5 with 4:8 groups: dict(colsq, score, meta, loss, map)."""
    s = colsq(xcal_bits) if colsq_in is None else np.ascontiguousarray(colsq_in, dtype=np.float64)
    sc = wanda_scores(w_bits, s)
    meta = select_4of8(sc)
    loss = tile_loss_4of8(sc, meta, tn, tk)
    if tile_map is None:
        tile_map = select_map(loss, n_sparse(fraction, loss.shape[0]))
    return {"colsq": s, "score": sc, "meta": meta, "loss": loss,
            "map": np.ascontiguousarray(tile_map, dtype=np.uint32)}


# ------------------------------------------------------ FP8 (e4m3) values

def e4m3_encode(v) -> np.ndarray:
    """e4m3 codes (uint8) of fp32 values: nearest, ties to the even code, saturating at 448."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """fp32 values of e4m3 codes."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float32)
    return table[codes]


def fp8_row_scales(x_bits) -> np.ndarray:
    """fp32 scale per row of a bf16 matrix: amax / 448 (1 for a zero row)."""
    x = _u16(x_bits)
    R, C = x.shape
    out = np.empty(R, dtype=np.float32)
    _load().oracle_fp8_row_scales(_ptr(x), R, C, _ptr(out))
    return out


def fp8_quantize(x_bits, scale) -> np.ndarray:
    """e4m3 codes of x / scale[row] (the quotient in fp32)."""
    x = _u16(x_bits)
    R, C = x.shape
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    out = np.empty((R, C), dtype=np.uint8)
    _load().oracle_fp8_quantize(_ptr(x), _ptr(scale), R, C, _ptr(out))
    return out


def gemm_fp8(qx, sx, qw, sw) -> np.ndarray:
    """y = sx[m] sw[n] sum_k dec(qx) dec(qw), fp64, k in order."""
    qx = np.ascontiguousarray(qx, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = qx.shape
    N = qw.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _load().oracle_gemm_fp8(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), M, N, K, _ptr(y))
    return y


def gemm_fp8_at(qx, sx, qw, sw, ms, ns) -> np.ndarray:
    qx = np.ascontiguousarray(qx, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    y = np.empty(ms.shape[0], dtype=np.float64)
    _load().oracle_gemm_fp8_at(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), qx.shape[1], _ptr(ms), _ptr(ns),
                               ms.shape[0], _ptr(y))
    return y


def pack_fp8(qw, meta, tile_map, tn: int, tk: int):
    """Packed bytes and k-step table of an FP8 handle from the codes of W_eff."""
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    N, K = qw.shape
    meta = np.ascontiguousarray(meta, dtype=np.uint32)
    tile_map = np.ascontiguousarray(tile_map, dtype=np.uint32)
    nbytes = int(_load().oracle_pack_bytes_fp8(_ptr(tile_map), N, K, tn, tk))
    out = np.zeros(nbytes, dtype=np.uint8)
    table = np.zeros((N // 128) * (K // 128), dtype=np.uint64)
    _load().oracle_pack_fp8(_ptr(qw), _ptr(meta), _ptr(tile_map), N, K, tn, tk, _ptr(out), _ptr(table))
    return out, table


def unpack_fp8(packed, table, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    table = np.ascontiguousarray(table, dtype=np.uint64)
    out = np.zeros((N, K), dtype=np.uint8)
    _load().oracle_unpack_fp8(_ptr(packed), _ptr(table), N, K, _ptr(out))
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
