"""Thin ctypes binding of ``libpatch_b200.so`` (include/patch.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  If the
library is missing or cannot be loaded, every call raises ``PatchLibraryError``;
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpatch_b200.so")

PATCH_OK = 0
STATUS_NAMES = {0: "PATCH_OK", 1: "PATCH_ERR_INVALID_ARG", 2: "PATCH_ERR_UNSUPPORTED",
                3: "PATCH_ERR_CUDA", 4: "PATCH_ERR_OOM", 5: "PATCH_ERR_TIMEOUT"}

# every symbol include/patch.h declares
EXPORTS = ("patch_score_mask", "patch_pack", "patch_hybrid_gemm", "patch_free",
           "patch_get_status", "patch_packed_info", "patch_packed_export",
           "patch_status_string", "patch_score_mask_noalloc",
           "patch_score_mask_noalloc_capacity", "patch_launch_count",
           "patch_select_maps_global", "patch_test_stall_first_kstep", "patch_pool_usage",
           "patch_colsq", "patch_colsq_partials", "patch_colsq_fold", "patch_test_prefill_kernel",
           "patch_score_mask_nm", "patch_pack_nm", "patch_pack_fp8", "patch_quantize_fp8",
           "patch_packed_fp8_scales", "patch_hybrid_gemm_group", "patch_pack_group")


class PatchLibraryError(RuntimeError):
    pass


class PatchError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


class PatchShape(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("tile_n", ctypes.c_int32), ("tile_k", ctypes.c_int32)]


class PatchPackedView(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("table", ctypes.c_void_p),
                ("packed_bytes", ctypes.c_size_t), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("tile_n", ctypes.c_int32), ("tile_k", ctypes.c_int32),
                ("sparse_ksteps", ctypes.c_int64), ("meta_blocks", ctypes.c_int64)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises PatchLibraryError when it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise PatchLibraryError(
            f"{path} is missing: build it with `python -m sparse_gemm_wanda_b200.build`")
    try:
        lib = ctypes.CDLL(path)
    except OSError as exc:
        raise PatchLibraryError(f"cannot load {path}: {exc}") from exc
    vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    lib.patch_score_mask.argtypes = [vp, vp, i64, vp, PatchShape, dbl, vp, vp, vp, vp, vp, vp]
    lib.patch_score_mask_noalloc.argtypes = [vp, vp, i64, vp, PatchShape, dbl, vp, vp, vp, vp, vp,
                                             vp]
    lib.patch_score_mask_noalloc.restype = ctypes.c_int
    lib.patch_score_mask_noalloc_capacity.argtypes = []
    lib.patch_score_mask_noalloc_capacity.restype = ctypes.c_size_t
    lib.patch_select_maps_global.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(i64), i32, dbl,
                                             ctypes.POINTER(vp), vp]
    lib.patch_select_maps_global.restype = ctypes.c_int
    lib.patch_launch_count.argtypes = []
    lib.patch_launch_count.restype = ctypes.c_uint64
    lib.patch_score_mask_nm.argtypes = [vp, vp, i64, vp, PatchShape, i32, i32, dbl, vp, vp, vp, vp,
                                        vp, vp]
    lib.patch_score_mask_nm.restype = ctypes.c_int
    lib.patch_pack_nm.argtypes = [vp, vp, vp, PatchShape, i32, i32, ctypes.POINTER(vp),
                                  ctypes.POINTER(ctypes.c_size_t), vp]
    lib.patch_pack_nm.restype = ctypes.c_int
    lib.patch_pack_fp8.argtypes = [vp, vp, vp, PatchShape, ctypes.POINTER(vp),
                                   ctypes.POINTER(ctypes.c_size_t), vp]
    lib.patch_pack_fp8.restype = ctypes.c_int
    lib.patch_quantize_fp8.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.patch_quantize_fp8.restype = ctypes.c_int
    lib.patch_packed_fp8_scales.argtypes = [vp, vp, vp]
    lib.patch_packed_fp8_scales.restype = ctypes.c_int
    lib.patch_colsq.argtypes = [vp, i64, i64, vp, vp]
    lib.patch_colsq_partials.argtypes = [vp, i64, i64, vp, vp]
    lib.patch_colsq_fold.argtypes = [vp, i64, i64, vp, vp]
    for name in ("patch_colsq", "patch_colsq_partials", "patch_colsq_fold"):
        getattr(lib, name).restype = ctypes.c_int
    lib.patch_test_prefill_kernel.argtypes = [i32]
    lib.patch_test_prefill_kernel.restype = None
    lib.patch_test_stall_first_kstep.argtypes = [i32]
    lib.patch_test_stall_first_kstep.restype = None
    lib.patch_pool_usage.argtypes = [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64),
                                     i32]
    lib.patch_pool_usage.restype = ctypes.c_int
    lib.patch_pack.argtypes = [vp, vp, vp, PatchShape, ctypes.POINTER(vp),
                               ctypes.POINTER(ctypes.c_size_t), vp]
    lib.patch_pack_group.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                     ctypes.POINTER(PatchShape), i32, ctypes.POINTER(vp),
                                     ctypes.POINTER(ctypes.c_size_t), vp]
    lib.patch_pack_group.restype = ctypes.c_int
    lib.patch_hybrid_gemm.argtypes = [vp, vp, i64, vp, i32, vp]
    lib.patch_hybrid_gemm_group.argtypes = [ctypes.POINTER(vp), i32, vp, i64, ctypes.POINTER(vp), i32, vp]
    lib.patch_hybrid_gemm_group.restype = ctypes.c_int
    lib.patch_free.argtypes = [vp, vp]
    lib.patch_free.restype = None
    lib.patch_get_status.argtypes = [vp]
    lib.patch_packed_info.argtypes = [vp, ctypes.POINTER(PatchPackedView)]
    lib.patch_packed_export.argtypes = [vp, vp, vp, vp]
    lib.patch_status_string.argtypes = [ctypes.c_int]
    lib.patch_status_string.restype = ctypes.c_char_p
    for name in ("patch_score_mask", "patch_pack", "patch_hybrid_gemm", "patch_get_status",
                 "patch_packed_info", "patch_packed_export"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def launch_count() -> int:
    """Kernels the library has enqueued so far in this process."""
    return int(load_library().patch_launch_count())


def test_stall_first_kstep(on: bool) -> None:
    """Failure-detection hook: while on, the first CTA of every GEMM never
    receives its first k-step, so its bounded wait runs out (tests only)."""
    load_library().patch_test_stall_first_kstep(1 if on else 0)


def test_prefill_kernel(which: int) -> None:
    """Test hook: 0 auto, 1 one-band, 2 band-pair, 3 two-SM, 4 two-SM four-band
    prefill kernel (M > 16)."""
    load_library().patch_test_prefill_kernel(int(which))


def pool_usage(reset_high: bool = False) -> tuple:
    """(bytes in use, high-water mark) of the library's device memory pool on
    the current device; reset_high restarts the mark from the current use."""
    now, high = ctypes.c_uint64(0), ctypes.c_uint64(0)
    _check("patch_pool_usage", load_library().patch_pool_usage(
        ctypes.byref(now), ctypes.byref(high), 1 if reset_high else 0))
    return int(now.value), int(high.value)


def _check(fn: str, code: int):
    if code != PATCH_OK:
        raise PatchError(fn, code)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        return ctypes.c_void_p(torch._C._cuda_getCurrentRawStream(torch.cuda.current_device()))
    return ctypes.c_void_p(stream.cuda_stream)


def _dptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def n_tiles(N: int, K: int, tile_n: int, tile_k: int) -> int:
    return (N // tile_n) * (K // tile_k)


def patch_score_mask(W: torch.Tensor, Xcal: torch.Tensor | None = None, *, tile_n: int = 128,
                     tile_k: int = 128, fraction: float = 0.0, map_in: torch.Tensor | None = None,
                     colsq_in: torch.Tensor | None = None, want_colsq: bool = False,
                     want_loss: bool = False, nm: tuple = (2, 4), stream=None) -> dict:
    """Wanda N:M codes (2:4 by default, or nm=(4, 8)), tile map (and optionally
    colsq, tile loss) for W[N,K] bf16."""
    lib = load_library()
    N, K = W.shape
    nt = n_tiles(N, K, tile_n, tile_k)
    dev = W.device
    meta = torch.empty((N, K // 32), dtype=torch.int32, device=dev)
    tmap = torch.empty(((nt + 31) // 32,), dtype=torch.int32, device=dev)
    colsq = torch.empty((K,), dtype=torch.float64, device=dev) if want_colsq else None
    loss = torch.empty((nt,), dtype=torch.float64, device=dev) if want_loss else None
    T = Xcal.shape[0] if Xcal is not None else 0
    if tuple(nm) == (2, 4):
        code = lib.patch_score_mask(
            _dptr(W, torch.bfloat16, "W"), _dptr(Xcal, torch.bfloat16, "Xcal"), T,
            _dptr(colsq_in, torch.float64, "colsq_in"), PatchShape(N, K, tile_n, tile_k),
            float(fraction), _dptr(map_in, (torch.int32, torch.uint32), "map_in"), _dptr(meta),
            _dptr(tmap), _dptr(colsq), _dptr(loss), _stream(stream))
        _check("patch_score_mask", code)
    else:
        code = lib.patch_score_mask_nm(
            _dptr(W, torch.bfloat16, "W"), _dptr(Xcal, torch.bfloat16, "Xcal"), T,
            _dptr(colsq_in, torch.float64, "colsq_in"), PatchShape(N, K, tile_n, tile_k),
            int(nm[0]), int(nm[1]), float(fraction),
            _dptr(map_in, (torch.int32, torch.uint32), "map_in"), _dptr(meta), _dptr(tmap),
            _dptr(colsq), _dptr(loss), _stream(stream))
        _check("patch_score_mask_nm", code)
    return {"meta": meta, "map": tmap, "colsq": colsq, "loss": loss}


COLSQ_CHUNK = 128  # calibration tokens per chunk partial of the column sums


def patch_colsq(Xcal: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """colsq[j] = sum_t Xcal[t, j]^2 (fp64, the fixed chunked order) for Xcal[T,K] bf16."""
    T, K = Xcal.shape
    if out is None:
        out = torch.empty((K,), dtype=torch.float64, device=Xcal.device)
    _check("patch_colsq", load_library().patch_colsq(
        _dptr(Xcal, torch.bfloat16, "Xcal"), T, K, _dptr(out, torch.float64, "colsq"), _stream(stream)))
    return out


def patch_colsq_partials(Xcal: torch.Tensor, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Chunk partials [ceil(T/128), K] fp64 of the column sums of squares."""
    T, K = Xcal.shape
    if out is None:
        out = torch.empty(((T + COLSQ_CHUNK - 1) // COLSQ_CHUNK, K), dtype=torch.float64,
                          device=Xcal.device)
    _check("patch_colsq_partials", load_library().patch_colsq_partials(
        _dptr(Xcal, torch.bfloat16, "Xcal"), T, K, _dptr(out, torch.float64, "partials"),
        _stream(stream)))
    return out


def patch_colsq_fold(partials: torch.Tensor, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Column sums of squares from chunk partials [chunks, K], added in chunk order."""
    chunks, K = partials.shape
    if out is None:
        out = torch.empty((K,), dtype=torch.float64, device=partials.device)
    _check("patch_colsq_fold", load_library().patch_colsq_fold(
        _dptr(partials, torch.float64, "partials"), chunks, K, _dptr(out, torch.float64, "colsq"),
        _stream(stream)))
    return out


def patch_score_mask_noalloc(W: torch.Tensor, Xcal: torch.Tensor | None = None, *,
                             tile_n: int = 128, tile_k: int = 128, fraction: float = 0.0,
                             map_in: torch.Tensor | None = None,
                             colsq_in: torch.Tensor | None = None, out: dict | None = None,
                             stream=None) -> dict:
    """patch_score_mask without any device allocation inside the library.

    For callers that cannot allocate device memory while they run (the
    library's scratch is a fixed 16 MiB array per device; see patch.h).  The
    outputs are the caller's: pass them in `out` (keys "meta", "map" and
    optionally "colsq", "loss", shaped as patch_score_mask returns them) to
    keep this call free of allocations on the Python side too.
    """
    lib = load_library()
    N, K = W.shape
    nt = n_tiles(N, K, tile_n, tile_k)
    if out is None:
        dev = W.device
        out = {"meta": torch.empty((N, K // 32), dtype=torch.int32, device=dev),
               "map": torch.empty(((nt + 31) // 32,), dtype=torch.int32, device=dev),
               "colsq": None, "loss": None}
    T = Xcal.shape[0] if Xcal is not None else 0
    code = lib.patch_score_mask_noalloc(
        _dptr(W, torch.bfloat16, "W"), _dptr(Xcal, torch.bfloat16, "Xcal"), T,
        _dptr(colsq_in, torch.float64, "colsq_in"), PatchShape(N, K, tile_n, tile_k),
        float(fraction), _dptr(map_in, (torch.int32, torch.uint32), "map_in"),
        _dptr(out["meta"]), _dptr(out["map"]), _dptr(out.get("colsq")), _dptr(out.get("loss")),
        _stream(stream))
    _check("patch_score_mask_noalloc", code)
    return out


class PackedWeight:
    """Owns a patch_packed handle; released by patch_free on close / deletion."""

    def __init__(self, handle: int, shape: tuple, packed_bytes: int, fp8: bool = False):
        self.handle = ctypes.c_void_p(handle)
        self.N, self.K, self.tile_n, self.tile_k = shape
        self.packed_bytes = packed_bytes
        self.fp8 = fp8

    def view(self) -> PatchPackedView:
        v = PatchPackedView()
        _check("patch_packed_info", load_library().patch_packed_info(self.handle, ctypes.byref(v)))
        return v

    def export(self, stream=None):
        """Copies of the packed bytes (uint8) and the k-step table (int64) as CUDA tensors."""
        v = self.view()
        packed = torch.empty((v.packed_bytes,), dtype=torch.uint8, device="cuda")
        steps = self.K // (128 if self.fp8 else 64)
        table = torch.empty(((self.N // 128) * steps,), dtype=torch.int64, device="cuda")
        _check("patch_packed_export", load_library().patch_packed_export(
            self.handle, _dptr(packed), _dptr(table), _stream(stream)))
        return packed, table

    def fp8_scales(self, stream=None) -> torch.Tensor:
        """The W_eff row scales of an FP8 handle ([N] fp32)."""
        out = torch.empty((self.N,), dtype=torch.float32, device="cuda")
        _check("patch_packed_fp8_scales", load_library().patch_packed_fp8_scales(
            self.handle, _dptr(out), _stream(stream)))
        return out

    def close(self, stream=None):
        if self.handle and self.handle.value:
            load_library().patch_free(self.handle, _stream(stream))
            self.handle = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def patch_select_maps_global(losses: list, fraction: float, stream=None) -> list:
    """Tile maps for several matrices at one block-wide target: the
    floor(fraction * all tiles) tiles of least loss over all matrices become
    2:4.  `losses` are the fp64 tile losses from patch_score_mask(want_loss=True)."""
    lib = load_library()
    count = len(losses)
    maps = [torch.empty(((l.numel() + 31) // 32,), dtype=torch.int32, device=l.device) for l in losses]
    lp = (ctypes.c_void_p * count)(*[_dptr(l, torch.float64, "loss").value for l in losses])
    mp = (ctypes.c_void_p * count)(*[m.data_ptr() for m in maps])
    nt = (ctypes.c_int64 * count)(*[l.numel() for l in losses])
    code = lib.patch_select_maps_global(lp, nt, count, float(fraction), mp, _stream(stream))
    _check("patch_select_maps_global", code)
    return maps


def patch_pack(W: torch.Tensor, meta: torch.Tensor, tile_map: torch.Tensor, *, tile_n: int = 128,
               tile_k: int = 128, nm: tuple = (2, 4), stream=None) -> PackedWeight:
    """Compress W (dense tiles + 2:4 tiles, or 4:8 tiles with nm=(4, 8)) into a
    library-owned handle."""
    lib = load_library()
    N, K = W.shape
    out = ctypes.c_void_p(0)
    nbytes = ctypes.c_size_t(0)
    if tuple(nm) == (2, 4):
        code = lib.patch_pack(_dptr(W, torch.bfloat16, "W"),
                              _dptr(meta, (torch.int32, torch.uint32), "meta"),
                              _dptr(tile_map, (torch.int32, torch.uint32), "map"),
                              PatchShape(N, K, tile_n, tile_k), ctypes.byref(out),
                              ctypes.byref(nbytes), _stream(stream))
        _check("patch_pack", code)
    else:
        code = lib.patch_pack_nm(_dptr(W, torch.bfloat16, "W"),
                                 _dptr(meta, (torch.int32, torch.uint32), "meta"),
                                 _dptr(tile_map, (torch.int32, torch.uint32), "map"),
                                 PatchShape(N, K, tile_n, tile_k), int(nm[0]), int(nm[1]),
                                 ctypes.byref(out), ctypes.byref(nbytes), _stream(stream))
        _check("patch_pack_nm", code)
    return PackedWeight(out.value, (N, K, tile_n, tile_k), nbytes.value)


def patch_pack_fp8(W: torch.Tensor, meta: torch.Tensor, tile_map: torch.Tensor, *, tile_n: int = 128,
                   tile_k: int = 128, stream=None) -> PackedWeight:
    """FP8 handle: W_eff quantised to e4m3 per output row, dense and 2:4 tiles."""
    lib = load_library()
    N, K = W.shape
    out = ctypes.c_void_p(0)
    nbytes = ctypes.c_size_t(0)
    code = lib.patch_pack_fp8(_dptr(W, torch.bfloat16, "W"), _dptr(meta, (torch.int32, torch.uint32), "meta"),
                              _dptr(tile_map, (torch.int32, torch.uint32), "map"),
                              PatchShape(N, K, tile_n, tile_k), ctypes.byref(out), ctypes.byref(nbytes),
                              _stream(stream))
    _check("patch_pack_fp8", code)
    return PackedWeight(out.value, (N, K, tile_n, tile_k), nbytes.value, fp8=True)


def patch_quantize_fp8(X: torch.Tensor, stream=None) -> tuple:
    """(codes uint8 [R, C], scales fp32 [R]) of the per-row e4m3 quantisation of X bf16."""
    R, C = X.shape
    codes = torch.empty((R, C), dtype=torch.uint8, device=X.device)
    scales = torch.empty((R,), dtype=torch.float32, device=X.device)
    _check("patch_quantize_fp8", load_library().patch_quantize_fp8(
        _dptr(X, torch.bfloat16, "X"), R, C, _dptr(codes), _dptr(scales), _stream(stream)))
    return codes, scales


def patch_hybrid_gemm(packed: PackedWeight, X: torch.Tensor, out: torch.Tensor | None = None,
                      out_fp32: bool = False, stream=None) -> torch.Tensor:
    """Y[M,N] = X[M,K] @ W_eff^T on the tensor cores (bf16 out, or fp32 out)."""
    lib = load_library()
    M, K = X.shape
    if K != packed.K:
        raise ValueError(f"X has {K} columns, the packed weight {packed.K}")
    if out is None:
        out = torch.empty((M, packed.N), dtype=torch.float32 if out_fp32 else torch.bfloat16,
                          device=X.device)
    want = torch.float32 if out_fp32 else torch.bfloat16
    code = lib.patch_hybrid_gemm(packed.handle, _dptr(X, torch.bfloat16, "X"), M,
                                 _dptr(out, want, "out"), 1 if out_fp32 else 0, _stream(stream))
    _check("patch_hybrid_gemm", code)
    return out


def patch_pack_group(Ws: list, metas: list, tile_maps: list, *, tile_n: int = 128, tile_k: int = 128,
                     stream=None) -> list:
    """patch_pack for several matrices (2:4 tiles) with one host wait; one
    handle per matrix, each equal to its patch_pack handle."""
    lib = load_library()
    n = len(Ws)
    if len(metas) != n or len(tile_maps) != n:
        raise ValueError("one meta and one map per weight")
    w_p = (ctypes.c_void_p * max(n, 1))(*[_dptr(w, torch.bfloat16, "W") for w in Ws])
    m_p = (ctypes.c_void_p * max(n, 1))(*[_dptr(m, (torch.int32, torch.uint32), "meta") for m in metas])
    t_p = (ctypes.c_void_p * max(n, 1))(*[_dptr(t, (torch.int32, torch.uint32), "map") for t in tile_maps])
    shps = (PatchShape * max(n, 1))(*[PatchShape(w.shape[0], w.shape[1], tile_n, tile_k) for w in Ws])
    outs = (ctypes.c_void_p * max(n, 1))()
    nbytes = (ctypes.c_size_t * max(n, 1))()
    code = lib.patch_pack_group(w_p, m_p, t_p, shps, n, outs, nbytes, _stream(stream))
    _check("patch_pack_group", code)
    return [PackedWeight(outs[i], (Ws[i].shape[0], Ws[i].shape[1], tile_n, tile_k), nbytes[i]) for i in range(n)]


def patch_hybrid_gemm_group(packed: list, X: torch.Tensor, outs: list | None = None,
                            out_fp32: bool = False, stream=None) -> list:
    """Ys[i] = X @ W_eff_i^T for handles that share the input X (same K), in
    one launch where the library can (see patch_hybrid_gemm_group in
    include/patch.h); returns the outputs."""
    lib = load_library()
    M, K = X.shape
    n = len(packed)
    for pk in packed:
        if pk.K != K:
            raise ValueError(f"X has {K} columns, a packed weight {pk.K}")
    want = torch.float32 if out_fp32 else torch.bfloat16
    if outs is None:
        outs = [torch.empty((M, pk.N), dtype=want, device=X.device) for pk in packed]
    if len(outs) != n:
        raise ValueError("one output per handle")
    handles = (ctypes.c_void_p * max(n, 1))(*[pk.handle for pk in packed])
    ys = (ctypes.c_void_p * max(n, 1))(*[_dptr(y, want, "out") for y in outs])
    code = lib.patch_hybrid_gemm_group(handles, n, _dptr(X, torch.bfloat16, "X"), M, ys,
                                       1 if out_fp32 else 0, _stream(stream))
    _check("patch_hybrid_gemm_group", code)
    return outs


def patch_free(packed: PackedWeight, stream=None) -> None:
    packed.close(stream)


def patch_get_status(packed: PackedWeight) -> int:
    """0 (ok) or 5 (a bounded device wait ran out); synchronises the device."""
    return int(load_library().patch_get_status(packed.handle))
