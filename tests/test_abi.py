"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/patch.h declares, and rejects bad arguments before touching the
device.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "patch.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_gemm_wanda_b200 import build, patch
    build.build()
    return patch.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(patch_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("patch_score_mask", "patch_pack", "patch_hybrid_gemm", "patch_free"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from sparse_gemm_wanda_b200 import patch
    names = declared_functions()
    assert set(names) == set(patch.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.patch_status_string(0) == b"ok"
    assert lib.patch_status_string(5) == b"bounded device wait ran out"


def test_gemm_rejects_null_handle(lib):
    assert lib.patch_hybrid_gemm(None, None, 1, None, 0, None) == 1
    assert lib.patch_hybrid_gemm(None, None, -1, None, 0, None) == 1


def test_score_mask_argument_checks(lib):
    from sparse_gemm_wanda_b200.patch import PatchShape
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: checks fail first
    # unsupported tile size
    assert lib.patch_score_mask(fake, fake, 8, None, PatchShape(256, 256, 32, 64), 0.5, None,
                                fake, fake, None, None, None) == 2
    # N not a multiple of the tile
    assert lib.patch_score_mask(fake, fake, 8, None, PatchShape(200, 256, 64, 64), 0.5, None,
                                fake, fake, None, None, None) == 1
    # null weight
    assert lib.patch_score_mask(None, fake, 8, None, PatchShape(256, 256, 64, 64), 0.5, None,
                                fake, fake, None, None, None) == 1
    # misaligned weight
    assert lib.patch_score_mask(ctypes.c_void_p(0x1002), fake, 8, None,
                                PatchShape(256, 256, 64, 64), 0.5, None, fake, fake, None, None,
                                None) == 1
    # no calibration and no colsq
    assert lib.patch_score_mask(fake, None, 8, None, PatchShape(256, 256, 64, 64), 0.5, None,
                                fake, fake, None, None, None) == 1
    # fraction out of range without a map
    assert lib.patch_score_mask(fake, fake, 8, None, PatchShape(256, 256, 64, 64), 1.5, None,
                                fake, fake, None, None, None) == 1
    # T < 1
    assert lib.patch_score_mask(fake, fake, 0, None, PatchShape(256, 256, 64, 64), 0.5, None,
                                fake, fake, None, None, None) == 1


def test_pack_argument_checks(lib):
    from sparse_gemm_wanda_b200.patch import PatchShape
    fake = ctypes.c_void_p(0x1000)
    out = ctypes.c_void_p(0)
    assert lib.patch_pack(fake, fake, fake, PatchShape(256, 256, 64, 64), None, None,
                          None) == 1
    # N not a multiple of 128 (64-row tiles allow N=192, the packed bands do not)
    assert lib.patch_pack(fake, fake, fake, PatchShape(192, 256, 64, 64), ctypes.byref(out),
                          None, None) == 1
    # K not a multiple of 128
    assert lib.patch_pack(fake, fake, fake, PatchShape(256, 192, 64, 64), ctypes.byref(out),
                          None, None) == 1
    # null map
    assert lib.patch_pack(fake, fake, None, PatchShape(256, 256, 64, 64), ctypes.byref(out),
                          None, None) == 1
    assert out.value is None


def test_select_maps_global_argument_checks(lib):
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: checks fail first
    vp3 = (ctypes.c_void_p * 3)(fake, fake, fake)
    nt3 = (ctypes.c_int64 * 3)(10, 1, 40)
    # null arrays
    assert lib.patch_select_maps_global(None, nt3, 3, 0.5, vp3, None) == 1
    assert lib.patch_select_maps_global(vp3, None, 3, 0.5, vp3, None) == 1
    assert lib.patch_select_maps_global(vp3, nt3, 3, 0.5, None, None) == 1
    # count outside 1..64
    assert lib.patch_select_maps_global(vp3, nt3, 0, 0.5, vp3, None) == 1
    many = (ctypes.c_void_p * 65)(*([fake] * 65))
    nt65 = (ctypes.c_int64 * 65)(*([4] * 65))
    assert lib.patch_select_maps_global(many, nt65, 65, 0.5, many, None) == 1
    # fraction outside [0, 1], NaN included
    assert lib.patch_select_maps_global(vp3, nt3, 3, -0.25, vp3, None) == 1
    assert lib.patch_select_maps_global(vp3, nt3, 3, float("nan"), vp3, None) == 1
    # a null loss array or a zero tile count among the matrices
    vp_null = (ctypes.c_void_p * 3)(fake, None, fake)
    assert lib.patch_select_maps_global(vp_null, nt3, 3, 0.5, vp3, None) == 1
    nt_zero = (ctypes.c_int64 * 3)(10, 0, 40)
    assert lib.patch_select_maps_global(vp3, nt_zero, 3, 0.5, vp3, None) == 1
    # more tiles than one ranking pass covers
    big = (ctypes.c_int64 * 3)(65535 * 256, 1, 1)
    assert lib.patch_select_maps_global(vp3, big, 3, 0.5, vp3, None) == 2


def test_handle_calls_reject_null(lib):
    assert lib.patch_get_status(None) == 1
    assert lib.patch_packed_info(None, None) == 1
    assert lib.patch_packed_export(None, None, None, None) == 1
    lib.patch_free(None, None)  # no-op


def test_binding_fails_loudly_without_library(tmp_path):
    from sparse_gemm_wanda_b200 import patch
    with pytest.raises(patch.PatchLibraryError):
        # a fresh loader pointed at a missing file must raise, not fall back
        saved = patch._lib
        try:
            patch._lib = None
            patch.load_library(str(tmp_path / "missing.so"))
        finally:
            patch._lib = saved


def test_pack_group_argument_checks(lib):
    # every member is checked before anything is allocated; no handle is left
    from sparse_gemm_wanda_b200.patch import PatchShape
    vp = ctypes.c_void_p
    fake = vp(0x1000)  # never dereferenced: checks fail first
    ws = (vp * 2)(fake, fake)
    outs = (vp * 2)(vp(0x55), vp(0x66))
    good = PatchShape(256, 256, 128, 128)
    shps = (PatchShape * 2)(good, PatchShape(256, 256, 32, 128))  # second: unsupported tile
    assert lib.patch_pack_group(ws, ws, ws, shps, 2, outs, None, None) == 2
    assert not outs[0] and not outs[1]
    shps = (PatchShape * 2)(good, PatchShape(200, 256, 64, 128))  # N not a multiple of 128
    assert lib.patch_pack_group(ws, ws, ws, shps, 2, outs, None, None) == 1
    shps = (PatchShape * 2)(good, good)
    nulls = (vp * 2)(fake, None)
    assert lib.patch_pack_group(nulls, ws, ws, shps, 2, outs, None, None) == 1
    assert lib.patch_pack_group(ws, ws, ws, shps, 0, outs, None, None) == 1
    assert lib.patch_pack_group(ws, ws, ws, shps, 9, outs, None, None) == 1
    assert lib.patch_pack_group(ws, ws, ws, shps, 2, None, None, None) == 1
