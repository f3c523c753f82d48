"""The allocation-free mask builder against the regular one.

patch_score_mask_noalloc serves callers that may not allocate device memory
while they run (a framework allocator that owns the whole GPU, a runtime that
reserves all memory up front, a latency-critical path where an allocation could
synchronise the device).  It works in a fixed scratch array inside the library
instead of the stream-ordered pool.  Here it must give exactly what
patch_score_mask gives, call after call: the array keeps the previous call's
contents, which must not leak into the next result.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_gemm_wanda_b200 import inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.fixture(scope="module")
def P():
    from sparse_gemm_wanda_b200 import build, patch
    build.build()
    patch.load_library()
    return patch


def problem(N, K, T, seed):
    w = inputs.weight(N, K, seed).cuda()
    o = inputs.outlier_channels(K, seed)
    xc = inputs.activations(T, K, seed, o).cuda()
    return w, xc


def call_noalloc(P, w, xc, tn, tk, frac, map_in=None, colsq_in=None, want_loss=True):
    """The new entry point through the C ABI, outputs allocated by the caller
    beforehand; checks that the call itself takes no memory from the library's
    pool (its high-water mark stays at the use before the call) nor from
    PyTorch's allocator."""
    lib = P.load_library()
    N, K = w.shape
    nt = (N // tn) * (K // tk)
    meta = torch.empty((N, K // 32), dtype=torch.int32, device="cuda")
    tmap = torch.empty(((nt + 31) // 32,), dtype=torch.int32, device="cuda")
    colsq = torch.empty((K,), dtype=torch.float64, device="cuda")
    loss = torch.empty((nt,), dtype=torch.float64, device="cuda") if want_loss else None
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    used0, _ = P.pool_usage(reset_high=True)
    # PyTorch's cumulative count of allocation requests (freeing garbage left
    # by earlier tests can change the bytes in use, never this count)
    torch_allocs = torch.cuda.memory_stats()["allocation.all.allocated"]
    code = lib.patch_score_mask_noalloc(
        ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(xc.data_ptr()) if xc is not None else None,
        xc.shape[0] if xc is not None else 0,
        ctypes.c_void_p(colsq_in.data_ptr()) if colsq_in is not None else None,
        P.PatchShape(N, K, tn, tk), float(frac),
        ctypes.c_void_p(map_in.data_ptr()) if map_in is not None else None,
        ctypes.c_void_p(meta.data_ptr()), ctypes.c_void_p(tmap.data_ptr()),
        ctypes.c_void_p(colsq.data_ptr()), ctypes.c_void_p(loss.data_ptr()) if want_loss else None,
        stream)
    assert code == 0, P.STATUS_NAMES.get(code, code)
    torch.cuda.synchronize()
    used1, high = P.pool_usage()
    # an allocation inside the call, even one freed before it returned, would
    # have lifted the mark above the use before the call (the reset may leave
    # the mark below that use, never above it)
    assert used1 == used0 and high <= used0, "the call took memory from the library's pool"
    assert torch.cuda.memory_stats()["allocation.all.allocated"] == torch_allocs
    return {"meta": meta, "map": tmap, "colsq": colsq, "loss": loss}


def assert_same(a, b, keys=("meta", "map", "colsq", "loss")):
    torch.cuda.synchronize()
    for key in keys:
        assert torch.equal(a[key], b[key]), key


def test_noalloc_matches_regular_two_calls_in_a_row(P):
    assert P.load_library().patch_score_mask_noalloc_capacity() == 16 << 20
    # the documented set-up: one small call first, at initialisation (it looks
    # up the scratch array's address and, under lazy module loading, reserves it)
    ws, xs = problem(128, 128, 16, seed=500)
    call_noalloc(P, ws, xs, 128, 128, 0.5)
    # first call: Llama-7B attention-shaped weight, 2048 calibration tokens
    w1, x1 = problem(4096, 4096, 2048, seed=501)
    ref1 = P.patch_score_mask(w1, x1, fraction=0.5, want_colsq=True, want_loss=True)
    got1 = call_noalloc(P, w1, x1, 128, 128, 0.5)
    assert_same(got1, ref1)
    # second call right after: other shapes, a ragged calibration set and a
    # given map, so stale scratch contents from the first call would show
    w2, x2 = problem(1024, 2048, 777, seed=502)
    nt = (1024 // 64) * (2048 // 128)
    m2 = inputs.random_map(nt, nt // 3, seed=502).cuda()
    ref2 = P.patch_score_mask(w2, x2, tile_n=64, tile_k=128, map_in=m2, want_colsq=True,
                              want_loss=True)
    got2 = call_noalloc(P, w2, x2, 64, 128, 0.0, map_in=m2)
    assert_same(got2, ref2)
    # and the first problem again: same answer as the first time
    got3 = call_noalloc(P, w1, x1, 128, 128, 0.5)
    assert_same(got3, ref1)


def test_noalloc_loss_kept_inside_and_norms_given(P):
    # tile_loss_out = NULL: the losses live in the fixed array and only the map
    # shows them; colsq_in given: the norms come from the caller's sums
    w1, x1 = problem(2048, 1024, 300, seed=511)
    ref = P.patch_score_mask(w1, x1, fraction=0.4, want_colsq=True, want_loss=True)
    got = call_noalloc(P, w1, x1, 128, 128, 0.4, want_loss=False)
    assert_same(got, ref, keys=("meta", "map", "colsq"))
    w2, _ = problem(1024, 1024, 1, seed=512)
    ref2 = P.patch_score_mask(w2, None, tile_n=64, tile_k=64, fraction=0.7,
                              colsq_in=ref["colsq"], want_colsq=True, want_loss=True)
    got2 = call_noalloc(P, w2, None, 64, 64, 0.7, colsq_in=ref["colsq"])
    assert_same(got2, ref2)
    got3 = call_noalloc(P, w2, None, 64, 64, 0.7, colsq_in=ref["colsq"], want_loss=False)
    assert_same(got3, ref2, keys=("meta", "map", "colsq"))


def test_noalloc_rejects_problems_beyond_its_scratch(P):
    # 66000 tokens x 4096 columns need 8*4096*516 bytes of chunk partials,
    # more than the 16 MiB array: refused before any work is enqueued
    w, _ = problem(256, 4096, 1, seed=503)
    xc = torch.zeros((66000, 4096), dtype=torch.bfloat16, device="cuda")
    lib = P.load_library()
    meta = torch.empty((256, 4096 // 32), dtype=torch.int32, device="cuda")
    tmap = torch.empty((2,), dtype=torch.int32, device="cuda")
    code = lib.patch_score_mask_noalloc(
        ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(xc.data_ptr()), xc.shape[0], None,
        P.PatchShape(256, 4096, 128, 128), 0.5, None, ctypes.c_void_p(meta.data_ptr()),
        ctypes.c_void_p(tmap.data_ptr()), None, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert code == 2  # PATCH_ERR_UNSUPPORTED
    del xc
    torch.cuda.empty_cache()
