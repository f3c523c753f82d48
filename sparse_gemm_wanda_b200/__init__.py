"""Tile-hybrid (dense / 2:4) Wanda-masked linear layers on NVIDIA B200 (sm_100a).

The compute lives in ``libpatch_b200.so`` (C ABI, include/patch.h); ``patch``
is its thin ctypes binding.  Importing this package does not load the CUDA
library; the first call does, and fails loudly if it is missing.
"""
from .patch import (PackedWeight, PatchError, PatchLibraryError, load_library,  # noqa: F401
                    patch_free, patch_get_status, patch_hybrid_gemm, patch_pack,
                    patch_score_mask)

__all__ = ["PackedWeight", "PatchError", "PatchLibraryError", "load_library", "patch_free",
           "patch_get_status", "patch_hybrid_gemm", "patch_pack", "patch_score_mask"]
