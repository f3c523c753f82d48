"""4:8 tiles on the GPU against the CPU oracle, through the C ABI.

Another N:M pattern for the sparse tiles ("PATCH: Learnable Tile-level Hybrid
Sparsity for LLMs", section 5: the tile scheme extends to 4:8): every group of
8 input channels of a 4:8 tile keeps its 4 weights of highest Wanda score
(ties to the lower index).  Bit-exact: keep masks, tile losses, maps, packed
bytes and k-step tables.  GEMM (the one-band kernel expanding 4:8 k-steps in
shared memory for dense MMAs): the tolerance reading of the 2:4 tests, with
W_eff from the oracle's own masks and map.
"""
import numpy as np
import pytest
import torch

from sparse_gemm_wanda_b200 import inputs
from tests.conftest import bf16_bits

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)

NM = (4, 8)


@pytest.fixture(scope="module")
def P():
    from sparse_gemm_wanda_b200 import build, patch
    build.build()
    patch.load_library()
    return patch


def u32(t):
    return t.cpu().numpy().view(np.uint32)


def check(y, yref, fp32_mode):
    y = y.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(yref ** 2)))
    err = np.abs(y - yref)
    if fp32_mode:
        assert err.max() <= 1e-2 * rms, (float(err.max()), rms)
    else:
        mag = np.maximum(np.abs(y), np.abs(yref))
        ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-30))) - 7)
        bad = ~(err <= 1e-2 * rms + 0.5 * ulp)
        assert not bad.any(), (int(bad.sum()), float(err.max()), rms)


def problem(N, K, T, M, seed):
    w = inputs.weight(N, K, seed)
    o = inputs.outlier_channels(K, seed)
    xc = inputs.activations(T, K, seed, o, role=0)
    x = inputs.activations(M, K, seed, o, role=1)
    return w, xc, x


@pytest.mark.parametrize("N,K,T,tn,tk,frac", [
    (256, 256, 64, 64, 64, 0.5),
    (512, 384, 300, 128, 128, 0.3),
    (384, 512, 129, 64, 128, 1.0),
    (4096, 4096, 2048, 128, 128, 0.5),
])
def test_mask_builder_4of8_bit_exact(P, oracle_mod, N, K, T, tn, tk, frac):
    w, xc, _ = problem(N, K, T, 1, seed=N + K + T + 8)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, fraction=frac,
                           want_colsq=True, want_loss=True, nm=NM)
    torch.cuda.synchronize()
    ref = oracle_mod.score_mask_4of8(bf16_bits(w), bf16_bits(xc), tn, tk, fraction=frac)
    assert np.array_equal(r["colsq"].cpu().numpy(), ref["colsq"])
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(r["loss"].cpu().numpy(), ref["loss"])
    assert np.array_equal(u32(r["map"]), ref["map"])


def test_mask_builder_4of8_ties(P, oracle_mod):
    # zero and duplicated calibration columns, equal magnitudes: exact ties
    w, xc, _ = problem(256, 256, 64, 1, seed=3)
    xc = xc.clone()
    xc[:, 0:64] = 0
    xc[:, 64:128] = xc[:, 128:192]
    w = w.clone()
    w[:, 200:256] = w[:, 200:201]
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=64, tile_k=64, fraction=0.5,
                           want_loss=True, nm=NM)
    torch.cuda.synchronize()
    ref = oracle_mod.score_mask_4of8(bf16_bits(w), bf16_bits(xc), 64, 64, fraction=0.5)
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(r["loss"].cpu().numpy(), ref["loss"])
    assert np.array_equal(u32(r["map"]), ref["map"])


@pytest.mark.parametrize("tn,tk", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.3, 1.0])
def test_pack_4of8_bit_exact(P, oracle_mod, tn, tk, frac):
    N, K = 512, 768
    w, xc, _ = problem(N, K, 64, 1, seed=tn + tk + int(frac * 100))
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), seed=tn * 3 + tk)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda(), nm=NM)
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk, nm=NM)
    packed, table = pk.export()
    torch.cuda.synchronize()
    ref = oracle_mod.score_mask_4of8(bf16_bits(w), bf16_bits(xc), tn, tk,
                                     tile_map=tmap.numpy().view(np.uint32))
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    ref_packed, ref_table = oracle_mod.pack_4of8(bf16_bits(w), ref["meta"], ref["map"], tn, tk)
    assert pk.packed_bytes == ref_packed.size
    assert np.array_equal(table.cpu().numpy().view(np.uint64), ref_table)
    assert np.array_equal(packed.cpu().numpy(), ref_packed)
    pk.close()


def run_gemm(P, oracle_mod, N, K, M, tn, tk, frac, seed, fp32_mode, sample=None, by_loss=False):
    w, xc, x = problem(N, K, 256, M, seed)
    nt = (N // tn) * (K // tk)
    if by_loss:
        r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, fraction=frac, nm=NM)
        ref = oracle_mod.score_mask_4of8(bf16_bits(w), bf16_bits(xc), tn, tk, fraction=frac)
    else:
        tmap = inputs.random_map(nt, int(frac * nt), seed=seed)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda(), nm=NM)
        ref = oracle_mod.score_mask_4of8(bf16_bits(w), bf16_bits(xc), tn, tk,
                                         tile_map=tmap.numpy().view(np.uint32))
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk, nm=NM)
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=fp32_mode)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(u32(r["map"]), ref["map"])
    weff = oracle_mod.weff_4of8(bf16_bits(w), ref["meta"], ref["map"], tn, tk)
    if sample is None:
        check(y, oracle_mod.gemm(bf16_bits(x), weff), fp32_mode)
    else:
        g = np.random.default_rng(seed)
        ms, ns = g.integers(0, M, sample), g.integers(0, N, sample)
        yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
        check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, fp32_mode)
        # one whole 128-row band, every token
        rows = slice(N - 128, N)
        check(y[:, rows], oracle_mod.gemm(bf16_bits(x), np.ascontiguousarray(weff[rows])), fp32_mode)
    pk.close()


@pytest.mark.parametrize("fp32_mode", [True, False])
@pytest.mark.parametrize("M", [1, 5, 16, 64, 100, 200])
def test_gemm_4of8_small_shapes(P, oracle_mod, M, fp32_mode):
    run_gemm(P, oracle_mod, 384, 512, M, 128, 128, 0.5, seed=M + 40, fp32_mode=fp32_mode)


@pytest.mark.parametrize("tn,tk", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_gemm_4of8_tiles_and_fractions(P, oracle_mod, tn, tk, frac):
    run_gemm(P, oracle_mod, 256, 512, 40, tn, tk, frac, seed=tn + tk + 9, fp32_mode=True)


@pytest.mark.parametrize("M", [1, 16, 2048])
def test_gemm_4of8_decode_shape_by_loss(P, oracle_mod, M):
    # Llama-7B MLP shape, half the tiles 4:8 by least Wanda tile loss
    run_gemm(P, oracle_mod, 11008, 4096, M, 128, 128, 0.5, seed=77 + M, fp32_mode=False,
             sample=4000 if M > 16 else None, by_loss=True)


def test_nm_rejects_other_patterns(P):
    w, xc, _ = problem(256, 256, 64, 1, seed=1)
    with pytest.raises(P.PatchError) as e:
        P.patch_score_mask(w.cuda(), xc.cuda(), fraction=0.5, nm=(1, 4))
    assert e.value.code == 2  # PATCH_ERR_UNSUPPORTED
    r = P.patch_score_mask(w.cuda(), xc.cuda(), fraction=0.5)
    with pytest.raises(P.PatchError) as e:
        P.patch_pack(w.cuda(), r["meta"], r["map"], nm=(8, 16))
    assert e.value.code == 2
