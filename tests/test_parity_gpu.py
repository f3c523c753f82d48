"""GPU path vs the CPU oracle, element by element, through the C ABI.

Bit-exact: column sums of squares, 2:4 codes, tile losses, tile maps, packed
bytes and k-step tables.  GEMM: fp32-output mode within the literal bound
max|y - y_ref| <= 1e-2 * RMS(y_ref); bf16-output mode per element within
1e-2 * RMS(y_ref) + half a bf16 ulp of max(|y|, |y_ref|) (the output rounding
alone can exceed the literal bound at |y| > ~2.6 RMS).
"""
import numpy as np
import pytest
import torch

from sparse_gemm_wanda_b200 import inputs
from tests.conftest import bf16_bits

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU machines, skipped there
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.fixture(scope="module")
def P():
    from sparse_gemm_wanda_b200 import build, patch
    build.build()
    patch.load_library()
    return patch


def u32(t):
    return t.cpu().numpy().view(np.uint32)


class forced_kernel:
    """Run the block's GEMMs (M > 16) on one prefill kernel: 1 one-band,
    2 band-pair, 3 two-SM (test hook of the library; 0 restores the choice)."""

    def __init__(self, P, which):
        self.P, self.which = P, which

    def __enter__(self):
        self.P.test_prefill_kernel(self.which)

    def __exit__(self, *exc):
        self.P.test_prefill_kernel(0)


def rel_rms_check(y, yref_f64, fp32_mode):
    y = y.double().cpu().numpy()
    rms = float(np.sqrt(np.mean(yref_f64 ** 2))) if yref_f64.size else 0.0
    err = np.abs(y - yref_f64)
    if fp32_mode:
        assert err.max() <= 1e-2 * rms, (err.max(), rms)
    else:
        mag = np.maximum(np.abs(y), np.abs(yref_f64))
        ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-30))) - 7)
        bad = ~(err <= 1e-2 * rms + 0.5 * ulp)  # NaN counts as bad
        assert not bad.any(), (int(bad.sum()), float(err.max()), rms)
    return float(err.max()), rms


def make_problem(N, K, T, M, seed, outliers=None):
    w = inputs.weight(N, K, seed)
    o = inputs.outlier_channels(K, seed, outliers)
    xc = inputs.activations(T, K, seed, o, role=0) if T else None
    x = inputs.activations(M, K, seed, o, role=1)
    return w, xc, x


def oracle_mask(oracle_mod, w, xc, tn, tk, frac=None, tmap=None):
    return oracle_mod.score_mask(bf16_bits(w), bf16_bits(xc), tn, tk,
                                 fraction=frac if frac is not None else 0.0,
                                 tile_map=tmap)


def oracle_weff_checked(oracle_mod, r, w, xc, tn, tk, tmap=None, frac=None):
    """W_eff from the oracle alone: its 2:4 codes and tile map for (w, xc),
    after asserting that the GPU's codes and map (in `r`) equal them.  With
    `tmap` (a caller map) the map is given; otherwise it is the oracle's
    least-loss map at `frac`."""
    tm = None if tmap is None else tmap.numpy().view(np.uint32)
    ref = oracle_mask(oracle_mod, w, xc, tn, tk, frac=frac, tmap=tm)
    assert np.array_equal(u32(r["meta"]), ref["meta"]), "2:4 codes differ from the oracle's"
    assert np.array_equal(u32(r["map"]), ref["map"]), "tile map differs from the oracle's"
    return oracle_mod.weff(bf16_bits(w), ref["meta"], ref["map"], tn, tk)


# ---------------------------------------------------------------- mask builder

@pytest.mark.parametrize("N,K,T,tn,tk,frac", [
    (256, 256, 64, 64, 64, 0.5),        # tiny config shape
    (256, 512, 300, 128, 128, 0.5),     # ragged calibration chunk
    (512, 384, 129, 64, 128, 0.3),
    (384, 256, 1, 128, 64, 1.0),        # single calibration token
    (256, 256, 64, 64, 64, 0.0),
    (4096, 4096, 2048, 128, 128, 0.5),  # decode config, attention-shaped
    (11008, 4096, 2048, 128, 128, 0.5), # decode config, MLP-shaped
])
def test_mask_builder_bit_exact(P, oracle_mod, N, K, T, tn, tk, frac):
    w, xc, _ = make_problem(N, K, T, 1, seed=N + K + T, outliers=3 if K == 256 else None)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, fraction=frac,
                           want_colsq=True, want_loss=True)
    torch.cuda.synchronize()
    ref = oracle_mask(oracle_mod, w, xc, tn, tk, frac=frac)
    assert np.array_equal(r["colsq"].cpu().numpy(), ref["colsq"])
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(r["loss"].cpu().numpy(), ref["loss"])
    assert np.array_equal(u32(r["map"]), ref["map"])


@pytest.mark.parametrize("T,K,cut", [(300, 512, 128), (2048, 4096, 1024), (129, 256, 0),
                                     (5000, 1024, 2560)])
def test_colsq_calls_bit_exact(P, oracle_mod, T, K, cut):
    # patch_colsq alone, and its halves over two pieces of the calibration set
    # cut at a multiple of 128 tokens (partials stacked in token order, then
    # folded): both bit-identical to the oracle's fixed-order sums
    o = inputs.outlier_channels(K, T + K)
    xc = inputs.activations(T, K, T + K, o, role=0)
    ref = oracle_mod.colsq(bf16_bits(xc))
    xd = xc.cuda()
    s = P.patch_colsq(xd)
    if cut:
        parts = torch.cat([P.patch_colsq_partials(xd[:cut]), P.patch_colsq_partials(xd[cut:])])
    else:
        parts = P.patch_colsq_partials(xd)
    assert parts.shape == ((T + 127) // 128, K)
    s2 = P.patch_colsq_fold(parts)
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), ref)
    assert np.array_equal(s2.cpu().numpy(), ref)


def test_mask_builder_given_map_and_colsq(P, oracle_mod):
    N, K, tn, tk = 512, 512, 128, 64
    w, xc, _ = make_problem(N, K, 200, 1, seed=7)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, nt // 3, seed=7)
    ref = oracle_mask(oracle_mod, w, xc, tn, tk, tmap=tmap.numpy().view(np.uint32))
    colsq = torch.from_numpy(ref["colsq"]).cuda()
    r = P.patch_score_mask(w.cuda(), None, tile_n=tn, tile_k=tk, map_in=tmap.cuda(),
                           colsq_in=colsq, want_colsq=True, want_loss=True)
    torch.cuda.synchronize()
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(u32(r["map"]), ref["map"])
    assert np.array_equal(r["colsq"].cpu().numpy(), ref["colsq"])
    assert np.array_equal(r["loss"].cpu().numpy(), ref["loss"])


def test_mask_builder_ties(P, oracle_mod):
    # zero and duplicated calibration columns: exact score ties everywhere
    N, K = 256, 256
    w, xc, _ = make_problem(N, K, 64, 1, seed=3)
    xc = xc.clone()
    xc[:, 0:64] = 0
    xc[:, 64:128] = xc[:, 128:192]
    w = w.clone()
    w[:, 200:256] = w[:, 200:201]  # equal magnitudes along rows
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=64, tile_k=64, fraction=0.5,
                           want_colsq=True, want_loss=True)
    torch.cuda.synchronize()
    ref = oracle_mask(oracle_mod, w, xc, 64, 64, frac=0.5)
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(u32(r["map"]), ref["map"])
    assert np.array_equal(r["loss"].cpu().numpy(), ref["loss"])


# ------------------------------------------------- global tile allocation

@pytest.mark.parametrize("frac", [0.0, 0.3, 0.6, 0.999, 1.0])
def test_global_maps_random_losses(P, oracle_mod, frac):
    # ragged tile counts (word boundaries, one-tile matrices) and many ties;
    # enough tiles in all that the rank kernel runs over several slices
    g = np.random.default_rng(11)
    sizes = [1, 31, 32, 33, 1000, 4095, 7, 64, 2500]
    losses = [np.round(g.standard_normal(n) * (1 + i % 3), 1) for i, n in enumerate(sizes)]
    maps = P.patch_select_maps_global([torch.from_numpy(l).cuda() for l in losses], frac)
    torch.cuda.synchronize()
    ref = oracle_mod.select_maps_global(losses, frac)
    for m, r in zip(maps, ref):
        assert np.array_equal(u32(m), r)


def test_global_maps_64_matrices(P, oracle_mod):
    g = np.random.default_rng(12)
    losses = [np.round(g.exponential(1.0 + (i % 5), int(g.integers(1, 300))), 2) for i in range(64)]
    maps = P.patch_select_maps_global([torch.from_numpy(l).cuda() for l in losses], 0.45)
    torch.cuda.synchronize()
    for m, r in zip(maps, oracle_mod.select_maps_global(losses, 0.45)):
        assert np.array_equal(u32(m), r)


def test_global_maps_one_matrix_equals_the_mask_builder_map(P, oracle_mod):
    w, xc, _ = make_problem(512, 768, 128, 1, seed=21)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=64, tile_k=64, fraction=0.4,
                           want_loss=True)
    (m,) = P.patch_select_maps_global([r["loss"]], 0.4)
    torch.cuda.synchronize()
    assert np.array_equal(u32(m), u32(r["map"]))


def test_global_maps_from_mask_builder_losses(P, oracle_mod):
    # three matrices of one block sharing a calibration set; the block-wide
    # map then feeds the mask builder's given-map mode and the packer
    K = 512
    o = inputs.outlier_channels(K, 31)
    xc = inputs.activations(256, K, 31, o, role=0)
    ws = [inputs.weight(n, K, 31 + n) for n in (256, 384, 640)]
    res = [P.patch_score_mask(w.cuda(), xc.cuda(), want_loss=True, want_colsq=True) for w in ws]
    maps = P.patch_select_maps_global([r["loss"] for r in res], 0.5)
    torch.cuda.synchronize()
    ref_losses = []
    for w in ws:
        ref = oracle_mask(oracle_mod, w, xc, 128, 128, frac=0.0)
        ref_losses.append(ref["loss"])
    for r, l in zip(res, ref_losses):
        assert np.array_equal(r["loss"].cpu().numpy(), l)
    ref_maps = oracle_mod.select_maps_global(ref_losses, 0.5)
    for w, m, rm in zip(ws, maps, ref_maps):
        assert np.array_equal(u32(m), rm)
        r2 = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=m)
        pk = P.patch_pack(w.cuda(), r2["meta"], r2["map"])
        torch.cuda.synchronize()
        assert np.array_equal(u32(r2["map"]), rm)
        pk.close()


def test_global_maps_bad_arguments(P):
    l = torch.zeros(10, dtype=torch.float64, device="cuda")
    for losses, f in [([l], -0.1), ([l], 1.5), ([l] * 65, 0.5)]:
        with pytest.raises(P.PatchError) as e:
            P.patch_select_maps_global(losses, f)
        assert e.value.code == 1  # PATCH_ERR_INVALID_ARG


# ----------------------------------------------------------------------- pack

@pytest.mark.parametrize("tn,tk", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.3, 0.5, 1.0])
def test_pack_bit_exact(P, oracle_mod, tn, tk, frac):
    N, K = 512, 768
    w, xc, _ = make_problem(N, K, 64, 1, seed=tn + tk + int(frac * 100))
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), seed=tn * 3 + tk)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk)
    packed, table = pk.export()
    torch.cuda.synchronize()
    ref_meta = oracle_mask(oracle_mod, w, xc, tn, tk, tmap=tmap.numpy().view(np.uint32))["meta"]
    ref_packed, ref_table = oracle_mod.pack(bf16_bits(w), ref_meta, tmap.numpy().view(np.uint32),
                                            tn, tk)
    assert pk.packed_bytes == ref_packed.size
    assert np.array_equal(table.cpu().numpy().view(np.uint64), ref_table)
    assert np.array_equal(packed.cpu().numpy(), ref_packed)
    pk.close()


@pytest.mark.parametrize("tn,tk", [(128, 128), (64, 64)])
def test_pack_group_bit_exact(P, oracle_mod, tn, tk):
    # several matrices of different shapes (an odd band count among them)
    # packed with one wait: every packed buffer and k-step table equal to the
    # oracle's, and the products equal to those of single-call handles
    shapes = [(512, 768, 0.5), (384, 1024, 1.0), (1024, 512, 0.3), (256, 256, 0.0)]
    ws, rs, tmaps = [], [], []
    for i, (N, K, frac) in enumerate(shapes):
        w, xc, _ = make_problem(N, K, 64, 1, seed=900 + i + tn)
        nt = (N // tn) * (K // tk)
        tmap = inputs.random_map(nt, int(frac * nt), seed=910 + i + tk)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda())
        ref_meta = oracle_mask(oracle_mod, w, xc, tn, tk, tmap=tmap.numpy().view(np.uint32))["meta"]
        assert np.array_equal(r["meta"].cpu().numpy().view(np.uint32), ref_meta)
        ws.append(w)
        rs.append((r, ref_meta))
        tmaps.append(tmap)
    pks = P.patch_pack_group([w.cuda() for w in ws], [r["meta"] for r, _ in rs], [r["map"] for r, _ in rs],
                             tile_n=tn, tile_k=tk)
    singles = [P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk) for w, (r, _) in zip(ws, rs)]
    for (N, K, _), w, (r, ref_meta), tmap, pk, pk1 in zip(shapes, ws, rs, tmaps, pks, singles):
        packed, table = pk.export()
        torch.cuda.synchronize()
        ref_packed, ref_table = oracle_mod.pack(bf16_bits(w), ref_meta, tmap.numpy().view(np.uint32), tn, tk)
        assert pk.packed_bytes == ref_packed.size
        assert np.array_equal(table.cpu().numpy().view(np.uint64), ref_table)
        assert np.array_equal(packed.cpu().numpy(), ref_packed)
        for M in (8, 300):
            x = inputs.activations(M, K, 920 + M, None).cuda()
            y = P.patch_hybrid_gemm(pk, x, out_fp32=True)
            y1 = P.patch_hybrid_gemm(pk1, x, out_fp32=True)
            torch.cuda.synchronize()
            assert torch.equal(y, y1)
        assert P.patch_get_status(pk) == 0
    for pk in pks + singles:
        pk.close()


def test_pack_group_bad_member_leaves_no_handle(P):
    # a member that fails its checks fails the call before anything is made
    w = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    meta = torch.zeros(256, 8, dtype=torch.int32, device="cuda")
    tmap = torch.zeros(1, dtype=torch.int32, device="cuda")
    w_bad = torch.zeros(200, 256, dtype=torch.bfloat16, device="cuda")  # N not a multiple of 128
    with pytest.raises(P.PatchError) as e:
        P.patch_pack_group([w, w_bad], [meta, meta], [tmap, tmap])
    assert e.value.code == 1


# ----------------------------------------------------------------------- GEMM

def run_case(P, oracle_mod, N, K, M, tn, tk, frac, seed, fp32_mode, sample=None):
    w, xc, x = make_problem(N, K, 64, M, seed)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(round(frac * nt)), seed=seed)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk)
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=fp32_mode)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    weff = oracle_weff_checked(oracle_mod, r, w, xc, tn, tk, tmap=tmap)
    if sample is None:
        yref = oracle_mod.gemm(bf16_bits(x), weff)
        out = rel_rms_check(y, yref, fp32_mode)
    else:
        g = np.random.default_rng(seed)
        ms = g.integers(0, M, sample)
        ns = g.integers(0, N, sample)
        yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
        # RMS of the reference over the sample stands in for the full matrix
        out = rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref,
                            fp32_mode)
    pk.close()
    return out


@pytest.mark.parametrize("fp32_mode", [True, False])
@pytest.mark.parametrize("M", [1, 3, 8, 16, 17, 64, 100, 128, 200, 256, 300])
def test_gemm_small_shapes(P, oracle_mod, M, fp32_mode):
    run_case(P, oracle_mod, 384, 512, M, 128, 128, 0.5, seed=M, fp32_mode=fp32_mode)


@pytest.mark.parametrize("tn,tk", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("M", [8, 160])
def test_gemm_tiles_and_fractions(P, oracle_mod, tn, tk, frac, M):
    run_case(P, oracle_mod, 256, 512, M, tn, tk, frac, seed=tn + tk + M, fp32_mode=True)


@pytest.mark.parametrize("N,K", [(128, 128), (128, 384), (256, 640), (384, 896), (128, 1152)])
@pytest.mark.parametrize("M", [1, 5, 16])
def test_gemm_decode_ragged_pair_counts(P, oracle_mod, N, K, M):
    # k-pairs per band of 1, 3, 5, 7, 9: chunks of fewer than four pairs,
    # stages holding a single k-pair, single-band matrices, fewer chunks than SMs
    run_case(P, oracle_mod, N, K, M, 128, 128, 0.5, seed=N + K + M, fp32_mode=True)


@pytest.mark.parametrize("N,K", [(128, 128), (128, 384), (256, 640), (384, 896), (128, 1152)])
@pytest.mark.parametrize("M", [17, 32, 33, 47, 64])
def test_gemm_skinny_ragged_pair_counts(P, oracle_mod, N, K, M):
    # the split-K path with 32- and 64-token tiles (17 <= M <= 64): ragged
    # token tiles, chunks of fewer than four pairs, single-pair stages
    run_case(P, oracle_mod, N, K, M, 128, 128, 0.5, seed=N + K + M, fp32_mode=True)


@pytest.mark.parametrize("tn,tk", [(64, 64), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 1.0])
@pytest.mark.parametrize("M", [24, 64])
def test_gemm_skinny_tiles_and_fractions(P, oracle_mod, tn, tk, frac, M):
    run_case(P, oracle_mod, 256, 512, M, tn, tk, frac, seed=tn + tk + M + 7, fp32_mode=False)


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("M", [32, 64])
def test_gemm_skinny_config_full(P, oracle_mod, N, K, M):
    # Llama-7B block shapes at M = 32 / 64, map by least Wanda tile loss at
    # f = 0.6, every output compared
    seed = inputs.BASE_SEED + 2
    w = inputs.weight(N, K, seed + N)
    o = inputs.outlier_channels(K, seed)
    xc = inputs.activations(1024, K, seed, o, role=0)
    x = inputs.activations(M, K, seed, o, role=1 + M)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), fraction=0.6)
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    y16 = P.patch_hybrid_gemm(pk, x.cuda())
    y32 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    y32b = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    # chunk partials are added in a fixed order: repeated calls agree bit for bit
    assert torch.equal(y32, y32b)
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, frac=0.6)
    yref = oracle_mod.gemm(bf16_bits(x), weff)
    rel_rms_check(y32, yref, True)
    rel_rms_check(y16, yref, False)
    pk.close()


@pytest.mark.parametrize("M", [40, 64])
def test_gemm_skinny_one_band_kernel_forced(P, oracle_mod, M):
    # the one-band stream-K kernel with 64-token tiles (test hook) at the
    # token counts the split-K path now serves
    with forced_kernel(P, 1):
        run_case(P, oracle_mod, 1024, 2048, M, 128, 128, 0.5, seed=M + 9, fp32_mode=True)


@pytest.mark.parametrize("M", [20, 64])
def test_gemm_skinny_bounded_wait_reports_timeout(P, oracle_mod, M):
    # the failure-detection hook on the 32- / 64-token split-K kernel
    N, K = 256, 512
    w, xc, x = make_problem(N, K, 64, M, seed=43 + M)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=43)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    P.test_stall_first_kstep(True)
    try:
        P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5  # PATCH_ERR_TIMEOUT, read and cleared
    assert P.patch_get_status(pk) == 0
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    pk.close()


def group_problem(P, oracle_mod, shapes, K, seed, frac=0.5):
    """Handles for matrices [N_i, K] that share one input, random maps."""
    pks, weffs = [], []
    for i, N in enumerate(shapes):
        w, xc, _ = make_problem(N, K, 64, 1, seed + 7 * i)
        nt = (N // 128) * (K // 128)
        tmap = inputs.random_map(nt, int(round(frac * nt)), seed=seed + i)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
        pks.append(P.patch_pack(w.cuda(), r["meta"], r["map"]))
        weffs.append(oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap))
    return pks, weffs


@pytest.mark.parametrize("M", [1, 5, 16, 24, 64])
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_group_equals_single_calls(P, oracle_mod, M, fp32_mode):
    # one launch over three matrices that read the same X gives, bit for bit,
    # what three calls give (the same chunks, added in the same order)
    K = 1152  # 9 k-pairs per band: a ragged last chunk
    pks, weffs = group_problem(P, oracle_mod, [512, 768, 256], K, seed=200 + M)
    x = inputs.activations(M, K, 300 + M, None)
    xd = x.cuda()
    ys = P.patch_hybrid_gemm_group(pks, xd, out_fp32=fp32_mode)
    singles = [P.patch_hybrid_gemm(pk, xd, out_fp32=fp32_mode) for pk in pks]
    torch.cuda.synchronize()
    for pk in pks:
        assert P.patch_get_status(pk) == 0
    for y, y1, weff in zip(ys, singles, weffs):
        assert torch.equal(y, y1)
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), fp32_mode)
    for pk in pks:
        pk.close()


@pytest.mark.parametrize("M", [1, 8, 64])
def test_gemm_group_block_shapes(P, oracle_mod, M):
    # q, k, v (3 x 4096x4096) and gate, up (2 x 11008x4096) of the Llama-7B
    # block, each group in one launch; equal to single calls, and to the
    # oracle on sampled outputs
    K = 4096
    for shapes, seed in (([4096, 4096, 4096], 410), ([11008, 11008], 420)):
        pks, weffs = group_problem(P, oracle_mod, shapes, K, seed=seed + M, frac=0.6)
        x = inputs.activations(M, K, seed + M, inputs.outlier_channels(K, seed))
        xd = x.cuda()
        ys = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
        singles = [P.patch_hybrid_gemm(pk, xd, out_fp32=True) for pk in pks]
        torch.cuda.synchronize()
        g = np.random.default_rng(seed + M)
        for y, y1, weff, pk in zip(ys, singles, weffs, pks):
            assert P.patch_get_status(pk) == 0
            assert torch.equal(y, y1)
            ms, ns = g.integers(0, M, 3000), g.integers(0, pk.N, 3000)
            yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
            rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
        for pk in pks:
            pk.close()


@pytest.mark.parametrize("M", [200, 700, 1300])
@pytest.mark.parametrize("forced", [False, True])
def test_gemm_group_prefill_one_launch(P, oracle_mod, M, forced):
    # above 128 tokens a group of handles whose band pairs agree in type runs
    # as one two-SM launch over all their band pairs (test hook 3 takes it at
    # every size; otherwise the estimate decides); each output against the
    # oracle, every element
    K = 1152
    pks, weffs = group_problem(P, oracle_mod, [512, 768, 256], K, seed=230 + M)
    x = inputs.activations(M, K, 330 + M, None)
    xd = x.cuda()
    if forced:
        with forced_kernel(P, 3):
            ys = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
            ys16 = P.patch_hybrid_gemm_group(pks, xd, out_fp32=False)
            ys2 = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
    else:
        ys = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
        ys16 = P.patch_hybrid_gemm_group(pks, xd, out_fp32=False)
        ys2 = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
    torch.cuda.synchronize()
    for y, y16, yb, weff, pk in zip(ys, ys16, ys2, weffs, pks):
        assert P.patch_get_status(pk) == 0
        assert torch.equal(y, yb)  # repeatable
        yref = oracle_mod.gemm(bf16_bits(x), weff)
        rel_rms_check(y, yref, True)
        rel_rms_check(y16, yref, False)
    for pk in pks:
        pk.close()


@pytest.mark.parametrize("M", [512, 4096])
def test_gemm_group_prefill_block_shapes(P, oracle_mod, M):
    # q/k/v and gate/up of the Llama-7B block at prefill token counts, each
    # group through the grouped entry point; sampled outputs (every band
    # pair's edge rows included) against the oracle
    K = 4096
    for shapes, seed in (([4096, 4096, 4096], 510), ([11008, 11008], 520)):
        pks, weffs = group_problem(P, oracle_mod, shapes, K, seed=seed + M, frac=0.6)
        x = inputs.activations(M, K, seed + M, inputs.outlier_channels(K, seed))
        ys = P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
        torch.cuda.synchronize()
        g = np.random.default_rng(seed + M)
        for y, weff, pk in zip(ys, weffs, pks):
            assert P.patch_get_status(pk) == 0
            N = pk.N
            ms = np.concatenate([g.integers(0, M, 2000), np.array([0, M - 1, M // 2, 0, M - 1, 0])])
            ns = np.concatenate([g.integers(0, N, 2000), np.array([0, N - 1, 255, N - 256, 0, 128])])
            yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
            rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
        for pk in pks:
            pk.close()


def test_gemm_group_falls_back_to_single_calls(P, oracle_mod):
    # handles that cannot share a launch (a 4:8 handle; M above the split-K
    # range) are run one after another with the same results
    K, M = 512, 200
    pks, weffs = group_problem(P, oracle_mod, [256, 384], K, seed=77)
    x = inputs.activations(M, K, 78, None)
    ys = P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    for y, weff in zip(ys, weffs):
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    w, xc, _ = make_problem(256, K, 64, 1, 79)
    r48 = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=inputs.random_map(8, 4, seed=79).cuda(), nm=(4, 8))
    pk48 = P.patch_pack(w.cuda(), r48["meta"], r48["map"], nm=(4, 8))
    x8 = inputs.activations(8, K, 80, None)
    mixed = [pks[0], pk48]
    ys = P.patch_hybrid_gemm_group(mixed, x8.cuda(), out_fp32=True)
    singles = [P.patch_hybrid_gemm(pk, x8.cuda(), out_fp32=True) for pk in mixed]
    torch.cuda.synchronize()
    for y, y1 in zip(ys, singles):
        assert torch.equal(y, y1)
    for pk in pks + [pk48]:
        pk.close()


def test_gemm_group_bounded_wait_raises_every_status(P, oracle_mod):
    K, M = 512, 8
    pks, weffs = group_problem(P, oracle_mod, [256, 128, 384], K, seed=91)
    x = inputs.activations(M, K, 92, None)
    P.test_stall_first_kstep(True)
    try:
        P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    for pk in pks:
        assert P.patch_get_status(pk) == 5  # PATCH_ERR_TIMEOUT, read and cleared
    ys = P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    for y, weff, pk in zip(ys, weffs, pks):
        assert P.patch_get_status(pk) == 0
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    for pk in pks:
        pk.close()


def test_gemm_group_prefill_bounded_wait_raises_every_status(P, oracle_mod):
    # the grouped two-SM launch: a k-pair that never lands ends the launch
    # through its bounded waits and raises every member's status word
    K, M = 512, 300
    pks, weffs = group_problem(P, oracle_mod, [256, 512], K, seed=93)
    x = inputs.activations(M, K, 94, None)
    P.test_stall_first_kstep(True)
    try:
        with forced_kernel(P, 3):
            P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    for pk in pks:
        assert P.patch_get_status(pk) == 5  # PATCH_ERR_TIMEOUT, read and cleared
    with forced_kernel(P, 3):
        ys = P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    for y, weff, pk in zip(ys, weffs, pks):
        assert P.patch_get_status(pk) == 0
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    for pk in pks:
        pk.close()


def test_gemm_group_bad_arguments(P, oracle_mod):
    import ctypes
    lib = P.load_library()
    pks, _ = group_problem(P, oracle_mod, [128], 256, seed=95)
    x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    h = (ctypes.c_void_p * 9)(*([pks[0].handle] * 9))
    ys = (ctypes.c_void_p * 9)(*([ctypes.c_void_p(y.data_ptr())] * 9))
    xp = ctypes.c_void_p(x.data_ptr())
    assert lib.patch_hybrid_gemm_group(h, 0, xp, 4, ys, 1, None) == 1
    assert lib.patch_hybrid_gemm_group(h, 9, xp, 4, ys, 1, None) == 1
    assert lib.patch_hybrid_gemm_group(None, 1, xp, 4, ys, 1, None) == 1
    assert lib.patch_hybrid_gemm_group(h, 1, None, 4, ys, 1, None) == 1
    assert lib.patch_hybrid_gemm_group(h, 1, xp, 4, ys, 2, None) == 1
    assert lib.patch_hybrid_gemm_group(h, 1, xp, 0, ys, 1, None) == 0  # empty batch
    torch.cuda.synchronize()
    pks[0].close()


def test_gemm_tiny_config(P, oracle_mod):
    # W 256x256, 64x64 tiles, 8 of 16 tiles 2:4, Xcal 64x256, X 8x256, 3 outlier channels
    wl = inputs.workloads()["tiny"]
    s = wl.seed
    w = inputs.weight(256, 256, s)
    o = inputs.outlier_channels(256, s, 3)
    xc = inputs.activations(64, 256, s, o, role=0)
    x = inputs.activations(8, 256, s, o, role=1)
    tmap = inputs.random_map(16, 8, s)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=64, tile_k=64, map_in=tmap.cuda(),
                           want_colsq=True, want_loss=True)
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"], tile_n=64, tile_k=64)
    y32 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    y16 = P.patch_hybrid_gemm(pk, x.cuda())
    torch.cuda.synchronize()
    ref = oracle_mask(oracle_mod, w, xc, 64, 64, tmap=tmap.numpy().view(np.uint32))
    assert np.array_equal(u32(r["meta"]), ref["meta"])
    assert np.array_equal(r["colsq"].cpu().numpy(), ref["colsq"])
    weff = oracle_mod.weff(bf16_bits(w), ref["meta"], ref["map"], 64, 64)
    yref = oracle_mod.gemm(bf16_bits(x), weff)
    rel_rms_check(y32, yref, True)
    rel_rms_check(y16, yref, False)
    # achieved sparsity: 8 of 16 tiles 2:4 -> 25%
    w_eff = oracle_mod.bf16_bits_to_f64(weff)
    assert abs(np.mean(w_eff == 0) - 0.25) < 1e-3


def test_gemm_all_dense_matches_cublas(P):
    N, K, M = 1024, 2048, 512
    w, xc, x = make_problem(N, K, 64, M, seed=99)
    nt = (N // 128) * (K // 128)
    tmap = torch.zeros(((nt + 31) // 32,), dtype=torch.int32)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    ref = x.cuda().float() @ w.cuda().float().t()  # fp32 library GEMM of the same operands
    torch.cuda.synchronize()
    err = (y - ref).abs().max().item()
    rms = ref.pow(2).mean().sqrt().item()
    assert err <= 1e-2 * rms
    pk.close()


def test_gemm_empty_batch(P, oracle_mod):
    w, xc, x = make_problem(256, 256, 64, 4, seed=5)
    nt = 4
    tmap = inputs.random_map(nt, 2, seed=5)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    y = P.patch_hybrid_gemm(pk, x.cuda()[:0])
    assert y.shape == (0, 256)
    pk.close()


@pytest.mark.parametrize("N", [4096, 11008])
@pytest.mark.parametrize("M", [1, 4, 16])
def test_gemm_decode_config_full(P, oracle_mod, N, M):
    # Llama-7B decode shapes, map by least Wanda tile loss at f = 0.5
    K = 4096
    seed = inputs.BASE_SEED + 1
    w = inputs.weight(N, K, seed + N)
    o = inputs.outlier_channels(K, seed)
    xc = inputs.activations(2048, K, seed, o, role=0)
    x = inputs.activations(M, K, seed, o, role=1 + M)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), fraction=0.5)
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    y16 = P.patch_hybrid_gemm(pk, x.cuda())
    y32 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    # codes AND least-loss map from the oracle (the GPU's asserted equal)
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, frac=0.5)
    yref = oracle_mod.gemm(bf16_bits(x), weff)
    rel_rms_check(y32, yref, True)
    rel_rms_check(y16, yref, False)
    pk.close()


@pytest.mark.parametrize("N,K", [(11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_gemm_prefill_config_sampled(P, oracle_mod, N, K, frac):
    # Llama-7B prefill shapes at M = 2048, seeded random maps; sampled outputs
    run_case(P, oracle_mod, N, K, 2048, 128, 128, frac, seed=N + int(frac * 4),
             fp32_mode=False, sample=4000)


@pytest.mark.parametrize("M", [8, 300, 2048])
def test_gemm_first_call_does_not_block_the_host(P, oracle_mod, M):
    # The first GEMM on a fresh handle (decode and prefill token counts) must
    # only enqueue: queued behind a ~1 s spin kernel, the call returns while
    # the stream is still busy.  The result is then checked as usual.
    import time
    N, K = 1024, 1024
    w, xc, x = make_problem(N, K, 64, M, seed=61 + M)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=61)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    xd = x.cuda()
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    torch.cuda._sleep(2_000_000_000)  # about a second of GPU cycles
    t0 = time.perf_counter()
    P.patch_hybrid_gemm(pk, xd, out=y, out_fp32=True)
    dt = time.perf_counter() - t0
    busy = not stream.query()
    torch.cuda.synchronize()
    assert busy, "the stream finished before the call returned: the call waited for it"
    assert dt < 0.25, dt
    assert P.patch_get_status(pk) == 0
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    if M <= 300:
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    else:
        g = np.random.default_rng(M)
        ms, ns = g.integers(0, M, 3000), g.integers(0, N, 3000)
        yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
        rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
    pk.close()


FIRST_CALL_SCRIPT = r"""
import sys, time, torch
sys.path.insert(0, {root!r})
from sparse_gemm_wanda_b200 import inputs, patch as P
P.load_library()
N, K = 1024, 1024
w = inputs.weight(N, K, 5).cuda()
xc = inputs.activations(64, K, 5, None).cuda()
tmap = inputs.random_map(64, 32, seed=5).cuda()
r = P.patch_score_mask(w, xc, map_in=tmap)
pk = P.patch_pack(w, r["meta"], r["map"])
stream = torch.cuda.current_stream()
for M in (8, 40, 300, 2048):  # split-K 16 / 64 tokens, one-band, two-SM
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    torch.cuda._sleep(1_000_000_000)
    t0 = time.perf_counter()
    P.patch_hybrid_gemm(pk, x, out=y, out_fp32=True)
    dt = time.perf_counter() - t0
    busy = not stream.query()
    torch.cuda.synchronize()
    assert busy and dt < 0.2, (M, busy, dt)
print("first calls ok")
"""


def test_gemm_first_calls_of_a_process_do_not_block_the_host():
    # In a fresh process every GEMM kernel is launched for the first time;
    # under lazy module loading a first launch would load the kernel and wait
    # for the device, so the pack call (which waits anyway) loads them all.
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", FIRST_CALL_SCRIPT.format(root=root)],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "first calls ok" in out.stdout


def test_gemm_repeated_calls_reset_tickets(P, oracle_mod):
    # stream-K tiles shared by several CTAs: every call must find its tickets at zero
    N, K, M = 1024, 2048, 5
    w, xc, _ = make_problem(N, K, 64, M, seed=31)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=31)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    for rep in range(3):
        x = inputs.activations(M, K, 100 + rep, None)
        y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
        torch.cuda.synchronize()
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    assert P.patch_get_status(pk) == 0
    pk.close()


def test_gemm_bounded_wait_reports_timeout(P, oracle_mod):
    # Failure detection without a GPU fault: the first CTA never receives its
    # first k-step; its bounded wait runs out, the kernel returns, the status
    # word reports the timeout, and the handle works again once cleared.
    N, K, M = 256, 256, 4
    w, xc, x = make_problem(N, K, 64, M, seed=41)
    tmap = inputs.random_map(4, 2, seed=41)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    P.test_stall_first_kstep(True)
    try:
        P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5  # PATCH_ERR_TIMEOUT, read and cleared
    assert P.patch_get_status(pk) == 0
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), weff), True)
    pk.close()


def test_gemm_chain_overlapped_matches_serialised(P, oracle_mod):
    # A layer chain where each GEMM reads the previous one's output as its X:
    # back to back on one stream, each GEMM may start (prologue and first
    # weight copies) while its predecessor still runs, and must still read X
    # only after it finished.  The chained results must equal the same calls
    # with a device synchronisation between them, bit for bit, for decode and
    # prefill token counts; the first GEMM is checked against the oracle.
    shapes = [(1024, 512), (768, 1024), (512, 768)]  # (N, K): K of each = N of the previous
    pks, weffs = [], []
    for i, (N, K) in enumerate(shapes):
        w, xc, _ = make_problem(N, K, 64, 1, seed=700 + i)
        nt = (N // 128) * (K // 128)
        tmap = inputs.random_map(nt, nt // 2, seed=700 + i)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
        pks.append(P.patch_pack(w.cuda(), r["meta"], r["map"]))
        weffs.append(oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap))
    for M in (3, 16, 200):
        x0 = inputs.activations(M, shapes[0][1], 800 + M, None)
        xs = x0.cuda()
        chained = []
        for pk in pks:
            xs = P.patch_hybrid_gemm(pk, xs)
            chained.append(xs)
        torch.cuda.synchronize()
        xs = x0.cuda()
        for i, pk in enumerate(pks):
            xs = P.patch_hybrid_gemm(pk, xs)
            torch.cuda.synchronize()
            assert torch.equal(xs, chained[i]), (M, i)
        rel_rms_check(chained[0], oracle_mod.gemm(bf16_bits(x0), weffs[0]), False)
    for pk in pks:
        assert P.patch_get_status(pk) == 0
        pk.close()


@pytest.mark.parametrize("N,K,M,tn,tk,frac", [
    (4096, 512, 1300, 128, 128, 0.5),   # band-pair kernel, 160-token tiles, ragged last tile
    (3968, 512, 1300, 128, 128, 1.0),   # odd band count: the last pair holds one band
    (4096, 1024, 2000, 128, 128, 0.0),  # all dense, 224-token tiles
    (4096, 512, 1300, 64, 64, 0.5),     # 64x64 tiles: mixed 64-row tiles inside a band
])
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_band_pair_kernel(P, oracle_mod, N, K, M, tn, tk, frac, fp32_mode):
    # the band-pair kernel (two bands per CTA sharing each X tile), forced
    with forced_kernel(P, 2):
        run_case(P, oracle_mod, N, K, M, tn, tk, frac, seed=N + M + tn, fp32_mode=fp32_mode,
                 sample=6000)


@pytest.mark.parametrize("M", [200, 1300])
def test_gemm_one_band_kernel_forced(P, oracle_mod, M):
    # the one-band kernel (stream-K below two waves of tiles) at prefill sizes
    with forced_kernel(P, 1):
        run_case(P, oracle_mod, 2048, 1024, M, 128, 128, 0.5, seed=M + 5, fp32_mode=True,
                 sample=6000)


def test_gemm_band_pair_kernel_bounded_wait(P, oracle_mod):
    # the failure-detection hook on the band-pair kernel: CTA 0's first stage
    # never lands, its waits run out, the status reports the timeout and the
    # handle computes correctly once the status is read
    N, K, M = 4096, 512, 1300
    w, xc, x = make_problem(N, K, 64, M, seed=43)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=43)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    P.test_stall_first_kstep(True)
    try:
        with forced_kernel(P, 2):
            P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5
    assert P.patch_get_status(pk) == 0
    with forced_kernel(P, 2):
        y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    g = np.random.default_rng(43)
    ms, ns = g.integers(0, M, 3000), g.integers(0, N, 3000)
    yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
    rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
    pk.close()


def band_aligned_map(n_rows_tiles, n_col_tiles, seed):
    """A map whose tile rows 2p and 2p+1 (bands 2p, 2p+1 for 128-row tiles)
    share one random dense / 2:4 pattern along K."""
    g = np.random.default_rng(seed)
    words = [0] * ((n_rows_tiles * n_col_tiles + 31) // 32)
    for rp in range(n_rows_tiles // 2):
        pat = g.integers(0, 2, n_col_tiles)
        for r in (2 * rp, 2 * rp + 1):
            for k in range(n_col_tiles):
                if pat[k]:
                    t = r * n_col_tiles + k
                    words[t // 32] |= 1 << (t % 32)
    return torch.from_numpy(np.array(words, dtype=np.uint32).view(np.int32))


@pytest.mark.parametrize("N,K,M,tn,frac", [
    (4096, 512, 1300, 128, 1.0),   # two-SM kernel: every tile 2:4, 160-token tiles, ragged
    (4096, 1024, 2000, 128, 0.0),  # every tile dense
    (4096, 512, 1300, 64, 1.0),    # 64x64 tiles, every tile 2:4
])
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_two_sm_kernel(P, oracle_mod, N, K, M, tn, frac, fp32_mode):
    # maps whose bands 2p and 2p+1 agree in type at every k-step run the
    # cta_group::2 kernel on the packed k-steps alone (one band per SM of a
    # CTA pair, M = 256 MMAs)
    with forced_kernel(P, 3):
        run_case(P, oracle_mod, N, K, M, tn, tn, frac, seed=N + M + 7 * tn, fp32_mode=fp32_mode,
                 sample=6000)


@pytest.mark.parametrize("N,K,M,tn,tk,frac", [
    (4096, 1024, 1300, 128, 128, 0.5),   # random map: half the k-pairs of a band pair differ
    (4096, 1024, 1300, 128, 128, 0.25),
    (4096, 1024, 1300, 64, 64, 0.5),     # 64-row tiles: mixed halves inside a band
    (4096, 1024, 1300, 128, 64, 0.5),    # 64-column tiles: k-pairs of mixed type
    (2048, 768, 700, 64, 128, 0.75),
])
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_two_sm_kernel_mixed_maps(P, oracle_mod, N, K, M, tn, tk, frac, fp32_mode):
    # any map runs the two-SM kernel through the prefill table: where the two
    # bands of an instruction differ in type, their k-pairs come from dense
    # copies of W_eff written by the packer after the packed bytes
    with forced_kernel(P, 3):
        run_case(P, oracle_mod, N, K, M, tn, tk, frac, seed=N + M + tn + tk, fp32_mode=fp32_mode,
                 sample=6000)


@pytest.mark.parametrize("N,K,M,frac", [
    (1024, 1024, 300, 0.5),    # fewer items than clusters
    (2048, 2048, 256, 0.6),
    (4096, 4096, 512, 0.6),    # Llama-7B block shapes at M = 512
    (11008, 4096, 512, 0.6),
    (4096, 11008, 512, 0.6),
    (4096, 1024, 4096, 0.5),   # many waves
])
def test_gemm_two_sm_kernel_block_shapes(P, oracle_mod, N, K, M, frac):
    # the two-SM kernel where its items fill one wave or less (M = 256 / 512
    # on the Llama-7B block shapes), a problem with fewer items than
    # clusters, and one of many waves; repeated calls agree bit for bit
    w, xc, x = make_problem(N, K, 64, M, seed=N + K + M)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, int(round(frac * nt)), seed=N + M)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    xd = x.cuda()
    with forced_kernel(P, 3):
        y16 = P.patch_hybrid_gemm(pk, xd)
        y32 = P.patch_hybrid_gemm(pk, xd, out_fp32=True)
        y32b = P.patch_hybrid_gemm(pk, xd, out_fp32=True)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    assert torch.equal(y32, y32b)
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    if M * N <= 300 * 1024:
        yref = oracle_mod.gemm(bf16_bits(x), weff)
        rel_rms_check(y32, yref, True)
        rel_rms_check(y16, yref, False)
    else:
        g = np.random.default_rng(N + M)
        # every row of the first band pair and the last, and random outputs
        ms = np.concatenate([g.integers(0, M, 3000), np.repeat(np.arange(M)[:: max(1, M // 16)], 4)])
        ns = np.concatenate([g.integers(0, N, 3000),
                             np.tile(np.array([0, 255, N - 256, N - 1]), len(np.arange(M)[:: max(1, M // 16)]))])
        yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
        mi, ni = torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()
        rel_rms_check(y32[mi, ni], yref, True)
        rel_rms_check(y16[mi, ni], yref, False)
    pk.close()


@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_two_sm_kernel_band_aligned_mixed_map(P, oracle_mod, fp32_mode):
    # dense and 2:4 k-steps alternate along K inside one item; both bands of
    # every instruction agree
    N, K, M = 4096, 1024, 1300
    w, xc, x = make_problem(N, K, 64, M, seed=91)
    tmap = band_aligned_map(N // 128, K // 128, seed=91)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=fp32_mode)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    g = np.random.default_rng(91)
    ms, ns = g.integers(0, M, 6000), g.integers(0, N, 6000)
    yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
    rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, fp32_mode)
    pk.close()


def test_gemm_two_sm_kernel_bounded_wait(P, oracle_mod):
    # the failure-detection hook on the two-SM kernel: the first CTA never
    # arms its first stage; both CTAs of its pair give up within their bounds,
    # meet at the final cluster barrier, and the handle works afterwards
    N, K, M = 4096, 512, 1300
    w, xc, x = make_problem(N, K, 64, M, seed=47)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt, seed=47)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    P.test_stall_first_kstep(True)
    try:
        P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5
    assert P.patch_get_status(pk) == 0
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    g = np.random.default_rng(47)
    ms, ns = g.integers(0, M, 3000), g.integers(0, N, 3000)
    yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
    rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
    pk.close()


# ------------------------------------------------- multi-GPU split, one GPU

@pytest.mark.parametrize("world,N,K,T,M,frac", [
    (2, 1024, 1024, 1000, 200, 0.5),
    (3, 4096, 4096, 2048, 16, 0.5),
])
def test_sharded_pieces_match_whole(P, oracle_mod, world, N, K, T, M, frac):
    # The pieces the multi-GPU split gives each rank (sparse_gemm_wanda_b200/
    # sharded.py), computed one after another on this GPU: the token pieces'
    # chunk partials folded in order equal the whole set's sums; each row
    # piece's codes and losses equal those rows of the whole matrix; the
    # least-loss selection over the pieces' losses (rank order) gives each
    # piece its slice of the whole map; each piece's GEMM matches the oracle.
    from sparse_gemm_wanda_b200 import sharded
    w, xc, x = make_problem(N, K, T, M, seed=900 + world)
    ref = oracle_mask(oracle_mod, w, xc, 128, 128, frac=frac)
    wd, xcd, xd = w.cuda(), xc.cuda(), x.cuda()
    parts = [P.patch_colsq_partials(xcd[t0:t1]) for t0, t1 in sharded.token_ranges(T, world) if t1 > t0]
    s = P.patch_colsq_fold(torch.cat(parts))
    torch.cuda.synchronize()
    assert np.array_equal(s.cpu().numpy(), ref["colsq"])
    rows = sharded.row_ranges(N, world)
    res = [P.patch_score_mask(wd[n0:n1], None, fraction=frac, colsq_in=s, want_loss=True)
           for n0, n1 in rows]
    maps = P.patch_select_maps_global([r["loss"] for r in res], frac)
    torch.cuda.synchronize()
    tiles_k = K // 128
    full_bits = np.unpackbits(ref["map"].view(np.uint8), bitorder="little")
    weff = oracle_mod.weff(bf16_bits(w), ref["meta"], ref["map"], 128, 128)
    for (n0, n1), r, m in zip(rows, res, maps):
        assert np.array_equal(u32(r["meta"]), ref["meta"][n0:n1])
        nt = (n1 - n0) // 128 * tiles_k
        g0 = n0 // 128 * tiles_k
        mine = np.unpackbits(u32(m).view(np.uint8), bitorder="little")[:nt]
        assert np.array_equal(mine, full_bits[g0:g0 + nt])
        pk = P.patch_pack(wd[n0:n1], r["meta"], m)
        y = P.patch_hybrid_gemm(pk, xd, out_fp32=True)
        torch.cuda.synchronize()
        assert P.patch_get_status(pk) == 0
        rel_rms_check(y, oracle_mod.gemm(bf16_bits(x), np.ascontiguousarray(weff[n0:n1])), True)
        pk.close()


# ------------------------------------------- two-SM kernel, two bands per SM

@pytest.mark.parametrize("N,K,M,tn,tk,frac", [
    (4096, 1024, 1300, 128, 128, 0.0),   # every tile dense
    (4096, 1024, 1300, 128, 128, 1.0),   # every tile 2:4
    (4096, 1024, 1300, 128, 128, 0.5),   # random map through the prefill table
    (4352, 512, 700, 64, 64, 0.5),       # 34 bands: the last quad holds one band pair
    (768, 1024, 333, 128, 64, 0.75),     # 6 bands, 64-column tiles, ragged token tile
    (2048, 768, 2000, 64, 128, 1.0),
])
@pytest.mark.parametrize("fp32_mode", [True, False])
def test_gemm_quad_kernel(P, oracle_mod, N, K, M, tn, tk, frac, fp32_mode):
    # four bands per CTA pair: bands 4q+2j (leader) and 4q+2j+1 (peer) in one
    # M = 256 instruction per pair j, both pairs sharing each SM's X half
    with forced_kernel(P, 4):
        run_case(P, oracle_mod, N, K, M, tn, tk, frac, seed=N + M + 3 * tn + tk,
                 fp32_mode=fp32_mode, sample=6000)


def test_gemm_quad_kernel_bounded_wait(P, oracle_mod):
    # the failure-detection hook on the four-band kernel: the first CTA never
    # arms its first stage; both CTAs of its pair give up within their bounds,
    # meet at the final cluster barrier, and the handle works afterwards
    N, K, M = 4096, 512, 1300
    w, xc, x = make_problem(N, K, 64, M, seed=53)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=53)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack(w.cuda(), r["meta"], r["map"])
    P.test_stall_first_kstep(True)
    try:
        with forced_kernel(P, 4):
            P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5
    assert P.patch_get_status(pk) == 0
    with forced_kernel(P, 4):
        y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    weff = oracle_weff_checked(oracle_mod, r, w, xc, 128, 128, tmap=tmap)
    g = np.random.default_rng(53)
    ms, ns = g.integers(0, M, 3000), g.integers(0, N, 3000)
    yref = oracle_mod.gemm_at(bf16_bits(x), weff, ms, ns)
    rel_rms_check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
    pk.close()
