"""FP8 (e4m3) values inside dense and 2:4 tiles on the GPU against the oracle,
through the C ABI ("SparseGPT vs Wanda", FAQ: prune first, then quantise).

Bit-exact: the e4m3 codes and fp32 scales of the per-row quantisation (X per
token, W_eff per output row), the packed bytes and the k-step table.  GEMM
(tcgen05 kind::f8f6f4, dense and sparse MMAs): against the oracle's fp64 sums
of the oracle's own codes, within the tolerance reading of the bf16 tests
(fp32 output: max err <= 1e-2 RMS; bf16 output: + half a bf16 ulp).
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


@pytest.mark.parametrize("R,C", [(1, 8), (5, 256), (300, 4096), (64, 11008)])
def test_quantize_fp8_bit_exact(P, oracle_mod, R, C):
    g = torch.Generator().manual_seed(R + C)
    x = torch.randn(R, C, generator=g) * 3
    x[:, : C // 16] *= 50              # outlier channels
    if R > 2:
        x[1] = 0.0                     # a zero row: scale 1, codes 0
        x[2, ::3] = -0.0               # negative zeros keep their sign
    xb = x.to(torch.bfloat16)
    codes, scales = P.patch_quantize_fp8(xb.cuda())
    torch.cuda.synchronize()
    ref_s = oracle_mod.fp8_row_scales(bf16_bits(xb))
    ref_q = oracle_mod.fp8_quantize(bf16_bits(xb), ref_s)
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    assert np.array_equal(codes.cpu().numpy(), ref_q)


def oracle_fp8(oracle_mod, w, xc, tmap, tn, tk):
    ref = oracle_mod.score_mask(bf16_bits(w), bf16_bits(xc), tn, tk,
                                tile_map=tmap.numpy().view(np.uint32))
    weff = oracle_mod.weff(bf16_bits(w), ref["meta"], ref["map"], tn, tk)
    sw = oracle_mod.fp8_row_scales(weff)
    qw = oracle_mod.fp8_quantize(weff, sw)
    return ref, sw, qw


@pytest.mark.parametrize("tn,tk", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_pack_fp8_bit_exact(P, oracle_mod, tn, tk, frac):
    N, K = 384, 512
    w = inputs.weight(N, K, 5 + tn + tk)
    o = inputs.outlier_channels(K, 5)
    xc = inputs.activations(64, K, 5, o, role=0)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), seed=tn + 3 * tk)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda())
    pk = P.patch_pack_fp8(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk)
    packed, table = pk.export()
    sw = pk.fp8_scales()
    torch.cuda.synchronize()
    ref, ref_sw, ref_qw = oracle_fp8(oracle_mod, w, xc, tmap, tn, tk)
    assert np.array_equal(sw.cpu().numpy(), ref_sw)
    ref_packed, ref_table = oracle_mod.pack_fp8(ref_qw, ref["meta"], ref["map"], tn, tk)
    assert pk.packed_bytes == ref_packed.size
    assert np.array_equal(table.cpu().numpy().view(np.uint64), ref_table)
    assert np.array_equal(packed.cpu().numpy(), ref_packed)
    pk.close()


class forced_kernel:
    """Select the prefill kernel for the calls inside the block (test hook)."""

    def __init__(self, P, which):
        self.P, self.which = P, which

    def __enter__(self):
        self.P.test_prefill_kernel(self.which)

    def __exit__(self, *exc):
        self.P.test_prefill_kernel(0)


def run_fp8_gemm(P, oracle_mod, N, K, M, tn, tk, frac, seed, fp32_mode, sample=None):
    w = inputs.weight(N, K, seed)
    o = inputs.outlier_channels(K, seed)
    xc = inputs.activations(128, K, seed, o, role=0)
    x = inputs.activations(M, K, seed, o, role=1)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), seed=seed)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), tile_n=tn, tile_k=tk, map_in=tmap.cuda())
    pk = P.patch_pack_fp8(w.cuda(), r["meta"], r["map"], tile_n=tn, tile_k=tk)
    y = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=fp32_mode)
    torch.cuda.synchronize()
    assert P.patch_get_status(pk) == 0
    ref, sw, qw = oracle_fp8(oracle_mod, w, xc, tmap, tn, tk)
    assert np.array_equal(r["meta"].cpu().numpy().view(np.uint32), ref["meta"])
    sx = oracle_mod.fp8_row_scales(bf16_bits(x))
    qx = oracle_mod.fp8_quantize(bf16_bits(x), sx)
    if sample is None:
        check(y, oracle_mod.gemm_fp8(qx, sx, qw, sw), fp32_mode)
    else:
        g = np.random.default_rng(seed)
        ms, ns = g.integers(0, M, sample), g.integers(0, N, sample)
        yref = oracle_mod.gemm_fp8_at(qx, sx, qw, sw, ms, ns)
        check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, fp32_mode)
        rows = slice(N - 128, N)  # one whole band, every token
        check(y[:, rows], oracle_mod.gemm_fp8(qx, sx, np.ascontiguousarray(qw[rows]), sw[rows]), fp32_mode)
    pk.close()


@pytest.mark.parametrize("fp32_mode", [True, False])
@pytest.mark.parametrize("M", [1, 7, 16, 64, 100, 200, 300])
def test_gemm_fp8_small_shapes(P, oracle_mod, M, fp32_mode):
    run_fp8_gemm(P, oracle_mod, 384, 512, M, 128, 128, 0.5, seed=M + 60, fp32_mode=fp32_mode)


@pytest.mark.parametrize("tn,tk", [(128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_gemm_fp8_tiles_and_fractions(P, oracle_mod, tn, tk, frac):
    run_fp8_gemm(P, oracle_mod, 256, 768, 150, tn, tk, frac, seed=tn + tk + 11, fp32_mode=True)


@pytest.mark.parametrize("M", [16, 2048])
@pytest.mark.parametrize("frac", [0.5, 1.0])
def test_gemm_fp8_llama_mlp_shape(P, oracle_mod, M, frac):
    run_fp8_gemm(P, oracle_mod, 11008, 4096, M, 128, 128, frac, seed=91 + M, fp32_mode=False,
                 sample=4000 if M > 16 else None)


@pytest.mark.parametrize("N,K,M,tn,tk,frac", [
    (1024, 1024, 700, 128, 128, 0.5),   # random map: side copies where a band pair differs
    (1024, 1024, 700, 128, 128, 1.0),   # every k-step 2:4 (the smaller weight slot)
    (1024, 1024, 700, 128, 128, 0.0),   # every k-step dense
    (768, 512, 333, 64, 64, 0.5),       # 64-row tiles: halves of a band differ
    (512, 1536, 1000, 128, 64, 0.75),   # 64-column tiles
    (256, 768, 129, 128, 128, 0.5),     # one band pair, a ragged second tile
])
@pytest.mark.parametrize("kernel", [1, 3])
def test_gemm_fp8_one_band_and_two_sm(P, oracle_mod, N, K, M, tn, tk, frac, kernel):
    # the same FP8 handle through the one-band kernel (1) and the two-SM
    # kernel on the prefill table (3), compared in full with the oracle
    with forced_kernel(P, kernel):
        run_fp8_gemm(P, oracle_mod, N, K, M, tn, tk, frac, seed=N + M + tn + tk + kernel, fp32_mode=True)


def test_gemm_fp8_odd_kstep_count_falls_back(P, oracle_mod):
    # an odd number of 128-column k-steps (K = 384) keeps the one-band kernel
    with forced_kernel(P, 3):
        run_fp8_gemm(P, oracle_mod, 512, 384, 300, 128, 128, 0.5, seed=17, fp32_mode=False)


@pytest.mark.parametrize("N,K", [(128, 256), (256, 1280), (384, 2304), (128, 3072)])
@pytest.mark.parametrize("M", [1, 5, 16, 33, 64])
def test_gemm_fp8_split_k_ragged_chunks(P, oracle_mod, N, K, M):
    # M <= 64 on FP8 handles with an even count of 128-column k-steps: the
    # split-K kernel; pairs per band 1, 5, 9, 12 (chunks of fewer than four
    # pairs, single-pair stages, single-band matrices), 16 / 32 / 64-token tiles
    run_fp8_gemm(P, oracle_mod, N, K, M, 128, 128, 0.5, seed=N + K + M, fp32_mode=True)


@pytest.mark.parametrize("M", [1, 16, 64])
def test_gemm_fp8_split_k_full_shapes(P, oracle_mod, M):
    # the Llama-7B decode shapes on FP8 handles: every output of one band and
    # sampled outputs everywhere; repeated calls agree bit for bit
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008)):
        run_fp8_gemm(P, oracle_mod, N, K, M, 128, 128, 0.5, seed=N + M, fp32_mode=False, sample=4000)


def test_gemm_fp8_split_k_repeatable_and_bounded_wait(P, oracle_mod):
    N, K, M = 512, 1024, 8
    w = inputs.weight(N, K, 71)
    xc = inputs.activations(128, K, 71, None, role=0)
    x = inputs.activations(M, K, 72, None, role=1)
    nt = (N // 128) * (K // 128)
    tmap = inputs.random_map(nt, nt // 2, seed=71)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pk = P.patch_pack_fp8(w.cuda(), r["meta"], r["map"])
    y0 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    y1 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)  # chunks added in a fixed order
    # failure detection: the first CTA never receives its first k-step; its
    # bounded wait runs out and the status word reports it
    P.test_stall_first_kstep(True)
    try:
        P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    finally:
        P.test_stall_first_kstep(False)
    assert P.patch_get_status(pk) == 5
    assert P.patch_get_status(pk) == 0
    y2 = P.patch_hybrid_gemm(pk, x.cuda(), out_fp32=True)
    torch.cuda.synchronize()
    assert torch.equal(y0, y2)
    pk.close()


@pytest.mark.parametrize("M", [1, 16, 64])
def test_gemm_fp8_group_equals_single_calls(P, oracle_mod, M):
    # FP8 handles that read one X: X quantised once, one split-K launch over
    # the group; every output equals its single call bit for bit
    K = 1024
    pks, refs = [], []
    x = inputs.activations(M, K, 500 + M, None, role=1)
    for i, N in enumerate((512, 256, 384)):
        w = inputs.weight(N, K, 510 + i)
        xc = inputs.activations(128, K, 510 + i, None, role=0)
        nt = (N // 128) * (K // 128)
        tmap = inputs.random_map(nt, nt // 2, seed=520 + i)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
        pks.append(P.patch_pack_fp8(w.cuda(), r["meta"], r["map"]))
        refs.append(oracle_fp8(oracle_mod, w, xc, tmap, 128, 128))
    xd = x.cuda()
    ys = P.patch_hybrid_gemm_group(pks, xd, out_fp32=True)
    singles = [P.patch_hybrid_gemm(pk, xd, out_fp32=True) for pk in pks]
    torch.cuda.synchronize()
    sx = oracle_mod.fp8_row_scales(bf16_bits(x))
    qx = oracle_mod.fp8_quantize(bf16_bits(x), sx)
    for y, y1, (ref, sw, qw), pk in zip(ys, singles, refs, pks):
        assert P.patch_get_status(pk) == 0
        assert torch.equal(y, y1)
        check(y, oracle_mod.gemm_fp8(qx, sx, qw, sw), True)
    # a group mixing an FP8 and a bf16 handle runs as single calls
    w = inputs.weight(256, K, 530)
    xc = inputs.activations(128, K, 530, None, role=0)
    tmap = inputs.random_map(16, 8, seed=530)
    r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
    pkb = P.patch_pack(w.cuda(), r["meta"], r["map"])
    mixed = [pks[0], pkb]
    ym = P.patch_hybrid_gemm_group(mixed, xd, out_fp32=True)
    ys1 = [P.patch_hybrid_gemm(pk, xd, out_fp32=True) for pk in mixed]
    torch.cuda.synchronize()
    for y, y1 in zip(ym, ys1):
        assert torch.equal(y, y1)
    for pk in pks + [pkb]:
        pk.close()


def fp8_group_problem(P, oracle_mod, shapes, K, fracs, seed):
    """FP8 handles for matrices [N_i, K] that share one input, random maps."""
    pks, refs = [], []
    for i, (N, frac) in enumerate(zip(shapes, fracs)):
        w = inputs.weight(N, K, seed + i)
        xc = inputs.activations(128, K, seed + i, None, role=0)
        nt = (N // 128) * (K // 128)
        tmap = inputs.random_map(nt, int(round(frac * nt)), seed=seed + 50 + i)
        r = P.patch_score_mask(w.cuda(), xc.cuda(), map_in=tmap.cuda())
        pks.append(P.patch_pack_fp8(w.cuda(), r["meta"], r["map"]))
        ref = oracle_fp8(oracle_mod, w, xc, tmap, 128, 128)
        assert np.array_equal(r["meta"].cpu().numpy().view(np.uint32), ref[0]["meta"])
        refs.append(ref)
    return pks, refs


@pytest.mark.parametrize("M", [200, 700])
@pytest.mark.parametrize("fracs", [(0.5, 1.0, 0.25), (1.0, 1.0, 1.0)])
@pytest.mark.parametrize("forced", [False, True])
def test_gemm_fp8_group_prefill_one_launch(P, oracle_mod, M, fracs, forced):
    # above 128 tokens FP8 handles that read one X: X quantised once and,
    # when the estimate takes it (always under test hook 3), one two-SM
    # launch over every matrix's band pairs; every element against the oracle
    # (a group whose matrices are all 2:4 gets the smaller weight slot)
    K = 1024
    pks, refs = fp8_group_problem(P, oracle_mod, (512, 768, 256), K, fracs, seed=600 + M)
    x = inputs.activations(M, K, 640 + M, None, role=1)
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
    sx = oracle_mod.fp8_row_scales(bf16_bits(x))
    qx = oracle_mod.fp8_quantize(bf16_bits(x), sx)
    for y, y16, yb, (ref, sw, qw), pk in zip(ys, ys16, ys2, refs, pks):
        assert P.patch_get_status(pk) == 0
        assert torch.equal(y, yb)  # repeatable
        yref = oracle_mod.gemm_fp8(qx, sx, qw, sw)
        check(y, yref, True)
        check(y16, yref, False)
    for pk in pks:
        pk.close()


def test_gemm_fp8_group_prefill_block_shapes(P, oracle_mod):
    # q/k/v and gate/up of the Llama-7B block on FP8 handles at M = 512
    # through the grouped entry point; sampled outputs (edge rows of the
    # first and last band pair included) against the oracle
    K, M = 4096, 512
    for shapes, seed in (((4096, 4096, 4096), 700), ((11008, 11008), 710)):
        pks, refs = fp8_group_problem(P, oracle_mod, shapes, K, (0.6,) * len(shapes), seed=seed)
        x = inputs.activations(M, K, seed + 5, inputs.outlier_channels(K, seed), role=1)
        ys = P.patch_hybrid_gemm_group(pks, x.cuda(), out_fp32=True)
        torch.cuda.synchronize()
        sx = oracle_mod.fp8_row_scales(bf16_bits(x))
        qx = oracle_mod.fp8_quantize(bf16_bits(x), sx)
        g = np.random.default_rng(seed)
        for y, (ref, sw, qw), pk in zip(ys, refs, pks):
            assert P.patch_get_status(pk) == 0
            N = pk.N
            ms = np.concatenate([g.integers(0, M, 2000), np.array([0, M - 1, M // 2, 0, M - 1, 0])])
            ns = np.concatenate([g.integers(0, N, 2000), np.array([0, N - 1, 255, N - 256, 0, 128])])
            yref = oracle_mod.gemm_fp8_at(qx, sx, qw, sw, ms, ns)
            check(y[torch.from_numpy(ms).cuda(), torch.from_numpy(ns).cuda()], yref, True)
        for pk in pks:
            pk.close()
