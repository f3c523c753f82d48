"""Pins of the CPU oracle to facts fixed outside the oracle itself.

Each oracle step is checked against something other than its own formula:
closed forms, exact rational brute force, invariants of 2:4 / tile sparsity,
hand-worked golden fixtures (tests/golden/, each citing its page), and library
routines (numpy fp64 matmul / sum) for the special cases that reduce to them.
The checks are chosen so that a dropped term, a swapped kept/pruned set, a
wrong tie rule, a transposed operand or a wrong tile index fails at least one.
"""
import os
from fractions import Fraction
from itertools import combinations

import numpy as np
import pytest
import torch

from tests.conftest import bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALLOWED_CODES = {4, 8, 12, 9, 13, 14}


def to_bits(values, shape=None):
    t = torch.tensor(np.asarray(values, dtype=np.float32))
    if shape is not None:
        t = t.reshape(shape)
    return bf16_bits(t.to(torch.bfloat16))


def codes_of(meta):
    """Unpack uint32 meta words into per-group 4-bit codes [N, K/4]."""
    meta = np.asarray(meta, dtype=np.uint32)
    shifts = (np.arange(8, dtype=np.uint32) * 4)
    c = (meta[..., None] >> shifts) & 0xF
    return c.reshape(meta.shape[0], -1)


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------
# column sum of squares
# ----------------------------------------------------------------------------

def test_colsq_constant_ones_ragged(oracle_mod):
    # X == 1 -> s_j = T exactly, with a ragged last chunk (300 = 2*128 + 44)
    x = to_bits(np.ones((300, 40)))
    s = oracle_mod.colsq(x)
    assert np.all(s == 300.0)


def test_colsq_one_hot(oracle_mod):
    x = np.zeros((257, 16), dtype=np.float32)
    x[200, 5] = 3.0
    x[0, 7] = -0.5
    s = oracle_mod.colsq(to_bits(x))
    expect = np.zeros(16)
    expect[5] = 9.0
    expect[7] = 0.25
    assert np.array_equal(s, expect)


def test_colsq_integer_exact(oracle_mod):
    rng = np.random.default_rng(0)
    xi = rng.integers(-8, 9, size=(1000, 64))
    s = oracle_mod.colsq(to_bits(xi.astype(np.float32)))
    assert np.array_equal(s, (xi.astype(np.int64) ** 2).sum(axis=0).astype(np.float64))


def test_colsq_matches_numpy_sum(oracle_mod):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(777, 96, generator=g) * 5).to(torch.bfloat16)
    s = oracle_mod.colsq(bf16_bits(x))
    ref = (x.double() ** 2).sum(0).numpy()
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=0)


# ----------------------------------------------------------------------------
# scores
# ----------------------------------------------------------------------------

def test_scores_hand_values(oracle_mod):
    # -0.5, 1.5, -0.0, 2.0 as bf16 bit patterns
    w = np.array([[0xBF00, 0x3FC0, 0x8000, 0x4000]], dtype=np.uint16)
    s = np.array([4.0, 9.0, 0.25, 0.0])
    sc = oracle_mod.wanda_scores(w, s)
    assert np.array_equal(sc, [[1.0, 4.5, 0.0, 0.0]])
    assert not np.signbit(sc[0, 2]), "|w| of -0 must be +0"


def test_golden_activation_outranks_magnitude(oracle_mod):
    rows = {r[0]: r[1:] for r in read_golden("wanda_activation_outranks_magnitude.txt")}
    w = to_bits([float(v) for v in rows["w"]], (1, 4))
    w = np.concatenate([w, np.zeros((1, 28), np.uint16)], axis=1)  # one 32-wide word
    s = np.concatenate([np.array([float(v) for v in rows["s"]]), np.ones(28)])
    sc = oracle_mod.wanda_scores(w, s)
    assert np.array_equal(sc[0, :4], [float(v) for v in rows["score"]])
    code = codes_of(oracle_mod.select_2of4(sc))[0, 0]
    assert code == int(rows["code"][0])
    # dropping the activation term (all norms 1) gives the magnitude-only code
    code_mag = codes_of(oracle_mod.select_2of4(oracle_mod.wanda_scores(w, np.ones(32))))[0, 0]
    assert code_mag == int(rows["magnitude_only_code"][0])


# ----------------------------------------------------------------------------
# top-2-of-4 selection
# ----------------------------------------------------------------------------

def brute_force_code(sc4):
    """Best of the 6 patterns by exact kept sum; ties -> lexicographically smallest pair."""
    best = None
    for pair in combinations(range(4), 2):  # already in lexicographic order
        total = Fraction(sc4[pair[0]]) + Fraction(sc4[pair[1]])
        if best is None or total > best[0]:
            best = (total, pair)
    a, b = best[1]
    return a | (b << 2)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_equals_bruteforce_with_ties(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    # few distinct values -> many exact ties
    sc = rng.choice([0.0, 0.5, 1.0, 1.5, 2.0], size=(64, 64)).astype(np.float64)
    codes = codes_of(oracle_mod.select_2of4(sc))
    for i in range(sc.shape[0]):
        for g in range(sc.shape[1] // 4):
            assert codes[i, g] == brute_force_code(sc[i, 4 * g:4 * g + 4]), (i, g)


def test_select_equals_bruteforce_random(oracle_mod):
    rng = np.random.default_rng(11)
    sc = np.abs(rng.standard_normal((32, 256)))
    codes = codes_of(oracle_mod.select_2of4(sc))
    for i in range(sc.shape[0]):
        for g in range(sc.shape[1] // 4):
            assert codes[i, g] == brute_force_code(sc[i, 4 * g:4 * g + 4])


@pytest.mark.parametrize("group,code", [((1, 1, 1, 1), 0x4), ((1, 3, 2, 0), 0x9),
                                        ((0, 0, 0, 1), 0xC), ((5, 1, 1, 5), 0xC),
                                        ((0, 2, 2, 2), 0x9), ((1, 0, 0, 1), 0xC),
                                        ((0, 0, 1, 1), 0xE), ((2, 0, 2, 0), 0x8)])
def test_select_special_cases(oracle_mod, group, code):
    sc = np.zeros((1, 32))
    sc[0, :4] = group
    assert codes_of(oracle_mod.select_2of4(sc))[0, 0] == code


def test_golden_patterns_all_reachable(oracle_mod):
    rows = read_golden("two_four_patterns.txt")
    assert len(rows) == 6
    seen = {}
    for idx0, idx1, code in rows:
        sc = np.zeros((1, 32))
        sc[0, int(idx0)] = 2.0
        sc[0, int(idx1)] = 1.0
        got = codes_of(oracle_mod.select_2of4(sc))[0, 0]
        assert got == int(code)
        seen[int(code)] = True
    assert set(seen) == ALLOWED_CODES


def test_select_dominance_and_alphabet(oracle_mod):
    rng = np.random.default_rng(5)
    sc = np.abs(rng.standard_normal((16, 128))).round(1)
    codes = codes_of(oracle_mod.select_2of4(sc))
    assert set(np.unique(codes)) <= ALLOWED_CODES
    for i in range(16):
        for g in range(32):
            c = codes[i, g]
            keep = {c & 3, c >> 2}
            grp = sc[i, 4 * g:4 * g + 4]
            for k in keep:
                for d in set(range(4)) - keep:
                    # kept beats dropped in the order (score desc, index asc)
                    assert grp[k] > grp[d] or (grp[k] == grp[d] and k < d)


# ----------------------------------------------------------------------------
# tile loss
# ----------------------------------------------------------------------------

def pruned_mask(codes, K):
    N = codes.shape[0]
    keep = np.zeros((N, K), dtype=bool)
    for g in range(K // 4):
        c = codes[:, g]
        for pos in range(4):
            keep[:, 4 * g + pos] = ((c & 3) == pos) | ((c >> 2) == pos)
    return ~keep


def test_tile_loss_exact_dyadic(oracle_mod):
    # dyadic scores with small magnitude: every partial sum is exact in fp64,
    # so the loss must equal the exact rational sum of the pruned scores,
    # whatever the order.
    rng = np.random.default_rng(7)
    N, K, tn, tk = 128, 192, 64, 64
    sc = rng.integers(0, 4096, size=(N, K)) / 8.0
    meta = oracle_mod.select_2of4(sc)
    loss = oracle_mod.tile_loss(sc, meta, tn, tk)
    pm = pruned_mask(codes_of(meta), K)
    tiles_k = K // tk
    for t in range(len(loss)):
        i0, j0 = (t // tiles_k) * tn, (t % tiles_k) * tk
        blk = sc[i0:i0 + tn, j0:j0 + tk][pm[i0:i0 + tn, j0:j0 + tk]]
        assert Fraction(loss[t]) == sum(Fraction(v) for v in blk)
        # exactly half of every tile is pruned
        assert blk.size == tn * tk // 2


def test_tile_loss_order_is_the_stated_tree(oracle_mod):
    # Row sums chosen so that fp64 rounding depends on the order: the stated
    # order (rows added as a balanced pairwise tree) must be the one used, not
    # a plain top-to-bottom sum.
    N, K, tn, tk = 4, 32, 4, 32
    sc = np.zeros((N, K))
    sc[:, 0::4] = 1e30        # positions 0 and 1 of every group are kept
    sc[:, 1::4] = 1e30
    r = [1.0, 2.0 ** 53, 1.0, 1.0]
    sc[:, 2] = r              # the only nonzero pruned score of each row
    meta = oracle_mod.select_2of4(sc)
    loss = oracle_mod.tile_loss(sc, meta, tn, tk)[0]
    tree = (r[0] + r[1]) + (r[2] + r[3])
    top_to_bottom = ((r[0] + r[1]) + r[2]) + r[3]
    assert tree != top_to_bottom  # 2**53 + 2 vs 2**53
    assert loss == tree


def test_tile_loss_plus_kept_is_total(oracle_mod):
    rng = np.random.default_rng(9)
    N, K, tn, tk = 256, 256, 128, 128
    sc = np.abs(rng.standard_normal((N, K)))
    meta = oracle_mod.select_2of4(sc)
    loss = oracle_mod.tile_loss(sc, meta, tn, tk)
    pm = pruned_mask(codes_of(meta), K)
    for t in range(4):
        i0, j0 = (t // 2) * tn, (t % 2) * tk
        blk = sc[i0:i0 + tn, j0:j0 + tk]
        kept_sum = blk[~pm[i0:i0 + tn, j0:j0 + tk]].sum()
        np.testing.assert_allclose(loss[t] + kept_sum, blk.sum(), rtol=1e-12)
        assert loss[t] <= kept_sum  # the kept half is the larger half


# ----------------------------------------------------------------------------
# map selection
# ----------------------------------------------------------------------------

def test_n_sparse_floor(oracle_mod):
    assert oracle_mod.n_sparse(0.6, 1024) == 614
    assert oracle_mod.n_sparse(0.6, 2752) == 1651
    assert oracle_mod.n_sparse(0.5, 16) == 8
    assert oracle_mod.n_sparse(1.0, 4320) == 4320
    assert oracle_mod.n_sparse(0.0, 4320) == 0
    assert oracle_mod.n_sparse(0.999, 10) == 9


def popcount(words):
    return int(sum(bin(int(w)).count("1") for w in np.asarray(words, dtype=np.uint32)))


def bits_of(words, n):
    words = np.asarray(words, dtype=np.uint32)
    return np.array([(int(words[t // 32]) >> (t % 32)) & 1 for t in range(n)], dtype=bool)


def test_map_invariants(oracle_mod):
    rng = np.random.default_rng(1)
    loss = rng.standard_normal(1000).round(2)  # with ties
    for ns in [0, 1, 313, 999, 1000]:
        m = oracle_mod.select_map(loss, ns)
        b = bits_of(m, 1000)
        assert b.sum() == ns == popcount(m)
        if 0 < ns < 1000:
            assert loss[b].max() <= loss[~b].min()
            # on the boundary value, lower indices were taken first
            v = loss[b].max()
            chosen = np.where(b & (loss == v))[0]
            left = np.where(~b & (loss == v))[0]
            if len(left):
                assert chosen.max() < left.min()


def test_map_all_ties_take_lowest_indices(oracle_mod):
    m = oracle_mod.select_map(np.full(70, 3.0), 33)
    b = bits_of(m, 70)
    assert b[:33].all() and not b[33:].any()


# ----------------------------------------------------------------------------
# global tile allocation over the matrices of a block (PATCH, section 4,
# ablation on a block-wide target against a per-layer one)


def test_global_maps_hand_example(oracle_mod):
    # two matrices, 3 + 2 tiles; 40 % of 5 tiles = 2 tiles of least loss:
    # 0.1 (matrix 1, tile 0) and 0.2 (matrix 0, tile 1)
    maps = oracle_mod.select_maps_global([np.array([0.5, 0.2, 0.9]), np.array([0.1, 0.7])], 0.4)
    assert [int(m[0]) for m in maps] == [0b010, 0b01]
    # 60 %: the next is 0.5 (matrix 0, tile 0)
    maps = oracle_mod.select_maps_global([np.array([0.5, 0.2, 0.9]), np.array([0.1, 0.7])], 0.6)
    assert [int(m[0]) for m in maps] == [0b011, 0b01]


def test_global_maps_single_matrix_is_the_per_matrix_map(oracle_mod):
    rng = np.random.default_rng(5)
    loss = rng.standard_normal(777).round(1)
    for f in [0.0, 0.3, 0.6, 1.0]:
        (m,) = oracle_mod.select_maps_global([loss], f)
        ref = oracle_mod.select_map(loss, oracle_mod.n_sparse(f, 777))
        assert np.array_equal(m, ref[:len(m)])


def test_global_maps_invariants(oracle_mod):
    rng = np.random.default_rng(6)
    sizes = [33, 1, 100, 64, 7]
    # different scales per matrix, so the shares differ from the target
    losses = [rng.standard_normal(n).round(1) * (1 + 2 * i) for i, n in enumerate(sizes)]
    total = sum(sizes)
    cat = np.concatenate(losses)
    for f in [0.0, 0.25, 0.5, 0.99, 1.0]:
        maps = oracle_mod.select_maps_global(losses, f)
        bits = np.concatenate([bits_of(m, n) for m, n in zip(maps, sizes)])
        ns = int(np.floor(f * total))
        assert bits.sum() == ns
        for m, n in zip(maps, sizes):
            assert len(m) == (n + 31) // 32
            assert popcount(m) == bits_of(m, n).sum()  # no bits past the last tile
        if 0 < ns < total:
            assert cat[bits].max() <= cat[~bits].min()
            v = cat[bits].max()
            chosen = np.where(bits & (cat == v))[0]
            left = np.where(~bits & (cat == v))[0]
            if len(left):
                assert chosen.max() < left.min()


def test_global_maps_ties_go_to_the_earlier_matrix(oracle_mod):
    maps = oracle_mod.select_maps_global([np.full(40, 1.0), np.full(40, 1.0)], 0.75)
    # 60 of 80 tied tiles: all of matrix 0, then tiles 0..19 of matrix 1
    assert bits_of(maps[0], 40).all()
    b1 = bits_of(maps[1], 40)
    assert b1[:20].all() and not b1[20:].any()


# ----------------------------------------------------------------------------
# effective weight and product
# ----------------------------------------------------------------------------

def rand_problem(seed, N, K, M=8):
    g = torch.Generator().manual_seed(seed)
    w = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    xc = torch.randn(32, K, generator=g).to(torch.bfloat16)
    return bf16_bits(w), bf16_bits(x), bf16_bits(xc)


def full_map(n_tiles, value):
    words = np.zeros((n_tiles + 31) // 32, dtype=np.uint32)
    if value:
        for t in range(n_tiles):
            words[t // 32] |= np.uint32(1 << (t % 32))
    return words


def test_all_dense_is_plain_gemm(oracle_mod):
    w, x, xc = rand_problem(0, 128, 256)
    r = oracle_mod.score_mask(w, xc, 64, 64, tile_map=full_map(8, False))
    weff = oracle_mod.weff(w, r["meta"], r["map"], 64, 64)
    assert np.array_equal(weff, w)
    y = oracle_mod.gemm(x, weff)
    xf, wf = oracle_mod.bf16_bits_to_f64(x), oracle_mod.bf16_bits_to_f64(w)
    bound = 1e-12 * (np.abs(xf) @ np.abs(wf).T)
    assert np.all(np.abs(y - xf @ wf.T) <= bound)
    # a transposed operand would not match
    assert not np.allclose(y, xf @ wf[:, ::-1].T)


def test_all_sparse_is_masked_gemm(oracle_mod):
    w, x, xc = rand_problem(1, 128, 256)
    r = oracle_mod.score_mask(w, xc, 64, 64, tile_map=full_map(8, True))
    weff = oracle_mod.weff(w, r["meta"], r["map"], 64, 64)
    # mask from brute-force selection on the same scores
    sc = r["score"]
    wf = oracle_mod.bf16_bits_to_f64(w)
    masked = wf.copy()
    for i in range(128):
        for g in range(64):
            c = brute_force_code(sc[i, 4 * g:4 * g + 4])
            for pos in range(4):
                if pos not in (c & 3, c >> 2):
                    masked[i, 4 * g + pos] = 0.0
    assert np.array_equal(oracle_mod.bf16_bits_to_f64(weff), masked)
    y = oracle_mod.gemm(x, weff)
    xf = oracle_mod.bf16_bits_to_f64(x)
    bound = 1e-12 * (np.abs(xf) @ np.abs(masked).T)
    assert np.all(np.abs(y - xf @ masked.T) <= bound)


def test_gemm_integer_exact_and_sampled(oracle_mod):
    rng = np.random.default_rng(4)
    xi = rng.integers(-4, 5, size=(5, 96))
    wi = rng.integers(-4, 5, size=(7, 96))
    y = oracle_mod.gemm(to_bits(xi), to_bits(wi))
    assert np.array_equal(y, (xi @ wi.T).astype(np.float64))
    ms, ns = np.array([0, 4, 2]), np.array([6, 0, 3])
    assert np.array_equal(oracle_mod.gemm_at(to_bits(xi), to_bits(wi), ms, ns), y[ms, ns])


@pytest.mark.parametrize("f_line", read_golden("tile_sparsity_endpoints.txt"))
def test_golden_achieved_sparsity(oracle_mod, f_line):
    f, s_expect = float(f_line[0]), float(f_line[1])
    N, K, tn, tk = 256, 512, 64, 64
    n_tiles = (N // tn) * (K // tk)
    w = np.full((N, K), 0x3F80, dtype=np.uint16)  # all ones: nothing is zero by chance
    sc = np.abs(np.random.default_rng(2).standard_normal((N, K)))
    meta = oracle_mod.select_2of4(sc)
    loss = oracle_mod.tile_loss(sc, meta, tn, tk)
    m = oracle_mod.select_map(loss, oracle_mod.n_sparse(f, n_tiles))
    weff = oracle_mod.weff(w, meta, m, tn, tk)
    achieved = np.count_nonzero(weff == 0) / weff.size
    assert achieved == s_expect
    # every 4-group of a 2:4 tile has exactly two nonzeros
    b = bits_of(m, n_tiles)
    for t in np.where(b)[0][:4]:
        i0, j0 = (t // (K // tk)) * tn, (t % (K // tk)) * tk
        blk = weff[i0:i0 + tn, j0:j0 + tk].reshape(tn, tk // 4, 4)
        assert np.all(np.count_nonzero(blk, axis=2) == 2)


# ----------------------------------------------------------------------------
# packed layout
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("tn,tk", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.3, 0.5, 1.0])
def test_pack_round_trip(oracle_mod, tn, tk, frac):
    N, K = 256, 384
    w, x, xc = rand_problem(int(frac * 10) + tn, N, K)
    n_tiles = (N // tn) * (K // tk)
    g = np.random.default_rng(tn + tk)
    chosen = g.permutation(n_tiles)[:int(frac * n_tiles)]
    m = np.zeros((n_tiles + 31) // 32, dtype=np.uint32)
    for t in chosen:
        m[t // 32] |= np.uint32(1 << (int(t) % 32))
    r = oracle_mod.score_mask(w, xc, tn, tk, tile_map=m)
    weff = oracle_mod.weff(w, r["meta"], m, tn, tk)
    packed, table = oracle_mod.pack(w, r["meta"], m, tn, tk)
    assert np.array_equal(oracle_mod.unpack(packed, table, N, K), weff)


@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_pack_bytes_closed_form(oracle_mod, frac):
    # 128x128 tiles: dense 32768 B, 2:4 16384 + 2048 B -> ratio 1 - 0.4375 f
    N, K = 512, 1024
    n_tiles = (N // 128) * (K // 128)
    ns = int(frac * n_tiles)
    m = np.zeros((n_tiles + 31) // 32, dtype=np.uint32)
    for t in range(ns):
        m[t // 32] |= np.uint32(1 << (t % 32))
    nbytes = oracle_mod.pack_bytes(m, N, K, 128, 128)
    assert nbytes == int(2 * N * K * (1 - 0.4375 * frac))
    w = np.zeros((N, K), dtype=np.uint16)
    meta = np.full((N, K // 32), 0x44444444, dtype=np.uint32)
    packed, table = oracle_mod.pack(w, meta, m, 128, 128)
    assert packed.size == nbytes
    sparse_steps = int(((table >> np.uint64(62)) & np.uint64(1)).sum())
    e_blocks = int((table >> np.uint64(63)).sum())
    assert sparse_steps == 2 * ns and e_blocks == ns


# ----------------------------------------------------------------------------
# 4:8 groups ("PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 5:
# the tile scheme extends to other N:M patterns such as 4:8)
# ----------------------------------------------------------------------------

def masks_of(meta):
    """Unpack uint32 meta words into per-group 8-bit keep masks [N, K/8]."""
    meta = np.asarray(meta, dtype=np.uint32)
    shifts = (np.arange(4, dtype=np.uint32) * 8)
    m = (meta[..., None] >> shifts) & 0xFF
    return m.reshape(meta.shape[0], -1)


def brute_4of8(group):
    """Among the 70 keep sets of size 4, the largest exact (rational) score sum;
    ties between sets go to the lexicographically smallest sorted index tuple.
    Returns the 8-bit mask."""
    best, best_key = None, None
    for subset in combinations(range(8), 4):
        s = sum(Fraction(float(group[q])) for q in subset)
        key = (-s, subset)
        if best_key is None or key < best_key:
            best_key, best = key, subset
    return sum(1 << q for q in best)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_4of8_equals_bruteforce_with_ties(oracle_mod, seed):
    g = np.random.default_rng(seed)
    # few distinct values: ties inside most groups
    score = g.choice(np.array([0.0, 0.25, 0.5, 1.0, 3.0]), size=(16, 64))
    masks = masks_of(oracle_mod.select_4of8(score))
    for i in range(score.shape[0]):
        for gi in range(score.shape[1] // 8):
            assert masks[i, gi] == brute_4of8(score[i, 8 * gi:8 * gi + 8]), (i, gi)


def test_select_4of8_equals_bruteforce_random(oracle_mod):
    g = np.random.default_rng(5)
    score = np.abs(g.standard_normal((8, 128))) * np.exp(g.standard_normal((1, 128)))
    masks = masks_of(oracle_mod.select_4of8(score))
    for i in range(score.shape[0]):
        for gi in range(score.shape[1] // 8):
            assert masks[i, gi] == brute_4of8(score[i, 8 * gi:8 * gi + 8])


@pytest.mark.parametrize("group,mask", [
    ([1.0] * 8, 0x0F),                                    # all equal: the four lowest indices
    ([8, 7, 6, 5, 4, 3, 2, 1], 0x0F),
    ([1, 2, 3, 4, 5, 6, 7, 8], 0xF0),
    ([0, 5, 0, 5, 0, 5, 0, 5], 0xAA),
    ([2, 2, 9, 2, 2, 2, 9, 2], 0x47),                      # 9s, then the two lowest 2s
])
def test_select_4of8_special_cases(oracle_mod, group, mask):
    score = np.zeros((1, 32))
    score[0, :8] = group
    assert masks_of(oracle_mod.select_4of8(score))[0, 0] == mask


def test_select_4of8_dominance_and_count(oracle_mod):
    g = np.random.default_rng(9)
    score = np.round(np.abs(g.standard_normal((32, 256))) * 4) / 4
    masks = masks_of(oracle_mod.select_4of8(score))
    for i in range(32):
        for gi in range(32):
            m = int(masks[i, gi])
            assert bin(m).count("1") == 4
            grp = score[i, 8 * gi:8 * gi + 8]
            kept = [q for q in range(8) if m >> q & 1]
            drop = [q for q in range(8) if not m >> q & 1]
            for a in kept:
                for b in drop:
                    assert grp[a] > grp[b] or (grp[a] == grp[b] and a < b)


def test_tile_loss_4of8_plus_kept_is_total(oracle_mod):
    # dyadic scores: every sum is exact, so pruned + kept = all, tile by tile
    g = np.random.default_rng(4)
    N, K, tn, tk = 128, 256, 64, 128
    score = g.integers(0, 64, size=(N, K)).astype(np.float64) / 8
    meta = oracle_mod.select_4of8(score)
    loss = oracle_mod.tile_loss_4of8(score, meta, tn, tk)
    bits = np.unpackbits(masks_of(meta).astype(np.uint8)[..., None], axis=-1, bitorder="little")
    keep = bits.reshape(N, K).astype(bool)
    for t in range(loss.shape[0]):
        i0, j0 = (t // (K // tk)) * tn, (t % (K // tk)) * tk
        sub, kp = score[i0:i0 + tn, j0:j0 + tk], keep[i0:i0 + tn, j0:j0 + tk]
        assert loss[t] == sub[~kp].sum()
        assert loss[t] + sub[kp].sum() == sub.sum()


def test_weff_4of8_all_sparse_is_masked_gemm(oracle_mod):
    g = torch.Generator().manual_seed(11)
    N, K, M = 256, 128, 5
    w = (torch.randn(N, K, generator=g) * 0.1).to(torch.bfloat16)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    wb, xb = bf16_bits(w), bf16_bits(x)
    score = np.abs(oracle_mod.bf16_bits_to_f64(wb)) * np.exp(np.linspace(0, 1, K))
    meta = oracle_mod.select_4of8(score)
    nt = (N // 64) * (K // 64)
    allmap = np.full((nt + 31) // 32, 0xFFFFFFFF, dtype=np.uint32)
    weff = oracle_mod.weff_4of8(wb, meta, allmap, 64, 64)
    wf = oracle_mod.bf16_bits_to_f64(wb)
    # the masks from brute force, not from the oracle's own codes
    keep = np.zeros((N, K), dtype=bool)
    for i in range(N):
        for gi in range(K // 8):
            m = brute_4of8(score[i, 8 * gi:8 * gi + 8])
            for q in range(8):
                keep[i, 8 * gi + q] = bool(m >> q & 1)
    assert np.array_equal(oracle_mod.bf16_bits_to_f64(weff), np.where(keep, wf, 0.0))
    y = oracle_mod.gemm(xb, weff)
    yref = oracle_mod.bf16_bits_to_f64(xb) @ np.where(keep, wf, 0.0).T
    assert np.allclose(y, yref, rtol=1e-12, atol=1e-12)
    # achieved sparsity of an all-4:8 map is exactly half (no zero weights drawn)
    assert np.mean(weff == 0) == 0.5


@pytest.mark.parametrize("tn,tk", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.4, 1.0])
def test_pack_4of8_round_trip_and_bytes(oracle_mod, tn, tk, frac):
    from sparse_gemm_wanda_b200 import inputs
    N, K = 256, 384
    w = inputs.weight(N, K, 3)
    wb = bf16_bits(w)
    score = np.abs(oracle_mod.bf16_bits_to_f64(wb))
    meta = oracle_mod.select_4of8(score)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), 5).numpy().view(np.uint32)
    packed, table = oracle_mod.pack_4of8(wb, meta, tmap, tn, tk)
    assert np.array_equal(oracle_mod.unpack_4of8(packed, table, N, K),
                          oracle_mod.weff_4of8(wb, meta, tmap, tn, tk))
    # closed form: a k-step is 4:8 iff every tile it overlaps is; 16384 or 9216 bytes
    sparse_steps = 0
    for b in range(N // 128):
        for c in range(K // 64):
            rows = range((128 * b) // tn, (128 * b + 127) // tn + 1)
            cols = range((64 * c) // tk, (64 * c + 63) // tk + 1)
            if all((tmap[(r * (K // tk) + q) // 32] >> ((r * (K // tk) + q) % 32)) & 1
                   for r in rows for q in cols):
                sparse_steps += 1
    total = (N // 128) * (K // 64)
    assert packed.size == 9216 * sparse_steps + 16384 * (total - sparse_steps)
    assert int(((table >> np.uint64(60)) & np.uint64(1)).sum()) == sparse_steps


# ----------------------------------------------------------------------------
# FP8 (e4m3) values ("SparseGPT vs Wanda", FAQ: prune first, then quantise)
# ----------------------------------------------------------------------------

def torch_e4m3(v):
    """PyTorch's float8_e4m3fn cast (nearest, ties to even), clamped to +-448
    first so that the library's overflow-to-NaN becomes the saturation the
    oracle defines."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_every_bf16_value(oracle_mod):
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[~np.isnan(v)]
    got = oracle_mod.e4m3_encode(v)
    ref = torch_e4m3(v)
    # +-0 and values rounding to zero: the library keeps the sign of zero too
    assert np.array_equal(got, ref)


def test_e4m3_encode_random_quotients(oracle_mod):
    g = np.random.default_rng(8)
    x = np.concatenate([g.uniform(-460, 460, 200000), g.uniform(-0.02, 0.02, 100000),
                        g.standard_normal(100000) * 30]).astype(np.float32)
    assert np.array_equal(oracle_mod.e4m3_encode(x), torch_e4m3(x))


def test_e4m3_decode_every_code(oracle_mod):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(oracle_mod.e4m3_decode(codes), ref)
    assert oracle_mod.e4m3_decode(np.array([0x7E], dtype=np.uint8))[0] == 448.0
    assert oracle_mod.e4m3_decode(np.array([0x01], dtype=np.uint8))[0] == 2.0 ** -9


def test_fp8_row_scales_closed_form(oracle_mod):
    x = np.zeros((3, 64), dtype=np.float32)
    x[0, 5] = -7.0
    x[0, 9] = 3.0
    x[2, :] = 448.0
    s = oracle_mod.fp8_row_scales(to_bits(x))
    assert s[0] == np.float32(7.0) / np.float32(448.0)
    assert s[1] == 1.0          # a zero row: scale 1, every code 0
    assert s[2] == 1.0          # amax 448: scale exactly 1
    q = oracle_mod.fp8_quantize(to_bits(x), s)
    assert np.all(q[1] == 0) and np.all(q[2] == 0x7E)
    assert oracle_mod.e4m3_decode(q[0, 5:6])[0] * s[0] == -7.0


def test_fp8_quantize_representable_values_exactly(oracle_mod):
    # rows whose largest magnitude is 448 have scale 1; values that e4m3 holds
    # exactly come back unchanged
    g = np.random.default_rng(2)
    codes = g.integers(0, 0x7F, size=(16, 128)).astype(np.uint8)
    codes[:, 0] = 0x7E  # 448 in every row
    vals = oracle_mod.e4m3_decode(codes) * np.where(g.random((16, 128)) < 0.5, -1, 1)
    q = oracle_mod.fp8_quantize(to_bits(vals), oracle_mod.fp8_row_scales(to_bits(vals)))
    assert np.array_equal(oracle_mod.e4m3_decode(q), vals.astype(np.float32))


def test_fp8_quantize_error_bound(oracle_mod):
    # |dec(q) s - x| <= s * (half the e4m3 spacing at |x/s|) + fp32 rounding
    g = torch.Generator().manual_seed(4)
    x = (torch.randn(64, 256, generator=g) * 0.05).to(torch.bfloat16)
    xb = bf16_bits(x)
    s = oracle_mod.fp8_row_scales(xb)
    q = oracle_mod.fp8_quantize(xb, s)
    xv = oracle_mod.bf16_bits_to_f64(xb)
    a = np.abs(xv / s[:, None])
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    spacing = np.exp2(e - 3)  # normal spacing; the subnormal spacing is 2^-9 = 2^(-6-3)
    err = np.abs(oracle_mod.e4m3_decode(q).astype(np.float64) * s[:, None] - xv)
    assert np.all(err <= s[:, None] * (0.5 * spacing * (1 + 1e-6)) + 1e-12)


def test_gemm_fp8_equals_numpy_on_decoded_codes(oracle_mod):
    g = np.random.default_rng(6)
    qx = g.integers(0, 0x7F, size=(5, 96)).astype(np.uint8) | (g.integers(0, 2, size=(5, 96)) << 7).astype(np.uint8)
    qw = g.integers(0, 0x7F, size=(7, 96)).astype(np.uint8)
    sx = g.uniform(0.01, 2, 5).astype(np.float32)
    sw = g.uniform(0.01, 2, 7).astype(np.float32)
    y = oracle_mod.gemm_fp8(qx, sx, qw, sw)
    ref = (sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)) * (
        oracle_mod.e4m3_decode(qx).astype(np.float64) @ oracle_mod.e4m3_decode(qw).astype(np.float64).T)
    assert np.allclose(y, ref, rtol=1e-12, atol=0)
    ms, ns = np.array([0, 4, 2]), np.array([6, 0, 3])
    assert np.array_equal(oracle_mod.gemm_fp8_at(qx, sx, qw, sw, ms, ns), y[ms, ns])


@pytest.mark.parametrize("tn,tk", [(128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_pack_fp8_round_trip_and_bytes(oracle_mod, tn, tk, frac):
    from sparse_gemm_wanda_b200 import inputs
    N, K = 256, 512
    w = inputs.weight(N, K, 4)
    wb = bf16_bits(w)
    sc = np.abs(oracle_mod.bf16_bits_to_f64(wb))
    meta = oracle_mod.select_2of4(sc)
    nt = (N // tn) * (K // tk)
    tmap = inputs.random_map(nt, int(frac * nt), 6).numpy().view(np.uint32)
    weff = oracle_mod.weff(wb, meta, tmap, tn, tk)
    qw = oracle_mod.fp8_quantize(weff, oracle_mod.fp8_row_scales(weff))
    packed, table = oracle_mod.pack_fp8(qw, meta, tmap, tn, tk)
    back = oracle_mod.unpack_fp8(packed, table, N, K)
    # pruned entries quantise to code 0 and come back as 0
    assert np.array_equal(back, qw)
    # a 2:4 k-step's metadata block: line m, bit k is bit k%4 of the 4-bit code
    # of row m's group k//4 (so the line's 32-bit words are the row's meta words)
    for b in range(N // 128):
        for c in range(K // 128):
            e = int(table[b * (K // 128) + c])
            if not (e >> 62) & 1:
                continue
            off = e & ((1 << 48) - 1)
            block = packed[off - 2048:off].view(np.uint32).reshape(128, 4)
            assert np.array_equal(block, meta[128 * b:128 * b + 128, 4 * c:4 * c + 4])
    sparse = 0
    for b in range(N // 128):
        for c in range(K // 128):
            rows = range((128 * b) // tn, (128 * b + 127) // tn + 1)
            cols = range((128 * c) // tk, (128 * c + 127) // tk + 1)
            if all((tmap[(r * (K // tk) + q) // 32] >> ((r * (K // tk) + q) % 32)) & 1
                   for r in rows for q in cols):
                sparse += 1
    total = (N // 128) * (K // 128)
    assert packed.size == 10240 * sparse + 16384 * (total - sparse)
