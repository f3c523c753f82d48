/*
 * patch_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * tile-hybrid (dense / 2:4) Wanda-masked linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or constant generator with the CUDA path.
 *
 * Arithmetic is IEEE fp64 throughout.  Build with -ffp-contract=off so that
 * no multiply-add is fused: every sum below is a chain of separately rounded
 * additions in the order written.  OpenMP splits work only across
 * independent output rows / columns, so the per-element order, and therefore
 * every bit of every result, is independent of the thread count.
 *
 * What is computed, and where it comes from:
 *   - Wanda importance |W_ij| * ||X_:,j||_2 over calibration tokens:
 *     "SparseGPT vs Wanda: one-shot LLM pruning without retraining",
 *     section "Wanda: simplicity of activation-aware pruning" (the page says
 *     the weight magnitude times the input activation of that channel; the
 *     activation term is read as the l2 norm over calibration tokens).
 *   - 2:4 groups (keep 2 of every 4 consecutive input channels) and the six
 *     possible keep patterns: "PATCH: Learnable Tile-level Hybrid Sparsity
 *     for LLMs", section 1 (problem statement, semi-structured 2:4) and
 *     section 2 (methodology, pattern choice among 6 permutations).
 *   - tiles of b1 x b2, each either dense (0% sparse) or 2:4 (50% sparse):
 *     same PATCH page, section 2, core mechanism.
 *   - the per-tile choice is learned in PATCH; here it is either given by the
 *     caller or taken as the tiles whose 2:4 pruning loses the least Wanda
 *     score (a data-free stand-in for the learned map; PATCH-Tile, section 2
 *     variants, freezes 2:4 patterns from a one-shot method).
 *   - a block-wide tile budget (one target over several matrices, left free
 *     to land unevenly): PATCH page, section 4, ablation on a global target
 *     against a per-layer one; here the least-loss tiles over all matrices.
 *   - compressed storage is required for any speedup: SparseGPT-vs-Wanda
 *     page, section on structured vs unstructured sparsity.  The packed
 *     layout itself is this library's own format (documented in
 *     include/patch.h); pack/unpack here are an independent restatement.
 *
 * Parity pins for every function live in tests/test_oracle.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16 helpers                                                        */
/* ------------------------------------------------------------------ */

/* Exact widening of a bf16 bit pattern to double (bf16 is the top half of
 * an IEEE binary32). */
static double bf16_bits_to_f64(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* |w| taken on the bits: clear the sign, so -0 becomes +0. */
static double bf16_abs_to_f64(uint16_t b) {
    return bf16_bits_to_f64((uint16_t)(b & 0x7FFFu));
}

/* ------------------------------------------------------------------ */
/* Step 1: column sum of squares of the calibration activations         */
/* ------------------------------------------------------------------ */

/*
 * s[j] = sum over calibration tokens t of x[t,j]^2, in this fixed order:
 *   tokens are cut into consecutive chunks of `chunk` tokens (the last
 *   chunk may be short); inside a chunk the squares are added one token
 *   after another, starting from 0.0; the chunk partials are then added one
 *   chunk after another, starting from 0.0.
 * A bf16 value squared is exact in fp64, so only the additions round.
 * Xcal is [T, K] row-major bf16 bits.
 */
void oracle_colsq(const uint16_t *Xcal, int64_t T, int64_t K, int64_t chunk,
                  double *s) {
    double *part = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t j = 0; j < K; ++j) s[j] = 0.0;
    for (int64_t c0 = 0; c0 < T; c0 += chunk) {
        int64_t c1 = c0 + chunk < T ? c0 + chunk : T;
        for (int64_t j = 0; j < K; ++j) part[j] = 0.0;
        for (int64_t t = c0; t < c1; ++t) {
            const uint16_t *row = Xcal + t * K;
#pragma omp parallel for schedule(static)
            for (int64_t j = 0; j < K; ++j) {
                double x = bf16_bits_to_f64(row[j]);
                part[j] = part[j] + x * x;
            }
        }
        for (int64_t j = 0; j < K; ++j) s[j] = s[j] + part[j];
    }
    free(part);
}

/* ------------------------------------------------------------------ */
/* Step 2: Wanda scores                                                 */
/* ------------------------------------------------------------------ */

/*
 * score[i,j] = |W[i,j]| * sqrt(s[j]).  sqrt is the correctly rounded IEEE
 * square root; the product is one rounded fp64 multiply.
 */
void oracle_wanda_scores(const uint16_t *W, const double *s, int64_t N,
                         int64_t K, double *score) {
    double *norm = (double *)malloc(sizeof(double) * (size_t)K);
    for (int64_t j = 0; j < K; ++j) norm[j] = sqrt(s[j]);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < K; ++j)
            score[i * K + j] = bf16_abs_to_f64(W[i * K + j]) * norm[j];
    free(norm);
}

/* ------------------------------------------------------------------ */
/* Step 3: top-2-of-4 selection and its 4-bit code                      */
/* ------------------------------------------------------------------ */

/*
 * For row i and group g (columns 4g..4g+3) keep the two candidates that come
 * first when ordered by (score descending, column index ascending): the
 * highest scores win and a tie goes to the lower index.  With idx0 < idx1 the
 * kept positions inside the group, the code is idx0 | (idx1 << 2).  Group g
 * of row i is stored in bits 4*(g%8) .. 4*(g%8)+3 of meta[i, g/8] (K/32 words
 * per row).
 */
static unsigned select_group(const double *sc) {
    /* first pick: the largest score, lowest index on ties (strict >) */
    int a = 0;
    for (int q = 1; q < 4; ++q)
        if (sc[q] > sc[a]) a = q;
    /* second pick: the largest among the other three, lowest index on ties */
    int b = -1;
    for (int q = 0; q < 4; ++q) {
        if (q == a) continue;
        if (b < 0 || sc[q] > sc[b]) b = q;
    }
    int lo = a < b ? a : b, hi = a < b ? b : a;
    return (unsigned)(lo | (hi << 2));
}

void oracle_select_2of4(const double *score, int64_t N, int64_t K,
                        uint32_t *meta) {
    int64_t words = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
        for (int64_t w = 0; w < words; ++w) {
            uint32_t word = 0;
            for (int g8 = 0; g8 < 8; ++g8) {
                int64_t col = w * 32 + g8 * 4;
                unsigned code = select_group(score + i * K + col);
                word |= (uint32_t)code << (4 * g8);
            }
            meta[i * words + w] = word;
        }
    }
}

/* Is column j of row i kept by the 2:4 code in meta? */
static int kept(const uint32_t *meta, int64_t K, int64_t i, int64_t j) {
    uint32_t word = meta[i * (K / 32) + j / 32];
    unsigned code = (word >> (4 * ((j % 32) / 4))) & 0xFu;
    unsigned pos = (unsigned)(j % 4);
    return pos == (code & 3u) || pos == (code >> 2);
}

/* ------------------------------------------------------------------ */
/* Step 4: per-tile loss of 2:4 pruning                                  */
/* ------------------------------------------------------------------ */

/*
 * Tiles are tn x tk, numbered row-major: t = (i/tn)*(K/tk) + (j/tk).
 * loss[t] = the Wanda score that 2:4 pruning would remove from tile t, added
 * in this fixed order (the pages fix none):
 *   - word sum: inside each 32-column word of a row, the pruned scores are
 *     added left to right, starting from 0.0;
 *   - row sum: the word sums of the row's tk/32 words inside the tile are
 *     added left to right, starting from 0.0;
 *   - tile sum: the tn row sums are added as a balanced binary tree: row
 *     sums (0,1), (2,3), ... are added pairwise, then those results
 *     pairwise, and so on until one value is left (tn is a power of two).
 */
static double word_pruned_sum(const double *score, const uint32_t *meta, int64_t K,
                              int64_t i, int64_t j0) {
    double w = 0.0;
    for (int64_t j = j0; j < j0 + 32; ++j)
        if (!kept(meta, K, i, j)) w = w + score[i * K + j];
    return w;
}

void oracle_tile_loss(const double *score, const uint32_t *meta, int64_t N,
                      int64_t K, int64_t tn, int64_t tk, double *loss) {
    int64_t tiles_k = K / tk, tiles_n = N / tn;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < tiles_n * tiles_k; ++t) {
        int64_t i0 = (t / tiles_k) * tn, j0 = (t % tiles_k) * tk;
        double *rows = (double *)malloc(sizeof(double) * (size_t)tn);
        for (int64_t r = 0; r < tn; ++r) {
            double row = 0.0;
            for (int64_t w = j0; w < j0 + tk; w += 32)
                row = row + word_pruned_sum(score, meta, K, i0 + r, w);
            rows[r] = row;
        }
        for (int64_t n = tn; n > 1; n /= 2)
            for (int64_t q = 0; q < n / 2; ++q) rows[q] = rows[2 * q] + rows[2 * q + 1];
        loss[t] = rows[0];
        free(rows);
    }
}

/* ------------------------------------------------------------------ */
/* Step 5: tile map                                                      */
/* ------------------------------------------------------------------ */

/* Number of 2:4 tiles for a target fraction f: floor(f * n_tiles). */
int64_t oracle_n_sparse(double f, int64_t n_tiles) {
    return (int64_t)floor(f * (double)n_tiles);
}

typedef struct { double loss; int64_t t; } keyed_tile;

static int cmp_keyed(const void *pa, const void *pb) {
    const keyed_tile *a = (const keyed_tile *)pa, *b = (const keyed_tile *)pb;
    if (a->loss < b->loss) return -1;
    if (a->loss > b->loss) return 1;
    return a->t < b->t ? -1 : (a->t > b->t ? 1 : 0);
}

/*
 * Order the tiles by (loss ascending, tile index ascending) and mark the
 * first n_sparse as 2:4.  Bit t%32 of map[t/32] is 1 for a 2:4 tile.
 */
void oracle_select_map(const double *loss, int64_t n_tiles, int64_t n_sparse,
                       uint32_t *map) {
    keyed_tile *kt = (keyed_tile *)malloc(sizeof(keyed_tile) * (size_t)n_tiles);
    for (int64_t t = 0; t < n_tiles; ++t) { kt[t].loss = loss[t]; kt[t].t = t; }
    qsort(kt, (size_t)n_tiles, sizeof(keyed_tile), cmp_keyed);
    for (int64_t w = 0; w < (n_tiles + 31) / 32; ++w) map[w] = 0;
    for (int64_t r = 0; r < n_sparse && r < n_tiles; ++r)
        map[kt[r].t / 32] |= 1u << (kt[r].t % 32);
    free(kt);
}

/*
 * Global tile allocation over several matrices (the ablation in section 4 of
 * "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs": one sparsity target
 * for a whole block, so each layer's share may vary, beats one target per
 * layer).  The pages learn that allocation; without training, the
 * n_sparse tiles of least Wanda tile loss over ALL matrices become 2:4.
 * Matrices are concatenated in the order given: tile t of matrix m has the
 * global index offset[m] + t, and ties in loss go to the lower global index.
 * loss: concatenated losses (total tiles); maps: the per-matrix bitmaps,
 * concatenated, matrix m's words starting at word_offset[m].
 */
void oracle_select_maps_global(const double *loss, const int64_t *n_tiles, int64_t count,
                               int64_t n_sparse, uint32_t *maps, const int64_t *word_offset) {
    int64_t total = 0;
    for (int64_t m = 0; m < count; ++m) total += n_tiles[m];
    uint32_t *global = (uint32_t *)malloc(sizeof(uint32_t) * (size_t)((total + 31) / 32 + 1));
    oracle_select_map(loss, total, n_sparse, global);
    int64_t base = 0;
    for (int64_t m = 0; m < count; ++m) {
        uint32_t *mm = maps + word_offset[m];
        for (int64_t w = 0; w < (n_tiles[m] + 31) / 32; ++w) mm[w] = 0;
        for (int64_t t = 0; t < n_tiles[m]; ++t) {
            const int64_t g = base + t;
            if ((global[g / 32] >> (g % 32)) & 1u) mm[t / 32] |= 1u << (t % 32);
        }
        base += n_tiles[m];
    }
    free(global);
}

static int tile_is_sparse(const uint32_t *map, int64_t t) {
    return (int)((map[t / 32] >> (t % 32)) & 1u);
}

/* ------------------------------------------------------------------ */
/* Step 6: effective weight                                              */
/* ------------------------------------------------------------------ */

/*
 * W_eff = W on dense tiles; on 2:4 tiles the kept entries of W and +0
 * elsewhere.  Output is bf16 bits.
 */
void oracle_weff(const uint16_t *W, const uint32_t *meta, const uint32_t *map,
                 int64_t N, int64_t K, int64_t tn, int64_t tk, uint16_t *weff) {
    int64_t tiles_k = K / tk;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < K; ++j) {
            int64_t t = (i / tn) * tiles_k + j / tk;
            uint16_t w = W[i * K + j];
            if (tile_is_sparse(map, t) && !kept(meta, K, i, j)) w = 0;
            weff[i * K + j] = w;
        }
}

/* ------------------------------------------------------------------ */
/* Step 7: the packed layout, restated independently                    */
/* ------------------------------------------------------------------ */

/*
 * Packed layout (this library's own format; the header include/patch.h is
 * its normative statement).  Geometry: bands of 128 rows, k-steps of 64
 * columns, k-pairs of 128 columns.
 *   - A k-step (band b, step c) is stored 2:4-compressed iff every tile of
 *     the map that overlaps rows [128b, 128b+128) x cols [64c, 64c+64) is a
 *     2:4 tile; otherwise it is stored dense, holding W_eff.
 *   - Bands are stored one after another; inside a band, k-steps in order.
 *   - dense k-step: 16384 bytes, element (r, k), r<128, k<64 at byte
 *       (r/8)*1024 + (r%8)*128 + (((k/8) ^ (r%8)) * 16) + (k%8)*2.
 *   - 2:4 k-step: 8192 bytes of kept values.  Kept value v (v<32, in
 *     increasing column order; two per group of 4) of row r at byte
 *       (r/8)*512 + (r%8)*64 + (((v/8) ^ ((r%8)/2)) * 16) + (v%8)*2.
 *   - metadata block: 2048 bytes per (band, k-pair) that holds at least one
 *     2:4 k-step, stored directly before the values of the first 2:4 k-step
 *     of that pair.  For row m = m0 + 8*m1 + 16*m2 (m0<8, m1<2, m2<8) and
 *     pair column k = k0 + 16*k1 + 32*k2 (k0<16, k1<2, k2<4), the code bit of
 *     logical column k lives in 16-byte line (m0 + 8*k1 + 16*m2) at bit
 *     (32*k2 + 16*m1 + k0); a group's 4-bit code occupies its four columns'
 *     bits, least significant bit first.  Bits of dense k-steps are zero.
 *   - table[b*(K/64) + c] (uint64): bits 0..47 byte offset of the k-step's
 *     data (values for 2:4, the matrix for dense); bit 62 set for 2:4;
 *     bit 63 set when the pair's metadata block sits right before it.
 */
#define BAND 128
#define KSTEP 64

static int kstep_sparse(const uint32_t *map, int64_t K, int64_t tn, int64_t tk,
                        int64_t b, int64_t c) {
    int64_t tiles_k = K / tk;
    for (int64_t ti = (b * BAND) / tn; ti <= (b * BAND + BAND - 1) / tn; ++ti)
        for (int64_t tj = (c * KSTEP) / tk; tj <= (c * KSTEP + KSTEP - 1) / tk;
             ++tj)
            if (!tile_is_sparse(map, ti * tiles_k + tj)) return 0;
    return 1;
}

/* Total packed bytes for this map. */
int64_t oracle_pack_bytes(const uint32_t *map, int64_t N, int64_t K, int64_t tn,
                          int64_t tk) {
    int64_t total = 0, steps = K / KSTEP;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            if (kstep_sparse(map, K, tn, tk, b, c)) {
                int first_in_pair = (c % 2 == 0) ||
                                    !kstep_sparse(map, K, tn, tk, b, c - 1);
                total += 8192 + (first_in_pair ? 2048 : 0);
            } else {
                total += 16384;
            }
        }
    return total;
}

void oracle_pack(const uint16_t *W, const uint32_t *meta, const uint32_t *map,
                 int64_t N, int64_t K, int64_t tn, int64_t tk, uint8_t *out,
                 uint64_t *table) {
    int64_t steps = K / KSTEP, off = 0;
    for (int64_t b = 0; b < N / BAND; ++b) {
        int64_t e_off = -1; /* metadata block of the current pair */
        for (int64_t c = 0; c < steps; ++c) {
            int sp = kstep_sparse(map, K, tn, tk, b, c);
            if (c % 2 == 0) e_off = -1;
            uint64_t entry = 0;
            if (!sp) {
                uint8_t *blk = out + off;
                for (int64_t r = 0; r < BAND; ++r)
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t i = b * BAND + r, j = c * KSTEP + k;
                        int64_t t = (i / tn) * (K / tk) + j / tk;
                        uint16_t w = W[i * K + j];
                        if (tile_is_sparse(map, t) && !kept(meta, K, i, j)) w = 0;
                        int64_t byte = (r / 8) * 1024 + (r % 8) * 128 +
                                       (((k / 8) ^ (r % 8)) * 16) + (k % 8) * 2;
                        memcpy(blk + byte, &w, 2);
                    }
                entry = (uint64_t)off;
                off += 16384;
            } else {
                if (e_off < 0) {
                    e_off = off;
                    memset(out + off, 0, 2048);
                    off += 2048;
                    entry |= 1ull << 63;
                }
                /* metadata bits for this k-step's half of the pair */
                uint8_t *eb = out + e_off;
                for (int64_t m = 0; m < BAND; ++m)
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t kp = (c % 2) * KSTEP + k; /* column in pair */
                        int64_t i = b * BAND + m, j = c * KSTEP + k;
                        uint32_t word = meta[i * (K / 32) + j / 32];
                        unsigned code = (word >> (4 * ((j % 32) / 4))) & 0xFu;
                        unsigned bit = (code >> (j % 4)) & 1u;
                        int64_t m0 = m % 8, m1 = (m / 8) % 2, m2 = m / 16;
                        int64_t k0 = kp % 16, k1 = (kp / 16) % 2, k2 = kp / 32;
                        int64_t line = m0 + 8 * k1 + 16 * m2;
                        int64_t pos = 32 * k2 + 16 * m1 + k0;
                        if (bit) eb[line * 16 + pos / 8] |= (uint8_t)(1u << (pos % 8));
                    }
                /* kept values, two per group, in column order */
                uint8_t *blk = out + off;
                for (int64_t r = 0; r < BAND; ++r) {
                    int64_t i = b * BAND + r;
                    int v = 0;
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t j = c * KSTEP + k;
                        if (!kept(meta, K, i, j)) continue;
                        uint16_t w = W[i * K + j];
                        int64_t byte = (r / 8) * 512 + (r % 8) * 64 +
                                       (((v / 8) ^ ((r % 8) / 2)) * 16) + (v % 8) * 2;
                        memcpy(blk + byte, &w, 2);
                        ++v;
                    }
                }
                entry |= (uint64_t)off | (1ull << 62);
                off += 8192;
            }
            table[b * steps + c] = entry;
        }
    }
}

/*
 * Inverse of oracle_pack: rebuild W_eff (bf16 bits, [N,K]) from the packed
 * bytes and the table alone.
 */
void oracle_unpack(const uint8_t *packed, const uint64_t *table, int64_t N,
                   int64_t K, uint16_t *weff) {
    int64_t steps = K / KSTEP;
    for (int64_t b = 0; b < N / BAND; ++b) {
        int64_t e_off = -1;
        for (int64_t c = 0; c < steps; ++c) {
            uint64_t entry = table[b * steps + c];
            int64_t off = (int64_t)(entry & ((1ull << 48) - 1));
            if (c % 2 == 0) e_off = -1;
            if (!(entry >> 62 & 1)) {
                for (int64_t r = 0; r < BAND; ++r)
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t byte = (r / 8) * 1024 + (r % 8) * 128 +
                                       (((k / 8) ^ (r % 8)) * 16) + (k % 8) * 2;
                        memcpy(&weff[(b * BAND + r) * K + c * KSTEP + k],
                               packed + off + byte, 2);
                    }
                continue;
            }
            if (entry >> 63) e_off = off - 2048;
            for (int64_t r = 0; r < BAND; ++r) {
                int v = 0;
                for (int64_t k = 0; k < KSTEP; ++k) {
                    int64_t kp = (c % 2) * KSTEP + k;
                    int64_t m0 = r % 8, m1 = (r / 8) % 2, m2 = r / 16;
                    int64_t k0 = kp % 16, k1 = (kp / 16) % 2, k2 = kp / 32;
                    int64_t line = m0 + 8 * k1 + 16 * m2;
                    int64_t pos = 32 * k2 + 16 * m1 + k0;
                    /* the group's code: its four bits starting at the group's
                     * first column */
                    int64_t gpos = pos - (k0 % 4);
                    unsigned code = 0;
                    for (int q = 0; q < 4; ++q) {
                        int64_t p = gpos + q;
                        code |= ((packed[e_off + line * 16 + p / 8] >> (p % 8)) & 1u) << q;
                    }
                    unsigned here = (unsigned)(k % 4);
                    uint16_t w = 0;
                    if (here == (code & 3u) || here == (code >> 2)) {
                        int64_t byte = (r / 8) * 512 + (r % 8) * 64 +
                                       (((v / 8) ^ ((r % 8) / 2)) * 16) + (v % 8) * 2;
                        memcpy(&w, packed + off + byte, 2);
                        ++v;
                    }
                    weff[(b * BAND + r) * K + c * KSTEP + k] = w;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Step 8: the product                                                   */
/* ------------------------------------------------------------------ */

/*
 * y[m,n] = sum_k X[m,k] * W_eff[n,k]: a naive triple loop, fp64 products of
 * the exact bf16 values, accumulated from 0.0 in increasing k.  The product
 * of two bf16 values is exact in fp64.
 */
void oracle_gemm(const uint16_t *X, const uint16_t *Weff, int64_t M, int64_t N,
                 int64_t K, double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc = acc + bf16_bits_to_f64(X[m * K + k]) *
                                bf16_bits_to_f64(Weff[n * K + k]);
            y[m * N + n] = acc;
        }
}

/* The same sum for a list of (m, n) output positions only. */
void oracle_gemm_at(const uint16_t *X, const uint16_t *Weff, int64_t K,
                    const int64_t *ms, const int64_t *ns, int64_t count,
                    double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < count; ++q) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc = acc + bf16_bits_to_f64(X[ms[q] * K + k]) *
                            bf16_bits_to_f64(Weff[ns[q] * K + k]);
        y[q] = acc;
    }
}

/* ------------------------------------------------------------------ */
/* Another N:M pattern: 4 of every 8 (4:8)                             */
/* ------------------------------------------------------------------ */

/*
 * PATCH's closing section ("PATCH: Learnable Tile-level Hybrid Sparsity for
 * LLMs", section 5, significance) says the tile-level scheme does not depend
 * on 2:4 and extends to other N:M patterns such as 4:8.  Here: inside a 4:8
 * tile every group of 8 consecutive input channels keeps the 4 weights with
 * the highest Wanda score, ties to the lower index (the same rule as 2:4,
 * with groups of 8).  Everything else (tile loss, map, W_eff) is the 2:4
 * definition with this kept set.
 *
 * Codes: group g of row i (columns 8g..8g+7) is an 8-bit mask with bit q set
 * for a kept position q (exactly four bits), at bits 8*(g%4) of meta[i, g/4]
 * (K/32 words per row, like the 2:4 codes).
 */
static unsigned select_group_4of8(const double *sc) {
    /* four picks, each the largest remaining score, lowest index on ties */
    unsigned mask = 0;
    for (int pick = 0; pick < 4; ++pick) {
        int best = -1;
        for (int q = 0; q < 8; ++q) {
            if ((mask >> q) & 1u) continue;
            if (best < 0 || sc[q] > sc[best]) best = q;
        }
        mask |= 1u << best;
    }
    return mask;
}

void oracle_select_4of8(const double *score, int64_t N, int64_t K, uint32_t *meta) {
    int64_t words = K / 32;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        for (int64_t w = 0; w < words; ++w) {
            uint32_t word = 0;
            for (int g4 = 0; g4 < 4; ++g4)
                word |= (uint32_t)select_group_4of8(score + i * K + w * 32 + g4 * 8) << (8 * g4);
            meta[i * words + w] = word;
        }
}

static int kept_4of8(const uint32_t *meta, int64_t K, int64_t i, int64_t j) {
    uint32_t word = meta[i * (K / 32) + j / 32];
    unsigned mask = (word >> (8 * ((j % 32) / 8))) & 0xFFu;
    return (int)((mask >> (j % 8)) & 1u);
}

/* Tile loss with the 4:8 kept set, in the order of oracle_tile_loss. */
void oracle_tile_loss_4of8(const double *score, const uint32_t *meta, int64_t N,
                           int64_t K, int64_t tn, int64_t tk, double *loss) {
    int64_t tiles_k = K / tk, tiles_n = N / tn;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < tiles_n * tiles_k; ++t) {
        int64_t i0 = (t / tiles_k) * tn, j0 = (t % tiles_k) * tk;
        double *rows = (double *)malloc(sizeof(double) * (size_t)tn);
        for (int64_t r = 0; r < tn; ++r) {
            double row = 0.0;
            for (int64_t w0 = j0; w0 < j0 + tk; w0 += 32) {
                double wsum = 0.0;
                for (int64_t j = w0; j < w0 + 32; ++j)
                    if (!kept_4of8(meta, K, i0 + r, j)) wsum = wsum + score[(i0 + r) * K + j];
                row = row + wsum;
            }
            rows[r] = row;
        }
        for (int64_t n = tn; n > 1; n /= 2)
            for (int64_t q = 0; q < n / 2; ++q) rows[q] = rows[2 * q] + rows[2 * q + 1];
        loss[t] = rows[0];
        free(rows);
    }
}

/* W_eff with 4:8 tiles: kept entries of W there, +0 elsewhere. */
void oracle_weff_4of8(const uint16_t *W, const uint32_t *meta, const uint32_t *map,
                      int64_t N, int64_t K, int64_t tn, int64_t tk, uint16_t *weff) {
    int64_t tiles_k = K / tk;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i)
        for (int64_t j = 0; j < K; ++j) {
            int64_t t = (i / tn) * tiles_k + j / tk;
            uint16_t w = W[i * K + j];
            if (tile_is_sparse(map, t) && !kept_4of8(meta, K, i, j)) w = 0;
            weff[i * K + j] = w;
        }
}

/*
 * Packed layout of a 4:8 handle (this library's own format, stated in
 * include/patch.h).  Bands of 128 rows and k-steps of 64 columns as for 2:4;
 * a k-step is 4:8-compressed iff every map tile overlapping it is a 4:8
 * tile, otherwise dense (the 2:4 handles' dense layout, holding W_eff).
 *   - 4:8 k-step: 9216 bytes.  Kept value v (v < 32, column order, four per
 *     group) of row r at byte r*64 + v*2; the keep mask of group g (g < 8)
 *     of row r at byte 8192 + r*8 + g (bit q: position q kept).
 *   - table[b*(K/64) + c] (uint64): bits 0..47 byte offset; bit 60 set for a
 *     4:8 k-step.
 */
#define STEP48_BYTES 9216

int64_t oracle_pack_bytes_4of8(const uint32_t *map, int64_t N, int64_t K, int64_t tn,
                               int64_t tk) {
    int64_t total = 0;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < K / KSTEP; ++c)
            total += kstep_sparse(map, K, tn, tk, b, c) ? STEP48_BYTES : 16384;
    return total;
}

void oracle_pack_4of8(const uint16_t *W, const uint32_t *meta, const uint32_t *map,
                      int64_t N, int64_t K, int64_t tn, int64_t tk, uint8_t *out,
                      uint64_t *table) {
    int64_t steps = K / KSTEP, off = 0;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            if (!kstep_sparse(map, K, tn, tk, b, c)) {
                for (int64_t r = 0; r < BAND; ++r)
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t i = b * BAND + r, j = c * KSTEP + k;
                        int64_t t = (i / tn) * (K / tk) + j / tk;
                        uint16_t w = W[i * K + j];
                        if (tile_is_sparse(map, t) && !kept_4of8(meta, K, i, j)) w = 0;
                        int64_t byte = (r / 8) * 1024 + (r % 8) * 128 +
                                       (((k / 8) ^ (r % 8)) * 16) + (k % 8) * 2;
                        memcpy(out + off + byte, &w, 2);
                    }
                table[b * steps + c] = (uint64_t)off;
                off += 16384;
            } else {
                for (int64_t r = 0; r < BAND; ++r) {
                    int64_t i = b * BAND + r;
                    int v = 0;
                    for (int64_t g = 0; g < KSTEP / 8; ++g) {
                        unsigned mask = 0;
                        for (int64_t q = 0; q < 8; ++q) {
                            int64_t j = c * KSTEP + g * 8 + q;
                            if (!kept_4of8(meta, K, i, j)) continue;
                            mask |= 1u << q;
                            memcpy(out + off + r * 64 + v * 2, &W[i * K + j], 2);
                            ++v;
                        }
                        out[off + 8192 + r * 8 + g] = (uint8_t)mask;
                    }
                }
                table[b * steps + c] = (uint64_t)off | (1ull << 60);
                off += STEP48_BYTES;
            }
        }
}

/* Inverse of oracle_pack_4of8: W_eff from the packed bytes and table alone. */
void oracle_unpack_4of8(const uint8_t *packed, const uint64_t *table, int64_t N, int64_t K,
                        uint16_t *weff) {
    int64_t steps = K / KSTEP;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            uint64_t e = table[b * steps + c];
            int64_t off = (int64_t)(e & ((1ull << 48) - 1));
            for (int64_t r = 0; r < BAND; ++r) {
                uint16_t *dst = weff + (b * BAND + r) * K + c * KSTEP;
                if (!((e >> 60) & 1u)) {
                    for (int64_t k = 0; k < KSTEP; ++k) {
                        int64_t byte = (r / 8) * 1024 + (r % 8) * 128 +
                                       (((k / 8) ^ (r % 8)) * 16) + (k % 8) * 2;
                        memcpy(&dst[k], packed + off + byte, 2);
                    }
                    continue;
                }
                int v = 0;
                for (int64_t g = 0; g < KSTEP / 8; ++g) {
                    unsigned mask = packed[off + 8192 + r * 8 + g];
                    for (int64_t q = 0; q < 8; ++q) {
                        uint16_t w = 0;
                        if ((mask >> q) & 1u) {
                            memcpy(&w, packed + off + r * 64 + v * 2, 2);
                            ++v;
                        }
                        dst[g * 8 + q] = w;
                    }
                }
            }
        }
}

/* ------------------------------------------------------------------ */
/* FP8 (e4m3) values inside dense and 2:4 tiles                         */
/* ------------------------------------------------------------------ */

/*
 * Prune first, then quantise ("SparseGPT vs Wanda: one-shot LLM pruning
 * without retraining", FAQ on combining pruning with quantisation: prune,
 * then quantise the surviving weights).  Here the Wanda 2:4 codes and the
 * tile map are decided on the bf16 weights exactly as above; W_eff (kept
 * entries, zeros elsewhere) is then quantised to FP8 e4m3 with one fp32
 * scale per output row, and the activations X with one fp32 scale per
 * token.  The product is
 *     y[m,n] = sx[m] * sw[n] * sum_k dec(qx[m,k]) * dec(qw[n,k]).
 *
 * e4m3 (the OCP 8-bit floating-point format, "fn" variant): sign, 4 exponent
 * bits (bias 7), 3 mantissa bits, no infinities; code 0x7F/0xFF is NaN; the
 * largest finite value is 448, the smallest subnormal 2^-9.  Encoding rounds
 * to nearest, ties to the even code, and saturates at +-448.
 *
 * Scales and the quotient x / s are fp32 (IEEE single, round to nearest):
 *     s = amax / 448 (amax = largest |value| of the row; s = 1 when amax = 0)
 *     q = enc(x / s).
 * Where floating point decides an integer code, both this oracle and the GPU
 * take that decision in fp32 with these exact operations.
 */
static float e4m3_decode_value(unsigned c) {
    unsigned e = (c >> 3) & 0xFu, m = c & 7u;
    float v = (e == 0) ? (float)m * 0.001953125f /* 2^-9 */
                       : ldexpf((float)(8u + m), (int)e - 10);
    return (c & 0x80u) ? -v : v;
}

/* The 127 non-negative finite values in increasing order: code i has value
 * table[i] for i = 0 .. 126 (0x7F is NaN). */
static float g_e4m3_table[127];
static int g_e4m3_ready = 0;

static void e4m3_init(void) {
    if (g_e4m3_ready) return;
    for (unsigned c = 0; c < 127; ++c) g_e4m3_table[c] = e4m3_decode_value(c);
    g_e4m3_ready = 1;
}

unsigned char oracle_e4m3_encode(float v) {
    e4m3_init();
    unsigned sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 0x80u : 0u;
    float a = fabsf(v);
    if (!(a == a)) return 0x7F; /* NaN in, NaN out (not used by the path) */
    if (a >= 448.0f) return (unsigned char)(sign | 0x7Eu);
    /* largest code with value <= a (binary search), then the nearer of it and
     * the next one; a tie goes to the even code */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (g_e4m3_table[mid] <= a) lo = mid; else hi = mid - 1;
    }
    unsigned c = (unsigned)lo;
    if (g_e4m3_table[c] != a) {
        double below = (double)a - (double)g_e4m3_table[c];
        double above = (double)g_e4m3_table[c + 1] - (double)a;
        if (above < below || (above == below && ((c + 1) & 1u) == 0)) c = c + 1;
    }
    return (unsigned char)(sign | c);
}

float oracle_e4m3_decode(unsigned char c) { return e4m3_decode_value(c); }

void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out) {
    e4m3_init();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* Row scales of a bf16 matrix [R, C]: s = amax / 448 in fp32 (1 for a zero row). */
void oracle_fp8_row_scales(const uint16_t *x, int64_t R, int64_t C, float *scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t c = 0; c < C; ++c) {
            float a = fabsf((float)bf16_bits_to_f64(x[r * C + c]));
            if (a > amax) amax = a;
        }
        scale[r] = amax > 0.0f ? amax / 448.0f : 1.0f;
    }
}

/* q[r,c] = enc(x[r,c] / scale[r]), the quotient in fp32. */
void oracle_fp8_quantize(const uint16_t *x, const float *scale, int64_t R, int64_t C, uint8_t *q) {
    e4m3_init();
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) {
            float v = (float)bf16_bits_to_f64(x[r * C + c]);
            float quot = v / scale[r];
            q[r * C + c] = oracle_e4m3_encode(quot);
        }
}

/* y[m,n] = sx[m] * sw[n] * sum_k dec(qx[m,k]) * dec(qw[n,k]); fp64, k in order. */
void oracle_gemm_fp8(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw,
                     int64_t M, int64_t N, int64_t K, double *y) {
    e4m3_init();
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc = acc + (double)e4m3_decode_value(qx[m * K + k]) *
                                (double)e4m3_decode_value(qw[n * K + k]);
            y[m * N + n] = (double)sx[m] * (double)sw[n] * acc;
        }
}

/* The same sums at listed (m, n) positions only. */
void oracle_gemm_fp8_at(const uint8_t *qx, const float *sx, const uint8_t *qw, const float *sw,
                        int64_t K, const int64_t *ms, const int64_t *ns, int64_t count, double *y) {
    e4m3_init();
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc = acc + (double)e4m3_decode_value(qx[ms[i] * K + k]) *
                            (double)e4m3_decode_value(qw[ns[i] * K + k]);
        y[i] = (double)sx[ms[i]] * (double)sw[ns[i]] * acc;
    }
}

/*
 * Packed layout of an FP8 handle (this library's own format, stated in
 * include/patch.h).  Bands of 128 rows; k-steps of 128 columns (128 bytes of
 * e4m3 per row).  A k-step is 2:4-compressed iff every map tile overlapping
 * it is a 2:4 tile; otherwise dense (the codes of W_eff).
 *   - dense k-step: 16384 bytes, code (r, k) at
 *       (r/8)*1024 + (r%8)*128 + ((k/16) ^ (r%8))*16 + k%16.
 *   - 2:4 k-step: a 2048-byte metadata block, then 8192 bytes of kept codes:
 *     kept code v (v < 64, column order, two per group) of row r at
 *       (r/8)*512 + (r%8)*64 + ((v/16) ^ ((r%8)/2))*16 + v%16;
 *     metadata: 16-byte line m holds row m; bit k (k < 128, LSB first) is the
 *     code bit of column k of the k-step (a group's 4-bit code over its four
 *     columns, LSB first).  This is the tensor-memory layout the sparse MMA
 *     for 8-bit inputs reads (one lane per row, one bit per K column), not
 *     the interleaved one of the 16-bit handles.
 *   - table[b*(K/128) + c] (uint64): bits 0..47 offset of the k-step's codes
 *     (after its metadata block for 2:4), bit 62 = 2:4.
 */
#define KSTEP8 128

static int kstep8_sparse(const uint32_t *map, int64_t K, int64_t tn, int64_t tk, int64_t b,
                         int64_t c) {
    int64_t tiles_k = K / tk;
    for (int64_t ti = (b * BAND) / tn; ti <= (b * BAND + BAND - 1) / tn; ++ti)
        for (int64_t tj = (c * KSTEP8) / tk; tj <= (c * KSTEP8 + KSTEP8 - 1) / tk; ++tj)
            if (!tile_is_sparse(map, ti * tiles_k + tj)) return 0;
    return 1;
}

int64_t oracle_pack_bytes_fp8(const uint32_t *map, int64_t N, int64_t K, int64_t tn, int64_t tk) {
    int64_t total = 0;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < K / KSTEP8; ++c)
            total += kstep8_sparse(map, K, tn, tk, b, c) ? 2048 + 8192 : 16384;
    return total;
}

/* qw: the e4m3 codes of W_eff [N, K] (pruned entries encode +0 = 0x00). */
void oracle_pack_fp8(const uint8_t *qw, const uint32_t *meta, const uint32_t *map, int64_t N,
                     int64_t K, int64_t tn, int64_t tk, uint8_t *out, uint64_t *table) {
    int64_t steps = K / KSTEP8, off = 0;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            if (!kstep8_sparse(map, K, tn, tk, b, c)) {
                for (int64_t r = 0; r < BAND; ++r)
                    for (int64_t k = 0; k < KSTEP8; ++k)
                        out[off + (r / 8) * 1024 + (r % 8) * 128 + (((k / 16) ^ (r % 8)) * 16) + k % 16] =
                            qw[(b * BAND + r) * K + c * KSTEP8 + k];
                table[b * steps + c] = (uint64_t)off;
                off += 16384;
                continue;
            }
            uint8_t *eb = out + off;
            memset(eb, 0, 2048);
            for (int64_t m = 0; m < BAND; ++m)
                for (int64_t k = 0; k < KSTEP8; ++k) {
                    int64_t i = b * BAND + m, j = c * KSTEP8 + k;
                    uint32_t word = meta[i * (K / 32) + j / 32];
                    unsigned code = (word >> (4 * ((j % 32) / 4))) & 0xFu;
                    unsigned bit = (code >> (j % 4)) & 1u;
                    if (bit) eb[m * 16 + k / 8] |= (uint8_t)(1u << (k % 8));
                }
            off += 2048;
            for (int64_t r = 0; r < BAND; ++r) {
                int64_t i = b * BAND + r;
                int v = 0;
                for (int64_t k = 0; k < KSTEP8; ++k) {
                    int64_t j = c * KSTEP8 + k;
                    if (!kept(meta, K, i, j)) continue;
                    out[off + (r / 8) * 512 + (r % 8) * 64 + (((v / 16) ^ ((r % 8) / 2)) * 16) + v % 16] =
                        qw[i * K + j];
                    ++v;
                }
            }
            table[b * steps + c] = (uint64_t)off | (1ull << 62);
            off += 8192;
        }
}

/* Inverse of oracle_pack_fp8: the codes of W_eff from the packed bytes and table. */
void oracle_unpack_fp8(const uint8_t *packed, const uint64_t *table, int64_t N, int64_t K,
                       uint8_t *qw) {
    int64_t steps = K / KSTEP8;
    for (int64_t b = 0; b < N / BAND; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            uint64_t e = table[b * steps + c];
            int64_t off = (int64_t)(e & ((1ull << 48) - 1));
            for (int64_t r = 0; r < BAND; ++r) {
                uint8_t *dst = qw + (b * BAND + r) * K + c * KSTEP8;
                if (!((e >> 62) & 1u)) {
                    for (int64_t k = 0; k < KSTEP8; ++k)
                        dst[k] = packed[off + (r / 8) * 1024 + (r % 8) * 128 + (((k / 16) ^ (r % 8)) * 16) + k % 16];
                    continue;
                }
                const uint8_t *eb = packed + off - 2048;
                int v = 0;
                for (int64_t k = 0; k < KSTEP8; ++k) {
                    int64_t gpos = k - (k % 4);
                    unsigned code = 0;
                    for (int q = 0; q < 4; ++q) {
                        int64_t p = gpos + q;
                        code |= ((eb[r * 16 + p / 8] >> (p % 8)) & 1u) << q;
                    }
                    unsigned here = (unsigned)(k % 4);
                    uint8_t w = 0;
                    if (here == (code & 3u) || here == (code >> 2)) {
                        w = packed[off + (r / 8) * 512 + (r % 8) * 64 + (((v / 16) ^ ((r % 8) / 2)) * 16) + v % 16];
                        ++v;
                    }
                    dst[k] = w;
                }
            }
        }
}
