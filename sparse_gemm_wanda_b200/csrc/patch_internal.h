// Launchers shared between the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace patchk {

cudaError_t launch_colsq(const void *Xcal, int64_t T, int64_t K, double *partial,
                         double *colsq_out, double *norm_out, cudaStream_t stream);
cudaError_t launch_norms_from_colsq(const double *colsq_in, int64_t K, double *colsq_out,
                                    double *norm_out, cudaStream_t stream);
cudaError_t launch_score_mask(const void *W, const double *norm, int64_t N, int64_t K, int tn,
                              int tk, uint32_t *meta, double *loss, cudaStream_t stream);
cudaError_t launch_select_map(const double *loss, int64_t n_tiles, int64_t n_sparse, int32_t *rank,
                              uint32_t *map, cudaStream_t stream);

cudaError_t launch_pack(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                        int64_t K, int tn, int tk, const uint64_t *table, uint8_t *out,
                        cudaStream_t stream);

struct GemmLaunch {
    const uint8_t *packed;
    const uint64_t *table;
    int64_t N, K;
    const void *X;
    int64_t M;
    void *Y;
    int y_fp32;
    float *workspace;         // split-K partials [splits][M][N] (fp32)
    int64_t workspace_floats; // capacity of `workspace`
    uint32_t *status;
    int num_sms;
};

// Picks the configuration (token tile, split-K) for M and launches.
cudaError_t launch_hybrid_gemm(const GemmLaunch &g, cudaStream_t stream);

// Number of split-K slices the decode configuration uses for N rows and K
// columns (k-pairs per slice are balanced; always >= 1).
int decode_splits(int64_t N, int64_t K, int num_sms);

}  // namespace patchk
