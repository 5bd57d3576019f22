/*
 * dgen probes -- measurement entry points of the tcgen05 GEMM core, built into
 * a separate library (block_denoising_step_b200/lib/libdgen_probe.so) so that
 * the shipping library carries only the denoising path.  C ABI; conventions as
 * in dgen.h.  (The pages have no counterpart: these measure this library's own
 * kernels.)
 */
#ifndef DGEN_PROBE_H
#define DGEN_PROBE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The product of dgen_gemm_bf16 (A[M][K] * B[N][K]^T, bf16 row-major device
 * arrays, K a multiple of 8) through the same GEMM core, but each thread writes
 * only the sum of its row of each BN-wide output tile, out_dev[M][ceil(N / BN)]
 * fp32, so the launch time is that of streaming the operands.  variant selects
 * the tile width BN, the shared-memory ring depth and how many TMA boxes make up
 * an A tile: 0 = (64, 8, 1), 1 = (64, 8, 8), 2 = (64, 4, 1), 3 = (32, 8, 1),
 * 4 = (128, 6, 1), 5 = (256, 4, 1).  stream: a cudaStream_t.  Asynchronous.
 * Errors: DGEN_EINVAL (-1) for bad sizes, pointers or variant, DGEN_ECUDA (-4). */
int dgen_gemm_rowsum_variant(const void* a_dev, const void* b_dev, float* out_dev, int32_t M, int32_t N, int32_t K,
                             int32_t variant, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DGEN_PROBE_H */
