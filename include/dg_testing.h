/*
 * dg_testing.h - test hooks of the DiffusionGemma denoising-step library.
 *
 * These entry points expose the tensor-core GEMM core of the library on its
 * own so that it can be checked element by element against a CPU product.
 * They are not part of the method; the pages have no counterpart.  Same
 * conventions as dg.h (device pointers, stream as void*, dg_status codes).
 */
#ifndef DG_TESTING_H
#define DG_TESTING_H

#include <stdint.h>
#include "dg.h"

#ifdef __cplusplus
extern "C" {
#endif

/* D[m, n] = sum_k A[m, k] B[n, k]: A bf16 [M, K], B bf16 [N, K] (both
   row-major, K contiguous), D fp32 [M, N] row-major.  Requirements:
   K % 64 == 0, M >= 128, N >= 16, 16-byte aligned pointers.  k_splits > 1
   splits the K loop into that many partial products written to
   D + s * M * N (D then holds k_splits matrices).  Synchronous. */
dg_status dg_test_gemm(const uint16_t* d_a, int32_t M, const uint16_t* d_b, int32_t N, int32_t K,
                       float* d_d, int32_t k_splits, void* stream);

/* Grouped product as used by the expert layers: group g multiplies A rows
   [g * rows_per_group, (g + 1) * rows_per_group) with B rows
   [off[g], off[g+1]) and writes D[r, f] (fp32, [n_rows, rows_per_group]) for
   each B row r of the group and each A row f of the group.  d_off is a
   device int32 array of n_groups + 1 non-decreasing offsets ending at n_rows.
   bn (16..256, power of two) is the number of B rows per pass.  Synchronous. */
dg_status dg_test_grouped_gemm(const uint16_t* d_a, int32_t rows_per_group, int32_t n_groups,
                               const uint16_t* d_b, int32_t n_rows, int32_t K, const int32_t* d_off,
                               float* d_d, int32_t bn, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_TESTING_H */
