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

/* dg_test_gemm with the unit shape chosen: mt (1 or 2) 128-row A tiles and
   bn (16..256, power of two) B rows per unit; bn = 0 picks the library's
   choice for N.  Same output layout and split convention.  Synchronous. */
dg_status dg_test_gemm_tiles(const uint16_t* d_a, int32_t M, const uint16_t* d_b, int32_t N, int32_t K,
                             float* d_d, int32_t k_splits, int32_t mt, int32_t bn, void* stream);

/* Grouped product as used by the expert layers: group g multiplies A rows
   [g * rows_per_group, (g + 1) * rows_per_group) with B rows
   [off[g], off[g+1]) and writes D[r, f] (fp32, [n_rows, rows_per_group]) for
   each B row r of the group and each A row f of the group.  d_off is a
   device int32 array of n_groups + 1 non-decreasing offsets ending at n_rows.
   bn (16..256, power of two) is the number of B rows per unit; d_chunk_off
   is caller-provided device scratch of n_groups + 1 int32.  As in the expert
   layers, bn <= 128 runs on CTA pairs (one 256-row tcgen05.mma.cta_group::2
   per pair of A tiles) and bn = 256 on single CTAs.  Synchronous. */
dg_status dg_test_grouped_gemm(const uint16_t* d_a, int32_t rows_per_group, int32_t n_groups,
                               const uint16_t* d_b, int32_t n_rows, int32_t K, const int32_t* d_off,
                               float* d_d, int32_t bn, int32_t* d_chunk_off, void* stream);

/* The work schedule of a grouped product, enumerated on the host (no GPU
   call): pair = 1 is the CTA-pair schedule (bn <= 128), pair = 0 the
   single-CTA one.  off is a HOST int32 array of n_groups + 1 non-decreasing B
   row offsets; chunk offsets are ceil(rows / bn) prefix sums as on the
   device.  For every unit u and CTA rank r (r = 0 only without pairs) one job
   of 10 int32 goes to jobs[(u * ranks + r) * 10]: u, r, group, A tile index
   within the group, first A row, valid A rows (<= 0 for the missing second
   tile of a pair), first B row, valid B rows, k blocks, B map index (pairs;
   -1 otherwise).  At most max_jobs jobs are written; *n_jobs receives the
   total.  DG_ERR_INVALID_ARG on bad sizes or decreasing offsets. */
dg_status dg_test_grouped_schedule(int32_t pair, int32_t rows_per_group, int32_t n_groups, const int32_t* off,
                                   int32_t K, int32_t bn, int32_t* jobs, int32_t max_jobs, int32_t* n_jobs);

/* The work schedule of a dense product D[M, N] = A[M, K] B[N, K]^T,
   enumerated on the host (no GPU call): bn B rows per unit (16..256, power of
   two), k_splits units along K (1..K/64), mt 128-row A tiles per unit (1 or
   2), n_fast != 0 when consecutive units walk the column tiles of one A tile.
   One job of 8 int32 per unit u goes to jobs[u * 8]: u, first A tile, A tiles
   in the unit, valid rows of its first tile, first B row, valid B rows, first
   and last (exclusive) k block.  At most max_jobs are written; *n_jobs
   receives the total.  DG_ERR_INVALID_ARG on bad sizes. */
dg_status dg_test_dense_schedule(int32_t M, int32_t N, int32_t K, int32_t bn, int32_t k_splits, int32_t mt,
                                 int32_t n_fast, int32_t* jobs, int32_t max_jobs, int32_t* n_jobs);

/* The library's attention kernel on its own (tcgen05 tensor cores):
   q bf16 packed by kv head [B][Hkv][nq][G][hd] (G = Hq / Hkv, query head
   g * G + j is row j of token t's group g), K cache bf16 [B][Hkv][c_max][hd],
   V cache transposed, fp16 [B][Hkv][hd][c_max], both holding keys
   [0, L0 + nq); c_max a multiple of 8; out bf16 [B * nq, Hq * hd]
   (token-major).  causal = 0: every query sees all L0 + nq keys; causal = 1:
   query i sees keys [0, L0 + i]; 1 < causal <= nq: queries i < causal are
   causal and the rest see all keys (a pass that appends a finished block
   ahead of a canvas, causal = 256).  splits (1..8; 0 means 1) key splits.  For
   splits > 1 with part_o and part_ml both NULL, the splits of each tile run
   as one thread-block cluster and merge through distributed shared memory
   (the form the layers use); otherwise the partial buffers come from the
   caller: part_o fp32 [splits * B * Hq * nq * hd] and part_ml fp32
   [splits * B * Hq * nq * 2], rows in packed query order
   [split][b][kv head][token * G + head in group], merged by a second kernel.
   head_dim one of 32, 64, 128, 176.  Synchronous. */
dg_status dg_test_attention(const uint16_t* d_q, const uint16_t* d_k, const uint16_t* d_v, uint16_t* d_out,
                            int32_t B, int32_t nq, int32_t L0, int32_t c_max, int32_t Hq, int32_t Hkv,
                            int32_t hd, int32_t causal, int32_t splits, float* d_part_o,
                            float* d_part_ml, void* stream);

/* Failure-path hook: one thread of a one-CTA kernel waits, with a bounded
   wait of limit_ns (0 < limit_ns <= 5e9), on an mbarrier that nothing arrives
   on.  The wait runs out, the kernel latches DG_ERR_TIMEOUT in the context's
   device error word and returns, so the next dg_check_device_error reports
   (and clears) it and the context stays usable.  Asynchronous on `stream`. */
dg_status dg_test_wait_timeout(dg_ctx* ctx, int64_t limit_ns, void* stream);

/* The top-k form of the expected embedding on its own (dg_sampler_config.
   selfcond_topk): for each of T rows of bf16 logits d_logits [T, V] (V a
   multiple of 256), the K (1 <= K <= min(1024, V)) largest (ties to the lower
   id), p = bf16(softmax over those K), d_out [T, d] bf16 = bf16(sum p_v
   E_emb[v]) with d_emb [V, d] bf16 (d a multiple of 64, at most 4096).
   Synchronous. */
dg_status dg_test_expected_embedding_topk(const uint16_t* d_logits, int64_t V, int32_t K, const uint16_t* d_emb,
                                          int32_t d, int32_t T, uint16_t* d_out, void* stream);

/* sizeof of one of the ABI's structs by its name ("dg_model_config",
   "dg_sampler_config", "dg_kv", "dg_canvas", "dg_step_args", "dg_step_out",
   "dg_block_stats", "dg_profile"), 0 for another name.  Host only: lets a
   binding check its mirrors of the structs against this build. */
size_t dg_test_struct_size(const char* name);

/* Device address and size of one named scratch buffer of a context's
   workspace (for inspecting the last layer's intermediates after a call):
   "x" fp32 residual [T, d], "xn" bf16 normed activations, "qkv" fp32,
   "q" bf16 [T, Hq*hd], "attn" bf16 [T, Hq*hd], "rpart" fp32 split-k router
   partial logits [splits, T, E], "off" int32 [E+1], "perm", "inv" int32 [T*k],
   "wperm" fp32 [T*k], "xperm" bf16 [T*k, d], "hperm" bf16 [T*k, f],
   "yperm" fp32 [T*k, d], "logits" bf16 [T, V], "probs" bf16 [T, V]. */
dg_status dg_test_workspace_buffer(dg_ctx* ctx, const char* name, void** d_ptr, size_t* bytes);

#ifdef __cplusplus
}
#endif
#endif /* DG_TESTING_H */
