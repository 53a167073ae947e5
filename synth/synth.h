/*
 * synth.h - seeded synthetic input generator shared by the CUDA library's
 * random-init entry point and by the CPU oracle.
 *
 * It holds none of the denoising method's arithmetic: it only turns
 * (seed, tensor id, element index) into input values (weights, token ids,
 * hidden states).  Two implementations exist, synth_host.c (CPU, threads)
 * and synth_device.cu (CUDA); both use integer arithmetic up to one
 * exactly rounded IEEE double multiply, so they produce identical bits.
 *
 * Recipe (the same on both sides):
 *   r[0..3] = Philox4x32-10(key = (lo32(seed), hi32(seed)),
 *                           ctr = (lo32(i), hi32(i), tid, SYNTH_CTR_TAG))
 *   Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and
 *   Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11), 10 rounds.
 *
 *   weight value  : s = r0 + r1 + r2 + r3 (exact, 64-bit), c = s - 2*(2^32-1)
 *                   x = (double)c * (std * sqrt(3) * 2^-32)
 *                   stored as bf16 (round to nearest even, straight from the
 *                   double).  The sum of four uniforms (Irwin-Hall, n = 4)
 *                   has mean 0 and standard deviation std, and is an
 *                   approximately normal N(0, std^2) draw.
 *   fp32 value    : same x, rounded to float (round to nearest even).
 *   token id      : (r0 * V) >> 32   (64-bit product, uniform over [0, V)).
 *
 * Tensor ids: global tensors use their kind, per-layer tensors use
 * ((layer + 1) << 5) | kind.  Element index i of a logical tensor is its
 * row-major index in the logical shape listed beside each kind.
 */
#ifndef DG_SYNTH_H
#define DG_SYNTH_H

#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SYNTH_CTR_TAG 0x53594E54u /* "SYNT": keeps input draws apart from the method's own draws */

/* global tensors */
#define SYNTH_KIND_EMB     1  /* E_emb  [V, d]                 */
#define SYNTH_KIND_LM      2  /* W_lm   [V, d]                 */
#define SYNTH_KIND_SC      3  /* W_sc   [d (out), d (in)]      */
#define SYNTH_KIND_CTX     4  /* context tokens [B, n], tid = SYNTH_KIND_CTX | (b << 8) */
#define SYNTH_KIND_HIDDEN  5  /* probe hidden states [T, d]    */
/* per-layer tensors */
#define SYNTH_KIND_WQ     16  /* [Hq*hd (out), d (in)]         */
#define SYNTH_KIND_WK     17  /* [Hkv*hd, d]                   */
#define SYNTH_KIND_WV     18  /* [Hkv*hd, d]                   */
#define SYNTH_KIND_WO     19  /* [d, Hq*hd]                    */
#define SYNTH_KIND_WR     20  /* router [E, d]                 */
#define SYNTH_KIND_WG     21  /* gate   [E, f, d]              */
#define SYNTH_KIND_WU     22  /* up     [E, f, d]              */
#define SYNTH_KIND_WD     23  /* down   [E, d, f]              */

static inline uint32_t synth_layer_tid(int layer, int kind) {
  return ((uint32_t)(layer + 1) << 5) | (uint32_t)kind;
}

/* ---- host implementation (synth_host.c) -------------------------------- */

/* dst[r*stride_r + c*stride_c] = bf16 value of element ((row0 + r)*cols + c),
   for r in [0, rows), c in [0, cols): rows [row0, row0 + rows) of a logical
   [*, cols] tensor.  Uses up to n_threads threads (<=0: all). */
int synth_fill_bf16_host(uint16_t* dst, int64_t row0, int64_t rows, int64_t cols,
                         int64_t stride_r, int64_t stride_c,
                         uint64_t seed, uint32_t tid, double std, int n_threads);
/* fp32 values of elements [0, n) */
int synth_fill_f32_host(float* dst, int64_t n, uint64_t seed, uint32_t tid,
                        double std, int n_threads);
/* token ids of elements [0, n), uniform over [0, V) */
int synth_fill_tokens_host(int32_t* dst, int64_t n, uint64_t seed, uint32_t tid,
                           int32_t V);
/* raw Philox4x32-10 block, exposed so the generator can be pinned to its
   published known-answer vectors */
void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* ---- device implementation (synth_device.cu) --------------------------- */
/* Same contracts as above; dst is device memory, work is queued on `stream`
   (a cudaStream_t passed as void*).  Return 0 or a cudaError_t code. */
int synth_fill_bf16_device(uint16_t* dst, int64_t row0, int64_t rows, int64_t cols,
                           int64_t stride_r, int64_t stride_c,
                           uint64_t seed, uint32_t tid, double std, void* stream);
int synth_fill_f32_device(float* dst, int64_t n, uint64_t seed, uint32_t tid,
                          double std, void* stream);
int synth_fill_tokens_device(int32_t* dst, int64_t n, uint64_t seed, uint32_t tid,
                             int32_t V, void* stream);

#ifdef __cplusplus
}
#endif
#endif
