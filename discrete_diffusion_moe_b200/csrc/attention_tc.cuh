// attention_tc.cuh - attention of one pass of queries over the keys of a
// KV cache on the tcgen05 tensor cores (sm_100a).
//
//   canvas pass (causal_n = 0): every query sees keys [0, L0 + nq)   (no mask:
//     bidirectional over the canvas, full view of the context)
//   context encoding (causal_n = nq): query i sees keys [0, L0 + i]
//   a finished block appended in the same pass as the next canvas round
//     (causal_n = 256): the block's queries causal, the canvas's see all keys
//
// One CTA computes one 128-row tile of packed queries against a range of
// 64-key tiles (a key split).  Grouped-query packing: the G = Hq / Hkv query
// heads of kv head g are stored as rows (token, head-in-group) of one
// [nq * G, hd] matrix, so one tile of K / V^T feeds every head of the group.
//
//   warp 0      TMA: the Q tile once, then K tile and V^T tile per stage
//               (three stages); the V^T map's key extent is the number of valid
//               keys, so keys past it arrive as zeros
//   warp 1      tensor memory owner and MMA issuer:
//                 S  = Q K^T            (M 128, N 64, K hd)    -> TMEM cols [0, 64)
//                 O += P V              (M 128, N hd, K 64)    -> TMEM cols [64, 64 + hd)
//                                       (V in fp16 from shared memory, P as
//                                        two fp16 parts from tensor memory:
//                                        O += P_hi V + P_lo V)
//               S of tile j + 1 is issued as soon as S of tile j has been read,
//               before P V of tile j, so the next scores overlap the softmax.
//   warps 2..9  softmax, two threads per query row (tensor-memory lane), each
//               taking 32 of the tile's 64 scores; the pair exchanges its
//               partial maxima through shared memory (bounded mbarrier wait),
//               keeps an online max / sum in the exp2 domain, rescales its
//               half of the row of O in tensor memory when the reference max
//               moved, writes P as P_hi = fp16(P) and P_lo = fp16(P - P_hi)
//               (about 22 significant bits together; scaled by 2^7 so that
//               the values lie in (0, 2^15])
//               into tensor memory, where the P V product takes its A
//               operand (the V^T cache holds the bf16-rounded values in
//               fp16, exact above 2^-14, for this product);
//               finally read O and write the normalised bf16 output, or
//               stage the split's unnormalised partial in the freed K/V
//               memory and store it with one bulk copy per 32 rows (with its
//               max and sum).
//
// Every mbarrier wait is bounded; a thread whose wait ran out sets the error
// word and stops issuing work, and the tensor memory is released only after
// the MMA issuer's last operations completed.
#pragma once

#include "common.cuh"

namespace dg {

struct AttnTcParams {
  uint16_t* out;       // [B * nq, Hq * hd] bf16 (splits == 1, or merged in the cluster)
  float* part_o;       // [splits][B][Hq][nq][hd] unnormalised (splits > 1 without cluster)
  float* part_ml;      // [splits][B][Hq][nq][2] (max in log2 units, sum)
  int B, nq, L0, c_max, Hq, Hkv, splits;
  int causal_n;        // queries of the first causal_n tokens of a canvas are causal
                       // (token i sees keys [0, L0 + i]); the others see every key
  float scale_log2;    // log2(e) / sqrt(hd)
  int* err;
  int cluster;         // splits > 1: the splits of a tile are one cluster and merge
                       // through distributed shared memory (no partials in global memory)
};

// P in the P V product: 1 = two fp16 parts, P_hi + P_lo (about 22 significant
// bits; two products per key tile), 0 = one fp16 part (11 bits).
#ifndef DG_ATTN_P_SPLIT
#define DG_ATTN_P_SPLIT 1
#endif
constexpr int kAttnPParts = DG_ATTN_P_SPLIT ? 2 : 1;

constexpr int kAttnThreads = 320;
constexpr int kAttnKeys = 64;   // keys per tile
constexpr int kAttnRows = 128;  // packed query rows per CTA
constexpr float kAttnLazyLog2 = 8.f;  // reference-max slack (log2 units)
// P is computed as 2^(s - m + 7): the values lie in (0, 2^15] (below the fp16
// maximum) and only those below 2^-21 of the reference fall to fp16
// subnormals.  The row sum carries the same factor, so it cancels.
constexpr float kAttnPScaleLog2 = 7.f;

template <int HD>
struct AttnTcShape {
  static constexpr int NA = (HD + 63) / 64;          // 64-wide atoms of the head dimension
  static constexpr uint32_t Q_BYTES = NA * 128 * 128;
  static constexpr uint32_t K_BYTES = NA * kAttnKeys * 128;
  static constexpr uint32_t V_BYTES = HD * 128;      // hd rows x 64 keys
  // P lives in tensor memory (the A operand of the P V product), not here
  static constexpr size_t FIXED = 1024 + Q_BYTES + 32 * 8 + 6 * 128 * 4;
  // K/V stages: three where they fit (the load of tile i + 3 is in flight while
  // tiles i + 1, i + 2 are multiplied), else two
  static constexpr int KV_STAGES = FIXED + 3 * (K_BYTES + V_BYTES) <= 227 * 1024 ? 3 : 2;
  static constexpr size_t SMEM = FIXED + KV_STAGES * (K_BYTES + V_BYTES);
  // the K/V stages hold the final O tile for its tensor stores: per lane
  // quarter, NCB boxes of 32 rows x 32 fp32 columns (128-byte swizzle)
  static constexpr int NCB = (HD + 31) / 32;
  // (the K/V stages: one contiguous region, free at the end)
  static_assert((size_t)KV_STAGES * (K_BYTES + V_BYTES) >= (size_t)4 * NCB * 4096, "O staging");
  // cluster merge: the unnormalised O tile staged row-major in the K/V stage
  // memory with a row pitch of HD + 4 floats (the 16-byte pieces of 8
  // consecutive rows fall in different bank groups), then (max, sum) per row
  static constexpr int OSTR = HD + 4;
  static constexpr uint32_t O_STAGE = 128u * OSTR * 4u;
  // then the merge weights, [at most 64 rows][8 splits]
  static constexpr uint32_t WTS_OFF = O_STAGE + 128 * 8;
  static_assert((size_t)KV_STAGES * (K_BYTES + V_BYTES) >= (size_t)WTS_OFF + 64 * 8 * 4, "cluster O staging");
  // tensor memory: S in columns [0, 64), O in [64, 64 + HD), then P from P_COL:
  // per tile parity P_hi (and P_lo) as 32 columns each, two fp16 keys per column
  static constexpr uint32_t P_COL = (64 + HD + 31) / 32 * 32;
  static constexpr uint32_t P_BUF_COLS = 32 * kAttnPParts;
  static constexpr uint32_t TMEM_NEED = P_COL + 2 * P_BUF_COLS;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 128 ? 128 : (TMEM_NEED <= 256 ? 256 : 512);
  static_assert(TMEM_NEED <= 512, "tensor memory");
};

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// 32 lanes x 16 consecutive 32-bit columns from registers (raw words)
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, fp16 inputs, fp32 accumulate; A is M rows
// in tensor-memory lanes, K packed two 16-bit elements per 32-bit column.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 consecutive fp32 columns in one load and one wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
#define DG_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : DG_R8(0), DG_R8(8), DG_R8(16), DG_R8(24)
      : "r"(taddr));
#undef DG_R8
#define DG_W8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
  asm volatile("tcgen05.wait::ld.sync.aligned;" : DG_W8(0), DG_W8(8), DG_W8(16), DG_W8(24) : : "memory");
#undef DG_W8
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 2^x on the special-function unit (PTX ex2.approx.ftz; 2^-inf = 0).
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 lanes x 64 consecutive fp32 columns in one load and one wait (the wait
// names every destination register so no use is scheduled before it).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
#define DG_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,"
      "%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : DG_R8(0), DG_R8(8), DG_R8(16), DG_R8(24), DG_R8(32), DG_R8(40), DG_R8(48), DG_R8(56)
      : "r"(taddr));
#undef DG_R8
#define DG_W8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7])
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : DG_W8(0), DG_W8(8), DG_W8(16), DG_W8(24), DG_W8(32), DG_W8(40), DG_W8(48), DG_W8(56)
               :
               : "memory");
#undef DG_W8
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// tmQ: packed queries [B * Hkv * nq * G rows, hd], box 64 x 128
// tmK: keys [B * Hkv * c_max rows, hd], box 64 x 64
// tmV: transposed values [B * Hkv * hd rows, keys] (key extent = valid keys), box 64 x hd
template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const AttnTcParams p) {
  using S = AttnTcShape<HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  constexpr int NS = S::KV_STAGES;
  uint8_t* sK = sQ + S::Q_BYTES;               // NS stages
  uint8_t* sV = sK + NS * S::K_BYTES;          // NS stages
  uint64_t* bars = (uint64_t*)(sV + NS * S::V_BYTES);
  uint64_t* q_full = bars;
  // K and V of a stage are released separately: K as soon as the scores of
  // its tile are computed (so the next K load overlaps the softmax), V after
  // the P V product
  uint64_t* k_full = bars + 1;          // [NS]
  uint64_t* k_empty = bars + 1 + NS;    // [NS]
  uint64_t* v_full = bars + 1 + 2 * NS; // [NS]
  uint64_t* v_empty = bars + 1 + 3 * NS;// [NS]
  uint64_t* s_full = bars + 1 + 4 * NS;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;      // [2] by tile parity
  uint64_t* pv_done = s_full + 4;     // [2] by tile parity
  uint64_t* drain = s_full + 6;
  uint64_t* pair_bar = s_full + 7;     // [4] per tensor-memory lane quarter: the two halves of a row
  uint32_t* tmem_slot = (uint32_t*)(s_full + 11);
  float* xchg = (float*)(s_full + 13);  // [2 tile parities][2 halves][128 rows] maxima, then [2][128] sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int rows_total = G * p.nq;
  const int r0 = blockIdx.x * kAttnRows;
  const int g = blockIdx.y;
  const int b = blockIdx.z / p.splits, split = blockIdx.z - b * p.splits;
  const int kv_len = p.L0 + p.nq;
  const int n_kt = (kv_len + kAttnKeys - 1) / kAttnKeys;
  const int kt0 = (int)((long long)n_kt * split / p.splits);
  int kt1 = (int)((long long)n_kt * (split + 1) / p.splits);
  {
    // the tile's last row sees the most keys (visibility grows with the token)
    const int r_last = min(r0 + kAttnRows - 1, rows_total - 1);
    if (r_last / G < p.causal_n) kt1 = min(kt1, (p.L0 + r_last / G) / kAttnKeys + 1);
  }
  const int n_tiles = max(0, kt1 - kt0);
  const int bg = b * p.Hkv + g;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_free), 256);
    mbar_init(smem_u32(&p_full[0]), 256);
    mbar_init(smem_u32(&p_full[1]), 256);
    for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&pair_bar[q]), 64);
    mbar_init(smem_u32(&pv_done[0]), 1);
    mbar_init(smem_u32(&pv_done[1]), 1);
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  grid_dep_wait();
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t t_s = tmem_base, t_o = tmem_base + 64, t_p = tmem_base + S::P_COL;

  if (warp == 0) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- TMA producer ----------------
      const uint32_t qb = smem_u32(q_full);
      mbar_arrive_expect_tx(qb, S::Q_BYTES);
      const int q_row0 = bg * rows_total + r0;
      for (int a = 0; a < S::NA; ++a) tma_load_2d(smem_u32(sQ + a * 16384), &tmQ, qb, a * 64, q_row0);
      int issued = 0;
      int issued_v = 0;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        const uint32_t par = ((i / NS) & 1) ^ 1;
        const int key0 = (kt0 + i) * kAttnKeys;
        if (!mbar_wait(smem_u32(&k_empty[s]), par, p.err)) break;
        const uint32_t kb = smem_u32(&k_full[s]);
        mbar_arrive_expect_tx(kb, S::K_BYTES);
        for (int a = 0; a < S::NA; ++a)
          tma_load_2d(smem_u32(sK + s * S::K_BYTES + a * kAttnKeys * 128), &tmK, kb, a * 64,
                      bg * p.c_max + key0);
        ++issued;
        if (!mbar_wait(smem_u32(&v_empty[s]), par, p.err)) break;
        const uint32_t vb = smem_u32(&v_full[s]);
        mbar_arrive_expect_tx(vb, S::V_BYTES);
        tma_load_2d(smem_u32(sV + s * S::V_BYTES), &tmV, vb, key0, bg * HD);
        ++issued_v;
      }
      // every issued copy must land before the CTA may exit
      mbar_wait(qb, 0, p.err);
      for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
        mbar_wait(smem_u32(&k_full[i % NS]), (i / NS) & 1, p.err);
      for (int i = issued_v > NS ? issued_v - NS : 0; i < issued_v; ++i)
        mbar_wait(smem_u32(&v_full[i % NS]), (i / NS) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t id_s = idesc_bf16_f32(128, kAttnKeys);
      const uint32_t id_o = idesc_f16_f32(128, HD);
      bool ok = mbar_wait(smem_u32(q_full), 0, p.err);
      auto issue_s = [&](int i) -> bool {
        const int s = i % NS;
        if (!mbar_wait(smem_u32(&k_full[s]), (i / NS) & 1, p.err)) return false;
        if (i > 0 && !mbar_wait(smem_u32(s_free), (i - 1) & 1, p.err)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK + s * S::K_BYTES);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint32_t off = (k & 3) * 32;
          umma_bf16(t_s, sdesc_k128(qa + (k >> 2) * 16384 + off), sdesc_k128(ka + (k >> 2) * kAttnKeys * 128 + off),
                    id_s, k > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(s_full));
        umma_commit(smem_u32(&k_empty[s]));  // K of this stage is consumed once the scores are
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 1 < n_tiles && !issue_s(i + 1)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&p_full[i & 1]), (i >> 1) & 1, p.err)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&v_full[i % NS]), (i / NS) & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t va = smem_u32(sV + (i % NS) * S::V_BYTES);
        // O += P_hi V + P_lo V: P to ~22 significant bits from two fp16 parts,
        // both read from tensor memory (8 columns of 16 keys per product)
        const uint32_t pa = t_p + (uint32_t)(i & 1) * S::P_BUF_COLS;
#pragma unroll
        for (int k = 0; k < kAttnKeys / 16; ++k)
          umma_f16_tmem_a(t_o, pa + k * 8, sdesc_k128(va + k * 32), id_o, (i > 0 || k > 0) ? 1u : 0u);
        if (kAttnPParts == 2) {
#pragma unroll
          for (int k = 0; k < kAttnKeys / 16; ++k) umma_f16_tmem_a(t_o, pa + 32 + k * 8, sdesc_k128(va + k * 32), id_o, 1u);
        }
        umma_commit(smem_u32(&pv_done[i & 1]));
        umma_commit(smem_u32(&v_empty[i % NS]));
      }
      umma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else {
    // ---------------- softmax + epilogue (warps 2..9) ----------------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;      // which 32 of the tile's 64 keys
    const int row = quarter * 32 + lane;   // tensor-memory lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int r = r0 + row;
    const int t_in = (r < rows_total ? r : rows_total - 1) / G;  // token within the pass
    const int lim = t_in < p.causal_n ? min(kv_len - 1, p.L0 + t_in) : kv_len - 1;
    const float scale = p.scale_log2;
    float m = -INFINITY, l = 0.f;  // reference max (scaled, log2 units) and this half's sum
    bool ok = true;
    const uint32_t pb = smem_u32(&pair_bar[quarter]);
    constexpr int NCH = HD / 16;
    const int oc0 = half ? (NCH + 1) / 2 : 0, oc1 = half ? NCH : (NCH + 1) / 2;  // this half's O chunks
    // waits are made warp-uniform: tensor-memory loads and stores are
    // warp-collective and must never run in a diverged warp
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.err)) != 0;
    };
    for (int i = 0; i < n_tiles && ok; ++i) {
      if (!wait_all(smem_u32(s_full), i & 1)) { ok = false; break; }
      tc_fence_after();
      float sv[32];
      tmem_ld32(t_s + lane_off + half * 32, sv);
      tc_fence_before();
      mbar_arrive(smem_u32(s_free));
      const int key0 = (kt0 + i) * kAttnKeys + half * 32;
      // raw maximum of this half (scale > 0 commutes with max); mask only a
      // tile that reaches past the row's last visible key
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (key0 + 31 <= lim) {
#pragma unroll
        for (int c = 0; c < 32; ++c) mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sv[c] = key0 + c <= lim ? sv[c] : -INFINITY;
          mq[c & 3] = fmaxf(mq[c & 3], sv[c]);
        }
      }
      // exchange the halves' maxima (double-buffered by tile parity)
      float* xm = xchg + (i & 1) * 256;
      xm[half * 128 + row] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      mbar_arrive(pb);
      if (!wait_all(pb, i & 1)) { ok = false; break; }
      const float raw = fmaxf(xm[row], xm[128 + row]);
      const float mx = raw * scale;  // -inf stays -inf
      // The reference max only moves when the tile's max exceeds it by more
      // than 2^8: the exponentials stay <= 256 (the same 16-bit P precision,
      // fp32 sums), and O is rescaled rarely instead of on nearly every tile.
      // The final normalisation divides by the sum taken against the same
      // reference, so the result is unchanged.
      const bool move = mx > m + kAttnLazyLog2 || (m == -INFINITY && mx != -INFINITY);
      const float m_new = move ? mx : m;
      const float alpha = (move && m != -INFINITY) ? ex2_fast(m - m_new) : 1.f;
      const float nref = m_new == -INFINITY ? 0.f : kAttnPScaleLog2 - m_new;
      float sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const float pv = ex2_fast(fmaf(sv[c], scale, nref));  // masked: 2^-inf = 0
        sv[c] = pv;
        sq[c & 3] += pv;
      }
      l = l * alpha + ((sq[0] + sq[1]) + (sq[2] + sq[3]));
      m = m_new;
      // O rescale: every product into O so far (up to tile i - 1) has completed
      if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_all(smem_u32(&pv_done[(i - 1) & 1]), ((i - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        {
          for (int c = oc0; c < oc1; ++c) {
            float v[16];
            tmem_ld16(t_o + lane_off + c * 16, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= alpha;
            tmem_st16(t_o + lane_off + c * 16, v);
          }
          tmem_wait_st();
        }
      }
      // this P buffer was last read by the product of tile i - 2
      if (i > 1) {
        if (!wait_all(smem_u32(&pv_done[i & 1]), ((i - 2) >> 1) & 1)) { ok = false; break; }
      }
      // P into tensor memory, the A operand of the P V product: the row's lane,
      // two keys per 32-bit column (the even key in the low half), this half's
      // 32 keys in columns [16 half, 16 half + 16); P_hi = fp16(P) and
      // P_lo = fp16(P - P_hi) (the difference is exact in fp32) 32 columns apart
      {
        uint32_t hv[16], lv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = sv[2 * e], b2 = sv[2 * e + 1];
          hv[e] = pack_f16x2(a, b2);
          const __half2 hh = *reinterpret_cast<const __half2*>(&hv[e]);
          lv[e] = pack_f16x2(a - __low2float(hh), b2 - __high2float(hh));
        }
        const uint32_t tp = t_p + lane_off + (uint32_t)(i & 1) * S::P_BUF_COLS + (uint32_t)half * 16;
        tmem_st16u(tp, hv);
        if (kAttnPParts == 2) tmem_st16u(tp + 32, lv);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&p_full[i & 1]));
    }
    if (ok && n_tiles > 0) ok = wait_all(smem_u32(&pv_done[(n_tiles - 1) & 1]), ((n_tiles - 1) >> 1) & 1);
    tc_fence_after();
    // total sum of the row: both halves used the same reference max
    float* xl = xchg + 512;
    xl[half * 128 + row] = l;
    mbar_arrive(pb);
    const bool have = ok && n_tiles > 0 && wait_all(pb, n_tiles & 1);  // uniform across the warp
    const float l_row = have ? xl[row] + xl[128 + row] : 0.f;
    const bool valid = r < rows_total;
    const int h = g * G + (valid ? r % G : 0);
    const float inv = (have && l_row > 0.f) ? 1.f / l_row : 0.f;
    if (p.splits == 1) {
      for (int c = oc0; c < oc1; ++c) {
        float v[16];
        if (have) {
          tmem_ld16(t_o + lane_off + c * 16, v);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0.f;
        }
        if (!valid) continue;
        uint16_t* dst = p.out + ((long long)(b * p.nq + t_in) * p.Hq + h) * HD + c * 16;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(v[2 * e] * inv, v[2 * e + 1] * inv);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(dst + 8) = make_uint4(w[4], w[5], w[6], w[7]);
      }
    } else if (p.cluster) {
      // cluster merge, part 1: stage this split's unnormalised O rows and the
      // row's (reference max, sum) for the other CTAs of the cluster (every
      // tensor-core operation and copy into the K/V stages has completed)
      float* so = reinterpret_cast<float*>(sK) + (size_t)row * S::OSTR;
      for (int c = oc0; c < oc1; ++c) {
        float v[16];
        if (have) {
          tmem_ld16(t_o + lane_off + c * 16, v);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<float4*>(so + c * 16 + 4 * e) = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
      }
      if (half == 0)
        reinterpret_cast<float2*>(sK + S::O_STAGE)[row] = make_float2(have ? m : -INFINITY, have ? l_row : 0.f);
    } else {
      // split partial: the unnormalised O rows (fp32) are staged in the K/V
      // stage memory (every tensor-core operation and copy into it has
      // completed) as 32 x 32 boxes with the 128-byte swizzle (16-byte piece k
      // of a box row r at k ^ (r % 8): the 8 rows of a quarter warp write 8
      // different bank groups) and leave in tensor stores, one per box; the
      // partial rows follow the packed query order [split][b][g][row]
      constexpr int MAXC = (NCH + 1) / 2;
      uint32_t rr[MAXC][16];
#pragma unroll
      for (int q = 0; q < MAXC; ++q)
#pragma unroll
        for (int e = 0; e < 16; ++e) rr[q][e] = 0u;
      if (have) {
#pragma unroll
        for (int q = 0; q < MAXC; ++q)
          if (oc0 + q < oc1) tmem_ld16_nowait(t_o + lane_off + (oc0 + q) * 16, rr[q]);
#pragma unroll
        for (int q = 0; q < MAXC; ++q)
          if (oc0 + q < oc1) tmem_wait_ld16(rr[q]);
      }
      uint8_t* qbox = sK + (size_t)quarter * S::NCB * 4096 + (size_t)lane * 128;
#pragma unroll
      for (int q = 0; q < MAXC; ++q)
        if (oc0 + q < oc1) {
          const int c = oc0 + q;
          uint8_t* bx = qbox + (size_t)(c >> 1) * 4096;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int piece = (c & 1) * 4 + e;
            *reinterpret_cast<float4*>(bx + ((piece ^ (lane & 7)) << 4)) =
                make_float4(__uint_as_float(rr[q][4 * e]), __uint_as_float(rr[q][4 * e + 1]),
                            __uint_as_float(rr[q][4 * e + 2]), __uint_as_float(rr[q][4 * e + 3]));
          }
        }
      const long long prow_g = (((long long)split * p.B + b) * p.Hkv + g) * rows_total + r;
      if (valid && half == 0) {
        p.part_ml[prow_g * 2] = have ? m : -INFINITY;
        p.part_ml[prow_g * 2 + 1] = have ? l_row : 0.f;
      }
      // each lane quarter's boxes leave once both halves have staged them
      // (rows past the pass's packed rows fall outside the tensor and are
      // not written)
      fence_proxy_async_smem();
      mbar_arrive(pb);
      const bool staged = wait_all(pb, (n_tiles + 1) & 1);
      const int q0 = r0 + quarter * 32;
      if (staged && half == 0 && lane == 0 && q0 < rows_total) {
        const int z = (split * p.B + b) * p.Hkv + g;
        for (int cb = 0; cb < S::NCB; ++cb)
          tma_store_3d(&tmO, smem_u32(sK + ((size_t)quarter * S::NCB + cb) * 4096), cb * 32, q0, z);
        bulk_commit_wait_read();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cluster && p.splits > 1) {
    // cluster merge, part 2: CTA `rank` of the cluster (= its key split)
    // finishes rows [q0, q1) of the tile from every split's staged rows, in
    // split order: O = sum_s w_s O_s with w_s = 2^(m_s - M) / sum_s' 2^(m_s' - M) l_s'
    cluster_sync_all();  // every split's rows and (max, sum) are staged
    if (warp >= 2) {
      const int S_ = p.splits;
      const int rank = (int)cluster_ctarank();
      const int per = (kAttnRows + S_ - 1) / S_;
      const int q0 = rank * per, q1 = min(kAttnRows, q0 + per);
      const int te = threadIdx.x - 64;
      float* wts = reinterpret_cast<float*>(sK + S::WTS_OFF);  // [per rows][8 splits] merge weights
      const uint32_t o_base = smem_u32(sK), ml_base = smem_u32(sK + S::O_STAGE);
      if (te < q1 - q0) {
        const int row = q0 + te;
        float2 ml[8];
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S_) {
            ml[s2] = ld_dsmem_f2(mapa_shared(ml_base + row * 8, (uint32_t)s2));
            M = fmaxf(M, ml[s2].x);
          }
        float w[8], L = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S_) {
            w[s2] = ml[s2].x == -INFINITY ? 0.f : ex2_fast(ml[s2].x - M);
            L += w[s2] * ml[s2].y;
          }
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          if (s2 < S_) wts[te * 8 + s2] = w[s2] * inv;
      }
      named_bar_sync(1, 256);
      constexpr int NC4 = HD / 4;
      const int n_items = (q1 - q0) * NC4;
      const int G = p.Hq / p.Hkv;
      const int rows_total = G * p.nq;
      // two items per pass: all of their remote loads are issued before the
      // first is used (a remote load's latency, not its bandwidth, bounds this)
      constexpr int kItems = 2;
      for (int it0 = te; it0 < n_items; it0 += 256 * kItems) {
        float4 v[kItems][8];
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
          const int it = it0 + u * 256;
          const int rr = it / NC4, c4 = it - rr * NC4;
          const uint32_t off = o_base + (uint32_t)((q0 + rr) * S::OSTR + c4 * 4) * 4u;
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            if (s2 < S_ && it < n_items) v[u][s2] = ld_dsmem_f4(mapa_shared(off, (uint32_t)s2));
        }
#pragma unroll
        for (int u = 0; u < kItems; ++u) {
          const int it = it0 + u * 256;
          if (it >= n_items) break;
          const int rr = it / NC4, c4 = it - rr * NC4;
          const int r = r0 + q0 + rr;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            if (s2 < S_) {
              const float ws = wts[rr * 8 + s2];
              acc.x += ws * v[u][s2].x; acc.y += ws * v[u][s2].y; acc.z += ws * v[u][s2].z; acc.w += ws * v[u][s2].w;
            }
          if (r < rows_total) {
            const int t_in = r / G, h = g * G + r % G;
            uint16_t* dst = p.out + ((long long)(b * p.nq + t_in) * p.Hq + h) * HD + c4 * 4;
            *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
          }
        }
      }
    }
    cluster_sync_all();  // no CTA leaves while another reads its shared memory
  }
  if (warp == 1) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

// Merge split-KV partials (fixed split order) -> bf16 output.  One warp per
// (canvas, head, query) row: the split maxima and sums are read once per row,
// the row's HD values are merged with 16-byte vector loads.  Partial rows are
// in packed query order: [split][b][g][token * G + head-in-group].
// MAXS: the largest split count the instantiation handles (4 or 8).
template <int MAXS>
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                    uint16_t* __restrict__ out, int splits, int B, int Hq, int Hkv, int nq,
                                    int HD) {
  grid_dep_wait();
  grid_dep_launch();
  const long long rows = (long long)B * Hq * nq;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int i = (int)(row % nq);
  const long long bh = row / nq;
  const int h = (int)(bh % Hq), b = (int)(bh / Hq);
  const int G = Hq / Hkv, g = h / G;
  const long long prow = (((long long)b * Hkv + g) * nq + i) * G + (h - g * G);
  // every load (the split maxima and sums, and this lane's partial O vectors
  // of every split) is issued before the first is used
  constexpr int kMaxVec = 2;  // 16-byte vectors per lane and split (HD <= 256)
  float2 ml[MAXS];
  float4 po[MAXS][kMaxVec];
#pragma unroll
  for (int s = 0; s < MAXS; ++s)
    if (s < splits) {
      ml[s] = *reinterpret_cast<const float2*>(part_ml + (s * rows + prow) * 2);
#pragma unroll
      for (int u = 0; u < kMaxVec; ++u) {
        const int c = lane * 4 + u * 128;
        if (c < HD) po[s][u] = *reinterpret_cast<const float4*>(part_o + (s * rows + prow) * HD + c);
      }
    }
  float mx = -INFINITY;
#pragma unroll
  for (int s = 0; s < MAXS; ++s)
    if (s < splits) mx = fmaxf(mx, ml[s].x);
  float wgt[MAXS];
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < MAXS; ++s) {
    wgt[s] = 0.f;
    if (s < splits) {
      if (ml[s].x != -INFINITY) wgt[s] = exp2f(ml[s].x - mx);
      den += wgt[s] * ml[s].y;
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  uint16_t* dst = out + ((long long)(b * nq + i) * Hq + h) * HD;
#pragma unroll
  for (int u = 0; u < kMaxVec; ++u) {
    const int c = lane * 4 + u * 128;
    if (c >= HD) break;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < MAXS; ++s)
      if (s < splits) {
        const float4 v = po[s][u];
        acc.x += wgt[s] * v.x; acc.y += wgt[s] * v.y; acc.z += wgt[s] * v.z; acc.w += wgt[s] * v.w;
      }
    uint2 o;
    o.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    o.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(dst + c) = o;
  }
}

}  // namespace dg
