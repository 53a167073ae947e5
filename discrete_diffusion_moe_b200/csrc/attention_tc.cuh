// attention_tc.cuh - attention of one pass of queries over the keys of a
// KV cache on the tcgen05 tensor cores (sm_100a).
//
//   canvas pass (causal = 0): every query sees keys [0, L0 + nq)   (no mask:
//     bidirectional over the canvas, full view of the context)
//   context encoding (causal = 1): query i sees keys [0, L0 + i]
//
// One CTA computes one 128-row tile of packed queries against a range of
// 64-key tiles (a key split).  Grouped-query packing: the G = Hq / Hkv query
// heads of kv head g are stored as rows (token, head-in-group) of one
// [nq * G, hd] matrix, so one tile of K / V^T feeds every head of the group.
//
//   warp 0      TMA: the Q tile once, then K tile and V^T tile per stage
//               (two stages); the V^T map's key extent is the number of valid
//               keys, so keys past it arrive as zeros
//   warp 1      tensor memory owner and MMA issuer:
//                 S  = Q K^T            (M 128, N 64, K hd)    -> TMEM cols [0, 64)
//                 O += P_hi V + P_lo V  (M 128, N hd, K 64)    -> TMEM cols [64, 64 + hd)
//               S of tile j + 1 is issued as soon as S of tile j has been read,
//               before P V of tile j, so the next scores overlap the softmax.
//   warps 2..5  softmax, one thread per query row (tensor-memory lane): read
//               its 64 scores, online max / sum in the exp2 domain, rescale its
//               row of O in tensor memory when the max grew, write P split
//               into a bf16 high part and a bf16 residual (P = P_hi + P_lo,
//               about 16 significant bits for the P V product) into shared
//               memory in the 128-byte-swizzled K-major layout the MMA reads;
//               finally read O and write the normalised bf16 output or the
//               split's unnormalised partial (with its max and sum).
//
// Every mbarrier wait is bounded; a thread whose wait ran out sets the error
// word and stops issuing work, and the tensor memory is released only after
// the MMA issuer's last operations completed.
#pragma once

#include "common.cuh"

namespace dg {

struct AttnTcParams {
  uint16_t* out;       // [B * nq, Hq * hd] bf16            (splits == 1)
  float* part_o;       // [splits][B][Hq][nq][hd] unnormalised (splits > 1)
  float* part_ml;      // [splits][B][Hq][nq][2] (max in log2 units, sum)
  int B, nq, L0, c_max, Hq, Hkv, splits, causal;
  float scale_log2;    // log2(e) / sqrt(hd)
  int* err;
};

constexpr int kAttnThreads = 192;
constexpr int kAttnKeys = 64;   // keys per tile
constexpr int kAttnRows = 128;  // packed query rows per CTA

template <int HD>
struct AttnTcShape {
  static constexpr int NA = (HD + 63) / 64;          // 64-wide atoms of the head dimension
  static constexpr uint32_t Q_BYTES = NA * 128 * 128;
  static constexpr uint32_t K_BYTES = NA * kAttnKeys * 128;
  static constexpr uint32_t V_BYTES = HD * 128;      // hd rows x 64 keys
  static constexpr uint32_t P_BYTES = kAttnRows * 128;
  static constexpr size_t SMEM = 1024 + Q_BYTES + 2 * (K_BYTES + V_BYTES) + 2 * P_BYTES + 16 * 8;
  static constexpr uint32_t TMEM_COLS = (64 + HD) <= 128 ? 128 : 256;
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

// tmQ: packed queries [B * Hkv * nq * G rows, hd], box 64 x 128
// tmK: keys [B * Hkv * c_max rows, hd], box 64 x 64
// tmV: transposed values [B * Hkv * hd rows, keys] (key extent = valid keys), box 64 x hd
template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnTcParams p) {
  using S = AttnTcShape<HD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + S::Q_BYTES;               // 2 stages
  uint8_t* sV = sK + 2 * S::K_BYTES;           // 2 stages
  uint8_t* sP = sV + 2 * S::V_BYTES;           // P_hi, P_lo
  uint64_t* bars = (uint64_t*)(sP + 2 * S::P_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* s_free = bars + 6;
  uint64_t* p_full = bars + 7;
  uint64_t* pv_done = bars + 8;
  uint64_t* drain = bars + 9;
  uint32_t* tmem_slot = (uint32_t*)(bars + 10);

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
  if (p.causal) {
    const int r_last = min(r0 + kAttnRows - 1, rows_total - 1);
    kt1 = min(kt1, (p.L0 + r_last / G) / kAttnKeys + 1);
  }
  const int n_tiles = max(0, kt1 - kt0);
  const int bg = b * p.Hkv + g;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_free), 128);
    mbar_init(smem_u32(p_full), 128);
    mbar_init(smem_u32(pv_done), 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t t_s = tmem_base, t_o = tmem_base + 64;

  if (warp == 0) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- TMA producer ----------------
      const uint32_t qb = smem_u32(q_full);
      mbar_arrive_expect_tx(qb, S::Q_BYTES);
      const int q_row0 = bg * rows_total + r0;
      for (int a = 0; a < S::NA; ++a) tma_load_2d(smem_u32(sQ + a * 16384), &tmQ, qb, a * 64, q_row0);
      int issued = 0;
      for (int i = 0; i < n_tiles; ++i, ++issued) {
        const int s = i & 1;
        if (!mbar_wait(smem_u32(&kv_empty[s]), ((i >> 1) & 1) ^ 1, p.err)) break;
        const uint32_t fb = smem_u32(&kv_full[s]);
        mbar_arrive_expect_tx(fb, S::K_BYTES + S::V_BYTES);
        const int key0 = (kt0 + i) * kAttnKeys;
        for (int a = 0; a < S::NA; ++a)
          tma_load_2d(smem_u32(sK + s * S::K_BYTES + a * kAttnKeys * 128), &tmK, fb, a * 64,
                      bg * p.c_max + key0);
        tma_load_2d(smem_u32(sV + s * S::V_BYTES), &tmV, fb, key0, bg * HD);
      }
      // every issued copy must land before the CTA may exit
      const int first = issued > 2 ? issued - 2 : 0;
      mbar_wait(qb, 0, p.err);
      for (int i = first; i < issued; ++i) mbar_wait(smem_u32(&kv_full[i & 1]), (i >> 1) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0 && n_tiles > 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t id_s = idesc_bf16_f32(128, kAttnKeys);
      const uint32_t id_o = idesc_bf16_f32(128, HD);
      bool ok = mbar_wait(smem_u32(q_full), 0, p.err);
      auto issue_s = [&](int i) -> bool {
        const int s = i & 1;
        if (!mbar_wait(smem_u32(&kv_full[s]), (i >> 1) & 1, p.err)) return false;
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
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int i = 0; i < n_tiles && ok; ++i) {
        if (i + 1 < n_tiles && !issue_s(i + 1)) { ok = false; break; }
        if (!mbar_wait(smem_u32(p_full), i & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t va = smem_u32(sV + (i & 1) * S::V_BYTES);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t pa = smem_u32(sP + part * S::P_BYTES);
#pragma unroll
          for (int k = 0; k < kAttnKeys / 16; ++k)
            umma_bf16(t_o, sdesc_k128(pa + k * 32), sdesc_k128(va + k * 32), id_o,
                      (i > 0 || part > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(pv_done));
        umma_commit(smem_u32(&kv_empty[i & 1]));
      }
      umma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else {
    // ---------------- softmax + epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // tensor-memory lane = query row of the tile
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int r = r0 + row;
    const int t_in = (r < rows_total ? r : rows_total - 1) / G;  // token within the pass
    const int lim = p.causal ? min(kv_len - 1, p.L0 + t_in) : kv_len - 1;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    uint8_t* p_hi = sP;
    uint8_t* p_lo = sP + S::P_BYTES;
    const uint32_t prow = (uint32_t)row * 128;
    // waits are made warp-uniform: tensor-memory loads and stores are
    // warp-collective and must never run in a diverged warp
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), parity, p.err)) != 0;
    };
    for (int i = 0; i < n_tiles && ok; ++i) {
      if (!wait_all(s_full, i & 1)) { ok = false; break; }
      tc_fence_after();
      float sv[kAttnKeys];
#pragma unroll
      for (int c = 0; c < kAttnKeys / 16; ++c) {
        float v[16];
        tmem_ld16(t_s + lane_off + c * 16, v);
#pragma unroll
        for (int e = 0; e < 16; ++e) sv[c * 16 + e] = v[e];
      }
      tc_fence_before();
      mbar_arrive(smem_u32(s_free));
      const int key0 = (kt0 + i) * kAttnKeys;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kAttnKeys; ++c) {
        const float v = key0 + c <= lim ? sv[c] * p.scale_log2 : -INFINITY;
        sv[c] = v;
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m - m_new);
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kAttnKeys; ++c) {
        const float pv = (m_new == -INFINITY) ? 0.f : exp2f(sv[c] - m_new);
        sv[c] = pv;
        sum += pv;
      }
      l = l * alpha + sum;
      m = m_new;
      // P of the previous tile has been consumed and O is up to date
      if (i > 0) {
        if (!wait_all(pv_done, (i - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          for (int c = 0; c < HD / 16; ++c) {
            float v[16];
            tmem_ld16(t_o + lane_off + c * 16, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] *= alpha;
            tmem_st16(t_o + lane_off + c * 16, v);
          }
          tmem_wait_st();
        }
      }
      // P_hi / P_lo rows into the swizzled K-major operand tiles
#pragma unroll
      for (int ch = 0; ch < kAttnKeys / 8; ++ch) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a0 = sv[ch * 8 + 2 * e], a1 = sv[ch * 8 + 2 * e + 1];
          hi[e] = pack_bf16x2(a0, a1);
          lo[e] = pack_bf16x2(a0 - bf16_to_f32(hi[e] & 0xFFFF), a1 - bf16_to_f32(hi[e] >> 16));
        }
        const uint32_t off = prow + (((uint32_t)ch ^ ((uint32_t)row & 7)) << 4);
        *reinterpret_cast<uint4*>(p_hi + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(p_lo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    if (ok && n_tiles > 0) ok = wait_all(pv_done, (n_tiles - 1) & 1);
    tc_fence_after();
    const bool have = ok && n_tiles > 0;  // uniform across the warp
    const bool valid = r < rows_total;
    const int h = g * G + (valid ? r % G : 0);
    const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
    const long long prow_g = (((long long)split * p.B + b) * p.Hq + h) * p.nq + t_in;
    for (int c = 0; c < HD / 16; ++c) {
      float v[16];
      if (have) {
        tmem_ld16(t_o + lane_off + c * 16, v);
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = 0.f;
      }
      if (!valid) continue;
      if (p.splits == 1) {
        uint16_t* dst = p.out + ((long long)(b * p.nq + t_in) * p.Hq + h) * HD + c * 16;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(v[2 * e] * inv, v[2 * e + 1] * inv);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(dst + 8) = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
        float* dst = p.part_o + prow_g * HD + c * 16;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          *reinterpret_cast<float4*>(dst + 4 * e) = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
      }
    }
    if (valid && p.splits > 1) {
      p.part_ml[prow_g * 2] = have ? m : -INFINITY;
      p.part_ml[prow_g * 2 + 1] = have ? l : 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

// Merge split-KV partials (fixed split order) -> bf16 output.  One warp per
// (canvas, head, query) row: the split maxima and sums are read once per row,
// the row's HD values are merged with 16-byte vector loads.
__global__ void attn_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                    uint16_t* __restrict__ out, int splits, int B, int Hq, int nq, int HD) {
  const long long rows = (long long)B * Hq * nq;
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, part_ml[(s * rows + row) * 2]);
  float wgt[8];
  float den = 0.f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    wgt[s] = 0.f;
    if (s < splits) {
      const float ms = part_ml[(s * rows + row) * 2];
      if (ms != -INFINITY) wgt[s] = exp2f(ms - mx);
      den += wgt[s] * part_ml[(s * rows + row) * 2 + 1];
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const int i = (int)(row % nq);
  const long long bh = row / nq;
  const int h = (int)(bh % Hq), b = (int)(bh / Hq);
  uint16_t* dst = out + ((long long)(b * nq + i) * Hq + h) * HD;
  for (int c = lane * 4; c < HD; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < 8; ++s)
      if (s < splits) {
        const float4 v = *reinterpret_cast<const float4*>(part_o + (s * rows + row) * HD + c);
        acc.x += wgt[s] * v.x; acc.y += wgt[s] * v.y; acc.z += wgt[s] * v.z; acc.w += wgt[s] * v.w;
      }
    uint2 o;
    o.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    o.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(dst + c) = o;
  }
}

}  // namespace dg
