// attention.cuh - attention of one pass of queries over the context KV cache
// plus the pass's own keys (already written into the cache at positions
// L0 .. L0 + nq - 1).
//
//   canvas pass (causal = 0): every query sees keys [0, L0 + nq)   (no mask:
//     bidirectional over the canvas, full view of the context)
//   context encoding (causal = 1): query i sees keys [0, L0 + i]
//
// Grouped-query layout: the G = Hq / Hkv query heads sharing kv head g are
// packed into G * nq rows, so one CTA's 64-row tile reuses each K/V tile for
// all heads of the group.  Flash-style online softmax in the exp2 domain;
// QK^T and PV run on bf16 mma.sync tensor-core instructions (m16n8k16, fp32
// accumulate).  The probabilities are split into a bf16 high part and a bf16
// residual (P = P_hi + P_lo, two PV products), so the PV operand carries about
// 16 significant bits instead of 8: the attention output of a long, nearly
// uniform softmax is a heavily cancelling average, and plain bf16 P would put
// a relative error of order 2^-9 on it.  Keys can be split across CTAs
// (split-KV); partial (m, l, O) are merged in a fixed order.
#pragma once

#include "common.cuh"

namespace dg {

struct AttnParams {
  const uint16_t* q;   // [B * nq, Hq * HD]
  const uint16_t* kc;  // this layer's K cache [B][Hkv][c_max][HD]
  const uint16_t* vc;
  uint16_t* out;       // [B * nq, Hq * HD]   (splits == 1)
  float* part_o;       // [splits][B][Hq][nq][HD]  (splits > 1, unnormalised)
  float* part_ml;      // [splits][B][Hq][nq][2]   (running max (log2 units), sum)
  int B, nq, L0, c_max, Hq, Hkv, splits, causal;
  float scale_log2;    // log2(e) / sqrt(HD)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int HD>
constexpr int attn_smem_bytes() {
  return (64 + 4 * 64) * (HD + 8) * 2;
}

template <int HD>
__global__ void __launch_bounds__(128) attn_kernel(const AttnParams p) {
  constexpr int LD = HD + 8;   // padded smem row (elements): conflict-free ldmatrix
  constexpr int NT = HD / 8;   // 8-wide dim tiles of O
  constexpr int KS = HD / 16;  // k steps of QK^T
  constexpr int CH = HD / 8;   // 16-byte chunks per row
  extern __shared__ __align__(16) uint16_t asmem[];
  uint16_t* sQ = asmem;
  uint16_t* sK = asmem + 64 * LD;
  uint16_t* sV = sK + 2 * 64 * LD;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int rows_total = G * p.nq;
  const int r0 = blockIdx.x * 64;
  const int g = blockIdx.y;
  const int b = blockIdx.z / p.splits, split = blockIdx.z - b * p.splits;
  const int kv_len = p.L0 + p.nq;
  const int n_kt = (kv_len + 63) / 64;
  const int kt0 = (int)((long long)n_kt * split / p.splits);
  int kt1 = (int)((long long)n_kt * (split + 1) / p.splits);
  if (p.causal) {
    const int r_last = min(r0 + 63, rows_total - 1);
    const int max_i = (r0 / p.nq == r_last / p.nq) ? (r_last % p.nq) : (p.nq - 1);
    kt1 = min(kt1, (p.L0 + max_i) / 64 + 1);
  }
  const uint16_t* kbase = p.kc + ((long long)b * p.Hkv + g) * p.c_max * HD;
  const uint16_t* vbase = p.vc + ((long long)b * p.Hkv + g) * p.c_max * HD;

  // Q tile
  for (int c = threadIdx.x; c < 64 * CH; c += 128) {
    const int row = c / CH, col = c - row * CH;
    const int r = r0 + row;
    const bool ok = r < rows_total;
    const int h = g * G + (ok ? r / p.nq : 0), i = ok ? r % p.nq : 0;
    const uint16_t* src = p.q + ((long long)(b * p.nq + i) * p.Hq + h) * HD + col * 8;
    cp_async16(smem_u32(sQ + row * LD + col * 8), src, ok);
  }
  auto load_kv = [&](int kt, int buf) {
    uint16_t* dk = sK + buf * 64 * LD;
    uint16_t* dv = sV + buf * 64 * LD;
    for (int c = threadIdx.x; c < 64 * CH; c += 128) {
      const int row = c / CH, col = c - row * CH;
      const int key = kt * 64 + row;
      const bool ok = key < kv_len;
      const long long off = (long long)(ok ? key : 0) * HD + col * 8;
      cp_async16(smem_u32(dk + row * LD + col * 8), kbase + off, ok);
      cp_async16(smem_u32(dv + row * LD + col * 8), vbase + off, ok);
    }
  };
  if (kt0 < kt1) load_kv(kt0, 0);
  cp_async_commit();

  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  // query position (within the pass) of this thread's two rows
  int qi[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = r0 + warp * 16 + (lane >> 2) + rr * 8;
    qi[rr] = r < rows_total ? r % p.nq : p.nq - 1;
  }

  for (int kt = kt0; kt < kt1; ++kt) {
    const int buf = (kt - kt0) & 1;
    if (kt + 1 < kt1) {
      load_kv(kt + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint16_t* cK = sK + buf * 64 * LD;
    const uint16_t* cV = sV + buf * 64 * LD;

    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(smem_u32(sQ + (warp * 16 + (lane & 15)) * LD + ks * 16 + (lane >> 4) * 8), a0, a1, a2, a3);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(cK + (np * 16 + (lane & 7) + ((lane >> 4) << 3)) * LD + ks * 16 +
                         ((lane >> 3) & 1) * 8),
                b0, b1, b2, b3);
        mma_bf16_16816(s[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(s[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // scale, mask, online softmax (per row: 4 threads share a row)
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int lim = p.causal ? min(kv_len - 1, p.L0 + qi[rr]) : kv_len - 1;
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int key = kt * 64 + n * 8 + (lane & 3) * 2 + c;
          float v = s[n][rr * 2 + c] * p.scale_log2;
          v = key <= lim ? v : -INFINITY;
          s[n][rr * 2 + c] = v;
          mx = fmaxf(mx, v);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[rr], mx);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_r[rr] - m_new);
      m_r[rr] = m_new;
      l_r[rr] *= alpha;
#pragma unroll
      for (int n = 0; n < NT; ++n) { o[n][rr * 2] *= alpha; o[n][rr * 2 + 1] *= alpha; }
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float v = s[n][rr * 2 + c];
          const float pv = (m_new == -INFINITY) ? 0.f : exp2f(v - m_new);
          s[n][rr * 2 + c] = pv;
          l_r[rr] += pv;
        }
    }
    // O += (P_hi + P_lo) V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t hi[4], lo[4];
      const float* pr[4] = {&s[2 * kk][0], &s[2 * kk][2], &s[2 * kk + 1][0], &s[2 * kk + 1][2]};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float p0 = pr[r][0], p1 = pr[r][1];
        hi[r] = pack_bf16x2(p0, p1);
        const float h0 = bf16_to_f32(hi[r] & 0xFFFF), h1 = bf16_to_f32(hi[r] >> 16);
        lo[r] = pack_bf16x2(p0 - h0, p1 - h1);
      }
#pragma unroll
      for (int dp = 0; dp < NT / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(cV + (kk * 16 + (lane & 15)) * LD + dp * 16 + (lane >> 4) * 8), b0, b1, b2, b3);
        mma_bf16_16816(o[2 * dp], hi[0], hi[1], hi[2], hi[3], b0, b1);
        mma_bf16_16816(o[2 * dp + 1], hi[0], hi[1], hi[2], hi[3], b2, b3);
        mma_bf16_16816(o[2 * dp], lo[0], lo[1], lo[2], lo[3], b0, b1);
        mma_bf16_16816(o[2 * dp + 1], lo[0], lo[1], lo[2], lo[3], b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    float l = l_r[rr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int r = r0 + warp * 16 + (lane >> 2) + rr * 8;
    if (r >= rows_total) continue;
    const int h = g * G + r / p.nq, i = r % p.nq;
    if (p.splits == 1) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* dst = p.out + ((long long)(b * p.nq + i) * p.Hq + h) * HD + (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<uint32_t*>(dst + n * 8) = pack_bf16x2(o[n][rr * 2] * inv, o[n][rr * 2 + 1] * inv);
    } else {
      const long long row = (((long long)split * p.B + b) * p.Hq + h) * p.nq + i;
      float* dst = p.part_o + row * HD + (lane & 3) * 2;
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(dst + n * 8) = make_float2(o[n][rr * 2], o[n][rr * 2 + 1]);
      if ((lane & 3) == 0) {
        p.part_ml[row * 2] = m_r[rr];
        p.part_ml[row * 2 + 1] = l;
      }
    }
  }
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
