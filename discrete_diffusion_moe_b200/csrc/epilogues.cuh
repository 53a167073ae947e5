// epilogues.cuh - per-thread epilogue functors of the tcgen05 GEMM core.
// Each epilogue thread owns one accumulator row (tile row `row`, 0..127) and
// receives its values 16 columns at a time.
#pragma once

#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace dg {

// Transposed store of a weight-stationary product (A = weights, one row per
// output feature; B = tokens): out[t * ld + f] for feature f = a_row0 + row and
// token t = n0 + column.  Consecutive threads write consecutive features, so
// each warp store is one contiguous 128-byte line.
//   mode 0: out  = D           (split k: out + ks * split_stride)
//   mode 1: out += D           (residual add)
//   mode 2: out  = E_emb[tok[t], f] + D   (canvas embedding + self-conditioning)
struct EpiStoreT {
  static constexpr int kEpiWarps = 8;
  float* out;
  long long ld;
  long long split_stride;
  int mode;
  const uint16_t* emb;   // mode 2: [V, ld] bf16
  const int* tokens;     // mode 2: [T]
  int vocab;             // mode 2
  int* err;
  // mode 2: token t goes to row (t / row_group) * row_pitch + row_off + t % row_group
  // (row_group 0: row t)
  int row_group = 0, row_pitch = 0, row_off = 0;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State&) const {
    if (row >= j.m_valid) return;
    const int f = j.m_tile * 128 + row;
    float* base = out + (long long)j.ks * split_stride + f;
    const int nv = j.n_valid - c0;  // valid columns in this chunk (may exceed 16)
    if (mode == 0) {
      // streaming stores (evict-first): the partial products are read once
      if (nv >= 16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) __stcs(base + (long long)(j.n0 + c0 + i) * ld, v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (i < nv) __stcs(base + (long long)(j.n0 + c0 + i) * ld, v[i]);
      }
    } else if (mode == 1) {
      // all loads first: the 16 read-modify-writes then overlap their latency
      float old[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) old[i] = i < nv ? base[(long long)(j.n0 + c0 + i) * ld] : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < nv) base[(long long)(j.n0 + c0 + i) * ld] = old[i] + v[i];
    } else {
      int tok[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) tok[i] = i < nv ? __ldg(tokens + j.n0 + c0 + i) : 0;
      float e[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        int t = tok[i];
        if (t < 0 || t >= vocab) { set_error(err, kDevErrBadToken); t = 0; }
        e[i] = bf16_to_f32(__ldg(emb + (long long)t * ld + f));
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < nv) {
          const int t = j.n0 + c0 + i;
          const long long r = row_group ? (long long)(t / row_group) * row_pitch + row_off + t % row_group : t;
          base[r * ld] = e[i] + v[i];
        }
    }
  }
};

// QKV projection with RoPE and the KV-cache write (the product's final values:
// it runs with the cluster split-k reduction).  A = Wqkv with the rows of every
// q and k head interleaved: head row j (j < hd/2) at physical row 2j and its
// rotation partner j + hd/2 at 2j + 1, so a rotated pair sits in adjacent
// accumulator lanes; v rows in natural order.  B = tokens t of the pass (B
// canvases x nq positions, position L0 + t % nq).  Per pair: the even lane
// outputs x_j cos - x_{j+hd/2} sin, the odd lane x_{j+hd/2} cos + x_j sin,
// rotated in double from the fp32 sums and rounded once to bf16 (the angle's
// (cos, sin) from the pass's table).  q goes to the packed grouped-query
// layout, k to the K cache, v (its bf16 value held in fp16) to the transposed
// V cache, each at the token's position.
struct EpiQKV {
  static constexpr int kEpiWarps = 8;
  const double2* rope;  // [nq][hd / 2] (cos, sin) of positions L0 .. L0 + nq - 1
  uint16_t* q;          // packed queries [B][Hkv][nq][G][hd] bf16
  uint16_t* kc;         // layer base of the K cache [B][Hkv][c_max][hd] bf16
  uint16_t* vc;         // layer base of the V^T cache [B][Hkv][hd][c_max] fp16
  int nq, L0, c_max, Hq, Hkv, hd;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State&) const {
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
    if (row >= j.m_valid) return;
    const int f = j.m_tile * 128 + row;
    const int qk_rows = (Hq + Hkv) * hd;
    const int half = hd >> 1;
    const int G = Hq / Hkv;
    const int nv = min(16, j.n_valid - c0);
    if (f < qk_rows) {
      const int h = f / hd, w = f - h * hd;
      const int jj = w >> 1, odd = w & 1;
      const int dim = jj + odd * half;
      const double sgn = odd ? 1.0 : -1.0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i >= nv) break;
        const int t = j.n0 + c0 + i;
        const int b = t / nq, pos = t - b * nq;
        const double2 cs = __ldg(rope + (long long)pos * half + jj);
        const uint16_t r = f32_to_bf16((float)((double)v[i] * cs.x + sgn * (double)o[i] * cs.y));
        if (h < Hq) {
          const int g = h / G, hh = h - g * G;
          q[((((long long)b * Hkv + g) * nq + pos) * G + hh) * hd + dim] = r;
        } else {
          const int g = h - Hq;
          kc[(((long long)b * Hkv + g) * c_max + L0 + pos) * hd + dim] = r;
        }
      }
    } else {
      const int g = (f - qk_rows) / hd, dim = (f - qk_rows) - g * hd;
      const int t0 = j.n0 + c0;
      const int b0 = t0 / nq, pos0 = t0 - b0 * nq;
      uint16_t hv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) hv[i] = bf16_to_f16(f32_to_bf16(v[i]));  // the bf16 value, held in fp16
      if (nv == 16 && pos0 + 15 < nq && ((L0 + pos0) & 7) == 0) {
        // 16 consecutive positions of one canvas: two 16-byte stores
        uint16_t* dst = vc + (((long long)b0 * Hkv + g) * hd + dim) * c_max + L0 + pos0;
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = (uint32_t)hv[2 * e] | ((uint32_t)hv[2 * e + 1] << 16);
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (i >= nv) break;
          const int t = t0 + i;
          const int b = t / nq, pos = t - b * nq;
          vc[(((long long)b * Hkv + g) * hd + dim) * c_max + L0 + pos] = hv[i];
        }
      }
    }
  }
};

// Grouped gate/up projection with SwiGLU.  The expert's [2 f, d] weight has
// gate row j at 2j and up row j at 2j+1, so the pair sits in adjacent lanes:
// h[slot, j] = bf16(silu(gate) * up) with silu(z) = z / (1 + e^-z).  The two
// lanes of a pair exchange their 16 values, then the even lane finishes the
// chunk's first 8 columns and the odd lane the last 8: every lane works, and
// all 8 activations are computed before any store, so the exponentials and
// divisions of different columns overlap instead of running one column at a
// time behind a branch.
struct EpiSwiGLU {
  static constexpr int kEpiWarps = 8;
  uint16_t* h;   // [rows, f_dim] bf16, rows in expert (permuted) order
  int f_dim;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State&) const {
    const int feat = (j.m_tile * 128 + row) >> 1;
    const bool odd = (row & 1) != 0;
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
    uint16_t r[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float g = odd ? o[q + 8] : v[q];
      const float u = odd ? v[q + 8] : o[q];
      r[q] = f32_to_bf16(__fdividef(g, 1.0f + __expf(-g)) * u);
    }
    if (row < j.m_valid) {
      const int nb = c0 + (odd ? 8 : 0);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (nb + q < j.n_valid) h[(long long)(j.n0 + nb + q) * f_dim + feat] = r[q];
    }
  }
};

// Grouped down projection: y[slot, f] = w[slot] * D (fp32), f = output feature.
struct EpiDown {
  static constexpr int kEpiWarps = 8;
  float* y;
  int d;
  const float* w_slot;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State&) const {
    if (row >= j.m_valid) return;
    const int f = j.m_tile * 128 + row;
    const int nv = j.n_valid - c0;
    float w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = i < nv ? __ldg(w_slot + j.n0 + c0 + i) : 0.f;
    // plain stores: the combine reads y next, from L2
    if (nv >= 16) {
#pragma unroll
      for (int i = 0; i < 16; ++i) y[(long long)(j.n0 + c0 + i) * d + f] = w[i] * v[i];
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i < nv) y[(long long)(j.n0 + c0 + i) * d + f] = w[i] * v[i];
    }
  }
};

// LM head (A = final normalised hidden states, one row per canvas position;
// B = W_lm rows = vocabulary ids).  Stores the logits in bf16 (the expected
// embedding's input; fp32 too when a debug buffer is given) and keeps, per
// position and per vocabulary tile, the online softmax statistics
//   m = max l, Z = sum e^(l - m), S = sum e^(l - m) l,
// the argmax (first maximum) and the Gumbel-max key argmax_v (l_v / T + g_v)
// with g = -ln(-ln u) from Philox (purpose 2, c0 = v / 4, word v % 4).  The
// inner logarithm uses the accurate logf: for u within ~1e-5 of 1, where the
// largest keys come from, the fast __logf has only absolute accuracy.
struct VocabPartials {
  float* m;
  float* z;
  float* s;
  float* amax_v;
  int* amax_i;
  float* gkey_v;
  int* gkey_i;
};

struct EpiLMHead {
  static constexpr int kEpiWarps = 4;
  uint16_t* logits_bf16; // [T, V] bf16: the expected embedding's input (a8)
  float* logits;         // optional [T, V] fp32 (debug output), may be null
  long long V;
  VocabPartials part;    // each [T, n_vt]
  int n_vt;              // vocabulary tiles (V / bn)
  int bn;
  const StepDev* sp;     // round parameters: Philox key, block, step, 1 / T_step
  int canvas;            // positions per canvas (256; 1 in the autoregressive mode)
  uint32_t purpose;      // Philox purpose of the Gumbel draw
  struct State {
    float m, z, s, av, gv;
    int ai, gi;
    uint32_t k0, k1, c2;
    float inv_t;
  };
  __device__ __forceinline__ void begin(const GemmJob&, int, State& st) const {
    st.m = -INFINITY; st.z = 0.f; st.s = 0.f;
    st.av = -INFINITY; st.ai = 0; st.gv = -INFINITY; st.gi = 0;
    st.k0 = sp->k0; st.k1 = sp->k1;
    st.c2 = (uint32_t)(sp->block * 256 + sp->step);
    st.inv_t = sp->inv_t;
  }
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State& st) const {
    if (row >= j.m_valid) return;
    const int t = j.m_tile * 128 + row;
    const int vb = j.n0 + c0;  // first vocabulary id of this chunk (multiple of 16)
    {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
      uint4* dst = reinterpret_cast<uint4*>(logits_bf16 + (long long)t * V + vb);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
    if (logits) {
      float4* dst = reinterpret_cast<float4*>(logits + (long long)t * V + vb);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }

    float cm = v[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) cm = fmaxf(cm, v[i]);
    if (cm > st.m) {
      const float sc = __expf(st.m - cm);  // 0 when st.m = -inf
      st.z *= sc;
      st.s *= sc;
      st.m = cm;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float e = __expf(v[i] - st.m);
      st.z += e;
      st.s = fmaf(e, v[i], st.s);
      if (v[i] > st.av) { st.av = v[i]; st.ai = vb + i; }
    }
    const int b = t / canvas, pos = t - b * canvas;
    const uint32_t c3 = (purpose << 24) | (uint32_t)b;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const Philox4 r = philox4x32_10((uint32_t)(vb >> 2) + q, (uint32_t)pos, st.c2, c3, st.k0, st.k1);
      const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float u = gumbel_u(w[e]);
        // -ln(u) needs relative accuracy for u near 1 (the largest Gumbel keys,
        // which decide the sample): the accurate logf there, the fast one outside
        const float g = -__logf(-logf(u));
        const float key = __fadd_rn(__fmul_rn(v[4 * q + e], st.inv_t), g);
        if (key > st.gv) { st.gv = key; st.gi = vb + 4 * q + e; }
      }
    }
  }
  __device__ __forceinline__ void end(const GemmJob& j, int row, State& st) const {
    if (row >= j.m_valid) return;
    const int t = j.m_tile * 128 + row;
    const long long idx = (long long)t * n_vt + j.n0 / bn;
    part.m[idx] = st.m;
    part.z[idx] = st.z;
    part.s[idx] = st.s;
    part.amax_v[idx] = st.av;
    part.amax_i[idx] = st.ai;
    part.gkey_v[idx] = st.gv;
    part.gkey_i[idx] = st.gi;
  }
};

// Plain row-major store D[m, n] -> out[m * ld + n] (the GEMM test hook).
struct EpiStoreRows {
  static constexpr int kEpiWarps = 8;
  float* out;
  long long ld;
  struct State {};
  __device__ __forceinline__ void begin(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void end(const GemmJob&, int, State&) const {}
  __device__ __forceinline__ void chunk(const GemmJob& j, int row, int c0, const float (&v)[16],
                                        State&) const {
    if (row >= j.m_valid) return;
    const long long m = (long long)j.m_tile * 128 + row;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (c0 + i < j.n_valid) out[m * ld + j.n0 + c0 + i] = v[i];
  }
};

}  // namespace dg
