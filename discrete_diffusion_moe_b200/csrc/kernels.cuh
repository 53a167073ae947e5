// kernels.cuh - bandwidth-bound kernels of the denoising step: embedding,
// RMSNorm, RoPE + KV write, router top-k, token permutation, expert combine,
// vocabulary statistics merge, softmax probabilities, split-k reduction of
// the expected embedding, the canvas update (entropy / lock / stop /
// re-noise) and canvas initialisation.  All reductions that carry results
// run in a fixed order (no atomics on values), so results are deterministic.
#pragma once

#include "common.cuh"

namespace dg {

// ---------------------------------------------------------------------------
// a1: x[t, :] = E_emb[tok[t], :]   (fp32 residual stream)
__global__ void embed_kernel(const uint16_t* __restrict__ emb, const int* __restrict__ tokens,
                             float* __restrict__ x, int T, int d, int vocab, int* err) {
  const int t = blockIdx.x;
  if (t >= T) return;
  int tok = tokens[t];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) set_error(err, kDevErrBadToken);
    tok = 0;
  }
  const uint16_t* src = emb + (long long)tok * d;
  float* dst = x + (long long)t * d;
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(src + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float4 a, b;
    a.x = bf16_to_f32(w[0] & 0xFFFF); a.y = bf16_to_f32(w[0] >> 16);
    a.z = bf16_to_f32(w[1] & 0xFFFF); a.w = bf16_to_f32(w[1] >> 16);
    b.x = bf16_to_f32(w[2] & 0xFFFF); b.y = bf16_to_f32(w[2] >> 16);
    b.z = bf16_to_f32(w[3] & 0xFFFF); b.w = bf16_to_f32(w[3] >> 16);
    *reinterpret_cast<float4*>(dst + c) = a;
    *reinterpret_cast<float4*>(dst + c + 4) = b;
  }
}

// ---------------------------------------------------------------------------
// RMSNorm: y = bf16(x / sqrt(mean(x^2) + eps) * g), one CTA per row.
template <int THREADS>
__global__ void __launch_bounds__(THREADS) rmsnorm_kernel(const float* __restrict__ x,
                                                          const uint16_t* __restrict__ gain,
                                                          uint16_t* __restrict__ y, int d, float eps) {
  const int t = blockIdx.x;
  const float* xr = x + (long long)t * d;
  float ss = 0.f;
  for (int c = threadIdx.x * 4; c < d; c += THREADS * 4) {
    const float4 v = *reinterpret_cast<const float4*>(xr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  __shared__ float red[THREADS / 32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < THREADS / 32; ++w) tot += red[w];
  const float r = rsqrtf(tot / (float)d + eps);
  uint16_t* yr = y + (long long)t * d;
  for (int c = threadIdx.x * 4; c < d; c += THREADS * 4) {
    const float4 v = *reinterpret_cast<const float4*>(xr + c);
    const uint2 gg = *reinterpret_cast<const uint2*>(gain + c);
    uint2 o;
    o.x = pack_bf16x2(v.x * r * bf16_to_f32(gg.x & 0xFFFF), v.y * r * bf16_to_f32(gg.x >> 16));
    o.y = pack_bf16x2(v.z * r * bf16_to_f32(gg.y & 0xFFFF), v.w * r * bf16_to_f32(gg.y >> 16));
    *reinterpret_cast<uint2*>(yr + c) = o;
  }
}

// ---------------------------------------------------------------------------
// x[t, :] += sum_s part[s, t, :] (split-k partials of the output projection, in
// split order), then xn = bf16(x / rms(x) * gain).  One CTA per token with
// one float4 of the row per thread (NV per thread when the row is longer than
// 4096): every load of the row is in flight at once and all tokens' CTAs are
// resident together; the row stays in registers between the two passes.
template <int NV>
__global__ void __launch_bounds__(1024) residual_norm_kernel(float* __restrict__ x, const float* __restrict__ part,
                                                             int ks, long long split_stride, int d,
                                                             const uint16_t* __restrict__ gain,
                                                             uint16_t* __restrict__ xn, float eps) {
  const int t = blockIdx.x;
  const int nt = blockDim.x;
  float* xr = x + (long long)t * d;
  float4 r[NV];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (q * nt + threadIdx.x) * 4;
    r[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c < d) {
      const float* pp = part + (long long)t * d + c;
      float4 sum = *reinterpret_cast<const float4*>(pp);
      for (int sp = 1; sp < ks; ++sp) {
        const float4 v = *reinterpret_cast<const float4*>(pp + sp * split_stride);
        sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
      }
      float4 acc = *reinterpret_cast<const float4*>(xr + c);
      acc.x += sum.x; acc.y += sum.y; acc.z += sum.z; acc.w += sum.w;
      *reinterpret_cast<float4*>(xr + c) = acc;
      r[q] = acc;
      ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
    }
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (nt >> 5); ++w) tot += red[w];
  const float rs = rsqrtf(tot / (float)d + eps);
  uint16_t* yr = xn + (long long)t * d;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (q * nt + threadIdx.x) * 4;
    if (c < d) {
      const uint2 gg = *reinterpret_cast<const uint2*>(gain + c);
      uint2 o;
      o.x = pack_bf16x2(r[q].x * rs * bf16_to_f32(gg.x & 0xFFFF), r[q].y * rs * bf16_to_f32(gg.x >> 16));
      o.y = pack_bf16x2(r[q].z * rs * bf16_to_f32(gg.y & 0xFFFF), r[q].w * rs * bf16_to_f32(gg.y >> 16));
      *reinterpret_cast<uint2*>(yr + c) = o;
    }
  }
}

// Threads and float4s per thread of the one-CTA-per-row kernels for a row of
// d floats (d a multiple of 4).
struct RowLaunch {
  int threads, nv;
};
inline RowLaunch row_launch(int d) {
  const int n4 = d / 4;
  const int nv = n4 <= 1024 ? 1 : (n4 <= 2048 ? 2 : 4);
  const int per = (n4 + nv - 1) / nv;
  return {(per + 31) / 32 * 32, nv};
}

// ---------------------------------------------------------------------------
// RoPE: pairs (i, i + hd/2) rotated by the angle pos * theta^(-2i/hd).  The
// cos/sin of each (position, pair) are computed once per pass in double
// (rope_table_kernel) and shared by all layers; the rotation is done in
// double from the fp32 projection and rounded once to bf16.
// q -> bf16 [T, Hq*hd]; k, v -> bf16 KV cache of this layer at position
// L0 + i of each canvas ([B][Hkv][c_max][hd]).
__global__ void rope_table_kernel(double2* __restrict__ tab, int nq, int L0, int half, int hd, double theta) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nq * half) return;
  const int pos_in = e / half, i = e - pos_in * half;
  const double inv_freq = pow(theta, -2.0 * (double)i / (double)hd);
  double sn, cs;
  sincos((double)(L0 + pos_in) * inv_freq, &sn, &cs);
  tab[e] = make_double2(cs, sn);
}

struct RopeParams {
  const float* qkv;   // [ks][T, (Hq + 2 Hkv) * hd] split-k partial products (summed in order)
  int ks;
  long long split_stride;
  const double2* tab; // [nq, hd/2] (cos, sin)
  uint16_t* q;        // packed queries [B][Hkv][nq][G][hd], G = Hq / Hkv
  uint16_t* kc;       // layer base of K cache   [B][Hkv][c_max][hd]
  uint16_t* vc;       // layer base of V^T cache [B][Hkv][hd][c_max] (fp16 holding the bf16 values)
  int T, nq, L0, c_max, Hq, Hkv, hd;
  int v_blocks;       // blocks [0, v_blocks) transpose v; the rest rotate q and k
};

constexpr int kRopeVTok = 16;          // tokens per v-transpose block
constexpr int kRopeHeadsPerBlock = 32; // q / k heads rotated per block

// Blocks [v_blocks, ...): one block per (token, group of up to 32 heads) rotates its
// q heads (into the packed grouped-query layout) and k heads (into the
// cache), one thread per rotated pair, the split-k partials summed in order.
// Blocks [0, v_blocks) (scheduled first: they are the long ones): one block per
// (canvas, kv head, 16 tokens) copies v into the transposed cache through
// shared memory, so both the reads (along the head dimension) and the writes
// (along positions) are contiguous; every thread issues the loads of several
// elements before it uses them, so the block is not a chain of dependent
// loads.
__global__ void __launch_bounds__(256) rope_kv_kernel(const RopeParams p) {
  const int half = p.hd / 2;
  const int row_w = (p.Hq + 2 * p.Hkv) * p.hd;
  const int parts = (p.Hq + p.Hkv + kRopeHeadsPerBlock - 1) / kRopeHeadsPerBlock;
  const int rot_blk = (int)blockIdx.x - p.v_blocks;
  if (rot_blk >= 0) {
    const int t = rot_blk / parts, part = rot_blk - t * parts;
    const int G = p.Hq / p.Hkv;
    const int b = t / p.nq, pos_in = t - b * p.nq;
    const int h0 = part * kRopeHeadsPerBlock;
    const int n_pairs = (min(p.Hq + p.Hkv, h0 + kRopeHeadsPerBlock) - h0) * half;
    const float* row = p.qkv + (long long)t * row_w;
    const double2* tab = p.tab + (long long)pos_in * half;
#pragma unroll 2
    for (int j = threadIdx.x; j < n_pairs; j += blockDim.x) {
      const int h = h0 + j / half, i = j - (h - h0) * half;
      const float* src = row + h * p.hd + i;
      float a1 = src[0], a2 = src[half];
      for (int q = 1; q < p.ks; ++q) { a1 += src[q * p.split_stride]; a2 += src[q * p.split_stride + half]; }
      const double2 cs = tab[i];
      const double x1 = a1, x2 = a2;
      const float o1 = (float)(x1 * cs.x - x2 * cs.y), o2 = (float)(x2 * cs.x + x1 * cs.y);
      uint16_t* dst;
      if (h < p.Hq) {
        const int g = h / G, hh = h - g * G;
        dst = p.q + ((((long long)b * p.Hkv + g) * p.nq + pos_in) * G + hh) * p.hd;
      } else {
        const int g = h - p.Hq;
        dst = p.kc + (((long long)b * p.Hkv + g) * p.c_max + p.L0 + pos_in) * p.hd;
      }
      dst[i] = f32_to_bf16(o1);
      dst[i + half] = f32_to_bf16(o2);
    }
  } else {
    __shared__ uint16_t tile[kRopeVTok * 256];  // [token][dim], hd <= 256
    const int tiles_per_seq = (p.nq + kRopeVTok - 1) / kRopeVTok;
    int blk = (int)blockIdx.x;
    const int tt = blk % tiles_per_seq;
    blk /= tiles_per_seq;
    const int g = blk % p.Hkv, b = blk / p.Hkv;
    const int pos0 = tt * kRopeVTok;
    const int ntok = min(kRopeVTok, p.nq - pos0);
    const int n = ntok * p.hd;
    const float* base = p.qkv + (long long)(b * p.nq + pos0) * row_w + (p.Hq + p.Hkv + g) * p.hd;
    constexpr int kPer = (kRopeVTok * 256 + 255) / 256;  // elements per thread at most
    float a[kPer];
    int off[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = threadIdx.x + u * 256;
      const int tok = e / p.hd, dim = e - tok * p.hd;
      off[u] = tok * row_w + dim;
      a[u] = e < n ? base[off[u]] : 0.f;
    }
    for (int q = 1; q < p.ks; ++q) {
#pragma unroll
      for (int u = 0; u < kPer; ++u)
        if (threadIdx.x + u * 256 < n) a[u] += base[q * p.split_stride + off[u]];
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = threadIdx.x + u * 256;
      if (e < n) tile[e] = bf16_to_f16(f32_to_bf16(a[u]));  // e = tok * hd + dim; the bf16 value, held in fp16
    }
    __syncthreads();
    uint16_t* dst = p.vc + ((long long)b * p.Hkv + g) * p.hd * p.c_max + p.L0 + pos0;
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const int dim = e / ntok, tok = e - dim * ntok;
      dst[(long long)dim * p.c_max + tok] = tile[tok * p.hd + dim];
    }
  }
}

// ---------------------------------------------------------------------------
// Router: sum the split-k partial logits (fixed order), pick the top-k
// experts by logit (ties to the lower id), softmax over the chosen k.
// One warp per token; E <= 256.
template <int KS>
__global__ void router_topk_kernel(const float* __restrict__ part, int T, int E, int k,
                                   int* __restrict__ idx, float* __restrict__ w,
                                   int* __restrict__ dbg_idx, float* __restrict__ dbg_w,
                                   float* __restrict__ dbg_logits) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  const int t = warp;
  float l[8];
  bool taken[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) { l[q] = 0.f; taken[q] = false; }
  // split-k partials summed in split order; the 8 expert slots of a lane are
  // independent, so their loads are issued together
#pragma unroll
  for (int p = 0; p < KS; ++p) {
    const float* row = part + ((long long)p * T + t) * E;
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = (lane + 32 * q < E) ? row[lane + 32 * q] : 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) l[q] += v[q];
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (lane + 32 * q >= E) l[q] = -INFINITY;
    else if (dbg_logits) dbg_logits[(long long)t * E + lane + 32 * q] = l[q];
  }
  float sel_l[8];
  int sel_e[8];
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = lane + 32 * q;
      if (e < E && !taken[q] && (l[q] > bv || (l[q] == bv && e < be))) { bv = l[q]; be = e; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (lane + 32 * q == be) taken[q] = true;
    sel_l[r] = bv;
    sel_e[r] = be;
  }
  if (lane == 0) {
    float den = 0.f;
    float ex[8];
    for (int r = 0; r < k; ++r) { ex[r] = expf(sel_l[r] - sel_l[0]); den += ex[r]; }
    for (int r = 0; r < k; ++r) {
      idx[t * k + r] = sel_e[r];
      w[t * k + r] = ex[r] / den;
      if (dbg_idx) dbg_idx[t * k + r] = sel_e[r];
      if (dbg_w) dbg_w[t * k + r] = ex[r] / den;
    }
  }
}

// ---------------------------------------------------------------------------
// Token permutation: stable counting sort of the T*k (token, slot) pairs by
// expert.  One CTA of 1024 threads.  Outputs off[E+1], perm[slot] = pair,
// inv[pair] = slot, w_perm[slot] = w[pair].  Within an expert, pairs keep
// ascending pair order (token-major), so the layout is deterministic.
constexpr int kPermThreads = 1024;
__global__ void __launch_bounds__(kPermThreads) permute_kernel(const int* __restrict__ idx,
                                                               const float* __restrict__ w, int P,
                                                               int E, int bn, int* __restrict__ off,
                                                               int* __restrict__ chunk_off,
                                                               int* __restrict__ perm,
                                                               int* __restrict__ inv,
                                                               float* __restrict__ w_perm, int* err) {
  extern __shared__ int sm[];
  int* cnt = sm;                    // [E]
  int* base = sm + E;               // [E] running base within expert
  int* wcnt = sm + 2 * E;           // [32 warps][E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  __syncthreads();
  for (int q = tid; q < P; q += kPermThreads) {
    int e = idx[q];
    if (e < 0 || e >= E) { set_error(err, kDevErrBadToken); e = 0; }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (warp == 0) {
    // exclusive scans of the counts and chunk counts, 8 experts per lane (E <= 256)
    int c8[8], k8[8], sc = 0, sk = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      c8[j] = e < E ? cnt[e] : 0;
      k8[j] = (c8[j] + bn - 1) / bn;
      sc += c8[j];
      sk += k8[j];
    }
    int ic = sc, ik = sk;  // inclusive lane sums
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, ic, o), b2 = __shfl_up_sync(0xffffffffu, ik, o);
      if (lane >= o) { ic += a; ik += b2; }
    }
    int pc = ic - sc, pk = ik - sk;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) { off[e] = pc; base[e] = pc; chunk_off[e] = pk; }
      pc += c8[j];
      pk += k8[j];
    }
    if (lane == 31) { off[E] = ic; chunk_off[E] = ik; }
  }
  __syncthreads();
  for (int c0 = 0; c0 < P; c0 += kPermThreads) {
    const int q = c0 + tid;
    int e = -1;
    if (q < P) { e = idx[q]; if (e < 0 || e >= E) e = 0; }
    for (int i = tid; i < 32 * E; i += kPermThreads) wcnt[i] = 0;
    __syncthreads();
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_in_warp = __popc(peers & ((1u << lane) - 1));
    if (e >= 0 && rank_in_warp == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    // exclusive scan over warps per expert (fixed order), then advance bases
    for (int ee = tid; ee < E; ee += kPermThreads) {
      int acc = base[ee];
      for (int wv = 0; wv < 32; ++wv) {
        const int c = wcnt[wv * E + ee];
        wcnt[wv * E + ee] = acc;
        acc += c;
      }
      base[ee] = acc;
    }
    __syncthreads();
    if (e >= 0) {
      const int slot = wcnt[warp * E + e] + rank_in_warp;
      perm[slot] = q;
      inv[q] = slot;
      w_perm[slot] = w[q];
    }
    __syncthreads();
  }
}

// chunk_off[g] = sum_{h < g} ceil((off[h+1] - off[h]) / bn)  (one thread)
__global__ void chunk_offsets_kernel(const int* __restrict__ off, int G, int bn, int* __restrict__ chunk_off) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int acc = 0;
  for (int g = 0; g < G; ++g) {
    chunk_off[g] = acc;
    const int n = off[g + 1] - off[g];
    acc += n > 0 ? (n + bn - 1) / bn : 0;
  }
  chunk_off[G] = acc;
}

// X_perm[slot, :] = xn[perm[slot] / k, :]  (bf16 rows, 16-byte vectors)
__global__ void gather_rows_kernel(const uint16_t* __restrict__ xn, const int* __restrict__ perm,
                                   uint16_t* __restrict__ xp, int P, int k, int d) {
  const int slot = blockIdx.x;
  if (slot >= P) return;
  const int t = perm[slot] / k;
  const uint4* src = reinterpret_cast<const uint4*>(xn + (long long)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xp + (long long)slot * d);
  for (int c = threadIdx.x; c < d / 8; c += blockDim.x) dst[c] = src[c];
}

// Mixture-of-experts combine + residual, fused with the next RMSNorm:
// x[t, :] += sum_{j < k} y[inv[t, j], :] (the expert outputs already carry
// their routing weights; fixed order j = 0..k-1), then, when xn is given,
// xn = bf16(x / rms(x) * gain).  One CTA per token, one float4 of the row per
// thread (NV when the row is longer than 4096).
template <int NV>
__global__ void __launch_bounds__(1024) moe_combine_norm_kernel(float* __restrict__ x, const float* __restrict__ y,
                                                                const int* __restrict__ inv, int T, int k, int d,
                                                                const uint16_t* __restrict__ gain,
                                                                uint16_t* __restrict__ xn, float eps) {
  const int t = blockIdx.x;
  if (t >= T) return;
  const int nt = blockDim.x;
  int slots[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) slots[j] = j < k ? inv[t * k + j] : 0;
  float* xr = x + (long long)t * d;
  float4 r[NV];
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (q * nt + threadIdx.x) * 4;
    r[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (c < d) {
      float4 acc = *reinterpret_cast<const float4*>(xr + c);
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k) v[j] = *reinterpret_cast<const float4*>(y + (long long)slots[j] * d + c);
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k) { sum.x += v[j].x; sum.y += v[j].y; sum.z += v[j].z; sum.w += v[j].w; }
      acc.x += sum.x; acc.y += sum.y; acc.z += sum.z; acc.w += sum.w;
      *reinterpret_cast<float4*>(xr + c) = acc;
      r[q] = acc;
      ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
    }
  }
  if (!xn) return;
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (nt >> 5); ++w) tot += red[w];
  const float rs = rsqrtf(tot / (float)d + eps);
  uint16_t* yr = xn + (long long)t * d;
#pragma unroll
  for (int q = 0; q < NV; ++q) {
    const int c = (q * nt + threadIdx.x) * 4;
    if (c < d) {
      const uint2 gg = *reinterpret_cast<const uint2*>(gain + c);
      uint2 o;
      o.x = pack_bf16x2(r[q].x * rs * bf16_to_f32(gg.x & 0xFFFF), r[q].y * rs * bf16_to_f32(gg.x >> 16));
      o.y = pack_bf16x2(r[q].z * rs * bf16_to_f32(gg.y & 0xFFFF), r[q].w * rs * bf16_to_f32(gg.y >> 16));
      *reinterpret_cast<uint2*>(yr + c) = o;
    }
  }
}

// ---------------------------------------------------------------------------
// Merge the per-tile vocabulary statistics of each position (fixed order:
// lane l folds tiles l, l+32, ...; then a fixed shuffle tree), in double.
// Writes m, 1/Z, entropy H = m + ln Z - S/Z (clamped to [0, ln V]), pmax = 1/Z,
// argmax and Gumbel sample.
struct PosStats {
  float* m;
  float* inv_z;
  float* entropy;
  float* pmax;
  int* argmax;
  int* sample;
};

__device__ __forceinline__ void merge_ms(double& m, double& z, double& s, double m2, double z2,
                                         double s2) {
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) { m = m2; z = z2; s = s2; return; }
  const double mn = fmax(m, m2);
  const double a = exp(m - mn), b = exp(m2 - mn);
  z = z * a + z2 * b;
  s = s * a + s2 * b;
  m = mn;
}

constexpr int kMergeThreads = 256;
// One CTA per position: thread i folds tiles i, i + 256, ... in order, then a
// fixed binary tree over the 256 partial states (shared memory) in double.
__global__ void __launch_bounds__(kMergeThreads) vocab_merge_kernel(
    const float* __restrict__ pm, const float* __restrict__ pz, const float* __restrict__ ps,
    const float* __restrict__ pav, const int* __restrict__ pai, const float* __restrict__ pgv,
    const int* __restrict__ pgi, int n_vt, int T, double log_v, PosStats out) {
  __shared__ double sm_m[kMergeThreads], sm_z[kMergeThreads], sm_s[kMergeThreads];
  __shared__ float sa_v[kMergeThreads], sg_v[kMergeThreads];
  __shared__ int sa_i[kMergeThreads], sg_i[kMergeThreads];
  const int t = blockIdx.x, tid = threadIdx.x;
  if (t >= T) return;
  const long long base = (long long)t * n_vt;
  double m = -INFINITY, z = 0.0, s_ = 0.0;
  float av = -INFINITY, gv = -INFINITY;
  int ai = 0x7fffffff, gi = 0x7fffffff;
  for (int v = tid; v < n_vt; v += kMergeThreads) {
    merge_ms(m, z, s_, (double)pm[base + v], (double)pz[base + v], (double)ps[base + v]);
    const float a = pav[base + v];
    const int a_i = pai[base + v];
    if (a > av || (a == av && a_i < ai)) { av = a; ai = a_i; }
    const float g = pgv[base + v];
    const int g_i = pgi[base + v];
    if (g > gv || (g == gv && g_i < gi)) { gv = g; gi = g_i; }
  }
  sm_m[tid] = m; sm_z[tid] = z; sm_s[tid] = s_;
  sa_v[tid] = av; sa_i[tid] = ai; sg_v[tid] = gv; sg_i[tid] = gi;
  __syncthreads();
  for (int h = kMergeThreads / 2; h > 0; h >>= 1) {
    if (tid < h) {
      double mm = sm_m[tid], zz = sm_z[tid], ss = sm_s[tid];
      merge_ms(mm, zz, ss, sm_m[tid + h], sm_z[tid + h], sm_s[tid + h]);
      sm_m[tid] = mm; sm_z[tid] = zz; sm_s[tid] = ss;
      if (sa_v[tid + h] > sa_v[tid] || (sa_v[tid + h] == sa_v[tid] && sa_i[tid + h] < sa_i[tid])) {
        sa_v[tid] = sa_v[tid + h]; sa_i[tid] = sa_i[tid + h];
      }
      if (sg_v[tid + h] > sg_v[tid] || (sg_v[tid + h] == sg_v[tid] && sg_i[tid + h] < sg_i[tid])) {
        sg_v[tid] = sg_v[tid + h]; sg_i[tid] = sg_i[tid + h];
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    const double mm = sm_m[0], zz = sm_z[0], ss = sm_s[0];
    double H = mm + log(zz) - ss / zz;
    H = fmin(fmax(H, 0.0), log_v);
    out.m[t] = (float)mm;
    out.inv_z[t] = (float)(1.0 / zz);
    out.entropy[t] = (float)H;
    out.pmax[t] = (float)(1.0 / zz);
    out.argmax[t] = sa_i[0];
    out.sample[t] = sg_i[0];
  }
}

// p[t, v] = bf16(exp(l[t, v] - m_t) / Z_t) — the softmax operand of the
// expected-embedding product.
__global__ void probs_kernel(const float* __restrict__ logits, const float* __restrict__ m,
                             const float* __restrict__ inv_z, uint16_t* __restrict__ p, int T,
                             long long V) {
  const long long n4 = (long long)T * V / 4;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n4;
       e += (long long)gridDim.x * blockDim.x) {
    const long long t = (e * 4) / V;
    const float mm = m[t], iz = inv_z[t];
    const float4 l = reinterpret_cast<const float4*>(logits)[e];
    uint2 o;
    o.x = pack_bf16x2(__expf(l.x - mm) * iz, __expf(l.y - mm) * iz);
    o.y = pack_bf16x2(__expf(l.z - mm) * iz, __expf(l.w - mm) * iz);
    reinterpret_cast<uint2*>(p)[e] = o;
  }
}

// e[t, f] = bf16(sum_s part[s, t, f]) for canvases that are still running.
__global__ void esum_kernel(const float* __restrict__ part, int ks, int T, int d, int canvas,
                            const uint8_t* __restrict__ done, uint16_t* __restrict__ sc_state) {
  const long long n = (long long)T * d;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(e / d);
    if (done[t / canvas]) continue;
    float acc = 0.f;
    for (int s = 0; s < ks; ++s) acc += part[(long long)s * n + e];
    sc_state[e] = f32_to_bf16(acc);
  }
}

// ---------------------------------------------------------------------------
// Per-round parameters read on the device (written by step_params_kernel as
// the first node of a round, so a captured round can be replayed for any step).
struct StepDev {
  int step, max_steps, block, policy;
  float lock_threshold, stop_entropy, inv_t;
  int require_stable;
  uint32_t k0, k1;
};

__global__ void step_params_kernel(StepDev* dst, const StepDev v) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *dst = v;
}

// Canvas update (a9), one CTA of 256 threads per canvas (thread = position).
struct UpdateParams {
  const float* entropy;
  const float* pmax;
  const int* argmax;
  const int* sample;
  int* tokens;          // canvas in/out
  int* prev_argmax;
  uint8_t* done;
  uint8_t* lock_out;    // may be null
  float* mean_out;      // may be null
  uint8_t* stop_out;    // may be null
  uint8_t* final_out;   // may be null
  uint8_t* flags;       // [B] internal copy of done after the update (host readback)
  const StepDev* sp;    // round parameters
  int vocab;
};

__global__ void __launch_bounds__(256) canvas_update_kernel(const UpdateParams p) {
  const int b = blockIdx.x, i = threadIdx.x;
  const int t = b * 256 + i;
  __shared__ float red[8];
  __shared__ int same_w[8];
  __shared__ float key[256];
  __shared__ int kid[256];
  __shared__ float csum[256];
  const StepDev sp = *p.sp;
  const float H = p.entropy[t];
  const float pm = p.pmax[t];
  const int am = p.argmax[t];
  const int smp = p.sample[t];
  const bool was_done = p.done[b] != 0;

  // mean entropy (fixed reduction order)
  float v = warp_sum(H);
  const int same = __all_sync(0xffffffffu, am == p.prev_argmax[t]);
  if ((i & 31) == 0) { red[i >> 5] = v; same_w[i >> 5] = same; }
  __syncthreads();
  float tot = 0.f;
  int all_same = 1;
#pragma unroll
  for (int w = 0; w < 8; ++w) { tot += red[w]; all_same &= same_w[w]; }
  const float meanH = tot / 256.0f;

  // lock mask
  bool lock;
  if (sp.policy == 0) {
    lock = pm > sp.lock_threshold;
  } else {
    // bitonic sort of (H, position) ascending, then a fixed-order running sum
    key[i] = H;
    kid[i] = i;
    __syncthreads();
    for (int size = 2; size <= 256; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const float a = key[i], c = key[j];
          const int ia = kid[i], ic = kid[j];
          const bool gt = (a > c) || (a == c && ia > ic);
          if (gt == up) { key[i] = c; key[j] = a; kid[i] = ic; kid[j] = ia; }
        }
        __syncthreads();
      }
    }
    if (i == 0) {
      float acc = 0.f;
      for (int r = 0; r < 256; ++r) { acc += key[r]; csum[r] = acc; }
    }
    __syncthreads();
    // rank of this position in sorted order
    lock = false;
    for (int r = 0; r < 256; ++r)
      if (kid[r] == i) { lock = csum[r] <= sp.lock_threshold; break; }
  }
  if (p.lock_out) p.lock_out[t] = lock ? 1 : 0;

  const bool stable = sp.step > 0 && all_same;
  const bool stop = !was_done && (meanH < sp.stop_entropy) && (!sp.require_stable || stable);
  const bool fin = !was_done && (stop || sp.step == sp.max_steps - 1);
  if (!was_done) {
    int nt;
    if (fin) {
      nt = am;
    } else if (lock) {
      nt = smp;
    } else {
      const Philox4 r = philox4x32_10(0u, (uint32_t)i, (uint32_t)(sp.block * 256 + sp.step),
                                      (kPurposeRenoise << 24) | (uint32_t)b, sp.k0, sp.k1);
      nt = uniform_token(r.x, (uint32_t)p.vocab);
    }
    p.tokens[t] = nt;
    p.prev_argmax[t] = am;
  }
  __syncthreads();
  if (i == 0) {
    if (p.mean_out) p.mean_out[b] = meanH;
    if (p.stop_out) p.stop_out[b] = stop ? 1 : 0;
    if (p.final_out) p.final_out[b] = fin ? 1 : 0;
    if (fin) p.done[b] = 1;
    p.flags[b] = (was_done || fin) ? 1 : 0;
  }
}

// Canvas initialisation: uniform tokens (purpose 1), prev_argmax = -1, done = 0.
__global__ void canvas_init_kernel(int* tokens, int* prev_argmax, uint8_t* done, int B, int block,
                                   uint32_t k0, uint32_t k1, int vocab) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= B * 256) return;
  const int b = t / 256, i = t % 256;
  const Philox4 r = philox4x32_10(0u, (uint32_t)i, (uint32_t)(block * 256),
                                  (kPurposeInit << 24) | (uint32_t)b, k0, k1);
  tokens[t] = uniform_token(r.x, (uint32_t)vocab);
  prev_argmax[t] = -1;
  if (i == 0) done[b] = 0;
}

__global__ void fill_u16_kernel(uint16_t* p, long long n, uint16_t v) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    p[e] = v;
}

}  // namespace dg
