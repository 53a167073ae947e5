// kernels.cuh - bandwidth-bound kernels of the denoising step: embedding,
// RMSNorm, RoPE table, router top-k, token permutation, expert combine,
// vocabulary statistics merge, softmax probabilities, split-k reduction of
// the expected embedding, the canvas update (entropy / lock / stop /
// re-noise) and canvas initialisation.  All reductions that carry results
// run in a fixed order (no atomics on values), so results are deterministic.
#pragma once

#include "common.cuh"
#include "l2_prefetch.cuh"

namespace dg {

// ---------------------------------------------------------------------------
// a1: x[t, :] = E_emb[tok[t], :]   (fp32 residual stream)
__global__ void embed_kernel(const uint16_t* __restrict__ emb, const int* __restrict__ tokens,
                             float* __restrict__ x, int T, int d, int vocab, int* err) {
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
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
// x[t, :] += sum_s part[s, t, :] (ks split-k partials, in split order; none
// when ks == 0), then xn = bf16(x / rms(x) * gain).  One CTA per token with
// one float4 of the row per thread (NV per thread when the row is longer than
// 4096): every load of the row is in flight at once and all tokens' CTAs are
// resident together; the row stays in registers between the two passes.
template <int NV>
__global__ void __launch_bounds__(1024) residual_norm_kernel(float* __restrict__ x, const float* __restrict__ part,
                                                             int ks, long long split_stride, int d,
                                                             const uint16_t* __restrict__ gain,
                                                             uint16_t* __restrict__ xn, float eps) {
  grid_dep_wait();
  grid_dep_launch();
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
      float4 acc = *reinterpret_cast<const float4*>(xr + c);
      if (ks > 0) {
        const float* pp = part + (long long)t * d + c;
        float4 sum = *reinterpret_cast<const float4*>(pp);
        for (int sp = 1; sp < ks; ++sp) {
          const float4 v = *reinterpret_cast<const float4*>(pp + sp * split_stride);
          sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        }
        acc.x += sum.x; acc.y += sum.y; acc.z += sum.z; acc.w += sum.w;
        *reinterpret_cast<float4*>(xr + c) = acc;
      }
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
// (rope_table_kernel) and shared by all layers; the rotation runs in double
// from the fp32 sums, rounded once to bf16: in the QKV projection's epilogue
// (EpiQKV, when the projection's k splits add up in a cluster) or in
// rope_kv_kernel from the projection's split-k partials.
__global__ void rope_table_kernel(double2* __restrict__ tab, int nq, int L0, int half, int hd, double theta) {
  grid_dep_wait();
  grid_dep_launch();
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

constexpr int kRopeMaxSplits = 3; // split-k partials of the projection read by the kernel

// Blocks [v_blocks, ...): one thread per (token, q or k head, 4 consecutive
// pairs) rotates the 4 pairs (i, i + hd/2) .. (i + 3, i + 3 + hd/2) (rows
// interleaved by pair, see EpiQKV): two 16-byte loads of every split-k
// partial (summed in split order) and the 4 (cos, sin), all issued before the
// first is used, then two 8-byte stores (q into the packed grouped-query
// layout, k into the cache).
// Threads [0, 256 v_blocks): one thread per (canvas, kv head, 4 consecutive
// dims, position) moves 4 values of v into the transposed cache; the lanes of
// a warp take consecutive positions, so each of the 4 stores of a warp is one
// contiguous run along the cache's position axis.
__global__ void __launch_bounds__(256) rope_kv_kernel(const RopeParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int half = p.hd / 2;
  const int row_w = (p.Hq + 2 * p.Hkv) * p.hd;
  const int rot_blk = (int)blockIdx.x - p.v_blocks;
  if (rot_blk >= 0) {
    const int n4 = half >> 2;  // groups of 4 pairs per head (hd % 8 == 0)
    const int per_tok = (p.Hq + p.Hkv) * n4;
    const long long gid = (long long)rot_blk * blockDim.x + threadIdx.x;
    if (gid >= (long long)p.T * per_tok) return;
    const int t = (int)(gid / per_tok);
    const int rem = (int)(gid - (long long)t * per_tok);
    const int h = rem / n4, i = (rem - h * n4) * 4;
    const int b = t / p.nq, pos_in = t - b * p.nq;
    // q / k rows are interleaved by rotation pair: dim j at physical row 2j,
    // dim j + hd/2 at 2j + 1, so pairs i .. i + 3 are 8 consecutive values
    const float* src = p.qkv + (long long)t * row_w + h * p.hd + 2 * i;
    float4 a1[kRopeMaxSplits], a2[kRopeMaxSplits];
#pragma unroll
    for (int q = 0; q < kRopeMaxSplits; ++q)
      if (q < p.ks) {
        a1[q] = __ldcg(reinterpret_cast<const float4*>(src + q * p.split_stride));
        a2[q] = __ldcg(reinterpret_cast<const float4*>(src + q * p.split_stride + 4));
      }
    const double2* tab = p.tab + (long long)pos_in * half + i;
    double2 cs[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) cs[u] = __ldg(tab + u);
    float x1[4] = {a1[0].x, a1[0].z, a2[0].x, a2[0].z}, x2[4] = {a1[0].y, a1[0].w, a2[0].y, a2[0].w};
#pragma unroll
    for (int q = 1; q < kRopeMaxSplits; ++q)
      if (q < p.ks) {
        x1[0] += a1[q].x; x1[1] += a1[q].z; x1[2] += a2[q].x; x1[3] += a2[q].z;
        x2[0] += a1[q].y; x2[1] += a1[q].w; x2[2] += a2[q].y; x2[3] += a2[q].w;
      }
    uint16_t o1[4], o2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const double y1 = x1[u], y2 = x2[u];
      o1[u] = f32_to_bf16((float)(y1 * cs[u].x - y2 * cs[u].y));
      o2[u] = f32_to_bf16((float)(y2 * cs[u].x + y1 * cs[u].y));
    }
    uint16_t* dst;
    if (h < p.Hq) {
      const int G = p.Hq / p.Hkv;
      const int g = h / G, hh = h - g * G;
      dst = p.q + ((((long long)b * p.Hkv + g) * p.nq + pos_in) * G + hh) * p.hd;
    } else {
      const int g = h - p.Hq;
      dst = p.kc + (((long long)b * p.Hkv + g) * p.c_max + p.L0 + pos_in) * p.hd;
    }
    *reinterpret_cast<uint2*>(dst + i) =
        make_uint2((uint32_t)o1[0] | ((uint32_t)o1[1] << 16), (uint32_t)o1[2] | ((uint32_t)o1[3] << 16));
    *reinterpret_cast<uint2*>(dst + i + half) =
        make_uint2((uint32_t)o2[0] | ((uint32_t)o2[1] << 16), (uint32_t)o2[2] | ((uint32_t)o2[3] << 16));
  } else {
    const int n4 = p.hd >> 2;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= (long long)(p.T / p.nq) * p.Hkv * n4 * p.nq) return;
    const int pos = (int)(gid % p.nq);
    long long rest = gid / p.nq;
    const int d4 = (int)(rest % n4);
    rest /= n4;
    const int g = (int)(rest % p.Hkv), b = (int)(rest / p.Hkv);
    const float* src = p.qkv + (long long)(b * p.nq + pos) * row_w + (p.Hq + p.Hkv + g) * p.hd + d4 * 4;
    float4 a[kRopeMaxSplits];
#pragma unroll
    for (int q = 0; q < kRopeMaxSplits; ++q)
      if (q < p.ks) a[q] = __ldcg(reinterpret_cast<const float4*>(src + q * p.split_stride));
    float v[4] = {a[0].x, a[0].y, a[0].z, a[0].w};
#pragma unroll
    for (int q = 1; q < kRopeMaxSplits; ++q)
      if (q < p.ks) { v[0] += a[q].x; v[1] += a[q].y; v[2] += a[q].z; v[3] += a[q].w; }
    uint16_t* dst = p.vc + (((long long)b * p.Hkv + g) * p.hd + d4 * 4) * p.c_max + p.L0 + pos;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      dst[(long long)u * p.c_max] = bf16_to_f16(f32_to_bf16(v[u]));  // the bf16 value, held in fp16
  }
}

// ---------------------------------------------------------------------------
// Routing of the mixture-of-experts block in one launch: router top-k, the
// stable counting sort of the (token, slot) pairs by expert, and the gather of
// the normalised rows into expert order.
//
// Top-k of one token (one warp): sum the split-k partial logits (fixed
// order), pick the k largest logits (ties to the lower expert id), softmax
// over the chosen k.  E <= 256, k <= 8.
template <int KS>
__device__ __forceinline__ void route_topk_token(const float* __restrict__ part, int T, int E, int k, int t,
                                                 int lane, int* sel_out, float* w_out, int dbg_t, int* dbg_idx,
                                                 float* dbg_w, float* dbg_logits) {
  float l[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) l[q] = 0.f;
  // the 8 expert slots of a lane are independent, so their loads issue together
#pragma unroll
  for (int p = 0; p < KS; ++p) {
    const float* row = part + ((long long)p * T + t) * E;
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = (lane + 32 * q < E) ? __ldcg(row + lane + 32 * q) : 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) l[q] += v[q];
  }
  // order-preserving integer keys of the logits (larger logit, larger key);
  // 0 marks an absent or already chosen expert
  uint32_t key[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const bool ok = lane + 32 * q < E;
    if (ok && dbg_logits) dbg_logits[(long long)dbg_t * E + lane + 32 * q] = l[q];
    const uint32_t u = __float_as_uint(l[q]);
    key[q] = ok ? ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) : 0u;
    if (ok && key[q] == 0u) key[q] = 1u;  // -NaN patterns: keep them selectable
  }
  // k rounds: the warp's largest key (one reduction), then the lowest expert
  // id holding it (a second reduction); that expert leaves the candidates
  uint32_t sel_k[8];
  int sel_e[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= k) break;
    uint32_t best = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) best = max(best, key[q]);
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
    uint32_t cand = 0xffffffffu;
#pragma unroll
    for (int q = 7; q >= 0; --q)
      if (key[q] == wmax && wmax != 0u) cand = (uint32_t)(lane + 32 * q);
    const uint32_t we = __reduce_min_sync(0xffffffffu, cand);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if ((uint32_t)(lane + 32 * q) == we) key[q] = 0u;
    sel_k[r] = wmax;
    sel_e[r] = (int)we;
  }
  // softmax over the chosen logits, lane r handling choice r
  float lr = 0.f;
  int er = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r == lane && r < k) {
      const uint32_t kk = sel_k[r];
      lr = __uint_as_float((kk & 0x80000000u) ? (kk & 0x7fffffffu) : ~kk);
      er = sel_e[r];
    }
  const float l0 = __shfl_sync(0xffffffffu, lr, 0);
  const float ex = lane < k ? expf(lr - l0) : 0.f;
  float den = ex;
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    const float wv = ex / den;
    sel_out[lane] = er;
    w_out[lane] = wv;
    if (dbg_idx) dbg_idx[dbg_t * k + lane] = er;
    if (dbg_w) dbg_w[dbg_t * k + lane] = wv;
  }
}

// All CTAs of the launch wait here until every CTA has arrived (the launch is
// cooperative, so they are co-resident).  bar[0] counts arrivals, bar[1]
// departures; the last CTA to leave zeroes both for the next launch and adds
// 1 to bar[2], the count of completed barriers.  Gives up after kWaitLimitNs
// (error word kDevErrTimeout, returns false).
__device__ __forceinline__ bool grid_barrier(int* bar, int nb, int* err) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    red_release_gpu_add(bar, 1);
    int ok = 1;
    if (ld_acquire_gpu_s32(bar) < nb) {
      const unsigned long long t0 = globaltimer_ns();
      while (ld_acquire_gpu_s32(bar) < nb) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          set_error(err, kDevErrTimeout);
          ok = 0;
          break;
        }
      }
    }
    if (atomicAdd(bar + 1, 1) == nb - 1) {
      atomicExch(bar, 0);
      atomicExch(bar + 1, 0);
      atomicAdd(bar + 2, 1);
    }
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

struct RouteParams {
  const float* part;      // [KS, T, E] split-k router logits
  const uint16_t* xn;     // [T, d] normalised rows (bf16)
  int T, E, k, d, bn;     // bn: token chunk width of the grouped products
  int tpc;                // tokens per CTA (CTA b owns tokens [b tpc, (b+1) tpc))
  int* off;               // [E+1] first slot of each expert
  int* chunk_off;         // [E+1] first chunk of each expert (chunks of bn slots)
  int* perm;              // [P] slot -> pair (pair = token * k + j)
  int* inv;               // [P] pair -> slot
  float* w_perm;          // [P] routing weight of the slot's pair
  uint16_t* xperm;        // [P, d] X_perm[slot] = xn[perm[slot] / k]
  int* fill;              // [2, E] slots claimed per expert, two buffers
  int* bar;               // [3] grid barrier counters and completed-barrier count
  int* dbg_idx;           // optional [T, k]
  float* dbg_w;           // optional [T, k]
  float* dbg_logits;      // optional [T, E]
  int dbg_nq, dbg_skip;   // dbg_nq > 0: of each dbg_nq tokens the first dbg_skip are not recorded
                          // (an appending pass: only the canvas rows, compacted)
  int* distinct;          // optional: += number of experts given at least one token
  int* dep;               // optional [dep_n]: zeroed (the fused expert kernel's chunk counters)
  int dep_n;
  int* err;
};

// The slots follow expert order.  Each CTA claims, per expert, a run of slots
// for its pairs of that expert with one atomic add on fill[e] (before the
// grid barrier, so the adds overlap the wait); after the barrier fill[] holds
// the expert totals, which give the expert offsets.  Launches alternate
// between the two fill buffers by the parity of the completed-barrier count;
// CTA 0 zeroes the buffer of the previous launch, which the next one uses.  Within a CTA's run the
// pairs keep ascending pair order; the order of the runs of different CTAs
// follows the atomics.  No result depends on it: every slot's expert row is
// computed on its own, and the combine adds a token's k expert outputs in
// the fixed order j = 0..k-1 through inv[].
constexpr int kRouteThreads = 256;
template <int KS>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ int rsm[];
  const int E = p.E, k = p.k;
  const int np_max = p.tpc * k;
  int* s_e = rsm;                        // [np_max] expert of each local pair
  float* s_w = (float*)(s_e + np_max);   // [np_max]
  int* s_rank = (int*)(s_w + np_max);    // [np_max] rank among the CTA's pairs of its expert
  int* s_slot = s_rank + np_max;         // [np_max]
  int* s_cnt = s_slot + np_max;          // [E] the CTA's pairs per expert
  int* s_bef = s_cnt + E;                // [E] first slot of the CTA's run within the expert
  int* s_off = s_bef + E;                // [E+1]
  int* s_tot = s_off + E + 1;            // [E]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = kRouteThreads / 32;
  const int b = blockIdx.x, nb = gridDim.x;
  const int t0 = b * p.tpc;
  const int nt = max(0, min(p.T, t0 + p.tpc) - t0);
  const int np = nt * k;
  const int ep = __ldcg(p.bar + 2) & 1;  // this launch's fill buffer
  int* fill = p.fill + ep * E;
  if (b == 0) {
    for (int e = tid; e < E; e += kRouteThreads) p.fill[(ep ^ 1) * E + e] = 0;
    if (p.dep)
      for (int i = tid; i < p.dep_n; i += kRouteThreads) p.dep[i] = 0;
  }

  // ---- top-k of the CTA's tokens ----
  for (int lt = warp; lt < nt; lt += nw) {
    const int t = t0 + lt;
    int r = t;
    bool rec = true;
    if (p.dbg_nq > 0) {
      const int in = t % p.dbg_nq;
      rec = in >= p.dbg_skip;
      r = (t / p.dbg_nq) * (p.dbg_nq - p.dbg_skip) + in - p.dbg_skip;
    }
    route_topk_token<KS>(p.part, p.T, E, k, t, lane, s_e + lt * k, s_w + lt * k, r, rec ? p.dbg_idx : nullptr,
                         rec ? p.dbg_w : nullptr, rec ? p.dbg_logits : nullptr);
  }
  for (int e = tid; e < E; e += kRouteThreads) s_cnt[e] = 0;
  __syncthreads();
  // ---- stable ranks within the CTA: 32 pairs at a time in pair order ----
  if (warp == 0) {
    for (int c0 = 0; c0 < np; c0 += 32) {
      const int i = c0 + lane;
      int e = i < np ? s_e[i] : -1;
      if (e >= E || (i < np && e < 0)) { set_error(p.err, kDevErrBadToken); e = 0; }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (i < np) {
        s_e[i] = e;
        s_rank[i] = s_cnt[e] + __popc(peers & ((1u << lane) - 1));
      }
      __syncwarp();
      if (i < np && (__ffs(peers) - 1) == lane) s_cnt[e] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kRouteThreads) {
    const int c = s_cnt[e];
    s_bef[e] = c ? atomicAdd(fill + e, c) : 0;
  }

  if (!grid_barrier(p.bar, nb, p.err)) return;

  // ---- expert totals ----
  for (int e = tid; e < E; e += kRouteThreads) s_tot[e] = __ldcg(fill + e);
  __syncthreads();
  // exclusive scans of the counts and of the chunk counts (8 experts per lane)
  if (warp == 0) {
    int c8[8], k8[8], sc = 0, sk = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      c8[j] = e < E ? s_tot[e] : 0;
      k8[j] = (c8[j] + p.bn - 1) / p.bn;
      sc += c8[j];
      sk += k8[j];
    }
    int ic = sc, ik = sk;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, ic, o), a2 = __shfl_up_sync(0xffffffffu, ik, o);
      if (lane >= o) { ic += a; ik += a2; }
    }
    int pc = ic - sc, pk = ik - sk;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e < E) {
        s_off[e] = pc;
        if (b == 0) { p.off[e] = pc; p.chunk_off[e] = pk; }
      }
      pc += c8[j];
      pk += k8[j];
    }
    if (lane == 31) {
      s_off[E] = ic;
      if (b == 0) { p.off[E] = ic; p.chunk_off[E] = ik; }
    }
    if (b == 0 && p.distinct) {
      int nz = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) nz += c8[j] > 0;
      nz = __reduce_add_sync(0xffffffffu, nz);
      if (lane == 0) atomicAdd(p.distinct, nz);
    }
  }
  __syncthreads();
  // ---- slots of the CTA's pairs ----
  const int P = p.T * k;
  for (int i = tid; i < np; i += kRouteThreads) {
    const int e = s_e[i];
    int slot = s_off[e] + s_bef[e] + s_rank[i];
    if (slot < 0 || slot >= P) { set_error(p.err, kDevErrBadToken); slot = 0; }
    const int q = t0 * k + i;
    p.perm[slot] = q;
    p.inv[q] = slot;
    p.w_perm[slot] = s_w[i];
    s_slot[i] = slot;
  }
  __syncthreads();
  // ---- gather: each 16-byte vector of a token row is loaded once and stored
  // to the token's k slots; a thread's loads are all issued before its stores ----
  const int nvec = p.d / 8;
  const int nv_all = nt * nvec;
  const uint4* src = reinterpret_cast<const uint4*>(p.xn + (long long)t0 * p.d);
  for (int v0 = tid; v0 < nv_all; v0 += 4 * kRouteThreads) {
    uint4 val[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * kRouteThreads;
      if (v < nv_all) val[u] = __ldcg(src + v);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * kRouteThreads;
      if (v < nv_all) {
        const int lt = v / nvec, cv = v - lt * nvec;
        for (int j = 0; j < k; ++j)
          reinterpret_cast<uint4*>(p.xperm + (long long)s_slot[lt * k + j] * p.d)[cv] = val[u];
      }
    }
  }
}

inline size_t route_smem_bytes(int tpc, int k, int E) {
  return (size_t)tpc * k * 16 + (size_t)(4 * E + 1) * 4;
}

// chunk_off[g] = sum_{h < g} ceil((off[h+1] - off[h]) / bn)  (one thread)
__global__ void chunk_offsets_kernel(const int* __restrict__ off, int G, int bn, int* __restrict__ chunk_off) {
  grid_dep_wait();
  grid_dep_launch();
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int acc = 0;
  for (int g = 0; g < G; ++g) {
    chunk_off[g] = acc;
    const int n = off[g + 1] - off[g];
    acc += n > 0 ? (n + bn - 1) / bn : 0;
  }
  chunk_off[G] = acc;
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
                                                                uint16_t* __restrict__ xn, float eps,
                                                                const void* pf, long long pf_bytes) {
  // the next projection's weights (pf, pf_bytes: none when null) into L2; they
  // depend on nothing, so this comes before the wait for the previous kernel
  if (threadIdx.x == 0) l2_prefetch_share(pf, pf_bytes, blockIdx.x, gridDim.x);
  grid_dep_wait();
  grid_dep_launch();
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
  grid_dep_wait();
  grid_dep_launch();
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

// p[t, v] = bf16(exp(l[t, v] - m_t) / Z_t) from the bf16 logits, with m_t
// and Z_t the statistics of the fp32 logits — the softmax operand of the
// expected-embedding product.  Eight values per thread (16-byte loads and
// stores).
__global__ void probs_kernel(const uint16_t* __restrict__ logits, const float* __restrict__ m,
                             const float* __restrict__ inv_z, uint16_t* __restrict__ p, int T,
                             long long V) {
  grid_dep_wait();
  grid_dep_launch();
  const long long n8 = (long long)T * V / 8;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n8;
       e += (long long)gridDim.x * blockDim.x) {
    const long long t = (e * 8) / V;
    const float mm = m[t], iz = inv_z[t];
    const uint4 l = reinterpret_cast<const uint4*>(logits)[e];
    const uint32_t w[4] = {l.x, l.y, l.z, l.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = pack_bf16x2(__expf(bf16_to_f32(w[q] & 0xFFFF) - mm) * iz, __expf(bf16_to_f32(w[q] >> 16) - mm) * iz);
    reinterpret_cast<uint4*>(p)[e] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// e[t, f] = bf16(sum_s part[s, t, f]) for canvases that are still running.
__global__ void esum_kernel(const float* __restrict__ part, int ks, int T, int d, int canvas,
                            const uint8_t* __restrict__ done, uint16_t* __restrict__ sc_state) {
  grid_dep_wait();
  grid_dep_launch();
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
  int persistent;   // a locked position keeps its token for the rest of the block
};

__global__ void step_params_kernel(StepDev* dst, const StepDev v) {
  grid_dep_wait();
  grid_dep_launch();
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
  uint8_t* locked;      // [B, 256] committed positions (persistent lock; null otherwise)
  const StepDev* sp;    // round parameters
  int vocab;
};

__global__ void __launch_bounds__(256) canvas_update_kernel(const UpdateParams p) {
  grid_dep_wait();
  grid_dep_launch();
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
  // persistent lock: a position committed in an earlier round keeps its token
  const bool committed = sp.persistent && p.locked && p.locked[t];
  lock = lock || committed;
  if (p.lock_out) p.lock_out[t] = lock ? 1 : 0;

  const bool stable = sp.step > 0 && all_same;
  const bool stop = !was_done && (meanH < sp.stop_entropy) && (!sp.require_stable || stable);
  const bool fin = !was_done && (stop || sp.step == sp.max_steps - 1);
  if (!was_done) {
    int nt;
    if (committed) {
      nt = p.tokens[t];
    } else if (fin) {
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
    if (sp.persistent && p.locked && lock) p.locked[t] = 1;
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

// Canvas initialisation: uniform tokens (purpose 1), prev_argmax = -1, done = 0,
// locked = 0 (when given).
__global__ void canvas_init_kernel(int* tokens, int* prev_argmax, uint8_t* done, uint8_t* locked, int B, int block,
                                   uint32_t k0, uint32_t k1, int vocab) {
  grid_dep_wait();
  grid_dep_launch();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= B * 256) return;
  const int b = t / 256, i = t % 256;
  const Philox4 r = philox4x32_10(0u, (uint32_t)i, (uint32_t)(block * 256),
                                  (kPurposeInit << 24) | (uint32_t)b, k0, k1);
  tokens[t] = uniform_token(r.x, (uint32_t)vocab);
  prev_argmax[t] = -1;
  if (locked) locked[t] = 0;
  if (i == 0) done[b] = 0;
}

__global__ void fill_u16_kernel(uint16_t* p, long long n, uint16_t v) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x)
    p[e] = v;
}

}  // namespace dg

namespace dg {

// ---------------------------------------------------------------------------
// a8, high-batch variant (top-k vocabulary truncation): per position, the K
// ids with the largest bf16-stored logits (ties to the lower id), weights
// p = bf16(exp(l - M) / sum_sel exp(l - M)) over those K (M their largest),
// e = bf16(sum_j p_j E_emb[id_j]) in ascending id order.  One CTA per
// position: a two-pass radix select on order-preserving 16-bit keys of the
// bf16 logits (per-warp histograms of the high, then the low byte), an
// index-ordered collect (each thread owns a contiguous id range; block scans
// give every thread its output slots), then the K-row gather-sum (fixed
// order).  Positions of canvases that are done keep their state.
constexpr int kTopkThreads = 1024;
constexpr int kTopkMax = 1024;     // largest K
constexpr int kTopkBins = 2048;    // first level: the key's top 11 bits (a quarter octave)
constexpr int kTopkBins2 = 32;     // second level: the 5 low bits
constexpr int kTopkStash = 8192;   // candidates held in shared memory after the second pass

__device__ __forceinline__ uint32_t bf16_order_key(uint16_t b) {
  return (b & 0x8000u) ? (~(uint32_t)b & 0xFFFFu) : ((uint32_t)b | 0x8000u);
}

// exclusive block scan of one int per thread (kTopkThreads threads); the
// total goes to *total.  Uses `ws` [kTopkThreads / 32 + 1] ints of shared memory.
__device__ __forceinline__ int block_excl_scan(int v, int* ws, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ws[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = lane < kTopkThreads / 32 ? ws[lane] : 0;
    int c = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, c, o);
      if (lane >= o) c += n;
    }
    if (lane < kTopkThreads / 32) ws[lane] = c - t;
    if (lane == 31) ws[kTopkThreads / 32] = c;
  }
  __syncthreads();
  const int r = ws[warp] + incl - v;
  *total = ws[kTopkThreads / 32];
  __syncthreads();
  return r;
}

// order keys of the two bf16 values packed in w (low half: the lower id)
__device__ __forceinline__ uint32_t bf16x2_order_keys(uint32_t w) {
  const uint32_t sgn = (w >> 15) & 0x00010001u;      // the halves' sign bits
  return w ^ ((sgn * 0x7FFFu) | 0x80008000u);        // negative: ~b, positive: b | 0x8000
}

// dynamic shared memory of topk_esum_kernel
struct TopkSmem {
  // lane-private histograms [bin][lane]: a warp's 32 adds never share an
  // address; the first level packs two 16-bit counters per word (a lane sees
  // at most V / 32 keys of a row)
  uint32_t lh[kTopkBins / 2 * 32];
  int lh2[kTopkBins2 * 32];
  int hist[kTopkBins];     // first level, summed over lanes
  int hist2[kTopkBins2];   // second level
  int sel_idx[kTopkMax];
  float sel_w[kTopkMax];
  int scan_ws[kTopkThreads / 32 + 1];
  float red[kTopkThreads / 32];
  int s_b1, s_above1, s_thr, s_above, s_cthr, s_ns, s_nsel, s_ntie, s_maxkey;
  union {
    struct {
      int id[kTopkStash];
      uint16_t key[kTopkStash];
    } stash;
    float part[8192];  // the gather's per-group partial sums [groups][d]
  } u;
};

// warp-aggregated append of up to 8 items per lane (bits of m8): returns the
// slot of this lane's first item (its items take consecutive slots); one
// atomic per warp
__device__ __forceinline__ int warp_append8(uint32_t m8, int* counter) {
  const int lane = threadIdx.x & 31;
  const int cnt = __popc(m8);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  int base = 0;
  if (lane == 31 && incl) base = atomicAdd(counter, incl);
  base = __shfl_sync(0xffffffffu, base, 31);
  return base + incl - cnt;
}

// warp-aggregated append: the lanes with `take` get consecutive slots of
// `counter` (one atomic per warp); returns this lane's slot (or -1)
__device__ __forceinline__ int warp_append(bool take, int* counter) {
  const unsigned mask = __ballot_sync(0xffffffffu, take);
  if (!mask) return -1;
  const int lane = threadIdx.x & 31, leader = __ffs(mask) - 1;
  int base = 0;
  if (lane == leader) base = atomicAdd(counter, __popc(mask));
  base = __shfl_sync(0xffffffffu, base, leader);
  return take ? base + __popc(mask & ((1u << lane) - 1u)) : -1;
}

// The high-batch variant of the self-conditioning input: per position t, the
// K largest bf16 logits (ties to the lower id), p_v = bf16(exp(l_v - M) /
// sum over the K of exp(l_u - M)) with M the row's largest, and
// e_t = bf16(sum_v p_v E_emb[v]) over those K rows only.  A persistent grid
// of one 1024-thread CTA per SM walks the positions, so the rows in flight
// (one 512 KB row of a 262144-id vocabulary per SM) stay in L2 between the
// passes.  Keys are the logits' bf16 bits mapped to an unsigned order; the
// histograms are lane-private ([bin][lane]) so that the many keys that share
// a bin never serialise a warp's shared-memory adds.
//   pass 1 (from DRAM): histogram of the key's top 11 bits (a quarter octave
//     per bin) and the row's largest key; the bin b1 holding the K-th largest;
//   pass 2 (from L2): histogram of the 5 low bits inside b1 (exact keys), and
//     every key in bins >= b1 appended (id, key) to a shared stash when they
//     fit (a second such pass with the exact threshold when they do not); the
//     K-th largest key thr follows, with the number of keys equal to it;
//   selection: the stashed keys above thr, then the lowest ids of the keys
//     equal to it (sorted when not all are taken); a third pass over the row in
//     id order only when more than 1024 keys tie at thr; the K ids sorted
//     ascending (bitonic) so that the sums below run in id order;
//   gather: 8 columns per thread, the K rows split over thread groups, the
//     groups' partial sums added in group order (deterministic).
// V is a multiple of 256, so the uint4 units of a warp are all in range or
// all out of it (the warp-collective steps below never diverge).
__global__ void __launch_bounds__(kTopkThreads, 1) topk_esum_kernel(const uint16_t* __restrict__ logits, long long V,
                                                                     int K, const uint16_t* __restrict__ emb, int d,
                                                                     int canvas, int T, const uint8_t* __restrict__ done,
                                                                     uint16_t* __restrict__ sc_state) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ __align__(16) uint8_t topk_smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(topk_smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long nv8 = V / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    if (done && done[t / canvas]) continue;  // block-uniform
    const uint4* lr = reinterpret_cast<const uint4*>(logits + (long long)t * V);
    // ---- pass 1: octave histogram and the largest key ----
    for (int e = tid; e < kTopkBins / 2 * 32 / 4; e += kTopkThreads) reinterpret_cast<int4*>(sm.lh)[e] = make_int4(0, 0, 0, 0);
    __syncthreads();
    uint32_t kmax2 = 0;
    for (long long u0 = tid; u0 < nv8; u0 += 4 * kTopkThreads) {
      uint4 w[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const long long u = u0 + (long long)r * kTopkThreads;
        w[r] = u < nv8 ? __ldcg(lr + u) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (u0 + (long long)r * kTopkThreads >= nv8) break;
        const uint32_t w4[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t k2 = bf16x2_order_keys(w4[q]);
          kmax2 = __vmaxu2(kmax2, k2);
          const uint32_t b_lo = (k2 & 0xFFFFu) >> 5, b_hi = k2 >> 21;
          atomicAdd(&sm.lh[((b_lo >> 1) << 5) | lane], 1u << ((b_lo & 1u) << 4));
          atomicAdd(&sm.lh[((b_hi >> 1) << 5) | lane], 1u << ((b_hi & 1u) << 4));
        }
      }
    }
    uint32_t kmax = max(kmax2 & 0xFFFFu, kmax2 >> 16);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) sm.red[warp] = __int_as_float((int)kmax);
    __syncthreads();
    for (int wi = warp; wi < kTopkBins / 2; wi += kTopkThreads / 32) {
      const uint32_t v = sm.lh[wi * 32 + lane];
      const int lo = (int)__reduce_add_sync(0xffffffffu, v & 0xFFFFu);
      const int hi = (int)__reduce_add_sync(0xffffffffu, v >> 16);
      if (lane == 0) { sm.hist[2 * wi] = lo; sm.hist[2 * wi + 1] = hi; }
    }
    __syncthreads();
    {
      // bins from the top: thread i owns bins 2047 - 2i and 2046 - 2i
      const int hb = kTopkBins - 1 - 2 * tid;
      const int c0 = sm.hist[hb], c1 = sm.hist[hb - 1];
      int total;
      const int before = block_excl_scan(c0 + c1, sm.scan_ws, &total);
      if (before < K && before + c0 + c1 >= K) {
        if (before + c0 >= K) { sm.s_b1 = hb;     sm.s_above1 = before; }
        else                  { sm.s_b1 = hb - 1; sm.s_above1 = before + c0; }
      }
      if (tid == 0) {
        uint32_t km = 0;
        for (int w_ = 0; w_ < kTopkThreads / 32; ++w_) km = max(km, (uint32_t)__float_as_int(sm.red[w_]));
        sm.s_maxkey = (int)km;
        sm.s_ns = 0;
        sm.s_nsel = 0;
      }
      for (int e = tid; e < kTopkBins2 * 32; e += kTopkThreads) sm.lh2[e] = 0;
    }
    __syncthreads();
    const uint32_t b1 = (uint32_t)sm.s_b1;
    const bool stash_ok = sm.s_above1 + sm.hist[b1] <= kTopkStash;
    // ---- pass 2: mantissa histogram inside b1; stash the candidates ----
    for (long long u0 = tid; u0 < nv8; u0 += 4 * kTopkThreads) {
      uint4 w[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const long long u = u0 + (long long)r * kTopkThreads;
        w[r] = u < nv8 ? __ldcg(lr + u) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const long long u = u0 + (long long)r * kTopkThreads;
        if (u >= nv8) break;  // warp-uniform
        const uint32_t w4[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
        uint32_t k2[4], mx2 = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          k2[q] = bf16x2_order_keys(w4[q]);
          mx2 = __vmaxu2(mx2, k2[q]);
        }
        // most 8-key groups hold no key in bins >= b1: one vote for the warp
        const bool cand = max(mx2 & 0xFFFFu, mx2 >> 16) >= (b1 << 5);
        if (__any_sync(0xffffffffu, cand)) {
          uint32_t m8 = 0;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t key = (k2[q >> 1] >> (16 * (q & 1))) & 0xFFFFu;
            const uint32_t bin = key >> 5;
            if (bin == b1) atomicAdd(&sm.lh2[((key & 31u) << 5) | lane], 1);
            m8 |= (uint32_t)(bin >= b1) << q;
          }
          if (stash_ok) {
            int pos = warp_append8(m8, &sm.s_ns);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (m8 & (1u << q)) {
                sm.u.stash.id[pos] = (int)(u * 8 + q);
                sm.u.stash.key[pos] = (uint16_t)((k2[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
                ++pos;
              }
          }
        }
      }
    }
    __syncthreads();
    for (int b = warp; b < kTopkBins2; b += kTopkThreads / 32) {
      const int v = __reduce_add_sync(0xffffffffu, sm.lh2[b * 32 + lane]);
      if (lane == 0) sm.hist2[b] = v;
    }
    __syncthreads();
    if (warp == 0) {
      // the K-th largest key: lane l owns the low-bit bin 31 - l
      const int c = sm.hist2[kTopkBins2 - 1 - lane];
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const int cum = sm.s_above1 + incl - c;
      if (cum < K && cum + c >= K) {
        sm.s_thr = (int)((b1 << 5) | (uint32_t)(kTopkBins2 - 1 - lane));
        sm.s_above = cum;   // keys larger than thr
        sm.s_cthr = c;      // keys equal to it
      }
      if (lane == 0) sm.s_ntie = 0;
    }
    __syncthreads();
    const uint32_t thr = (uint32_t)sm.s_thr;
    const int above = sm.s_above, c_thr = sm.s_cthr, ties_needed = K - above;
    // the stash holds every key >= thr when it took all of bins >= b1; else one
    // more pass collects exactly the keys >= thr when they fit
    bool have = stash_ok;
    if (!have && above + c_thr <= kTopkStash) {
      if (tid == 0) sm.s_ns = 0;
      __syncthreads();
      for (long long u0 = tid; u0 < nv8; u0 += 4 * kTopkThreads) {
        uint4 w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const long long u = u0 + (long long)r * kTopkThreads;
          w[r] = u < nv8 ? __ldcg(lr + u) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const long long u = u0 + (long long)r * kTopkThreads;
          if (u >= nv8) break;  // warp-uniform
          const uint32_t w4[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
          uint32_t k2[4], mx2 = 0;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            k2[q] = bf16x2_order_keys(w4[q]);
            mx2 = __vmaxu2(mx2, k2[q]);
          }
          if (__any_sync(0xffffffffu, max(mx2 & 0xFFFFu, mx2 >> 16) >= thr)) {
            uint32_t m8 = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) m8 |= (uint32_t)(((k2[q >> 1] >> (16 * (q & 1))) & 0xFFFFu) >= thr) << q;
            int pos = warp_append8(m8, &sm.s_ns);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (m8 & (1u << q)) {
                sm.u.stash.id[pos] = (int)(u * 8 + q);
                sm.u.stash.key[pos] = (uint16_t)((k2[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
                ++pos;
              }
          }
        }
      }
      __syncthreads();
      have = true;
    }
    if (have && c_thr <= kTopkMax) {
      // ---- selection from the stash: the keys above thr, then the ties_needed
      // lowest ids of the keys equal to it; finally the K ids ascending ----
      int* tie_ids = reinterpret_cast<int*>(sm.sel_w);  // free until the weights
      const int ns = sm.s_ns;
      for (int e0 = 0; e0 < ns; e0 += kTopkThreads) {
        const int e = e0 + tid;
        const uint32_t key = e < ns ? (uint32_t)sm.u.stash.key[e] : 0u;
        const int pos = warp_append(e < ns && key > thr, &sm.s_nsel);
        if (pos >= 0) sm.sel_idx[pos] = sm.u.stash.id[e];
        const int pt = warp_append(e < ns && key == thr, &sm.s_ntie);
        if (pt >= 0) tie_ids[pt] = sm.u.stash.id[e];
      }
      __syncthreads();
      if (ties_needed < c_thr) {
        int n2 = 1;
        while (n2 < c_thr) n2 <<= 1;
        for (int e = c_thr + tid; e < n2; e += kTopkThreads) tie_ids[e] = 0x7FFFFFFF;
        __syncthreads();
        for (int k2 = 2; k2 <= n2; k2 <<= 1)
          for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
            const int e = tid, f = e ^ j2;
            if (e < n2 && f > e) {
              const int a = tie_ids[e], b = tie_ids[f];
              if (((e & k2) == 0) == (a > b)) { tie_ids[e] = b; tie_ids[f] = a; }
            }
            __syncthreads();
          }
      }
      for (int e = tid; e < ties_needed; e += kTopkThreads) sm.sel_idx[above + e] = tie_ids[e];
      int n2 = 1;
      while (n2 < K) n2 <<= 1;
      for (int e = K + tid; e < n2; e += kTopkThreads) sm.sel_idx[e] = 0x7FFFFFFF;
      __syncthreads();
      for (int k2 = 2; k2 <= n2; k2 <<= 1)
        for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
          const int e = tid, f = e ^ j2;
          if (e < n2 && f > e) {
            const int a = sm.sel_idx[e], b = sm.sel_idx[f];
            if (((e & k2) == 0) == (a > b)) { sm.sel_idx[e] = b; sm.sel_idx[f] = a; }
          }
          __syncthreads();
        }
    } else {
      // ---- pass 3 (more than kTopkMax keys tie at thr, or too many above it):
      // collect in id order, each thread a contiguous id range ----
      const long long per = (nv8 + kTopkThreads - 1) / kTopkThreads;  // uint4 units per thread
      const long long v0 = min(nv8, (long long)tid * per), v1 = min(nv8, v0 + per);
      int n_gt = 0, n_eq = 0;
      for (long long u = v0; u < v1; ++u) {
        const uint4 w = __ldcg(lr + u);
        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint32_t key = bf16_order_key((uint16_t)(w4[q >> 1] >> (16 * (q & 1))));
          n_gt += key > thr;
          n_eq += key == thr;
        }
      }
      int total;
      const int eq_before = block_excl_scan(n_eq, sm.scan_ws, &total);
      const int take_eq = max(0, min(n_eq, ties_needed - eq_before));
      int slot = block_excl_scan(n_gt + take_eq, sm.scan_ws, &total);
      int eq_taken = 0;
      const uint16_t* lr16 = logits + (long long)t * V;
      for (long long i = v0 * 8; i < v1 * 8 && slot < K; ++i) {
        const uint32_t key = bf16_order_key(lr16[i]);
        if (key > thr || (key == thr && eq_taken < take_eq)) {
          if (key == thr) ++eq_taken;
          sm.sel_idx[slot++] = (int)i;
        }
      }
      __syncthreads();
    }
    // ---- weights: softmax over the selected bf16 logits (fixed-order sum) ----
    const uint16_t* lr16 = logits + (long long)t * V;
    const uint32_t mk = (uint32_t)sm.s_maxkey;
    const uint16_t mbits = (uint16_t)((mk & 0x8000u) ? (mk & 0x7FFFu) : (~mk & 0xFFFFu));
    const float M = bf16_to_f32(mbits);
    float part = 0.f;
    for (int j = tid; j < K; j += kTopkThreads) {
      const float w = expf(bf16_to_f32(lr16[sm.sel_idx[j]]) - M);
      sm.sel_w[j] = w;
      part += w;
    }
    part = warp_sum(part);
    if (lane == 0) sm.red[warp] = part;
    __syncthreads();
    float den = 0.f;
#pragma unroll
    for (int w_ = 0; w_ < kTopkThreads / 32; ++w_) den += sm.red[w_];
    for (int j = tid; j < K; j += kTopkThreads) sm.sel_w[j] = bf16_to_f32(f32_to_bf16(sm.sel_w[j] / den));
    __syncthreads();
    // ---- e = sum_j p_j E_emb[id_j]: groups of d/8 threads, group g takes j = g, g + G, ... ----
    const int cpt = d / 8, G = min(kTopkThreads / cpt, (int)(8192 / d));
    const int g = tid / cpt, c8 = tid - g * cpt;
    if (g < G) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int j = g;
      for (; j + 3 * G < K; j += 4 * G) {
        uint4 w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
          w[r] = __ldg(reinterpret_cast<const uint4*>(emb + (long long)sm.sel_idx[j + r * G] * d) + c8);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float p = sm.sel_w[j + r * G];
          const uint32_t w4[4] = {w[r].x, w[r].y, w[r].z, w[r].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] = fmaf(p, bf16_to_f32(w4[q] & 0xFFFF), acc[2 * q]);
            acc[2 * q + 1] = fmaf(p, bf16_to_f32(w4[q] >> 16), acc[2 * q + 1]);
          }
        }
      }
      for (; j < K; j += G) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(emb + (long long)sm.sel_idx[j] * d) + c8);
        const float p = sm.sel_w[j];
        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = fmaf(p, bf16_to_f32(w4[q] & 0xFFFF), acc[2 * q]);
          acc[2 * q + 1] = fmaf(p, bf16_to_f32(w4[q] >> 16), acc[2 * q + 1]);
        }
      }
      float* dst = sm.u.part + (long long)g * d + c8 * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = acc[q];
    }
    __syncthreads();
    if (tid < cpt) {
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = sm.u.part[tid * 8 + q];
      for (int g2 = 1; g2 < G; ++g2) {
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += sm.u.part[(long long)g2 * d + tid * 8 + q];
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(sc_state + (long long)t * d)[tid] = o;
    }
    __syncthreads();  // the shared buffers are reused by the next position
  }
}

}  // namespace dg
