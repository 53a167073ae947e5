// gemm_tc.cuh - persistent, warp-specialised tcgen05 GEMM core for sm_100a.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      (bf16 inputs, fp32 accumulate)
//
// A and B are K-major bf16 matrices read through 2-D TMA tensor maps with the
// 128-byte swizzle (box: 64 elements of K x 128 rows for A).  B comes with
// three tensor maps of 16, min(64, bn) and bn rows per box: every stage loads
// its B rows with ONE copy, the smallest box that covers the unit's columns.
// Each copy costs about a hundred cycles to issue, so each stage is exactly
// two copies.  Two CTAs per SM (tiles of at most 128 columns) measured faster
// than one CTA with twice the stages for every product: a CTA's main loop
// advances at a near-fixed time per k block, whatever its bytes.  Each CTA
// loops over work units:
//   warp 0      TMA producer (one elected lane) filling a ring of smem stages
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma (M = 128,
//               N = the unit's columns rounded up to 16) into one of two
//               accumulator buffers and commits stage / accumulator barriers
//   warps 2..5  epilogue: tcgen05.ld of the 128 x N accumulator (warp w owns
//               TMEM lanes 32*(w%4) .. +31, i.e. tile rows) into registers and
//               a caller-supplied functor; the second accumulator buffer lets
//               the next unit's MMAs overlap this epilogue.
//
// Two schedules:
//   dense    units = (m_tile, n_tile, k_split); B rows [n_tile*bn, +bn)
//   grouped  units = (group, m_tile, chunk); group g uses A rows
//            [g * a_rows_per_group + m_tile*128, +128) and B rows
//            [group_off[g], group_off[g+1]) in chunks of at most bn rows
//            (a mixture-of-experts layer: one group per expert, B rows are the
//            tokens routed to it).  chunk_off[g] = sum over groups < g of
//            ceil(rows / bn), built on the device; units are ordered group,
//            then m_tile, then chunk, so the CTAs that run at the same time
//            share each weight tile through L2 instead of re-reading HBM.
//
// Every mbarrier wait is bounded (see mbar_wait); a unit whose wait ran out
// is abandoned, the error word is set, in-flight copies are drained and the
// tensor memory is released before the CTA exits.
#pragma once

#include "common.cuh"

namespace dg {

struct GemmPlan {
  int K;                 // reduction length, multiple of 64
  int a_rows;            // dense: rows of A (M); grouped: rows per group actually valid
  int m_tiles;           // dense: ceil(M / 128); grouped: tiles per group
  int n_total;           // dense: rows of B (N)
  int bn;                // columns per pass: multiple of 16, <= 256
  int b_rows[3];         // rows per box of the three B tensor maps (ascending, last covers bn)
  int k_splits;          // dense: K loop split into this many units (>= 1)
  int n_fast;            // dense: 1 = consecutive units walk the N tiles of one A tile
  const int* group_off;  // grouped when non-null: [n_groups + 1] B row offsets
  const int* chunk_off;  // grouped: [n_groups + 1] prefix sums of ceil(rows / bn)
  int n_groups;
  int a_rows_per_group;  // grouped: A row stride between groups
  int a_hint, b_hint;    // L2 policy of the A / B loads: 0 none, 1 evict_first, 2 evict_last
  int mt;                // dense: 128-row A tiles per unit (1 or 2; grouped: 1)
  int cluster_k;         // dense, > 1: the k_splits (== cluster_k) units of a tile are one
                         // cluster and add their accumulators through distributed shared
                         // memory before a single epilogue (one unit per CTA)
  int* err;              // device error word
};

struct GemmJob {
  int m_tile;    // tile index within the group (grouped) or within A (dense)
  int a_row0;    // first A row of the tile
  int m_valid;   // valid rows in this tile (<= 128)
  int group;     // grouped: group id; dense: -1
  int n0;        // first B row of this pass
  int n_local0;  // first column of this pass relative to the group / matrix start
  int n_valid;   // valid columns (B rows) in this pass, 1..bn
  int ks;        // k split index
  int kb0, kb1;  // k blocks [kb0, kb1) of 64
  int mt_eff;    // A tiles in this unit (dense units may cover two, tiles m_tile, m_tile + 1)
};

// The grouped schedule's offset tables are copied into shared memory at the
// start of the kernel (a binary search over them in global memory would be a
// chain of dependent loads before the first copy is issued).
constexpr int kGemmMaxGroups = 256;
struct GemmTables {
  int chunk_off[kGemmMaxGroups + 1];
  int group_off[kGemmMaxGroups + 1];
};
// static shared memory set aside for the tables (and rounding) when sizing
// the dynamic part
constexpr size_t kGemmStaticSmem = 4096;
static_assert(sizeof(GemmTables) <= kGemmStaticSmem, "offset tables");

__host__ __device__ __forceinline__ int gemm_num_units(const GemmPlan& p, const GemmTables& tb) {
  if (p.group_off) return p.m_tiles * tb.chunk_off[p.n_groups];
  const int n_tiles = (p.n_total + p.bn - 1) / p.bn;
  const int m_units = (p.m_tiles + p.mt - 1) / p.mt;
  return m_units * n_tiles * p.k_splits;
}

// Every unit is one pass (kept as a loop level so a unit could be split).
__host__ __device__ __forceinline__ int gemm_unit_passes(const GemmPlan&, int) { return 1; }

__host__ __device__ __forceinline__ GemmJob gemm_job(const GemmPlan& p, const GemmTables& tb, int u, int) {
  GemmJob j;
  const int kb_total = p.K / 64;
  if (p.group_off) {
    // group g with m_tiles * chunk_off[g] <= u < m_tiles * chunk_off[g + 1]
    int lo = 0, hi = p.n_groups;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.m_tiles * tb.chunk_off[mid] <= u) lo = mid;
      else hi = mid;
    }
    const int g = lo;
    const int c0 = tb.chunk_off[g];
    const int nch = tb.chunk_off[g + 1] - c0;
    const int r = u - p.m_tiles * c0;
    j.m_tile = r / nch;
    const int ch = r - j.m_tile * nch;
    j.group = g;
    j.a_row0 = g * p.a_rows_per_group + j.m_tile * 128;
    j.m_valid = min(128, p.a_rows - j.m_tile * 128);
    const int off0 = tb.group_off[g], off1 = tb.group_off[g + 1];
    j.n_local0 = ch * p.bn;
    j.n0 = off0 + j.n_local0;
    j.n_valid = min(p.bn, off1 - j.n0);
    j.ks = 0;
    j.kb0 = 0;
    j.kb1 = kb_total;
    j.mt_eff = 1;
  } else {
    const int n_tiles = (p.n_total + p.bn - 1) / p.bn;
    const int m_units = (p.m_tiles + p.mt - 1) / p.mt;
    const int ks = u % p.k_splits;
    const int r = u / p.k_splits;
    int mu, nt;
    if (p.n_fast) { nt = r % n_tiles; mu = r / n_tiles; }
    else          { mu = r % m_units; nt = r / m_units; }
    const int mt = mu * p.mt;
    j.mt_eff = min(p.mt, p.m_tiles - mt);
    j.m_tile = mt;
    j.group = -1;
    j.a_row0 = mt * 128;
    j.m_valid = min(128, p.a_rows - mt * 128);
    j.n_local0 = nt * p.bn;
    j.n0 = j.n_local0;
    j.n_valid = min(p.bn, p.n_total - j.n0);
    j.ks = ks;
    j.kb0 = kb_total * ks / p.k_splits;         // K / 64 * k_splits < 2^31
    j.kb1 = kb_total * (ks + 1) / p.k_splits;
  }
  return j;
}

// The plan's scalars sit in the kernel's parameter bank, whose first read on
// an SM misses; each job derives from several of them through divisions.
// Reading them all at entry (an empty asm use forces the loads there) lets the
// misses overlap the CTA's set-up and the wait for the previous kernel instead
// of delaying the first copy.
__device__ __forceinline__ void touch_plan(const GemmPlan& p) {
  asm volatile("" ::"r"(p.K), "r"(p.a_rows), "r"(p.m_tiles), "r"(p.n_total), "r"(p.bn), "r"(p.b_rows[0]),
               "r"(p.b_rows[1]), "r"(p.b_rows[2]), "r"(p.k_splits), "r"(p.n_fast), "l"(p.group_off),
               "l"(p.chunk_off), "r"(p.n_groups), "r"(p.a_rows_per_group), "r"(p.a_hint), "r"(p.b_hint),
               "r"(p.mt), "r"(p.cluster_k), "l"(p.err));
}

// Threads of a CTA: warp 0 copies, warp 1 issues the MMAs, Epi::kEpiWarps
// warps (4 or 8) drain the accumulators.  With 8, warps w and w + 4 read the
// same tensor-memory lane quarter (rows) and take alternate 16-column chunks.
template <class Epi>
__host__ __device__ constexpr int gemm_threads() { return 64 + 32 * Epi::kEpiWarps; }
constexpr int kATileBytes = 128 * 128;  // 128 rows x 64 bf16

// B tensor maps: boxes of b_rows[0] / b_rows[1] / b_rows[2] rows
struct BMaps {
  CUtensorMap m[3];
};

template <class Epi>
__global__ void __launch_bounds__(gemm_threads<Epi>(), 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
                   const GemmPlan p, const Epi epi, const int stages) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmTables tabs;
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int b_stage_bytes = p.bn * 128;
  const int a_stage_bytes = p.mt * kATileBytes;
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)stages * a_stage_bytes;
  uint64_t* bars = (uint64_t*)(sB + (size_t)stages * b_stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + stages;
  uint64_t* acc_full = bars + 2 * stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  touch_plan(p);
  // a dense plan's first job needs no table: computed before any wait
  const bool dense = p.group_off == nullptr;
  const GemmJob j_first = dense ? gemm_job(p, tabs, blockIdx.x, 0) : GemmJob{};
  const int U_dense = dense ? gemm_num_units(p, tabs) : 0;
  // accumulator buffers: two (the next unit's MMAs overlap this unit's
  // epilogue) unless two A tiles of 256 columns fill the tensor memory
  const uint32_t buf_cols = (uint32_t)(p.mt * p.bn);
  const int nbuf = buf_cols <= 256u ? 2 : 1;
  const uint32_t tmem_need = buf_cols * nbuf;
  const uint32_t tmem_cols = tmem_need <= 32u ? 32u : (tmem_need <= 64u ? 64u : (tmem_need <= 128u ? 128u : (tmem_need <= 256u ? 256u : 512u)));

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 32 * Epi::kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    for (int i = 0; i < 3; ++i) tma_prefetch_desc(&tmB.m[i]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  grid_dep_wait();
  grid_dep_launch();
  if (p.group_off && warp >= 2) {
    for (int g = threadIdx.x - 64; g <= p.n_groups; g += gemm_threads<Epi>() - 64) {
      tabs.chunk_off[g] = __ldg(p.chunk_off + g);
      tabs.group_off[g] = __ldg(p.group_off + g);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int U = dense ? U_dense : gemm_num_units(p, tabs);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t it = 0;
      bool ok = true;
      const uint64_t pol_first = l2_policy_evict_first(), pol_last = l2_policy_evict_last();
      const uint64_t pol_a = p.a_hint == 1 ? pol_first : pol_last;
      const uint64_t pol_b = p.b_hint == 1 ? pol_first : pol_last;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const int np = gemm_unit_passes(p, u);
        for (int pass = 0; pass < np && ok; ++pass) {
          const GemmJob j = (dense && u == (int)blockIdx.x && pass == 0) ? j_first : gemm_job(p, tabs, u, pass);
          const int n_mma = (j.n_valid + 15) & ~15;
          const int bi = n_mma <= p.b_rows[0] ? 0 : (n_mma <= p.b_rows[1] ? 1 : 2);
          const CUtensorMap* mb = &tmB.m[bi];
          const uint32_t tx = (uint32_t)j.mt_eff * kATileBytes + (uint32_t)p.b_rows[bi] * 128;
          for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
            const int s = it % stages;
            const uint32_t ph = (it / stages) & 1;
            if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, p.err)) { ok = false; break; }
            const uint32_t fb = smem_u32(&full[s]);
            mbar_arrive_expect_tx(fb, tx);
            for (int t = 0; t < j.mt_eff; ++t) {
              const uint32_t dA = smem_u32(sA + (size_t)s * a_stage_bytes + t * kATileBytes);
              if (p.a_hint) tma_load_2d_hint(dA, &tmA, fb, kb * 64, j.a_row0 + t * 128, pol_a);
              else          tma_load_2d(dA, &tmA, fb, kb * 64, j.a_row0 + t * 128);
            }
            const uint32_t dB = smem_u32(sB + (size_t)s * b_stage_bytes);
            if (p.b_hint) tma_load_2d_hint(dB, mb, fb, kb * 64, j.n0, pol_b);
            else          tma_load_2d(dB, mb, fb, kb * 64, j.n0);
          }
        }
      }
      // drain: wait until every issued copy has landed before the CTA may exit
      const uint32_t n_issued = it;
      const uint32_t first = n_issued > (uint32_t)stages ? n_issued - stages : 0;
      for (uint32_t q = first; q < n_issued; ++q)
        mbar_wait(smem_u32(&full[q % stages]), (q / stages) & 1, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t it = 0, jc = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const int np = gemm_unit_passes(p, u);
        for (int pass = 0; pass < np && ok; ++pass, ++jc) {
          const GemmJob j = (dense && u == (int)blockIdx.x && pass == 0) ? j_first : gemm_job(p, tabs, u, pass);
          const int n_mma = (j.n_valid + 15) & ~15;
          const uint32_t idesc = idesc_bf16_f32(128, n_mma);
          const uint32_t acc = nbuf == 2 ? (jc & 1) : 0;
          const uint32_t use = nbuf == 2 ? (jc >> 1) : jc;
          if (!mbar_wait(smem_u32(&acc_empty[acc]), (use & 1) ^ 1, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * buf_cols;
          for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
            const int s = it % stages;
            const uint32_t ph = (it / stages) & 1;
            if (!mbar_wait(smem_u32(&full[s]), ph, p.err)) { ok = false; break; }
            tc_fence_after();
            const uint32_t b0 = smem_u32(sB + (size_t)s * b_stage_bytes);
            for (int t = 0; t < j.mt_eff; ++t) {
              const uint32_t a0 = smem_u32(sA + (size_t)s * a_stage_bytes + t * kATileBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16(d_tmem + t * (uint32_t)p.bn, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                          (kb > j.kb0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(smem_u32(&empty[s]));
          }
          if (ok) umma_commit(smem_u32(&acc_full[acc]));
        }
      }
      // all issued tensor-core work must finish before the memory is released
      umma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else if (p.cluster_k > 1) {
    // ---------------- cluster split-k, part 1: stage the accumulator ----------------
    // (one unit per CTA; every copy into the stage ring has been consumed and
    // every MMA has completed once acc_full fires, so the ring is free)
    constexpr int CSTEP = Epi::kEpiWarps / 4;
    const int quarter = warp & 3;
    const int cfirst = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const GemmJob j = gemm_job(p, tabs, blockIdx.x, 0);
    const bool ok = blockIdx.x < (unsigned)U && __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[0]), 0, p.err));
    tc_fence_after();
    const int pitch = p.bn + 4;
    float* stg = reinterpret_cast<float*>(sA) + (size_t)row * pitch;
    const int nch = (j.n_valid + 15) >> 4;
    for (int c = cfirst; c < nch; c += CSTEP) {
      float v[16];
      if (ok) {
        tmem_ld16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(c * 16), v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        *reinterpret_cast<float4*>(stg + c * 16 + 4 * e) = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    static_assert(Epi::kEpiWarps == 4 || Epi::kEpiWarps == 8, "epilogue warps");
    constexpr int CSTEP = Epi::kEpiWarps / 4;  // chunk stride of a warp
    const int quarter = warp & 3;
    const int cfirst = (warp - 2) >> 2;       // first chunk of this warp
    const int row = quarter * 32 + lane;
    uint32_t jc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const int np = gemm_unit_passes(p, u);
      for (int pass = 0; pass < np && ok; ++pass, ++jc) {
        const GemmJob ju = (dense && u == (int)blockIdx.x && pass == 0) ? j_first : gemm_job(p, tabs, u, pass);
        const uint32_t acc = nbuf == 2 ? (jc & 1) : 0;
        const uint32_t use = nbuf == 2 ? (jc >> 1) : jc;
        if (!mbar_wait(smem_u32(&acc_full[acc]), use & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int t = 0; t < ju.mt_eff; ++t) {
        GemmJob j = ju;
        j.m_tile = ju.m_tile + t;
        j.a_row0 = ju.a_row0 + t * 128;
        j.m_valid = min(128, p.a_rows - j.m_tile * 128);
        const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * buf_cols + t * (uint32_t)p.bn;
        typename Epi::State st;
        epi.begin(j, row, st);
        const int nch = (j.n_valid + 15) >> 4;
        // the load of this warp's next chunk is in flight while the current
        // one is processed
        uint32_t ra[16], rb[16];
        if (cfirst < nch) {
          tmem_ld16_nowait(t0 + cfirst * 16, ra);
          tmem_wait_ld16(ra);
        }
        for (int c = cfirst; c < nch; c += CSTEP) {
          if (c + CSTEP < nch) tmem_ld16_nowait(t0 + (c + CSTEP) * 16, rb);
          float v[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(ra[i]);
          epi.chunk(j, row, c * 16, v, st);
          if (c + CSTEP < nch) {
            tmem_wait_ld16(rb);
#pragma unroll
            for (int i = 0; i < 16; ++i) ra[i] = rb[i];
          }
        }
        epi.end(j, row, st);
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&acc_empty[acc]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (p.cluster_k > 1) {
    // ---------------- cluster split-k, part 2: reduce and run the epilogue ----------------
    // CTA `rank` of the cluster (its k split) takes the 16-column chunks
    // c == rank (mod cluster_k) of the tile: each thread adds its row of the
    // chunk from every CTA's staged accumulator in rank order (a fixed order:
    // deterministic) and hands the sum to the functor, as split 0.
    cluster_sync_all();  // every CTA's accumulator is staged
    if (warp >= 2) {
      constexpr int CSTEP = Epi::kEpiWarps / 4;
      const int quarter = warp & 3;
      const int cfirst = (warp - 2) >> 2;
      const int row = quarter * 32 + lane;
      const int rank = (int)cluster_ctarank();
      GemmJob j = gemm_job(p, tabs, blockIdx.x, 0);
      j.ks = 0;
      j.kb0 = 0;
      j.kb1 = p.K / 64;
      const int nch = (j.n_valid + 15) >> 4;
      const uint32_t stg = smem_u32(sA) + (uint32_t)(row * (p.bn + 4)) * 4u;
      typename Epi::State st;
      epi.begin(j, row, st);
      int idx = 0;
      for (int c = rank; c < nch; c += p.cluster_k, ++idx) {
        if ((idx % CSTEP) != cfirst) continue;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
        for (int r = 0; r < p.cluster_k; ++r) {
          const uint32_t src = mapa_shared(stg + (uint32_t)c * 64u, (uint32_t)r);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 a = ld_dsmem_f4(src + 16u * e);
            v[4 * e] += a.x; v[4 * e + 1] += a.y; v[4 * e + 2] += a.z; v[4 * e + 3] += a.w;
          }
        }
        epi.chunk(j, row, c * 16, v, st);
      }
      epi.end(j, row, st);
    }
    cluster_sync_all();  // no CTA leaves while another reads its shared memory
  }
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// Dynamic shared memory of one CTA for `stages` stages.
inline size_t gemm_smem_bytes(int bn, int stages, int mt = 1) {
  return 1024 + (size_t)stages * ((size_t)mt * kATileBytes + (size_t)bn * 128) + (2 * stages + 5) * 8 + 16;
}

// CTAs per SM: two when both fit (tensor memory: 2 buffers x mt x bn columns
// <= 256 each; shared memory: at least three stages each), else one.
inline int gemm_ctas_per_sm(int bn, int mt = 1) { return mt * bn <= 128 ? 2 : 1; }

// Stages that fit `ctas` CTAs in one SM's 228 KB (1 KB of each CTA's share is
// reserved by the system).
inline int gemm_pick_stages(int bn, int ctas, int max_stages = 8, int mt = 1) {
  const size_t budget = (size_t)228 * 1024 / ctas - 1024 - kGemmStaticSmem;
  int s = max_stages;
  while (s > 2 && gemm_smem_bytes(bn, s, mt) > budget) --s;
  return s;
}

}  // namespace dg
