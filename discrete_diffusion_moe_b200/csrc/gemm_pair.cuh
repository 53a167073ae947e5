// gemm_pair.cuh - the grouped (mixture-of-experts) schedule of the tcgen05
// GEMM core run on CTA pairs: one tcgen05.mma.cta_group::2 instruction of
// M = 256 rows spans the two CTAs of a 2-CTA cluster, which sit on the two
// SMs of one TPC.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      (bf16 inputs, fp32 accumulate)
//
// A unit is (group, pair of 128-row A tiles, chunk of at most bn B rows); a
// dense plan (no groups, the LM head) has units (pair of A tiles, column tile).
// CTA rank r of the pair copies its own A tile (tile 2 * pair + r) and half
// of the unit's B rows (rows [r * N / 2, (r + 1) * N / 2) of the N = the
// chunk's rows rounded up to 16); the MMA reads A from each CTA for its 128
// rows and B from both, and leaves each CTA's 128 x N accumulator in that
// CTA's tensor memory.  Per 64-wide k block a CTA therefore copies 16 KB of
// weights and N / 2 rows of tokens instead of N rows: for 128-row chunks a
// quarter fewer bytes per output, the copy stream of each CTA being what
// bounds these products when few experts share many tokens.  Two clusters
// share each SM pair (two CTAs per SM).
//
// Protocol (rank 0 is the leader and issues every MMA):
//   full[s]       rank 0's only: the leader's producer posts the stage's
//                 bytes of both CTAs (arrive.expect_tx); both CTAs' copies
//                 complete their bytes on it (.cta_group::2 loads).
//   empty[s]      both CTAs: the leader's MMA commit arrives on both (one
//                 multicast commit); each producer waits on its own.
//   acc_full[a]   both CTAs: multicast commit after a unit's last MMA.
//   acc_empty[a]  rank 0's only: one arrival per epilogue warp of each CTA
//                 (release / acquire at cluster scope).
// Tensor memory is allocated and freed by warp 1 of both CTAs together
// (cta_group::2).  A cluster barrier after the barrier set-up and another
// before the tensor memory is freed keep either CTA from signalling a barrier
// the other has not initialised or has left.  Every mbarrier wait is bounded.
#pragma once

#include "gemm_tc.cuh"

namespace dg {

// ---- CTA-pair PTX (cluster rank, mapa and the cluster barrier are in common.cuh) ----------
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded like mbar_wait, acquiring what the arrivals of both CTAs released
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, int* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_error(err, kDevErrTimeout);
      return false;
    }
  }
}
// 2-D tiled load into this CTA's shared memory whose bytes complete on an
// mbarrier of this CTA or of its pair peer (`bar` is a shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(map), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T, M = 256
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive once on the mbarrier at this shared-memory offset in every CTA of
// `mask` when the pair's tensor-core work issued so far has completed
__device__ __forceinline__ void umma_commit_pair_mc(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// ---- schedule ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ int pair_tiles(const GemmPlan& p) { return (p.m_tiles + 1) >> 1; }

__host__ __device__ __forceinline__ int pair_num_units(const GemmPlan& p, const GemmTables& tb) {
  if (!p.group_off) return pair_tiles(p) * ((p.n_total + p.bn - 1) / p.bn) * p.k_splits;
  return pair_tiles(p) * tb.chunk_off[p.n_groups];
}

// The job of CTA `rank` in unit u: group g with P * chunk_off[g] <= u <
// P * chunk_off[g + 1] (P tile pairs per group), then pair, then chunk.
// m_valid <= 0 marks the missing second tile of a group with an odd tile count.
__host__ __device__ __forceinline__ GemmJob pair_job(const GemmPlan& p, const GemmTables& tb, int u, int rank) {
  const int P = pair_tiles(p);
  if (!p.group_off) {
    // dense: unit u = (k split u % k_splits, then tile pair, then column
    // tile); consecutive units share a column tile (its B rows are read from
    // L2 after the first)
    GemmJob j;
    const int ks = u % p.k_splits, r = u / p.k_splits;
    const int pr = r % P, nt = r / P;
    j.m_tile = 2 * pr + rank;
    j.group = -1;
    j.a_row0 = j.m_tile * 128;
    j.m_valid = min(128, p.a_rows - j.m_tile * 128);
    j.n_local0 = nt * p.bn;
    j.n0 = j.n_local0;
    j.n_valid = min(p.bn, p.n_total - j.n0);
    j.ks = ks;
    j.kb0 = (p.K / 64) * ks / p.k_splits;       // K / 64 * k_splits < 2^31
    j.kb1 = (p.K / 64) * (ks + 1) / p.k_splits;
    j.mt_eff = 1;
    return j;
  }
  int lo = 0, hi = p.n_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (P * tb.chunk_off[mid] <= u) lo = mid;
    else hi = mid;
  }
  const int g = lo;
  const int c0 = tb.chunk_off[g];
  const int nch = tb.chunk_off[g + 1] - c0;
  const int r = u - P * c0;
  const int pr = r / nch;
  const int ch = r - pr * nch;
  GemmJob j;
  j.m_tile = 2 * pr + rank;
  j.group = g;
  j.a_row0 = g * p.a_rows_per_group + j.m_tile * 128;
  j.m_valid = min(128, p.a_rows - j.m_tile * 128);
  const int off0 = tb.group_off[g], off1 = tb.group_off[g + 1];
  j.n_local0 = ch * p.bn;
  j.n0 = off0 + j.n_local0;
  j.n_valid = min(p.bn, off1 - j.n0);
  j.ks = 0;
  j.kb0 = 0;
  j.kb1 = p.K / 64;
  j.mt_eff = 1;
  return j;
}

// B box rows of a pair unit: the smallest of the three maps (boxes of
// b_rows[0] < b_rows[1] < b_rows[2] rows, the last bn / 2) that covers half
// of the unit's columns rounded up to 16.
__host__ __device__ __forceinline__ int pair_b_map(const GemmPlan& p, int n_valid) {
  const int half = ((n_valid + 15) & ~15) >> 1;
  return half <= p.b_rows[0] ? 0 : (half <= p.b_rows[1] ? 1 : 2);
}

template <class Epi>
__global__ void __launch_bounds__(gemm_threads<Epi>(), 2)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BMaps tmB,
                     const GemmPlan p, const Epi epi, const int stages) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmTables tabs;
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int b_stage_bytes = (p.bn / 2) * 128;  // a multiple of 1024 (bn >= 16): swizzled tiles stay aligned
  uint8_t* sA = smem;
  uint8_t* sB = smem + (size_t)stages * kATileBytes;
  uint64_t* bars = (uint64_t*)(sB + (size_t)stages * b_stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + stages;
  uint64_t* acc_full = bars + 2 * stages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  touch_plan(p);
  const uint32_t rank = cluster_ctarank();
  const int cidx = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  // a dense plan's first job needs no table: computed before any wait
  const bool dense = p.group_off == nullptr;
  const GemmJob j_first = dense ? pair_job(p, tabs, cidx, (int)rank) : GemmJob{};
  const GemmJob j_first0 = dense ? pair_job(p, tabs, cidx, 0) : GemmJob{};
  const int U_dense = dense ? pair_num_units(p, tabs) : 0;
  const uint32_t buf_cols = (uint32_t)p.bn;
  const uint32_t tmem_cols = 2u * buf_cols <= 32u ? 32u : (2u * buf_cols <= 64u ? 64u : (2u * buf_cols <= 128u ? 128u : (2u * buf_cols <= 256u ? 256u : 512u)));
  const uint32_t acc_stride = tmem_cols / 2;  // two accumulator buffers

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 2 * Epi::kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA);
    for (int i = 0; i < 3; ++i) tma_prefetch_desc(&tmB.m[i]);
  }
  grid_dep_wait();
  grid_dep_launch();
  if (warp >= 2 && p.group_off) {
    for (int g = threadIdx.x - 64; g <= p.n_groups; g += gemm_threads<Epi>() - 64) {
      tabs.chunk_off[g] = __ldg(p.chunk_off + g);
      tabs.group_off[g] = __ldg(p.group_off + g);
    }
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before either signals one
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int U = dense ? U_dense : pair_num_units(p, tabs);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      uint32_t it = 0;
      bool ok = true;
      const uint64_t pol_first = l2_policy_evict_first(), pol_last = l2_policy_evict_last();
      const uint64_t pol_a = p.a_hint == 1 ? pol_first : pol_last;
      const uint64_t pol_b = p.b_hint == 1 ? pol_first : pol_last;
      for (int u = cidx; u < U && ok; u += ncl) {
        const GemmJob j = (dense && u == cidx) ? j_first : pair_job(p, tabs, u, (int)rank);
        const int bi = pair_b_map(p, j.n_valid);
        const int half = ((j.n_valid + 15) & ~15) >> 1;
        const bool a_mine = j.m_valid > 0;
        const bool a_peer = 2 * (j.m_tile >> 1) + 1 < p.m_tiles;  // the odd tile of the pair exists
        const uint32_t tx = (uint32_t)(a_peer ? 2 : 1) * kATileBytes + 2u * (uint32_t)p.b_rows[bi] * 128u;
        for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
          const int s = it % stages;
          const uint32_t ph = (it / stages) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, p.err)) { ok = false; break; }
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
          if (a_mine) tma_load_2d_pair(smem_u32(sA + (size_t)s * kATileBytes), &tmA, fb, kb * 64, j.a_row0, pol_a);
          tma_load_2d_pair(smem_u32(sB + (size_t)s * b_stage_bytes), &tmB.m[bi], fb, kb * 64,
                           j.n0 + (int)rank * half, pol_b);
        }
      }
      // drain: the leader's full barriers count both CTAs' bytes
      if (rank == 0) {
        const uint32_t n_issued = it;
        const uint32_t first = n_issued > (uint32_t)stages ? n_issued - stages : 0;
        for (uint32_t q = first; q < n_issued; ++q)
          mbar_wait(smem_u32(&full[q % stages]), (q / stages) & 1, p.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader) ----------------
      uint32_t it = 0, jc = 0;
      bool ok = true;
      for (int u = cidx; u < U && ok; u += ncl, ++jc) {
        const GemmJob j = (dense && u == cidx) ? j_first0 : pair_job(p, tabs, u, 0);
        const int n_mma = (j.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(256, n_mma);
        const uint32_t acc = jc & 1, use = jc >> 1;
        if (!mbar_wait_cluster(smem_u32(&acc_empty[acc]), (use & 1) ^ 1, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * acc_stride;
        for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
          const int s = it % stages;
          const uint32_t ph = (it / stages) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + (size_t)s * kATileBytes);
          const uint32_t b0 = smem_u32(sB + (size_t)s * b_stage_bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_pair(d_tmem, sdesc_k128(a0 + kk * 32), sdesc_k128(b0 + kk * 32), idesc,
                           (kb > j.kb0 || kk > 0) ? 1u : 0u);
          umma_commit_pair_mc(smem_u32(&empty[s]), (uint16_t)3);
        }
        if (ok) umma_commit_pair_mc(smem_u32(&acc_full[acc]), (uint16_t)3);
      }
      umma_commit_pair(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, p.err);
    }
  } else {
    // ---------------- epilogue (both CTAs; warps 2..) ----------------
    static_assert(Epi::kEpiWarps == 4 || Epi::kEpiWarps == 8, "epilogue warps");
    constexpr int CSTEP = Epi::kEpiWarps / 4;
    const int quarter = warp & 3;
    const int cfirst = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t release_to = lane == 0 ? mapa_shared(smem_u32(&acc_empty[0]), 0) : 0u;
    uint32_t jc = 0;
    bool ok = true;
    for (int u = cidx; u < U && ok; u += ncl, ++jc) {
      const GemmJob j = (dense && u == cidx) ? j_first : pair_job(p, tabs, u, (int)rank);
      const uint32_t acc = jc & 1, use = jc >> 1;
      if (!mbar_wait(smem_u32(&acc_full[acc]), use & 1, p.err)) { ok = false; break; }
      tc_fence_after();
      if (j.m_valid > 0) {
        const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * acc_stride;
        typename Epi::State st;
        epi.begin(j, row, st);
        const int nch = (j.n_valid + 15) >> 4;
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
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(release_to + acc * 8u);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, loads and tensor-memory reads are all done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, tmem_cols);
  __syncthreads();
  cluster_sync_all();
}

// Dynamic shared memory of one pair CTA: stages of one A tile and bn / 2 B rows.
inline size_t gemm_pair_smem_bytes(int bn, int stages) {
  return 1024 + (size_t)stages * ((size_t)kATileBytes + (size_t)(bn / 2) * 128) + (2 * stages + 5) * 8 + 16;
}

// CTAs per SM of the pair kernel: two, unless the two 256-column accumulator
// buffers of a CTA take the whole tensor memory.
inline int gemm_pair_ctas_per_sm(int bn) { return bn <= 128 ? 2 : 1; }

// Stages that fit the pair CTAs of one SM in its 228 KB.
inline int gemm_pair_stages(int bn, int max_stages = 8) {
  const size_t budget = (size_t)228 * 1024 / gemm_pair_ctas_per_sm(bn) - 1024 - kGemmStaticSmem;
  int s = max_stages;
  while (s > 2 && gemm_pair_smem_bytes(bn, s) > budget) --s;
  return s;
}

}  // namespace dg
