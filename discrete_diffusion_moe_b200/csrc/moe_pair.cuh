// moe_pair.cuh - the two grouped products of the expert block in one
// persistent launch on CTA pairs: the gate/up product with SwiGLU (phase 1)
// and the down product with the routing weight (phase 2).
//
// Units are numbered phase 1 first (every (expert, tile pair, token chunk) of
// the gate/up product), then phase 2 (the same for the down product); each
// pair takes units cidx, cidx + ncl, ... in increasing order.  A down unit
// reads the SwiGLU outputs of its (expert, token chunk), which every gate/up
// tile pair of that expert and chunk writes: when a CTA has stored its part of
// a gate/up unit it adds one to the chunk's counter (release), and the copy
// warp of a down unit waits (acquire, bounded) until all 2 x tile-pairs CTAs of
// the chunk have, before it copies the chunk's rows.  Deadlock-free: the grid
// is resident as a whole (one launch of at most the CTAs the SMs hold), a pair
// waiting in a down unit has finished all of its own earlier units, and the
// units it waits for are gate/up units, which never wait; they belong to pairs
// that reach them before any down unit of theirs.  The counters are zeroed by
// the routing kernel of the same layer, which runs before this launch.
//
// The down product of an (expert, chunk) thus starts as soon as its inputs
// exist, overlapping the other gate/up units' epilogues and the tail of the
// phase, and the second launch's set-up is gone.  Otherwise the protocol
// (stages, accumulators, the leader's MMAs, tensor memory) is the pair
// kernel's (gemm_pair.cuh).
#pragma once

#include <type_traits>

#include "gemm_pair.cuh"

namespace dg {

struct MoePlan {
  GemmPlan up;    // phase 1: grouped gate/up (K = d_model, 2 d_ff rows per expert)
  GemmPlan down;  // phase 2: grouped down (K = d_ff, d_model rows per expert); same groups and chunks
  int* dep;       // [chunks] CTAs of phase 1 that finished a token chunk (zero at launch)
};

// orders this thread's later async-proxy (TMA) reads of global memory after
// what its generic-proxy acquire made visible
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// bounded wait until *cnt >= target
__device__ __forceinline__ bool wait_count(const int* cnt, int target, int* err) {
  if (ld_acquire_gpu_s32(cnt) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      __nanosleep(64);
      if (ld_acquire_gpu_s32(cnt) >= target) return true;
    }
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_error(err, kDevErrTimeout);
      return false;
    }
  }
}

struct MoeUnit {
  GemmJob j;
  int phase;   // 0 gate/up, 1 down
  int chunk;   // global token chunk: chunk_off[expert] + chunk within the expert
};

__device__ __forceinline__ MoeUnit moe_unit(const MoePlan& mp, const GemmTables& tb, int u, int rank, int U1) {
  MoeUnit m;
  m.phase = u >= U1;
  m.j = m.phase ? pair_job(mp.down, tb, u - U1, rank) : pair_job(mp.up, tb, u, rank);
  m.chunk = tb.chunk_off[m.j.group] + m.j.n_local0 / mp.up.bn;
  return m;
}

template <class EpiU, class EpiD>
__global__ void __launch_bounds__(gemm_threads<EpiU>(), 2)
    moe_pair_kernel(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ BMaps tmB1,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ BMaps tmB2,
                    const __grid_constant__ MoePlan mp, const EpiU e1, const EpiD e2, const int stages) {
  static_assert(EpiU::kEpiWarps == EpiD::kEpiWarps, "one epilogue warp count for both phases");
  constexpr int kEW = EpiU::kEpiWarps;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmTables tabs;
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int bn = mp.up.bn;
  const int b_stage_bytes = (bn / 2) * 128;
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
  touch_plan(mp.up);
  touch_plan(mp.down);
  int* const err = mp.up.err;
  const uint32_t rank = cluster_ctarank();
  const int cidx = (int)(blockIdx.x >> 1), ncl = (int)(gridDim.x >> 1);
  const uint32_t buf_cols = (uint32_t)bn;
  const uint32_t tmem_cols = 2u * buf_cols <= 32u ? 32u : (2u * buf_cols <= 64u ? 64u : (2u * buf_cols <= 128u ? 128u : (2u * buf_cols <= 256u ? 256u : 512u)));
  const uint32_t acc_stride = tmem_cols / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 2 * kEW);
    }
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmA2);
    for (int i = 0; i < 3; ++i) {
      tma_prefetch_desc(&tmB1.m[i]);
      tma_prefetch_desc(&tmB2.m[i]);
    }
  }
  grid_dep_wait();
  grid_dep_launch();
  if (warp >= 2) {
    for (int g = threadIdx.x - 64; g <= mp.up.n_groups; g += gemm_threads<EpiU>() - 64) {
      tabs.chunk_off[g] = __ldg(mp.up.chunk_off + g);
      tabs.group_off[g] = __ldg(mp.up.group_off + g);
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

  const int chunks = tabs.chunk_off[mp.up.n_groups];
  const int U1 = pair_tiles(mp.up) * chunks;
  const int U = U1 + pair_tiles(mp.down) * chunks;
  const int dep_target = 2 * pair_tiles(mp.up);  // both CTAs of every gate/up tile pair of a chunk

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      uint32_t it = 0;
      bool ok = true;
      const uint64_t pol_first = l2_policy_evict_first(), pol_last = l2_policy_evict_last();
      for (int u = cidx; u < U && ok; u += ncl) {
        const MoeUnit m = moe_unit(mp, tabs, u, (int)rank, U1);
        const GemmPlan& p = m.phase ? mp.down : mp.up;
        const CUtensorMap* ta = m.phase ? &tmA2 : &tmA1;
        const BMaps* tb = m.phase ? &tmB2 : &tmB1;
        const uint64_t pol_a = p.a_hint == 1 ? pol_first : pol_last;
        const uint64_t pol_b = p.b_hint == 1 ? pol_first : pol_last;
        if (m.phase) {
          // the chunk's SwiGLU outputs are complete and visible to the copies
          if (!wait_count(mp.dep + m.chunk, dep_target, err)) { ok = false; break; }
          fence_proxy_async_global();
        }
        const GemmJob& j = m.j;
        const int bi = pair_b_map(p, j.n_valid);
        const int half = ((j.n_valid + 15) & ~15) >> 1;
        const bool a_mine = j.m_valid > 0;
        const bool a_peer = 2 * (j.m_tile >> 1) + 1 < p.m_tiles;  // the odd tile of the pair exists
        const uint32_t tx = (uint32_t)(a_peer ? 2 : 1) * kATileBytes + 2u * (uint32_t)p.b_rows[bi] * 128u;
        for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
          const int s = it % stages;
          const uint32_t ph = (it / stages) & 1;
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, err)) { ok = false; break; }
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
          if (a_mine) tma_load_2d_pair(smem_u32(sA + (size_t)s * kATileBytes), ta, fb, kb * 64, j.a_row0, pol_a);
          tma_load_2d_pair(smem_u32(sB + (size_t)s * b_stage_bytes), &tb->m[bi], fb, kb * 64,
                           j.n0 + (int)rank * half, pol_b);
        }
      }
      // drain: the leader's full barriers count both CTAs' bytes
      if (rank == 0) {
        const uint32_t n_issued = it;
        const uint32_t first = n_issued > (uint32_t)stages ? n_issued - stages : 0;
        for (uint32_t q = first; q < n_issued; ++q)
          mbar_wait(smem_u32(&full[q % stages]), (q / stages) & 1, err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader) ----------------
      uint32_t it = 0, jc = 0;
      bool ok = true;
      for (int u = cidx; u < U && ok; u += ncl, ++jc) {
        const MoeUnit m = moe_unit(mp, tabs, u, 0, U1);
        const GemmJob& j = m.j;
        const int n_mma = (j.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(256, n_mma);
        const uint32_t acc = jc & 1, use = jc >> 1;
        if (!mbar_wait_cluster(smem_u32(&acc_empty[acc]), (use & 1) ^ 1, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * acc_stride;
        for (int kb = j.kb0; kb < j.kb1; ++kb, ++it) {
          const int s = it % stages;
          const uint32_t ph = (it / stages) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, err)) { ok = false; break; }
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
      mbar_wait(smem_u32(drain), 0, err);
    }
  } else {
    // ---------------- epilogue (both CTAs; warps 2..) ----------------
    static_assert(kEW == 4 || kEW == 8, "epilogue warps");
    constexpr int CSTEP = kEW / 4;
    const int quarter = warp & 3;
    const int cfirst = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t release_to = lane == 0 ? mapa_shared(smem_u32(&acc_empty[0]), 0) : 0u;
    uint32_t jc = 0;
    bool ok = true;
    auto drain_acc = [&](const auto& epi, const GemmJob& j, uint32_t acc) {
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * acc_stride;
      typename std::remove_reference_t<decltype(epi)>::State st;
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
    };
    // Every epilogue warp walks every unit (after a failed wait it stops waiting
    // and working, but still takes each gate/up unit's barrier), so the named
    // barrier below always sees all of them.
    for (int u = cidx; u < U; u += ncl, ++jc) {
      const MoeUnit m = moe_unit(mp, tabs, u, (int)rank, U1);
      const uint32_t acc = jc & 1, use = jc >> 1;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&acc_full[acc]), use & 1, err)) != 0;
      if (ok) {
        tc_fence_after();
        if (m.j.m_valid > 0) {
          if (m.phase) drain_acc(e2, m.j, acc);
          else         drain_acc(e1, m.j, acc);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(release_to + acc * 8u);
      }
      if (!m.phase) {
        // this CTA's part of the chunk's SwiGLU outputs is stored: publish it
        __threadfence();
        named_bar_sync(1, 32 * kEW);
        if (warp == 2 && lane == 0 && ok) red_release_gpu_add(mp.dep + m.chunk, 1);
      }
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

}  // namespace dg
