// l2_prefetch.cuh - asynchronous prefetch of a weight range into L2, split
// over the CTAs of a launch.  A kernel that leaves DRAM mostly idle (the
// expert combine) asks L2 for the weights the next projection streams, so
// that projection's loads hit L2 instead of waiting on DRAM.  The prefetch
// uses no shared memory and has no completion to wait for.
#pragma once

#include <cstdint>

namespace dg {

// 1: the expert combine prefetches the next layer's QKV weights into L2 (0: off)
#ifndef DG_L2_PREFETCH
#define DG_L2_PREFETCH 1
#endif

// CTA `cta` of `ctas` asks L2 for its share of [base, base + bytes) (base
// 16-byte aligned; a last piece shorter than 16 bytes is left out), in pieces
// of at most 64 KB.  A null base or an empty range does nothing.
__device__ __forceinline__ void l2_prefetch_share(const void* base, long long bytes, int cta, int ctas) {
  bytes &= ~15LL;
  if (!DG_L2_PREFETCH || base == nullptr || bytes <= 0 || ctas <= 0 || ((uintptr_t)base & 15)) return;
  const long long share = ((bytes + ctas - 1) / ctas + 15) & ~15LL;
  long long lo = (long long)cta * share;
  const long long hi = lo + share < bytes ? lo + share : bytes;
  for (; lo < hi; lo += 65536) {
    const uint32_t n = (uint32_t)(hi - lo < 65536 ? hi - lo : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"((const char*)base + lo), "r"(n) : "memory");
  }
}

}  // namespace dg
