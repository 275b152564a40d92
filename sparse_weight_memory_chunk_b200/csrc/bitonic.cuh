// bitonic.cuh -- register-resident bitonic sorts of 64-bit keys (ascending).
//
// Keys are unique in every use (an index sits in the low bits), so the sorted order is
// fully determined.  Layout is "blocked": thread t holds elements t*VPT .. t*VPT+VPT-1.
// Compare-exchange partners closer than VPT stay in registers, partners within a warp
// are reached with shuffles, and only longer strides go through shared memory.
#pragma once

#include <stdint.h>

namespace fwpkm {

typedef unsigned long long u64;

__device__ __forceinline__ u64 umin64(u64 a, u64 b) { return a < b ? a : b; }
__device__ __forceinline__ u64 umax64(u64 a, u64 b) { return a < b ? b : a; }

// In-register stage with a compile-time partner distance JJ < VPT.
template <int VPT, int JJ>
__device__ __forceinline__ void bitonic_reg_stage(u64 (&x)[VPT], int base, int kk) {
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int pu = u ^ JJ;
    if (pu > u) {
      const bool up = ((base + u) & kk) == 0;
      const u64 a = x[u], b = x[pu];
      const bool sw = (a > b) == up;
      x[u] = sw ? b : a;
      x[pu] = sw ? a : b;
    }
  }
}

template <int VPT>
__device__ __forceinline__ void bitonic_reg_stages(u64 (&x)[VPT], int base, int kk, int jj_hi) {
  // all in-register distances jj = min(jj_hi, VPT/2) .. 1
  if (VPT >= 16 && jj_hi >= 8) bitonic_reg_stage<VPT, (VPT >= 16 ? 8 : 0)>(x, base, kk);
  if (VPT >= 8 && jj_hi >= 4) bitonic_reg_stage<VPT, (VPT >= 8 ? 4 : 0)>(x, base, kk);
  if (VPT >= 4 && jj_hi >= 2) bitonic_reg_stage<VPT, (VPT >= 4 ? 2 : 0)>(x, base, kk);
  if (VPT >= 2 && jj_hi >= 1) bitonic_reg_stage<VPT, (VPT >= 2 ? 1 : 0)>(x, base, kk);
}

// Shuffle stage: partner is lane ^ lj, same register slot.
template <int VPT>
__device__ __forceinline__ void bitonic_shfl_stage(u64 (&x)[VPT], int base, int lane, int kk, int lj) {
  const bool lower = (lane & lj) == 0;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const u64 other = __shfl_xor_sync(0xffffffffu, x[u], lj);
    const bool up = ((base + u) & kk) == 0;
    x[u] = (lower == up) ? umin64(x[u], other) : umax64(x[u], other);
  }
}

// Sort 32*VPT keys held by one warp (ascending).
template <int VPT>
__device__ __forceinline__ void warp_sort_asc(u64 (&x)[VPT], int lane) {
  constexpr int S = 32 * VPT;
  const int base = lane * VPT;
#pragma unroll
  for (int kk = 2; kk <= S; kk <<= 1) {
#pragma unroll
    for (int jj = kk >> 1; jj >= VPT; jj >>= 1) bitonic_shfl_stage<VPT>(x, base, lane, kk, jj / VPT);
    if (VPT > 1) bitonic_reg_stages<VPT>(x, base, kk, (kk >> 1) < VPT ? (kk >> 1) : VPT / 2);
  }
}

// Sort S keys (power of two, S >= 32*VPT) held by the first S/VPT threads of the block.
// Every thread of the block must call it (it contains __syncthreads); threads beyond
// S/VPT pass dummy registers.  `sm` must hold S keys.
template <int VPT>
__device__ void block_sort_asc(u64 (&x)[VPT], u64* sm, int S) {
  const int tid = threadIdx.x, lane = tid & 31;
  const bool active = tid * VPT < S;
  const int base = tid * VPT;
  const int warp_span = 32 * VPT;
  for (int kk = 2; kk <= S; kk <<= 1) {
    int jj = kk >> 1;
    for (; jj >= warp_span; jj >>= 1) {  // partner in another warp: exchange through shared memory
      // striped layout (slot u of thread t at u*nthr + t): conflict-free for both the
      // stores and the partner loads, whose thread index differs only above the lane bits
      const int nthr = S / VPT;
      if (active)
#pragma unroll
        for (int u = 0; u < VPT; ++u) sm[u * nthr + tid] = x[u];
      __syncthreads();
      if (active) {
        const int ptid = tid ^ (jj / VPT);
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
          const int i = base + u;
          const u64 other = sm[u * nthr + ptid];
          const bool up = (i & kk) == 0;
          const bool lower = (i & jj) == 0;
          x[u] = (lower == up) ? umin64(x[u], other) : umax64(x[u], other);
        }
      }
      __syncthreads();
    }
    if (active) {
      for (; jj >= VPT; jj >>= 1) bitonic_shfl_stage<VPT>(x, base, lane, kk, jj / VPT);
      if (VPT > 1) bitonic_reg_stages<VPT>(x, base, kk, jj);
    }
  }
}

// Total order on floats as an unsigned key and its inverse.
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

}  // namespace fwpkm
