// topk.cuh -- per-half top-k of one distance row by one warp (used by the fused selection
// kernel).
//
// Fast-weight Product Key Memory (paperlayer summary) §2.2: each half keeps the k
// sub-keys nearest to its half-query; (rainbus summary) PKM prerequisite.  Order: distance
// ascending, ties to the lower sub-key index.
//
// The row is held in registers (NPL values per lane, column lane + 32u).  Float compares
// throughout except for the final ranking:
//  1. each lane keeps its two smallest values m1 <= m2;
//  2. the 32 m1 and the 32 m2 are bitonic-sorted across the warp (1 shuffle per stage),
//     and a merge-path split of the two sorted lists gives tau = the k-th smallest of
//     those 64 values -- so at least k row values are <= tau (about 36 for k = 32);
//  3. the values <= tau are compacted into shared memory as (distance, index) keys and
//     ranked by comparing each with every other candidate; the k lowest ranks are the
//     answer, written in rank order.
// If more than 128 values pass (heavy ties) the warp falls back to k rounds of warp-wide
// minimum extraction over the row (re-read from memory).
#pragma once

#include "bitonic.cuh"
#include "fwpkm_internal.cuh"

namespace fwpkm {


// ascending bitonic sort of one float per lane
__device__ __forceinline__ float warp_sort32(float x, int lane) {
#pragma unroll
  for (int kk = 2; kk <= 32; kk <<= 1) {
#pragma unroll
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, x, jj);
      const bool up = (lane & kk) == 0;
      const bool lower = (lane & jj) == 0;
      x = (lower == up) ? fminf(x, o) : fmaxf(x, o);
    }
  }
  return x;
}

// The k nearest sub-keys of `row` (n distances) in rank order: out_sub[r], out_d[r] for
// r < k (global or shared memory).  `cand` is this warp's 128-key shared scratch.
template <int NPL>
__device__ __forceinline__ void row_topk(const float* __restrict__ row, int n, int k, int lane, u64* cand,
                                         int* out_sub, float* out_d) {
  const float INF = __int_as_float(0x7f800000);
  float v[NPL];
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int a = lane + 32 * u;
    v[u] = a < n ? row[a] : INF;
  }
  float m1 = INF, m2 = INF;
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    m2 = fminf(m2, fmaxf(m1, v[u]));
    m1 = fminf(m1, v[u]);
  }
  const float A = warp_sort32(m1, lane);
  const float B = warp_sort32(m2, lane);
  // merge path: lane l tests taking l values from A and k-l from B (lane 31 also tests
  // taking all 32 from A when k == 32)
  const float a_prev = __shfl_up_sync(0xffffffffu, A, 1);
  const int jb = k - lane;  // values taken from B
  const float b_at = __shfl_sync(0xffffffffu, B, jb < 32 ? (jb < 0 ? 0 : jb) : 31);
  const float b_prev = __shfl_sync(0xffffffffu, B, jb - 1 < 0 ? 0 : (jb - 1 > 31 ? 31 : jb - 1));
  const float Ai = A, Aim1 = lane == 0 ? -INF : a_prev;
  const float Bj = jb >= 32 ? INF : b_at, Bjm1 = jb <= 0 ? -INF : b_prev;
  const bool valid = lane <= k && jb <= 32 && Aim1 <= Bj && Bjm1 <= Ai;
  const float cand_tau = fmaxf(Aim1, Bjm1);
  // split i = 32 (k == 32: all of A, none of B) needs A[31] <= B[0]
  const float A31 = __shfl_sync(0xffffffffu, A, 31);
  const float B0 = __shfl_sync(0xffffffffu, B, 0);
  const unsigned bal = __ballot_sync(0xffffffffu, valid);
  float tau;
  if (bal) tau = __shfl_sync(0xffffffffu, cand_tau, __ffs(bal) - 1);
  else tau = (k == 32 && A31 <= B0) ? A31 : INF;  // INF: no split found (NaN rows) -> fallback

  // padding columns (index >= n) never become candidates, whatever tau is
  auto is_cand = [&](int u) { return lane + 32 * u < n && v[u] <= tau; };
  int c = 0;
#pragma unroll
  for (int u = 0; u < NPL; ++u) c += is_cand(u) ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total >= k && total <= 128) {
    int pos = incl - c;
#pragma unroll
    for (int u = 0; u < NPL; ++u)
      if (is_cand(u)) cand[pos++] = ((u64)float_key(v[u]) << 32) | (unsigned)(lane + 32 * u);
    __syncwarp();
    if (total <= 64) {
      u64 mine[2];
      int rk[2] = {0, 0};
#pragma unroll
      for (int j = 0; j < 2; ++j) mine[j] = lane + 32 * j < total ? cand[lane + 32 * j] : ~0ull;
      for (int t = 0; t < total; ++t) {
        const u64 o = cand[t];
        rk[0] += o < mine[0] ? 1 : 0;
        rk[1] += o < mine[1] ? 1 : 0;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j)
        if (lane + 32 * j < total && rk[j] < k) {
          out_sub[rk[j]] = (int)(mine[j] & 0xffffffffu);
          out_d[rk[j]] = key_float((uint32_t)(mine[j] >> 32));
        }
    } else {
      u64 mine[4];
      int rk[4] = {0, 0, 0, 0};
#pragma unroll
      for (int j = 0; j < 4; ++j) mine[j] = lane + 32 * j < total ? cand[lane + 32 * j] : ~0ull;
      for (int t = 0; t < total; ++t) {
        const u64 o = cand[t];
#pragma unroll
        for (int j = 0; j < 4; ++j) rk[j] += o < mine[j] ? 1 : 0;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (lane + 32 * j < total && rk[j] < k) {
          out_sub[rk[j]] = (int)(mine[j] & 0xffffffffu);
          out_d[rk[j]] = key_float((uint32_t)(mine[j] >> 32));
        }
    }
  } else {  // rare: re-read the row (cached) instead of keeping it live in registers
    u64 last = 0;
    for (int r = 0; r < k; ++r) {
      u64 best = ~0ull;
      for (int a = lane; a < n; a += 32) {
        const u64 key = ((u64)float_key(row[a]) << 32) | (unsigned)a;
        if ((r == 0 || key > last) && key < best) best = key;
      }
      last = warp_min_u64(best);
      if (lane == 0) {
        out_sub[r] = (int)(last & 0xffffffffu);
        out_d[r] = key_float((uint32_t)(last >> 32));
      }
    }
  }
}

}  // namespace fwpkm
