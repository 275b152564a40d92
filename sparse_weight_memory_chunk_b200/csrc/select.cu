// select.cu -- restricted Cartesian top-k with softmax weights, and the per-chunk
// (slot, token) sort that drives the atomic-free write.
//
// Fast-weight Product Key Memory (rainbus summary), PKM prerequisite and method
// step 2; (paperlayer summary) §2.2: the final top-k is searched in the Cartesian
// product of the two halves' top-k, and the k selected slots get normalised weights.
#include "fwpkm_internal.cuh"

namespace fwpkm {

// ---------------------------------------------------------------------------
// Cartesian top-k: one warp per (memory, token).
//
// sigma_j = -log(eps + D_j) on the 2k survivors.  Each half is put in (sigma desc,
// sub-key asc) order; then a pair of ranks (i, j) can only be in the final top-k if
// (i+1)(j+1) <= k, because every pair (i' <= i, j' <= j) scores at least as high
// and wins exact ties on the slot index.  Lane i owns row i of that staircase and
// the k winners are extracted in (score desc, slot asc) order.  Weights are the
// softmax of the k scores.
// ---------------------------------------------------------------------------
constexpr int CART_WARPS = 8;

__global__ void __launch_bounds__(CART_WARPS * 32)
cartesian_kernel(Dims dm, Work w, int wt0, int len, int32_t* __restrict__ idx_out,
                 float* __restrict__ w_out) {
  __shared__ float s_sig[CART_WARPS][2][32];
  __shared__ int s_sub[CART_WARPS][2][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i_tok = blockIdx.x * CART_WARPS + warp;
  const int m = blockIdx.y;
  if (i_tok >= len) return;
  const int k = dm.k, n = dm.n;
  const long long tok = (long long)wt0 + i_tok;

  for (int j = 0; j < 2; ++j) {
    const size_t base = (((size_t)m * 2 + j) * w.max_T + tok) * k;
    float sig = 0.f;
    int sub = 0;
    unsigned long long key = ~0ull;
    if (lane < k) {
      sub = w.A[base + lane];
      sig = -logf(dm.eps_idw + w.Dsv[base + lane]);
      key = ((unsigned long long)(~orderable(sig)) << 32) | (unsigned)sub;  // sigma desc, sub asc
    }
    int rank = 0;
    for (int o = 0; o < 32; ++o) {
      unsigned long long other = __shfl_sync(0xffffffffu, key, o);
      rank += (other < key) ? 1 : 0;
    }
    if (lane < k) {
      s_sig[warp][j][rank] = sig;
      s_sub[warp][j][rank] = sub;
    }
  }
  __syncwarp();

  // candidate keys of row `lane`: (score desc, slot asc) packed so that smaller = better
  const int rowlen = lane < k ? k / (lane + 1) : 0;
  const float sig1 = lane < k ? s_sig[warp][0][lane] : 0.f;
  const int a = lane < k ? s_sub[warp][0][lane] : 0;
  auto cand = [&](int jj) -> unsigned long long {
    float S = sig1 + s_sig[warp][1][jj];
    unsigned slot = (unsigned)(a * n + s_sub[warp][1][jj]);
    return ((unsigned long long)(~orderable(S)) << 32) | slot;
  };
  unsigned long long best = ~0ull;
  for (int jj = 0; jj < rowlen; ++jj) {
    unsigned long long c = cand(jj);
    best = c < best ? c : best;
  }
  unsigned long long mine = ~0ull;  // lane r keeps the r-th winner
  for (int r = 0; r < k; ++r) {
    unsigned long long win = warp_min_u64(best);
    if (lane == r) mine = win;
    if (best == win) {
      best = ~0ull;
      for (int jj = 0; jj < rowlen; ++jj) {
        unsigned long long c = cand(jj);
        if (c > win && c < best) best = c;
      }
    }
  }
  // unpack, softmax over the k scores (max is rank 0)
  float S = 0.f;
  int slot = 0;
  if (lane < k) {
    uint32_t o = ~(uint32_t)(mine >> 32);
    uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
    S = __uint_as_float(u);
    slot = (int)(mine & 0xffffffffu);
  }
  const float smax = __shfl_sync(0xffffffffu, S, 0);
  float e = lane < k ? expf(S - smax) : 0.f;
  const float z = warp_sum(e);
  if (lane < k) {
    const float wt = e / z;
    const size_t o = ((size_t)m * w.max_T + tok) * k + lane;
    w.idx[o] = slot;
    w.w[o] = wt;
    if (idx_out) idx_out[((size_t)m * len + i_tok) * k + lane] = slot;
    if (w_out) w_out[((size_t)m * len + i_tok) * k + lane] = wt;
  }
}

int launch_cartesian(const Dims& d, const Work& w, int wt0, int len, int32_t* idx_out, float* w_out,
                     cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + CART_WARPS - 1) / CART_WARPS, d.M);
  cartesian_kernel<<<grid, CART_WARPS * 32, 0, s>>>(d, w, wt0, len, idx_out, w_out);
  return 1;
}

// ---------------------------------------------------------------------------
// Per-chunk sort of the (slot, token) read pairs: one CTA per (memory, chunk).
//
// Keys are (slot << 32) | (t_local * k + r); ascending order groups each slot's
// readers in token order, which is the summation order of the write.  Segment
// boundaries give N_read,i (paperlayer §3.3 read-count consensus).  Bitonic sort in
// shared memory; all orders are fixed, so the result is deterministic.
// ---------------------------------------------------------------------------
constexpr int SORT_THREADS = 1024;

__global__ void __launch_bounds__(SORT_THREADS)
sort_pairs_kernel(Dims dm, Work w, int wt0, int total_len, int last_has_target) {
  extern __shared__ unsigned long long s_keys[];
  __shared__ int s_warp[SORT_THREADS / 32];
  __shared__ int s_base;
  const int m = blockIdx.y;
  const int cc = blockIdx.x;
  const int C = dm.C, k = dm.k;
  const int tc0 = cc * C;  // relative to wt0
  const int clen = min(C, total_len - tc0);
  int npair = clen;
  if (!last_has_target && tc0 + clen == total_len) npair = clen - 1;
  const int P = npair * k;
  int Ppad = 1;
  while (Ppad < P) Ppad <<= 1;
  const int cslot = (wt0 + tc0) / C;
  const size_t cbase = (size_t)m * w.max_chunks + cslot;

  for (int i = threadIdx.x; i < Ppad; i += SORT_THREADS) {
    unsigned long long key = ~0ull;
    if (i < P) {
      int t_local = i / k, r = i - t_local * k;
      int slot = w.idx[((size_t)m * w.max_T + wt0 + tc0 + t_local) * k + r];
      key = ((unsigned long long)(unsigned)slot << 32) | (unsigned)i;
    }
    s_keys[i] = key;
  }
  __syncthreads();
  for (int kk = 2; kk <= Ppad; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < Ppad; i += SORT_THREADS) {
        int ixj = i ^ jj;
        if (ixj > i) {
          unsigned long long a = s_keys[i], b = s_keys[ixj];
          bool up = (i & kk) == 0;
          if ((a > b) == up) {
            s_keys[i] = b;
            s_keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // segments: compaction of the positions where the slot changes
  uint32_t* pair_tr = w.pair_tr + (size_t)m * w.max_chunks * C * k + (size_t)cslot * C * k;
  int32_t* seg_start = w.seg_start + cbase * (C * k + 1);
  int32_t* seg_slot = w.seg_slot + cbase * (C * k);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  for (int i0 = 0; i0 < P; i0 += SORT_THREADS) {
    const int i = i0 + threadIdx.x;
    bool head = false;
    unsigned long long key = 0;
    if (i < P) {
      key = s_keys[i];
      pair_tr[i] = (uint32_t)(key & 0xffffffffu);
      head = (i == 0) || ((s_keys[i - 1] >> 32) != (key >> 32));
    }
    unsigned bal = __ballot_sync(0xffffffffu, head);
    if (lane == 0) s_warp[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
      int v = s_warp[lane];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      s_warp[lane] = incl - v;  // exclusive
    }
    __syncthreads();
    if (head) {
      int pos = s_base + s_warp[warp] + __popc(bal & ((1u << lane) - 1u));
      seg_start[pos] = i;
      seg_slot[pos] = (int32_t)(key >> 32);
    }
    __syncthreads();
    if (threadIdx.x == SORT_THREADS - 1) {
      // last thread: total heads in this tile = exclusive prefix of last warp + its count
      s_base += s_warp[SORT_THREADS / 32 - 1] + __popc(bal);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    seg_start[s_base] = P;
    w.nseg[cbase] = s_base;
  }
}

int launch_sort_pairs(const Dims& d, const Work& w, int wt0, int total_len, bool last_has_target,
                      cudaStream_t s) {
  if (total_len <= 0) return 0;
  const int nchunks = (total_len + d.C - 1) / d.C;
  int Ppad = 1;
  while (Ppad < d.C * d.k) Ppad <<= 1;
  size_t smem = sizeof(unsigned long long) * (size_t)Ppad;
  cudaFuncSetAttribute(sort_pairs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  dim3 grid(nchunks, d.M);
  sort_pairs_kernel<<<grid, SORT_THREADS, smem, s>>>(d, w, wt0, total_len, last_has_target ? 1 : 0);
  return 1;
}

}  // namespace fwpkm
