// selection.cu -- restricted Cartesian top-k with softmax weights, and the per-chunk
// (slot, token) sort that drives the atomic-free write.
//
// Fast-weight Product Key Memory (rainbus summary), PKM prerequisite and method
// step 2; (paperlayer summary) §2.2: the final top-k is searched in the Cartesian
// product of the two halves' top-k, and the k selected slots get normalised weights.
#include "topk.cuh"

namespace fwpkm {

// ---------------------------------------------------------------------------
// Cartesian top-k: one warp per (memory, token).
//
// sigma_j = -log(eps + D_j) on the 2k survivors.  Each half must be in (sigma desc,
// sub-key asc) order; the per-half top-k delivers its survivors by (D asc, sub-key asc),
// which is that order unless two distances map to one sigma (or the logarithm's rounding
// inverts a pair), so the warp checks neighbours and sorts only when the check fails.
// Then a pair of ranks (i, j) can only be in the final top-k if (i+1)(j+1) <= k, because
// every pair (i' <= i, j' <= j) scores at least as high and wins exact ties on the slot
// index.  Those ~k ln k candidates (a table built once per CTA maps candidate c to its
// (i, j)) are spread evenly over the lanes as (score desc, slot asc) keys,
// bitonic-sorted, and the first k are the answer.  Weights are the softmax of the k
// scores.
// ---------------------------------------------------------------------------
constexpr int CART_WARPS = 8;

template <int VPT>
__device__ __forceinline__ void sort_cand(u64 (&x)[4], u64* cand, int lane) {
  u64 y[VPT];
#pragma unroll
  for (int u = 0; u < VPT; ++u) y[u] = x[u];
  warp_sort_asc<VPT>(y, lane);
#pragma unroll
  for (int u = 0; u < VPT; ++u) cand[lane * VPT + u] = y[u];
}

// Staircase table, built by one warp: candidate c -> (i << 8) | j, where lane i owns rank
// i of half 1 and ranks 0 .. k/(i+1)-1 of half 2.  Returns the candidate count in *total.
__device__ __forceinline__ void build_staircase(int k, int lane, unsigned short* tab, int* total) {
  const int rowlen = lane < k ? k / (lane + 1) : 0;
  int incl = rowlen;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  for (int jj = 0; jj < rowlen; ++jj) tab[incl - rowlen + jj] = (unsigned short)((lane << 8) | jj);
  if (lane == 31) *total = incl;
}

// Restricted Cartesian top-k + softmax of one token, by one warp.  Survivors of half j
// arrive in rank order (D asc, sub-key asc) at sub[j][r], dist[j][r] (r < k).  Writes
// slot/weight r of the token to idx_o[r], w_o[r] (and to the optional user copies).
__device__ __noinline__ void cartesian_token(const Dims& dm, const int* const (&sub)[2],
                                                const float* const (&dist)[2], float (*s_sig)[32],
                                                int (*s_sub)[32], u64* cand, const unsigned short* tab,
                                                int total, int lane, int32_t* idx_o, float* w_o,
                                                int32_t* idx_u, float* w_u) {
  const int k = dm.k, n = dm.n;
  for (int j = 0; j < 2; ++j) {
    u64 key[1] = {~0ull};
    if (lane < k) {
      const float sig = -logf(dm.eps_idw + dist[j][lane]);
      key[0] = ((u64)(~float_key(sig)) << 32) | (unsigned)sub[j][lane];  // sigma desc, sub asc
    }
    const u64 nxt = __shfl_down_sync(0xffffffffu, key[0], 1);
    if (__any_sync(0xffffffffu, lane < 31 && nxt < key[0])) warp_sort_asc<1>(key, lane);
    __syncwarp();
    if (lane < k) {
      s_sig[j][lane] = key_float(~(uint32_t)(key[0] >> 32));
      s_sub[j][lane] = (int)(key[0] & 0xffffffffu);
    }
  }
  __syncwarp();

  u64 x[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane * 4 + u;
    x[u] = ~0ull;
    if (c < total) {
      const int t = tab[c], i1 = t >> 8, i2 = t & 255;
      const float S = s_sig[0][i1] + s_sig[1][i2];
      const unsigned slot = (unsigned)s_sub[0][i1] * (unsigned)n + (unsigned)s_sub[1][i2];
      x[u] = ((u64)(~float_key(S)) << 32) | slot;
    }
  }
  // the sorts take the elements lane * VPT + u, u < VPT: repack for VPT < 4
  const int Sz = total <= 32 ? 32 : total <= 64 ? 64 : 128;
  if (Sz == 128) {
    sort_cand<4>(x, cand, lane);
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) cand[lane * 4 + u] = x[u];
    __syncwarp();
    u64 y[4];
    const int vpt = Sz / 32;
    for (int u = 0; u < 4; ++u) y[u] = u < vpt ? cand[lane * vpt + u] : ~0ull;
    __syncwarp();
    if (Sz == 64) sort_cand<2>(y, cand, lane);
    else sort_cand<1>(y, cand, lane);
  }
  __syncwarp();

  float S = 0.f;
  int slot = 0;
  if (lane < k) {
    const u64 key = cand[lane];
    S = key_float(~(uint32_t)(key >> 32));
    slot = (int)(key & 0xffffffffu);
  }
  const float smax = __shfl_sync(0xffffffffu, S, 0);
  const float e = lane < k ? expf(S - smax) : 0.f;
  const float z = warp_sum(e);
  if (lane < k) {
    const float wt = e / z;
    idx_o[lane] = slot;
    w_o[lane] = wt;
    if (idx_u) idx_u[lane] = slot;
    if (w_u) w_u[lane] = wt;
  }
}

// Survivors from the per-half top-k arrays A/Dsv.
__global__ void __launch_bounds__(CART_WARPS * 32)
cartesian_kernel(Dims dm, Work w, int wt0, int len, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_sig[CART_WARPS][2][32];
  __shared__ int s_sub[CART_WARPS][2][32];
  __shared__ u64 s_cand[CART_WARPS][128];
  __shared__ unsigned short s_tab[128];
  __shared__ int s_total;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = dm.k;
  if (warp == 0) build_staircase(k, lane, s_tab, &s_total);
  __syncthreads();
  const int i_tok = blockIdx.x * CART_WARPS + warp;
  const int m = blockIdx.y;
  if (i_tok >= len) return;
  const long long tok = (long long)wt0 + i_tok;
  const size_t b0 = (((size_t)m * 2 + 0) * w.max_T + tok) * k, b1 = (((size_t)m * 2 + 1) * w.max_T + tok) * k;
  const int* const sub[2] = {w.A + b0, w.A + b1};
  const float* const dist[2] = {w.Dsv + b0, w.Dsv + b1};
  const size_t o = ((size_t)m * w.max_T + tok) * k;
  const size_t ou = ((size_t)m * len + i_tok) * k;
  cartesian_token(dm, sub, dist, s_sig[warp], s_sub[warp], s_cand[warp], s_tab, s_total, lane, w.idx + o, w.w + o,
                  idx_out ? idx_out + ou : nullptr, w_out ? w_out + ou : nullptr);
}

// Fused per-half top-k + Cartesian search (tensor-core path): a CTA takes SEL_TOK tokens of
// one memory; warps 2i and 2i+1 take the two halves of token i from the distance rows,
// leave their survivors in shared memory, and warp 2i then finishes the token.
constexpr int SEL_TOK = 4;
template <int NPL>
__global__ void __launch_bounds__(SEL_TOK * 64, 3)
select_kernel(Dims dm, Work w, int wt0, int len, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ u64 s_cand[2 * SEL_TOK][128];
  __shared__ int s_hsub[SEL_TOK][2][32];
  __shared__ float s_hd[SEL_TOK][2][32];
  __shared__ float s_sig[SEL_TOK][2][32];
  __shared__ int s_sub[SEL_TOK][2][32];
  __shared__ unsigned short s_tab[128];
  __shared__ int s_total;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tl = warp >> 1, j = warp & 1;
  const int i_tok = blockIdx.x * SEL_TOK + tl;
  const int m = blockIdx.y;
  const int k = dm.k;
  if (warp == 0) build_staircase(k, lane, s_tab, &s_total);
  if (i_tok < len) {
    const float* row = w.Dfull + ((size_t)(m * 2 + j) * w.drows + i_tok) * dm.n;
    row_topk<NPL>(row, dm.n, k, lane, s_cand[warp], s_hsub[tl][j], s_hd[tl][j]);
  }
  __syncthreads();
  if (j != 0 || i_tok >= len) return;
  const long long tok = (long long)wt0 + i_tok;
  const int* const sub[2] = {s_hsub[tl][0], s_hsub[tl][1]};
  const float* const dist[2] = {s_hd[tl][0], s_hd[tl][1]};
  const size_t o = ((size_t)m * w.max_T + tok) * k;
  const size_t ou = ((size_t)m * len + i_tok) * k;
  cartesian_token(dm, sub, dist, s_sig[tl], s_sub[tl], s_cand[warp], s_tab, s_total, lane, w.idx + o, w.w + o,
                  idx_out ? idx_out + ou : nullptr, w_out ? w_out + ou : nullptr);
}

int launch_select(const Dims& d, const Work& w, int wt0, int len, int32_t* idx_out, float* w_out, cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + SEL_TOK - 1) / SEL_TOK, d.M);
  const int npl = (d.n + 31) / 32;
  const int th = SEL_TOK * 64;
  if (npl <= 2) launch_k(select_kernel<2>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else if (npl <= 4) launch_k(select_kernel<4>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else if (npl <= 8) launch_k(select_kernel<8>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else if (npl <= 16) launch_k(select_kernel<16>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else if (npl <= 32) launch_k(select_kernel<32>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else if (npl <= 64) launch_k(select_kernel<64>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  else launch_k(select_kernel<128>, grid, th, 0, s, d, w, wt0, len, idx_out, w_out);
  return 1;
}

int launch_cartesian(const Dims& d, const Work& w, int wt0, int len, int32_t* idx_out, float* w_out,
                     cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + CART_WARPS - 1) / CART_WARPS, d.M);
  launch_k(cartesian_kernel, grid, CART_WARPS * 32, 0, s, d, w, wt0, len, idx_out, w_out);
  return 1;
}

// ---------------------------------------------------------------------------
// Per-chunk sort of the (slot, token) read pairs.
//
// Keys are (slot << 32) | (t_local * k + r).  The write needs every slot's readers
// contiguous and in token order (its summation order); segment boundaries then give
// N_read,i (paperlayer §3.3 read-count consensus).  A global slot order is not needed,
// so keys are bucketed by a multiplicative hash of the slot (~64 keys per bucket; a slot
// falls in exactly one bucket), laid out bucket after bucket, and ordered inside each
// bucket by their full key.
//
// `split` CTAs (a power of two, at most SORT_SPLIT) share one (memory, chunk): each counts
// all buckets (so all agree on the bucket offsets), keeps the keys of its own share of the
// buckets in shared memory, and one warp per bucket ranks each key by comparing it with every other key
// of the bucket and stores it at its rank.  The scatter into buckets may land keys in
// any order; ranking by the full unique key makes the output independent of it.  A
// bucket of more than 128 keys (strongly skewed slot use: a row read by many tokens) is
// ranked by the whole CTA that owns it instead of one warp.
// ---------------------------------------------------------------------------
constexpr int SORT_THREADS = 1024;
constexpr int SORT_SPLIT = 16;
constexpr int SORT_BUCKET_KEYS = 64;   // average keys per bucket
constexpr int SORT_BUCKET_CAP = 128;   // largest bucket the ranking path handles

// HEADS: the memories of a sequence share its value table (dm.H > 1); false compiles the
// one-head kernel, whose pair i is offset i of the chunk's [C][k] slot block.
template <int VPT, bool HEADS>
__global__ void __launch_bounds__(SORT_THREADS)
sort_pairs_kernel(Dims dm, Work w, int wt0, int total_len, int last_has_target, int split) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ u64 s_keys[];
  __shared__ int s_cnt[512], s_off[513], s_cur[512];
  const int m = blockIdx.y;  // the value table (sequence); its heads are memories m H .. m H + H - 1
  const int cc = blockIdx.x / split, part = blockIdx.x % split;
  const int C = dm.C, k = dm.k, H = HEADS ? dm.H : 1, kh = k * H;
  const int tc0 = cc * C;  // relative to wt0
  const int clen = min(C, total_len - tc0);
  int npair = clen;
  if (!last_has_target && tc0 + clen == total_len) npair = clen - 1;
  const int P = npair * kh;
  int Ppad = 32 * VPT;
  while (Ppad < P) Ppad <<= 1;
  const int NB = Ppad / SORT_BUCKET_KEYS;  // a power of two, <= 512
  const int nb_log2 = 31 - __clz(NB);
  const int b_lo = part * NB / split, b_hi = (part + 1) * NB / split;
  const int cslot = (wt0 + tc0) / C;
  const size_t cbase = (size_t)m * w.max_chunks + cslot;
  u64* out = w.sk + cbase * (size_t)(C * kh);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int b = tid; b < NB; b += SORT_THREADS) s_cnt[b] = 0;
  __syncthreads();
  u64 x[VPT];
  int bk[VPT];
  // every slot of this thread's pairs is loaded before the counting
  unsigned sl[VPT];
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = tid * VPT + u;
    sl[u] = 0u;
    if (i < P) {
      if (!HEADS) {
        sl[u] = (unsigned)w.idx[((size_t)m * w.max_T + wt0 + tc0) * k + i];
      } else {
        // pair i = (t_local H + head) k + r: slot r of the head's selection for token t_local
        const int t = i / kh, hr = i - t * kh, hd = hr / k, r = hr - hd * k;
        sl[u] = (unsigned)w.idx[(((size_t)m * H + hd) * w.max_T + wt0 + tc0 + t) * k + r];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = tid * VPT + u;
    u64 key = ~0ull;
    bk[u] = -1;
    if (i < P) {
      const unsigned slot = sl[u];
      key = ((u64)slot << 32) | (unsigned)i;
      bk[u] = NB > 1 ? (int)((slot * 2654435761u) >> (32 - nb_log2)) : 0;  // multiplicative hash
      atomicAdd(&s_cnt[bk[u]], 1);
    }
    x[u] = key;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the bucket sizes
    int run = 0;
    for (int b0 = 0; b0 < NB; b0 += 32) {
      const int v = b0 + lane < NB ? s_cnt[b0 + lane] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b0 + lane < NB) {
        s_off[b0 + lane] = run + incl - v;
        s_cur[b0 + lane] = run + incl - v;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[NB] = run;
  }
  __syncthreads();
  if (part == 0 && tid == 0) w.npairs[cbase] = P;
  // this CTA's buckets [b_lo, b_hi) occupy key positions [s_off[b_lo], s_off[b_hi])
  const int base0 = s_off[b_lo];
#pragma unroll
  for (int u = 0; u < VPT; ++u)
    if (bk[u] >= b_lo && bk[u] < b_hi) s_keys[atomicAdd(&s_cur[bk[u]], 1) - base0] = x[u];
  __syncthreads();
  // buckets of up to SORT_BUCKET_CAP keys: one warp each, every key ranked against the others
  for (int b = b_lo + warp; b < b_hi; b += SORT_THREADS / 32) {
    const int base = s_off[b] - base0, cnt = s_off[b + 1] - s_off[b];
    if (cnt == 0 || cnt > SORT_BUCKET_CAP) continue;
    u64 mine[SORT_BUCKET_CAP / 32];
    int rk[SORT_BUCKET_CAP / 32];
#pragma unroll
    for (int j = 0; j < SORT_BUCKET_CAP / 32; ++j) {
      const int i = lane + 32 * j;
      mine[j] = i < cnt ? s_keys[base + i] : ~0ull;
      rk[j] = 0;
    }
    if (cnt <= 64) {
      for (int t = 0; t < cnt; ++t) {
        const u64 o = s_keys[base + t];
        rk[0] += o < mine[0] ? 1 : 0;
        rk[1] += o < mine[1] ? 1 : 0;
      }
    } else {
      for (int t = 0; t < cnt; ++t) {
        const u64 o = s_keys[base + t];
#pragma unroll
        for (int j = 0; j < SORT_BUCKET_CAP / 32; ++j) rk[j] += o < mine[j] ? 1 : 0;
      }
    }
#pragma unroll
    for (int j = 0; j < SORT_BUCKET_CAP / 32; ++j)
      if (lane + 32 * j < cnt) out[s_off[b] + rk[j]] = mine[j];
  }
  // larger buckets (skewed slot use: a row read by many tokens of the chunk): the whole CTA
  // ranks each one, every thread a strided share of its keys against all of them (the
  // comparison reads are broadcasts); the output is the same as the warps' ranking
  for (int b = b_lo; b < b_hi; ++b) {
    const int base = s_off[b] - base0, cnt = s_off[b + 1] - s_off[b];
    if (cnt <= SORT_BUCKET_CAP) continue;
    for (int i0 = 0; i0 < cnt; i0 += 4 * SORT_THREADS) {
      u64 mine[4];
      int rk[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = i0 + tid + j * SORT_THREADS;
        mine[j] = i < cnt ? s_keys[base + i] : ~0ull;
        rk[j] = 0;
      }
      for (int t = 0; t < cnt; ++t) {
        const u64 o = s_keys[base + t];
#pragma unroll
        for (int j = 0; j < 4; ++j) rk[j] += o < mine[j] ? 1 : 0;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (i0 + tid + j * SORT_THREADS < cnt) out[s_off[b] + rk[j]] = mine[j];
    }
  }
}

int launch_sort_pairs(const Dims& d, const Work& w, int wt0, int total_len, bool last_has_target,
                      cudaStream_t s) {
  if (total_len <= 0) return 0;
  const int nchunks = (total_len + d.C - 1) / d.C;
  const int P = d.C * d.k * d.H;
  // CTAs per (table, chunk): a launch of several chunks (a frozen-key addressing window)
  // takes about one wave of 1024-thread CTAs (each CTA counts all of its chunk's keys, so
  // more CTAs than SMs only repeat that work: mid 30 against 136 us per window); a
  // one-chunk launch keeps SORT_SPLIT, which finishes sooner beside the gather it overlaps
  // (layer 2.745 against 2.89 ms per step).  FWPKM_SORT_SPLIT overrides both.
  static const int forced = [] {
    const char* e = getenv("FWPKM_SORT_SPLIT");
    return e ? atoi(e) : 0;
  }();
  static const int sms = [] {
    int dev = 0, v = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  int split = 1;
  const long long units = (long long)nchunks * d.B;
  if (nchunks == 1) split = SORT_SPLIT;
  while (split < SORT_SPLIT && units * split * 2 <= sms) split <<= 1;
  if (forced > 0) {
    split = 1;
    while (split < SORT_SPLIT && split * 2 <= forced) split <<= 1;
  }
  dim3 grid(nchunks * split, d.B);
  auto go = [&](auto kern, int vpt) {
    int Ppad = 32 * vpt;
    while (Ppad < P) Ppad <<= 1;
    const size_t smem = sizeof(u64) * (size_t)Ppad;
    if (!raise_smem_limit((const void*)kern, smem)) return -1;
    launch_k(kern, grid, SORT_THREADS, smem, s, d, w, wt0, total_len, last_has_target ? 1 : 0, split);
    return 1;
  };
  int rc;
  if (P <= 8 * SORT_THREADS)
    rc = d.H > 1 ? go(sort_pairs_kernel<8, true>, 8) : go(sort_pairs_kernel<8, false>, 8);
  else
    rc = d.H > 1 ? go(sort_pairs_kernel<16, true>, 16) : go(sort_pairs_kernel<16, false>, 16);
  if (rc < 0) return -1;
  return 1;
}

}  // namespace fwpkm
