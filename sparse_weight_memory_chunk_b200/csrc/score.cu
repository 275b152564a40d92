// score.cu -- sub-key distances and per-half top-k (SIMT path).
//
// Fast-weight Product Key Memory (paperlayer summary), §2.2: each half-query is
// scored against its own sub-key codebook; §A.2: the score is inverse-distance
// weighting on the Euclidean distance.  The per-half top-k keeps the k sub-keys of
// smallest squared distance, ties to the lower index.
//
// One CTA handles TQ tokens of one (memory, half).  It computes the squared
// distances to all n sub-keys in the direct form sum_e (q_e - K[a][e])^2 (fp32,
// one fused multiply-add per term, no cancellation), keeps the [TQ][n] rows in
// shared memory, and then each warp selects the k smallest of its rows.  With the
// key update enabled the rows (and sum_a 1/(eps + D)) are also written out for
// the entropy step, which needs every sub-key's distance.
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int SCORE_THREADS = 256;
constexpr int SCORE_KT = 64;  // sub-keys per shared-memory tile

template <typename QT, int TQ>
__global__ void __launch_bounds__(SCORE_THREADS)
score_topk_simt(Dims dm, Work w, const float* __restrict__ K1, const float* __restrict__ K2,
                const QT* __restrict__ q, long long q_stride, int wt0, int len, int key_update) {
  extern __shared__ float smem[];
  const int h = dm.h, n = dm.n, k = dm.k;
  const int m = blockIdx.y >> 1, j = blockIdx.y & 1;
  const int tt0 = blockIdx.x * TQ;
  const int ntok = min(TQ, len - tt0);
  const int hp = h + 1;  // padded row: conflict-free column reads
  float* q_s = smem;                 // [TQ][h]
  float* k_s = q_s + TQ * h;         // [KT][h+1]
  float* D_s = k_s + SCORE_KT * hp;  // [TQ][n]
  const float* K = (j == 0 ? K1 : K2) + (size_t)m * n * h;

  for (int i = threadIdx.x; i < TQ * h; i += SCORE_THREADS) {
    int tq = i / h, e = i - tq * h;
    float val = 0.f;
    if (tq < ntok) val = load_qv(q, ((long long)m * q_stride + tt0 + tq) * dm.d + (long long)j * h + e);
    q_s[i] = val;
  }
  constexpr int TPT = TQ / 4;  // tokens per thread
  const int kx = threadIdx.x % SCORE_KT, ty = threadIdx.x / SCORE_KT;
  for (int a0 = 0; a0 < n; a0 += SCORE_KT) {
    __syncthreads();
    const int nk = min(SCORE_KT, n - a0);
    for (int i = threadIdx.x; i < SCORE_KT * h; i += SCORE_THREADS) {
      int kk = i / h, e = i - kk * h;
      k_s[kk * hp + e] = kk < nk ? K[(size_t)(a0 + kk) * h + e] : 0.f;
    }
    __syncthreads();
    float acc[TPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i) acc[i] = 0.f;
    for (int e = 0; e < h; ++e) {
      const float kv = k_s[kx * hp + e];
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        float df = q_s[(ty + 4 * i) * h + e] - kv;
        acc[i] = fmaf(df, df, acc[i]);
      }
    }
    if (kx < nk) {
#pragma unroll
      for (int i = 0; i < TPT; ++i) D_s[(ty + 4 * i) * n + a0 + kx] = acc[i];
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = warp; row < ntok; row += SCORE_THREADS / 32) {
    const float* Drow = D_s + (size_t)row * n;
    const long long tok = (long long)wt0 + tt0 + row;
    if (key_update) {
      float z = 0.f;
      float* out = w.Dfull + (((size_t)m * 2 + j) * dm.C + tt0 + row) * n;
      for (int a = lane; a < n; a += 32) {
        float dv = Drow[a];
        out[a] = dv;
        z += 1.f / (dm.eps_idw + dv);
      }
      z = warp_sum(z);
      if (lane == 0) w.Z[((size_t)m * 2 + j) * dm.C + tt0 + row] = z;
    }
    // k smallest by (distance, index): keys are unique, so each round the winning
    // lane advances to its smallest key above the last winner.
    unsigned long long best = ~0ull;
    for (int a = lane; a < n; a += 32) {
      unsigned long long key = ((unsigned long long)orderable(Drow[a]) << 32) | (unsigned)a;
      best = key < best ? key : best;
    }
    const size_t obase = (((size_t)m * 2 + j) * w.max_T + tok) * k;
    for (int r = 0; r < k; ++r) {
      unsigned long long win = warp_min_u64(best);
      int a = (int)(win & 0xffffffffu);
      if (lane == 0) {
        w.A[obase + r] = a;
        w.Dsv[obase + r] = Drow[a];
      }
      if ((a & 31) == lane) {
        best = ~0ull;
        for (int b = lane; b < n; b += 32) {
          unsigned long long key = ((unsigned long long)orderable(Drow[b]) << 32) | (unsigned)b;
          if (key > win && key < best) best = key;
        }
      }
    }
  }
}

template <typename QT, int TQ>
static int launch_tq(const Dims& d, const Work& w, const float* K1, const float* K2, const void* q,
                     long long q_stride, int wt0, int len, bool key_update, cudaStream_t s) {
  size_t smem = sizeof(float) * ((size_t)TQ * d.h + (size_t)SCORE_KT * (d.h + 1) + (size_t)TQ * d.n);
  auto kern = score_topk_simt<QT, TQ>;
  if (!raise_smem_limit((const void*)kern, smem)) return -1;
  dim3 grid((len + TQ - 1) / TQ, d.M * 2);
  kern<<<grid, SCORE_THREADS, smem, s>>>(d, w, K1, K2, (const QT*)q, q_stride, wt0, len,
                                        key_update ? 1 : 0);
  return 1;
}

int launch_score_topk(const Dims& d, const Work& w, const float* K1, const float* K2, const void* q,
                      long long q_stride, int wt0, int len, bool key_update, cudaStream_t s) {
  if (len <= 0) return 0;
  // shared memory budget: TQ rows of n distances plus one sub-key tile
  int tq = 32;
  while (tq > 4 && (size_t)tq * d.n * 4 + (size_t)tq * d.h * 4 + (size_t)SCORE_KT * (d.h + 1) * 4 > 200 * 1024)
    tq >>= 1;
  if (d.qv_bf16) {
    if (tq == 32) return launch_tq<__nv_bfloat16, 32>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
    if (tq == 16) return launch_tq<__nv_bfloat16, 16>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
    if (tq == 8) return launch_tq<__nv_bfloat16, 8>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
    return launch_tq<__nv_bfloat16, 4>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
  }
  if (tq == 32) return launch_tq<float, 32>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
  if (tq == 16) return launch_tq<float, 16>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
  if (tq == 8) return launch_tq<float, 8>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
  return launch_tq<float, 4>(d, w, K1, K2, q, q_stride, wt0, len, key_update, s);
}

}  // namespace fwpkm
