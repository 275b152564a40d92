// address.cu -- entropy (anti-collapse) step on the sub-key codebooks.
//
// Fast-weight Product Key Memory (rainbus summary), method step 5: minimise
// L_addr = -H(pbar_1) - H(pbar_2) to update K1 and K2; (paperlayer summary) §3.4:
// pbar_j is the marginal slot-usage distribution of half j over the chunk.
// Reading: P_j[t] = softmax_a(-log(eps + D_j[t][a])) over all n sub-keys, i.e.
// P_j[t][a] = (eps + D)^-1 / Z_t, and pbar_j = mean_t P_j[t].  By the chain rule
//   dL/dsigma[t][b] = (1/len) P[t][b] (log pbar[b] - L_t),  L_t = sum_a P[t][a] log pbar[a]
//   dsigma/dK[b]    = 2 (q_t - K[b]) / (eps + D[t][b])
// so with W[t][b] = dL/dsigma[t][b] / (eps + D[t][b]):
//   dL/dK[b] = 2 (sum_t W[t][b] q_t - (sum_t W[t][b]) K[b]).
// The distances are those the chunk was read with (written by the scoring kernel).
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int ADDR_THREADS = 256;
constexpr int ADDR_KB = 8;  // sub-keys per CTA in the gradient kernel

// pbar and its log: one thread per (memory, half, sub-key), summing over the chunk.
__global__ void __launch_bounds__(ADDR_THREADS)
addr_pbar_kernel(Dims dm, Work w, int len) {
  __shared__ float s_invz[1024];
  const int mj = blockIdx.y;
  const float* Z = w.Z + (size_t)mj * dm.C;
  for (int t = threadIdx.x; t < len; t += ADDR_THREADS) s_invz[t] = 1.f / Z[t];
  __syncthreads();
  const int a = blockIdx.x * ADDR_THREADS + threadIdx.x;
  if (a >= dm.n) return;
  const float* D = w.Dfull + (size_t)mj * dm.C * dm.n;
  float s = 0.f;
  for (int t = 0; t < len; ++t) s += (1.f / (dm.eps_idw + D[(size_t)t * dm.n + a])) * s_invz[t];
  w.lp[(size_t)mj * dm.n + a] = logf(s / (float)len);
}

// L_t = sum_a P[t][a] log pbar[a]: one warp per (memory, half, token).
__global__ void __launch_bounds__(ADDR_THREADS)
addr_rowL_kernel(Dims dm, Work w, int len) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (ADDR_THREADS / 32) + warp;
  const int mj = blockIdx.y;
  if (t >= len) return;
  const float* D = w.Dfull + ((size_t)mj * dm.C + t) * dm.n;
  const float* lp = w.lp + (size_t)mj * dm.n;
  float s = 0.f;
  for (int a = lane; a < dm.n; a += 32) s += lp[a] / (dm.eps_idw + D[a]);
  s = warp_sum(s);
  if (lane == 0) w.Lt[(size_t)mj * dm.C + t] = s / w.Z[(size_t)mj * dm.C + t];
}

// Gradient and step for ADDR_KB sub-keys of one (memory, half).
template <typename QT>
__global__ void __launch_bounds__(ADDR_THREADS)
addr_update_kernel(Dims dm, Work w, float* __restrict__ K1, float* __restrict__ K2,
                   const QT* __restrict__ q, long long q_stride, int len) {
  __shared__ float s_W[ADDR_KB][1024];
  __shared__ float s_wsum[ADDR_KB];
  const int mj = blockIdx.y, m = mj >> 1, j = mj & 1;
  const int b0 = blockIdx.x * ADDR_KB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = dm.n, h = dm.h;
  const float inv_len = 1.f / (float)len;
  {  // warp `warp` builds W for sub-key b0 + warp
    const int b = b0 + warp;
    float part = 0.f;
    if (b < n) {
      const float* D = w.Dfull + (size_t)mj * dm.C * n;
      const float lpb = w.lp[(size_t)mj * n + b];
      for (int t = lane; t < len; t += 32) {
        const float inv = 1.f / (dm.eps_idw + D[(size_t)t * n + b]);
        const float P = inv / w.Z[(size_t)mj * dm.C + t];
        const float Wt = inv_len * P * (lpb - w.Lt[(size_t)mj * dm.C + t]) * inv;
        s_W[warp][t] = Wt;
        part += Wt;
      }
    }
    part = warp_sum(part);
    if (lane == 0) s_wsum[warp] = part;
  }
  __syncthreads();
  float* K = (j == 0 ? K1 : K2) + (size_t)m * n * h;
  const int kg = threadIdx.x >> 7;  // two groups of 128 threads, ADDR_KB/2 keys each
  for (int e = threadIdx.x & 127; e < h; e += 128) {
    float acc[ADDR_KB / 2];
#pragma unroll
    for (int i = 0; i < ADDR_KB / 2; ++i) acc[i] = 0.f;
    for (int t = 0; t < len; ++t) {
      const float qv = load_qv(q, ((long long)m * q_stride + t) * dm.d + (long long)j * h + e);
#pragma unroll
      for (int i = 0; i < ADDR_KB / 2; ++i) acc[i] = fmaf(s_W[kg * (ADDR_KB / 2) + i][t], qv, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < ADDR_KB / 2; ++i) {
      const int bl = kg * (ADDR_KB / 2) + i;
      const int b = b0 + bl;
      if (b < n) {
        float kv = K[(size_t)b * h + e];
        float grad = 2.f * (acc[i] - s_wsum[bl] * kv);
        K[(size_t)b * h + e] = kv - dm.lr_key * grad;
      }
    }
  }
}

int launch_address(const Dims& d, const Work& w, float* K1, float* K2, const void* q, long long q_stride,
                   int len, cudaStream_t s) {
  if (len <= 0) return 0;
  addr_pbar_kernel<<<dim3((d.n + ADDR_THREADS - 1) / ADDR_THREADS, d.M * 2), ADDR_THREADS, 0, s>>>(d, w, len);
  addr_rowL_kernel<<<dim3((len + 7) / 8, d.M * 2), ADDR_THREADS, 0, s>>>(d, w, len);
  dim3 grid((d.n + ADDR_KB - 1) / ADDR_KB, d.M * 2);
  if (d.qv_bf16)
    addr_update_kernel<__nv_bfloat16><<<grid, ADDR_THREADS, 0, s>>>(d, w, K1, K2, (const __nv_bfloat16*)q,
                                                                   q_stride, len);
  else
    addr_update_kernel<float><<<grid, ADDR_THREADS, 0, s>>>(d, w, K1, K2, (const float*)q, q_stride, len);
  return 3;
}

}  // namespace fwpkm
