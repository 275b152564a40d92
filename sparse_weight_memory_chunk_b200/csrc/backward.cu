// backward.cu -- the read path's backward: the gradient that reaches the slow weights'
// inputs q, v, g from dL/do.
//
// Fast-weight Product Key Memory (paperlayer summary) §2 / Figure 1 (slow weights learn
// during training, the fast key/value parameters online), §3.1-§3.2 (the slow-weight
// projections supply q, v, g; the read D_j[a] = ||q_j - K_j[a]||^2, sigma = -log(eps + D),
// S = sigma_1[a] + sigma_2[b], s' = softmax(S), vhat = sum s' V_i, o = g vhat + (1-g) v).
// The fast weights as they were at the chunk's read are constants here and the discrete
// selection passes no gradient, so per token with slots I (rank order):
//   dg = <dL/do, vhat - v>,  dv = (1 - g) dL/do,  ds_r = <g dL/do, V_{I_r}>,
//   dS_r = s'_r (ds_r - sum s' ds),  dq_j = sum_r dS_r (-2 / (eps + D_j)) (q_j - K_j[row_r]).
//
// One CTA of BW_WARPS warps per (memory, token); warp w takes a contiguous share of the
// ranks.  Pass 1: per rank, the two sub-key distances and dsraw_r = <dL/do, V_{I_r}> (lanes
// over the features and over d_v, warp sums), into shared memory.  Then one warp forms s',
// dS and the per-rank coefficients; dg needs no vhat: dg = sum_r s'_r dsraw_r - <dL/do, v>.
// Pass 2: each warp adds its ranks' terms of dq (the key rows come back from L2), and the
// partial rows are summed in warp order.
//
// The kernel is bound by the latency of its dependent rounds, not by bytes: on uniformly
// random slots at 1M slots, d = d_v = 256, k = 32 (2048 token-memories, L2 flushed), two
// warps per token took 39 us, four 41, eight 53, one warp per token with a serial rank loop
// 68; keeping pass 1's key differences in registers for pass 2 (fewer CTAs resident) and
// issuing the loads of 4-8 ranks unconditionally were both slower.
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int BW_WARPS = 2;  // warps per (memory, token)

template <typename VT>
__device__ __forceinline__ float ld_elem(const VT* p);
template <>
__device__ __forceinline__ float ld_elem<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float bw_warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float bw_warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// HPL: features per lane of one half (h <= 32 HPL); VPL: 16-byte vectors per lane of a
// value row (d_v <= 128 VPL).
template <typename VT, int HPL, int VPL>
__global__ void __launch_bounds__(BW_WARPS * 32)
read_backward_kernel(Dims dm, const float* __restrict__ K1, const float* __restrict__ K2,
                     const float* __restrict__ V, const VT* __restrict__ q, const VT* __restrict__ v,
                     const float* __restrict__ g, const int32_t* __restrict__ idx, const float* __restrict__ d_o,
                     int len, long long stride, float* __restrict__ dq, float* __restrict__ dv,
                     float* __restrict__ dg) {
  __shared__ float sD1[32], sD2[32], sDS[32], sC1[32], sC2[32];
  __shared__ float sdq[BW_WARPS][64 * HPL];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int m = blockIdx.y;
  const int k = dm.k, n = dm.n, h = dm.h, dv4 = dm.dv >> 2;
  const float eps = dm.eps_idw;
  const long long row = (long long)m * stride + i;
  const float* K1m = K1 + (size_t)m * n * h;
  const float* K2m = K2 + (size_t)m * n * h;
  const float4* Vm = reinterpret_cast<const float4*>(V + (size_t)m * dm.N * dm.dv);

  // the token's slots, one per lane (slots outside [0, N) contribute nothing)
  int slot = -1;
  if (lane < k) slot = idx[((size_t)m * len + i) * k + lane];
  const bool slot_ok = slot >= 0 && (long long)slot < dm.N;
  const int safe_slot = slot_ok ? slot : 0;
  float q1[HPL], q2[HPL];
#pragma unroll
  for (int u = 0; u < HPL; ++u) {
    const int e = lane + 32 * u;
    q1[u] = e < h ? ld_elem<VT>(q + row * dm.d + e) : 0.f;
    q2[u] = e < h ? ld_elem<VT>(q + row * dm.d + h + e) : 0.f;
  }
  float4 dO[VPL];
  const float4* dor = reinterpret_cast<const float4*>(d_o + row * dm.dv);
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    const int e4 = lane + 32 * c;
    dO[c] = e4 < dv4 ? dor[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int rpw = (k + BW_WARPS - 1) / BW_WARPS;  // ranks per warp
  const int r_lo = warp * rpw, r_hi = min(k, r_lo + rpw);

  // pass 1: D1_r, D2_r, dsraw_r for this warp's ranks, four at a time
  for (int r0 = r_lo; r0 < r_hi; r0 += 4) {
    float p1[4], p2[4], p3[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      p1[j] = p2[j] = p3[j] = 0.f;
      const int r = r0 + j;
      const int sr = __shfl_sync(0xffffffffu, safe_slot, r & 31);
      if (r < r_hi) {
        const int a = sr / n, b = sr - a * n;
#pragma unroll
        for (int u = 0; u < HPL; ++u) {
          const int e = lane + 32 * u;
          if (e < h) {
            const float d1 = q1[u] - K1m[(size_t)a * h + e];
            const float d2 = q2[u] - K2m[(size_t)b * h + e];
            p1[j] = fmaf(d1, d1, p1[j]);
            p2[j] = fmaf(d2, d2, p2[j]);
          }
        }
        const float4* vr = Vm + (size_t)sr * dv4;
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
          const int e4 = lane + 32 * c;
          if (e4 < dv4) {
            const float4 x = vr[e4];
            p3[j] = fmaf(dO[c].x, x.x, p3[j]); p3[j] = fmaf(dO[c].y, x.y, p3[j]);
            p3[j] = fmaf(dO[c].z, x.z, p3[j]); p3[j] = fmaf(dO[c].w, x.w, p3[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      p1[j] = bw_warp_sum(p1[j]);
      p2[j] = bw_warp_sum(p2[j]);
      p3[j] = bw_warp_sum(p3[j]);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (r0 + j < r_hi) {
          sD1[r0 + j] = p1[j];
          sD2[r0 + j] = p2[j];
          sDS[r0 + j] = p3[j];
        }
      }
    }
  }
  __syncthreads();

  // s', dS_r = g s'_r (dsraw_r - sum s' dsraw), the dq coefficients; dg and dv
  if (warp == 0) {
    const bool live = lane < k && slot_ok;
    const float D1 = live ? sD1[lane] : 0.f, D2 = live ? sD2[lane] : 0.f;
    const float dsr = live ? sDS[lane] : 0.f;
    const float S = live ? -logf(eps + D1) - logf(eps + D2) : -INFINITY;
    const float smax = bw_warp_max(S);
    const float ex = live ? expf(S - smax) : 0.f;
    const float s = ex / bw_warp_sum(ex);
    const float sds = bw_warp_sum(live ? s * dsr : 0.f);
    const float gt = g[row];
    const float dS = live ? gt * s * (dsr - sds) : 0.f;
    sC1[lane] = live ? -2.f * dS / (eps + D1) : 0.f;
    sC2[lane] = live ? -2.f * dS / (eps + D2) : 0.f;
    // dg = <dL/do, vhat - v> = sum s' dsraw - <dL/do, v>;  dv = (1 - g) dL/do
    float pv = 0.f;
    float4* dvr = reinterpret_cast<float4*>(dv + row * dm.dv);
    const float og = 1.f - gt;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const int e4 = lane + 32 * c;
      if (e4 < dv4) {
        const VT* vr = v + row * dm.dv + 4 * e4;
        pv = fmaf(dO[c].x, ld_elem<VT>(vr), pv); pv = fmaf(dO[c].y, ld_elem<VT>(vr + 1), pv);
        pv = fmaf(dO[c].z, ld_elem<VT>(vr + 2), pv); pv = fmaf(dO[c].w, ld_elem<VT>(vr + 3), pv);
        dvr[e4] = make_float4(og * dO[c].x, og * dO[c].y, og * dO[c].z, og * dO[c].w);
      }
    }
    pv = bw_warp_sum(pv);
    if (lane == 0) dg[row] = sds - pv;
  }
  __syncthreads();

  // pass 2: this warp's share of dq_j = sum_r c_j,r (q_j - K_j[row_r])
  float g1[HPL], g2[HPL];
#pragma unroll
  for (int u = 0; u < HPL; ++u) g1[u] = g2[u] = 0.f;
  for (int r0 = r_lo; r0 < r_hi; r0 += 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + j;
      const int sr = __shfl_sync(0xffffffffu, safe_slot, r & 31);
      if (r < r_hi) {
        const float cr1 = sC1[r], cr2 = sC2[r];
        const int a = sr / n, b = sr - a * n;
#pragma unroll
        for (int u = 0; u < HPL; ++u) {
          const int e = lane + 32 * u;
          if (e < h) {
            g1[u] = fmaf(cr1, q1[u] - K1m[(size_t)a * h + e], g1[u]);
            g2[u] = fmaf(cr2, q2[u] - K2m[(size_t)b * h + e], g2[u]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < HPL; ++u) {
    sdq[warp][lane + 32 * u] = g1[u];
    sdq[warp][32 * HPL + lane + 32 * u] = g2[u];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 2 * h; e += BW_WARPS * 32) {
    const int half = e >= h, f = e - half * h;
    const int o = half * 32 * HPL + f;
    float acc = sdq[0][o];
#pragma unroll
    for (int w = 1; w < BW_WARPS; ++w) acc += sdq[w][o];
    dq[row * dm.d + e] = acc;
  }
}

int launch_read_backward(const Dims& d, const float* K1, const float* K2, const float* V, const void* q,
                         const void* v, const float* g, const int32_t* idx, const float* d_o, int len,
                         long long stride, float* dq, float* dv, float* dg, cudaStream_t s) {
  if (len <= 0) return 0;
  const dim3 grid(len, d.M);
  const int hpl = (d.h + 31) / 32;
  const int vpl = (d.dv / 4 + 31) / 32;
  const int H = hpl <= 1 ? 1 : hpl <= 2 ? 2 : hpl <= 4 ? 4 : 8;
  const int W = vpl <= 1 ? 1 : vpl <= 2 ? 2 : vpl <= 4 ? 4 : 8;
#define FWPKM_BW_GO(VTT, HV, WV)                                                                                \
  launch_k(read_backward_kernel<VTT, HV, WV>, grid, BW_WARPS * 32, 0, s, d, K1, K2, V, (const VTT*)q,         \
           (const VTT*)v, g, idx, d_o, len, stride, dq, dv, dg)
#define FWPKM_BW_W(VTT, HV)                         \
  switch (W) {                                      \
    case 1: FWPKM_BW_GO(VTT, HV, 1); break;         \
    case 2: FWPKM_BW_GO(VTT, HV, 2); break;         \
    case 4: FWPKM_BW_GO(VTT, HV, 4); break;         \
    default: FWPKM_BW_GO(VTT, HV, 8); break;        \
  }
#define FWPKM_BW_H(VTT)                             \
  switch (H) {                                      \
    case 1: FWPKM_BW_W(VTT, 1); break;              \
    case 2: FWPKM_BW_W(VTT, 2); break;              \
    case 4: FWPKM_BW_W(VTT, 4); break;              \
    default: FWPKM_BW_W(VTT, 8); break;             \
  }
  if (d.qv_bf16) {
    FWPKM_BW_H(__nv_bfloat16);
  } else {
    FWPKM_BW_H(float);
  }
#undef FWPKM_BW_H
#undef FWPKM_BW_W
#undef FWPKM_BW_GO
  return 1;
}

}  // namespace fwpkm
