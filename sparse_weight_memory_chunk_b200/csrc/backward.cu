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
// One warp per (memory, token).  Pass 1 walks the ranks: the two sub-key distances of
// each selected slot (direct form, lanes over the features, a warp sum) and, with the
// softmax weights, the gathered row for vhat and ds (16-byte vector loads, lanes over
// d_v).  Pass 2 walks the ranks again for dq (the key rows are re-read from L1/L2).
#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int BW_WARPS = 8;

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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * BW_WARPS + warp;
  const int m = blockIdx.y;
  if (i >= len) return;
  const int k = dm.k, n = dm.n, h = dm.h, dv4 = dm.dv >> 2;
  const float eps = dm.eps_idw;
  const long long row = (long long)m * stride + i;
  const float* K1m = K1 + (size_t)m * n * h;
  const float* K2m = K2 + (size_t)m * n * h;
  const float4* Vm = reinterpret_cast<const float4*>(V + (size_t)m * dm.N * dm.dv);

  float q1[HPL], q2[HPL];
#pragma unroll
  for (int u = 0; u < HPL; ++u) {
    const int e = lane + 32 * u;
    q1[u] = e < h ? ld_elem<VT>(q + row * dm.d + e) : 0.f;
    q2[u] = e < h ? ld_elem<VT>(q + row * dm.d + h + e) : 0.f;
  }
  const float gt = g[row];
  float4 dO[VPL], xv[VPL];
  const float4* dor = reinterpret_cast<const float4*>(d_o + row * dm.dv);
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    const int e4 = lane + 32 * c;
    dO[c] = e4 < dv4 ? dor[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    if (e4 < dv4) {
      const VT* vr = v + row * dm.dv + 4 * e4;
      xv[c] = make_float4(ld_elem<VT>(vr), ld_elem<VT>(vr + 1), ld_elem<VT>(vr + 2), ld_elem<VT>(vr + 3));
    } else {
      xv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  // the token's slots, one per lane (slots outside [0, N) contribute nothing)
  int slot = -1;
  if (lane < k) slot = idx[((size_t)m * len + i) * k + lane];
  const bool slot_ok = slot >= 0 && (long long)slot < dm.N;

  // pass 1a: the two distances of every rank (lane r keeps rank r's)
  float myD1 = 0.f, myD2 = 0.f;
  for (int r = 0; r < k; ++r) {
    const int sr = __shfl_sync(0xffffffffu, slot_ok ? slot : 0, r);
    const int a = sr / n, b = sr - a * n;
    float p1 = 0.f, p2 = 0.f;
#pragma unroll
    for (int u = 0; u < HPL; ++u) {
      const int e = lane + 32 * u;
      if (e < h) {
        const float d1 = q1[u] - K1m[(size_t)a * h + e];
        const float d2 = q2[u] - K2m[(size_t)b * h + e];
        p1 = fmaf(d1, d1, p1);
        p2 = fmaf(d2, d2, p2);
      }
    }
    p1 = bw_warp_sum(p1);
    p2 = bw_warp_sum(p2);
    if (lane == r) {
      myD1 = p1;
      myD2 = p2;
    }
  }
  const bool live = lane < k && slot_ok;
  const float S = live ? -logf(eps + myD1) - logf(eps + myD2) : -INFINITY;
  const float smax = bw_warp_max(S);
  const float ex = live ? expf(S - smax) : 0.f;
  const float s = ex / bw_warp_sum(ex);

  // pass 1b: vhat and ds_r = <g dL/do, V_{slot_r}>
  float4 vhat[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) vhat[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  float myds = 0.f;
  for (int r = 0; r < k; ++r) {
    const int sr = __shfl_sync(0xffffffffu, slot_ok ? slot : 0, r);
    const float wr = __shfl_sync(0xffffffffu, s, r);
    const float4* vr = Vm + (size_t)sr * dv4;
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const int e4 = lane + 32 * c;
      if (e4 < dv4) {
        const float4 x = vr[e4];
        vhat[c].x = fmaf(wr, x.x, vhat[c].x); vhat[c].y = fmaf(wr, x.y, vhat[c].y);
        vhat[c].z = fmaf(wr, x.z, vhat[c].z); vhat[c].w = fmaf(wr, x.w, vhat[c].w);
        part = fmaf(dO[c].x, x.x, part); part = fmaf(dO[c].y, x.y, part);
        part = fmaf(dO[c].z, x.z, part); part = fmaf(dO[c].w, x.w, part);
      }
    }
    part = gt * bw_warp_sum(part);
    if (lane == r) myds = part;
  }
  // dg, dv
  float pg = 0.f;
  float4* dvr = reinterpret_cast<float4*>(dv + row * dm.dv);
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    const int e4 = lane + 32 * c;
    if (e4 < dv4) {
      pg = fmaf(dO[c].x, vhat[c].x - xv[c].x, pg); pg = fmaf(dO[c].y, vhat[c].y - xv[c].y, pg);
      pg = fmaf(dO[c].z, vhat[c].z - xv[c].z, pg); pg = fmaf(dO[c].w, vhat[c].w - xv[c].w, pg);
      const float og = 1.f - gt;
      dvr[e4] = make_float4(og * dO[c].x, og * dO[c].y, og * dO[c].z, og * dO[c].w);
    }
  }
  pg = bw_warp_sum(pg);
  if (lane == 0) dg[row] = pg;
  // dS_r = s'_r (ds_r - sum s' ds)
  const float sds = bw_warp_sum(live ? s * myds : 0.f);
  const float dS = live ? s * (myds - sds) : 0.f;
  const float c1 = live ? -2.f * dS / (eps + myD1) : 0.f;
  const float c2 = live ? -2.f * dS / (eps + myD2) : 0.f;

  // pass 2: dq_j = sum_r c_j,r (q_j - K_j[row_r]), in rank order
  float g1[HPL], g2[HPL];
#pragma unroll
  for (int u = 0; u < HPL; ++u) g1[u] = g2[u] = 0.f;
  for (int r = 0; r < k; ++r) {
    const int sr = __shfl_sync(0xffffffffu, slot_ok ? slot : 0, r);
    const float cr1 = __shfl_sync(0xffffffffu, c1, r), cr2 = __shfl_sync(0xffffffffu, c2, r);
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
#pragma unroll
  for (int u = 0; u < HPL; ++u) {
    const int e = lane + 32 * u;
    if (e < h) {
      dq[row * dm.d + e] = g1[u];
      dq[row * dm.d + h + e] = g2[u];
    }
  }
}

int launch_read_backward(const Dims& d, const float* K1, const float* K2, const float* V, const void* q,
                         const void* v, const float* g, const int32_t* idx, const float* d_o, int len,
                         long long stride, float* dq, float* dv, float* dg, cudaStream_t s) {
  if (len <= 0) return 0;
  const dim3 grid((len + BW_WARPS - 1) / BW_WARPS, d.M);
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
