// value_kernels.cu -- the HBM-bound value path: sparse read + gated output, reconstruction
// residuals, and the atomic-free fast-weight write.
//
// Fast-weight Product Key Memory (rainbus summary), method steps 2-4:
//   vhat_t = sum_{i in I_t} s'_{t,i} V_i;  o_t = g_t vhat_t + (1 - g_t) v_t;
//   L_mem = 1/2 sum_t g_t ||target_t - vhat_t||^2;  V_i -= (dL_mem/dV_i) / N_read,i.
// (paperlayer summary) §A.1 target = v_{t+1}; §A.3 z-scored target, no clipping;
// §A.4 summed (not averaged) loss, so the step is exactly the gradient; §A.5 gate
// weighting; §3.3 read-count averaging.
//
// Rows are moved as 16-byte vectors: a warp covers 512 contiguous bytes per load.  Both
// kernels are bound by HBM latency x bytes in flight, so each warp keeps many row loads
// outstanding before it consumes any of them.
#include <climits>
#include <cstdlib>
#include <mutex>

#include "fwpkm_internal.cuh"

namespace fwpkm {

constexpr int VAL_WARPS = 8;

template <typename VT>
__device__ __forceinline__ float4 load4(const VT* p, long long i4);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p, long long i4) {
  return reinterpret_cast<const float4*>(p)[i4];
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p, long long i4) {
  const __nv_bfloat162* q = reinterpret_cast<const __nv_bfloat162*>(p) + 2 * i4;
  float2 a = __bfloat1622float2(q[0]), b = __bfloat1622float2(q[1]);
  return make_float4(a.x, a.y, b.x, b.y);
}

// The gather streams V rows through L2 (64 MB per chunk, mostly read once): its loads
// carry an evict-first policy so that they do not push the addressing chain's working set
// (distance rows, key pieces, W) out of L2.  (The write's rows are left at the default:
// with the policy on its loads and stores the step was slower.)
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// COHERENT: the row may have been written earlier in the same launch by another SM (the
// persistent value loop), so the load goes to L2 (.cg) and never hits a stale L1 line.
template <bool COHERENT>
__device__ __forceinline__ float4 ld_stream(const float4* p, uint64_t pol) {
  float4 v;
  if (COHERENT)
    asm volatile("ld.global.cg.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
  else
    asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(pol));
  return v;
}
template <bool COHERENT>
__device__ __forceinline__ float4 ld_row4(const float4* p) {
  return COHERENT ? __ldcg(p) : *p;
}
// r = gw * (vhat - tau), tau = z(u) or u.  Shared by the fused and the streaming path
// so both give the same bits.
template <typename VT, int VPL>
__device__ __forceinline__ void load_row(const Dims& dm, const VT* u, float4 (&x)[VPL], int lane) {
  const int dv4 = dm.dv >> 2;
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    int e4 = lane + 32 * c;
    x[c] = (u && e4 < dv4) ? load4<VT>(u, e4) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// r from vhat and the target row already in registers (x, overwritten).
template <int VPL>
__device__ __forceinline__ void residual_of(const Dims& dm, const float4 (&vhat)[VPL], float4 (&x)[VPL],
                                            float gw, float4 (&r)[VPL], int lane) {
  const int dv4 = dm.dv >> 2;
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < VPL; ++c) s += (x[c].x + x[c].y) + (x[c].z + x[c].w);
  if (dm.flags & FWPKM_TARGET_NORM) {
    const float mean = warp_sum(s) / (float)dm.dv;
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      int e4 = lane + 32 * c;
      if (e4 < dv4) {
        float a = x[c].x - mean, b = x[c].y - mean, cc = x[c].z - mean, dd = x[c].w - mean;
        ss += (a * a + b * b) + (cc * cc + dd * dd);
      }
    }
    const float var = warp_sum(ss) / (float)dm.dv;
    const float inv = 1.0f / sqrtf(var + dm.eps_norm);
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      x[c].x = (x[c].x - mean) * inv; x[c].y = (x[c].y - mean) * inv;
      x[c].z = (x[c].z - mean) * inv; x[c].w = (x[c].w - mean) * inv;
    }
  }
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    r[c].x = gw * (vhat[c].x - x[c].x); r[c].y = gw * (vhat[c].y - x[c].y);
    r[c].z = gw * (vhat[c].z - x[c].z); r[c].w = gw * (vhat[c].w - x[c].w);
  }
}

template <typename VT, int VPL>
__device__ __forceinline__ void residual(const Dims& dm, const float4 (&vhat)[VPL], const VT* u,
                                         float gw, float4 (&r)[VPL], int lane) {
  float4 x[VPL];
  load_row<VT, VPL>(dm, u, x, lane);
  residual_of<VPL>(dm, vhat, x, gw, r, lane);
}

// Lookahead source of local token i, or nullptr if it has no target.
template <typename VT>
__device__ __forceinline__ const VT* target_src(const Dims& dm, const VT* v, const VT* v_next,
                                                long long stride, int m, int i, int len) {
  if (!(dm.flags & FWPKM_LOOKAHEAD)) return v + ((long long)m * stride + i) * dm.dv;
  if (i + 1 < len) return v + ((long long)m * stride + i + 1) * dm.dv;
  if (v_next) return v_next + (long long)m * stride * dm.dv;
  return nullptr;
}

// ---------------------------------------------------------------------------
// Gather: two warps per (memory, token), GATHER_TOK tokens per CTA.  Warp half h reads the
// rows of ranks [16h, 16h + 16) with 16-byte loads, all in flight at once, and sums them in
// rank order; warp half 0 adds half 1's sum (a fixed order), then forms o and the residual.
// With at most 16 rows per token half 1 would read nothing, so one warp takes the token
// (split = false: VAL_WARPS tokens per CTA); the sum is the same, since half 0 would only
// have added half 1's +0.
// The token's own value row and gate are loaded before the rows so that their latency
// overlaps the gather.
// ---------------------------------------------------------------------------
constexpr int GATHER_TOK = VAL_WARPS / 2;
__host__ __device__ __forceinline__ bool gather_split(const Dims& dm) { return dm.k * (dm.H > 1 ? dm.H : 1) > 16; }
// HEADS: the memories of a sequence share its value table (dm.H > 1, up to 64 rows per
// token); false compiles the one-head kernel (k <= 32 rows, one entry per lane).
//
// gather_token is one token's read by its two warps (`half` 0 and 1; with split false by one
// warp, half 0): every thread of the CTA calls it, inactive tokens too, since it holds a CTA
// barrier when split.  s_tok is the token's slot of the CTA's partial-sum array.  m is the
// value table (sequence); its heads are memories m H .. m H + H - 1.
template <typename VT, int VPL, bool HEADS, bool COHERENT, bool SPLIT>
__device__ __forceinline__ void gather_token(const Dims& dm, const Work& w, const float* __restrict__ V,
                                             const VT* __restrict__ v, const float* __restrict__ g,
                                             long long stride, int wt0, int len, float* __restrict__ o,
                                             int fuse_resid, const VT* __restrict__ v_next, int m, int i,
                                             bool active, int half, int lane, float4 (*s_tok)[32]) {
  const int k = dm.k, dv4 = dm.dv >> 2, H = HEADS ? dm.H : 1;
  const int R = H * k;       // rows read by the token: entry e = (head e / k, rank e % k)
  const long long tok = (long long)wt0 + i;
  // lane l holds entries l and l + 32: slot and weight s'/H (H = 1: the weight itself)
  int myslot = 0, myslot2 = 0;
  float myw = 0.f, myw2 = 0.f;
  const float invH = 1.f / (float)H;
  if (active && !HEADS) {
    if (lane < k) {
      myslot = w.idx[((size_t)m * w.max_T + tok) * k + lane];
      myw = w.w[((size_t)m * w.max_T + tok) * k + lane];
    }
  } else if (active) {
    if (lane < R) {
      const size_t o = (((size_t)m * H + lane / k) * w.max_T + tok) * k + lane % k;
      myslot = w.idx[o];
      myw = w.w[o] * invH;
    }
    if (lane + 32 < R) {
      const size_t o = (((size_t)m * H + (lane + 32) / k) * w.max_T + tok) * k + (lane + 32) % k;
      myslot2 = w.idx[o];
      myw2 = w.w[o] * invH;
    }
  }
  // half 0 prefetches the token's value row, gate and write target (no V row is needed for
  // them, so their loads overlap the gather instead of following it)
  float4 xv[VPL], tv[VPL];
  float gt = 0.f;
  const VT* u = (active && fuse_resid) ? target_src<VT>(dm, v, v_next, stride, m, i, len) : nullptr;
  if (active && half == 0) {
    gt = g[(long long)m * stride + i];
    load_row<VT, VPL>(dm, v + ((long long)m * stride + i) * dm.dv, xv, lane);
    load_row<VT, VPL>(dm, u, tv, lane);
  }
  const float4* Vm = reinterpret_cast<const float4*>(V + (size_t)m * dm.N * dm.dv);
  float4 acc[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  // warp half 0 sums entries [0, HALF), half 1 [HALF, R) (HALF = 16 when R <= 32)
  const int HALF = R <= 32 ? 16 : (R + 1) / 2;
  const int r0 = half * HALF, r1 = min(R, r0 + HALF);
  const uint64_t pol = evict_first_policy();
  if (active) {
#pragma unroll 16
    for (int r = r0; r < r1; ++r) {
      const int slot = __shfl_sync(0xffffffffu, (!HEADS || r < 32) ? myslot : myslot2, r & 31);
      const float wr = __shfl_sync(0xffffffffu, (!HEADS || r < 32) ? myw : myw2, r & 31);
      const float4* row = Vm + (size_t)slot * dv4;
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        int e4 = lane + 32 * c;
        if (e4 < dv4) {
          float4 x = ld_stream<COHERENT>(row + e4, pol);
          acc[c].x = fmaf(wr, x.x, acc[c].x); acc[c].y = fmaf(wr, x.y, acc[c].y);
          acc[c].z = fmaf(wr, x.z, acc[c].z); acc[c].w = fmaf(wr, x.w, acc[c].w);
        }
      }
    }
  }
  if (SPLIT) {
    if (half == 1) {
#pragma unroll
      for (int c = 0; c < VPL; ++c) s_tok[c][lane] = acc[c];
    }
    __syncthreads();
    if (half == 1 || !active) return;
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      const float4 b = s_tok[c][lane];
      acc[c].x += b.x; acc[c].y += b.y; acc[c].z += b.z; acc[c].w += b.w;
    }
  } else if (!active) {
    return;
  }
  float4* orow = reinterpret_cast<float4*>(o + ((long long)m * stride + i) * dm.dv);
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    int e4 = lane + 32 * c;
    if (e4 < dv4) {
      const float4 x = xv[c];
      float4 y;
      y.x = gt * acc[c].x + (1.f - gt) * x.x; y.y = gt * acc[c].y + (1.f - gt) * x.y;
      y.z = gt * acc[c].z + (1.f - gt) * x.z; y.w = gt * acc[c].w + (1.f - gt) * x.w;
      orow[e4] = y;
    }
  }
  // resid rows are chunk-local: a call may start inside a chunk (token-at-a-time reads)
  float4* rrow = reinterpret_cast<float4*>(w.resid + ((size_t)m * dm.C + wt0 % dm.C + i) * dm.dv);
  if (fuse_resid) {
    if (u == nullptr) return;
    const float gw = (dm.flags & FWPKM_GATE_WEIGHT) ? gt : 1.f;
    float4 r[VPL];
    residual_of<VPL>(dm, acc, tv, gw, r, lane);
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      int e4 = lane + 32 * c;
      if (e4 < dv4) rrow[e4] = r[c];
    }
  } else {
#pragma unroll
    for (int c = 0; c < VPL; ++c) {
      int e4 = lane + 32 * c;
      if (e4 < dv4) rrow[e4] = acc[c];
    }
  }
}

template <typename VT, int VPL, bool HEADS, bool SPLIT>
__global__ void __launch_bounds__(VAL_WARPS * 32, 4)
gather_kernel(Dims dm, Work w, const float* __restrict__ V, const VT* __restrict__ v,
              const float* __restrict__ g, long long stride, int wt0, int len, float* __restrict__ o,
              int fuse_resid, const VT* __restrict__ v_next) {
  pdl_wait();
  pdl_trigger();
  __shared__ float4 s_part[GATHER_TOK][VPL][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tl = SPLIT ? warp >> 1 : warp;
  const int i = blockIdx.x * (SPLIT ? GATHER_TOK : VAL_WARPS) + tl;
  gather_token<VT, VPL, HEADS, false, SPLIT>(dm, w, V, v, g, stride, wt0, len, o, fuse_resid, v_next, blockIdx.y, i,
                                             i < len, SPLIT ? warp & 1 : 0, lane, s_part[SPLIT ? tl : 0]);
}

// Streaming path: resid holds vhat from the forward call; turn it into r_t in place.
template <typename VT, int VPL>
__global__ void __launch_bounds__(VAL_WARPS * 32)
resid_kernel(Dims dm, Work w, const VT* __restrict__ v, const float* __restrict__ g, long long stride,
             int len, const VT* __restrict__ v_next) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * VAL_WARPS + warp;
  const int m = blockIdx.y;
  if (i >= len) return;
  const int dv4 = dm.dv >> 2;
  const VT* u = target_src<VT>(dm, v, v_next, stride, m, i, len);
  if (u == nullptr) return;
  float4* rrow = reinterpret_cast<float4*>(w.resid + ((size_t)m * dm.C + i) * dm.dv);
  float4 vh[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    int e4 = lane + 32 * c;
    vh[c] = e4 < dv4 ? rrow[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float gt = g[(long long)m * stride + i];
  const float gw = (dm.flags & FWPKM_GATE_WEIGHT) ? gt : 1.f;
  float4 r[VPL];
  residual<VT, VPL>(dm, vh, u, gw, r, lane);
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    int e4 = lane + 32 * c;
    if (e4 < dv4) rrow[e4] = r[c];
  }
}

// ---------------------------------------------------------------------------
// Write: the chunk's read pairs are sorted so that each touched row's pairs are
// contiguous and in token order.  Each warp owns G consecutive list positions; a
// position whose slot differs from its predecessor's starts a segment (one touched row)
// and that segment belongs to the warp, even where it runs past the warp's positions.
// The warp issues the value-row loads of all its segments before consuming any, then for
// each row sums G_i = sum s'_{t,i} r_t in token order and stores V_i - G_i / N_read,i.
// Rows are disjoint, so there are no atomics and the result does not depend on
// scheduling.
// ---------------------------------------------------------------------------
template <int VPL, int G>
__global__ void __launch_bounds__(VAL_WARPS * 32)
write_kernel(Dims dm, Work w, float* __restrict__ V, int wt0) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.y;
  const int C = dm.C, k = dm.k, dv4 = dm.dv >> 2;
  const int kshift = (k & (k - 1)) == 0 ? __popc(k - 1) : -1;  // t = pair / k by a shift when k is 2^s
  const int cslot = wt0 / C;
  const size_t cbase = (size_t)m * w.max_chunks + cslot;
  const int P = w.npairs[cbase];
  const unsigned long long* sk = w.sk + cbase * (size_t)(C * k);
  const float* wrow = w.w + ((size_t)m * w.max_T + wt0) * k;  // pair t*k + r of the chunk at wrow[t*k + r]
  float* Vm = V + (size_t)m * dm.N * dm.dv;
  // the CTAs of a memory cover its list in strides (grid sized to the resident CTAs)
  for (int pos0 = (blockIdx.x * VAL_WARPS + warp) * G; pos0 < P; pos0 += gridDim.x * VAL_WARPS * G) {
    unsigned long long my_key = ~0ull;
    bool head = false;
    if (lane < G && pos0 + lane < P) {
      const int pos = pos0 + lane;
      my_key = sk[pos];
      head = pos == 0 || (sk[pos - 1] >> 32) != (my_key >> 32);
    }
    const unsigned heads = __ballot_sync(0xffffffffu, head);
    const int my_slot = (int)(my_key >> 32);
    float4 Vr[G][VPL];
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      const int slot = __shfl_sync(0xffffffffu, my_slot, gi);
      const bool ok = ((heads >> gi) & 1u) && slot >= 0 && (long long)slot < dm.N;
      const float4* row = reinterpret_cast<const float4*>(Vm + (size_t)(ok ? slot : 0) * dm.dv);
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        const int e4 = lane + 32 * c;
        Vr[gi][c] = (ok && e4 < dv4) ? row[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int gi = 0; gi < G; ++gi) {
      const unsigned long long key0 = __shfl_sync(0xffffffffu, my_key, gi);
      if (!((heads >> gi) & 1u)) continue;
      const int slot = (int)(key0 >> 32);
      if (slot < 0 || (long long)slot >= dm.N) {
        if (lane == 0) raise_status(w.status, w.hstat, DEV_BAD_SLOT);
        continue;
      }
      float4 Gs[VPL];
#pragma unroll
      for (int c = 0; c < VPL; ++c) Gs[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      int p = pos0 + gi;
      unsigned long long key = key0;
      for (;;) {
        const uint32_t tr = (uint32_t)(key & 0xffffffffu);
        const int t_local = kshift >= 0 ? (int)(tr >> kshift) : (int)(tr / (uint32_t)k);
        const float wt = wrow[tr];
        const float4* rrow = reinterpret_cast<const float4*>(w.resid + ((size_t)m * C + t_local) * dm.dv);
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
          const int e4 = lane + 32 * c;
          if (e4 < dv4) {
            const float4 x = rrow[e4];
            Gs[c].x = fmaf(wt, x.x, Gs[c].x); Gs[c].y = fmaf(wt, x.y, Gs[c].y);
            Gs[c].z = fmaf(wt, x.z, Gs[c].z); Gs[c].w = fmaf(wt, x.w, Gs[c].w);
          }
        }
        if (++p >= P) break;
        key = sk[p];
        if ((int)(key >> 32) != slot) break;
      }
      const float inv = 1.f / (float)(p - (pos0 + gi));
      float4* row = reinterpret_cast<float4*>(Vm + (size_t)slot * dm.dv);
#pragma unroll
      for (int c = 0; c < VPL; ++c) {
        const int e4 = lane + 32 * c;
        if (e4 < dv4) {
          float4 x = Vr[gi][c];
          x.x = fmaf(-Gs[c].x, inv, x.x); x.y = fmaf(-Gs[c].y, inv, x.y);
          x.z = fmaf(-Gs[c].z, inv, x.z); x.w = fmaf(-Gs[c].w, inv, x.w);
          row[e4] = x;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Write, batched: each warp owns a contiguous range [r0, r1) of one memory's sorted pair
// list and every segment (touched row) whose first pair lies in it, even where the
// segment runs past r1; positions before its first head belong to a peer's segment.  The
// warp reads the list in windows of 32 positions (one key per lane and the key before it,
// in one round trip: a position is a segment head where the slot changes) and consumes
// each window in batches of WB positions: it issues the residual-row and weight loads of
// the batch's pairs and the V-row loads of the segments that start in it, all at once,
// then accumulates G_i = sum s'_{t,i} r_t in list order (token order within a segment) and
// stores V_i - G_i / N_read,i at each segment's last pair.  A segment still open at the end
// of a window is carried (V row, partial sum, count) into the next window, so the additions
// happen in the same order as in a serial walk of the segment.
// ---------------------------------------------------------------------------
constexpr int WR_WARPS = 4;

template <int VPL>
__device__ __forceinline__ void store_row(float* Vm, int slot, const Dims& dm, const float4 (&cv)[VPL],
                                          const float4 (&acc)[VPL], int nr, int lane) {
  float4* row = reinterpret_cast<float4*>(Vm + (size_t)slot * dm.dv);
  // one reciprocal per row (exact for the common N_read = 1, 2, 4)
  const float inv = 1.f / (float)nr;
  const int dv4 = dm.dv >> 2;
#pragma unroll
  for (int c = 0; c < VPL; ++c) {
    const int e4 = lane + 32 * c;
    if (e4 < dv4) {
      float4 x = cv[c];
      x.x = fmaf(-acc[c].x, inv, x.x); x.y = fmaf(-acc[c].y, inv, x.y);
      x.z = fmaf(-acc[c].z, inv, x.z); x.w = fmaf(-acc[c].w, inv, x.w);
      row[e4] = x;
    }
  }
}

// HEADS: the memories of a sequence share its value table (dm.H > 1): weights s'/H and
// N_read counted in distinct tokens; false compiles the one-head kernel (N_read = pairs).
// write_warp is the work of warp wi of table m's warps_per_mem warps.
template <int VPL, int WB, bool HEADS, bool COHERENT>
__device__ __forceinline__ void write_warp(const Dims& dm, const Work& w, float* __restrict__ V, int wt0, int m,
                                           int wi, int warps_per_mem, int lane) {
  const int C = dm.C, k = dm.k, dv4 = dm.dv >> 2, H = HEADS ? dm.H : 1, kh = k * H;
  const int kshift = (kh & (kh - 1)) == 0 ? __popc(kh - 1) : -1;
  const float invH = 1.f / (float)H;
  const size_t cbase = (size_t)m * w.max_chunks + wt0 / C;
  const int P = w.npairs[cbase];
  const int r0 = (int)((long long)P * wi / warps_per_mem), r1 = (int)((long long)P * (wi + 1) / warps_per_mem);
  if (r0 >= r1) return;
  const unsigned long long* sk = w.sk + cbase * (size_t)(C * kh);
  const float* wrow = w.w + ((size_t)m * w.max_T + wt0) * k;  // one head: pair t k + r at wrow[t k + r]
  const float4* resid = reinterpret_cast<const float4*>(w.resid + (size_t)m * C * dm.dv);
  float* Vm = V + (size_t)m * dm.N * dm.dv;
  // the open segment: cur = its slot (-1: none open; -2: a slot outside [0, N), skipped),
  // its V row cv, partial sum acc, and N_read = the tokens it has met (a token may read
  // the row through several heads; their pairs are adjacent) with the last of them
  int cur = -1, nr = 0, last_t = -1;
  float4 cv[VPL], acc[VPL];
#pragma unroll
  for (int c = 0; c < VPL; ++c) cv[c] = acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  bool started = false;
  for (int pos0 = r0; pos0 < P; pos0 += 32) {
    const int pos = pos0 + lane;
    unsigned long long key = ~0ull, prv = ~0ull;
    if (pos < P) {
      key = sk[pos];
      if (pos > 0) prv = sk[pos - 1];
    }
    const bool head = pos < P && (pos == 0 || (prv >> 32) != (key >> 32));
    const unsigned hm = __ballot_sync(0xffffffffu, head);
    // the segment carried from the previous window ends before this window's first head
    if (cur != -1 && (hm & 1u)) {
      if (cur >= 0) store_row<VPL>(Vm, cur, dm, cv, acc, nr, lane);
      cur = -1;
    }
    // heads at positions >= r1 start peers' segments: the first of them ends this warp's work
    const int rel = r1 - pos0;
    const unsigned beyond = rel >= 32 ? 0u : (rel <= 0 ? 0xffffffffu : (0xffffffffu << rel));
    const unsigned stop_heads = hm & beyond;
    const int stop = stop_heads ? pos0 + __ffs(stop_heads) - 1 : P;  // first position not this warp's
    int first = 0;
    if (!started) {
      if (!hm) {
        if (rel <= 32) break;  // no head left in [r0, r1): the range is a peer's tail
        continue;
      }
      first = __ffs(hm) - 1;
      if (pos0 + first >= r1) break;  // likewise
      started = true;
    }
    const int lim = stop - pos0 < 32 ? stop - pos0 : 32;  // positions [first, lim) of this window are ours
#pragma unroll 1
    for (int b0 = first; b0 < lim; b0 += WB) {
      // ---- issue every load of the batch ----
      float4 R[WB][VPL], Vh[WB][VPL];
      float wt[WB];
      int tl_[HEADS ? WB : 1];
#pragma unroll
      for (int u = 0; u < WB; ++u) {
        const int l = b0 + u;
        const bool in = l < lim;
        const unsigned long long ku = __shfl_sync(0xffffffffu, key, l & 31);
        const bool hd = in && ((hm >> (l & 31)) & 1u);
        const uint32_t tr = (uint32_t)(ku & 0xffffffffu);
        const int slot = (int)(ku >> 32);
        const bool okslot = slot >= 0 && (long long)slot < dm.N;
        // pair tr = (t_local H + head) k + r: weight s'/H of the head's rank r for the token
        const int t_local = kshift >= 0 ? (int)(tr >> kshift) : (int)(tr / (uint32_t)kh);
        if (HEADS) {
          const int hr = (int)tr - t_local * kh, head = hr / k, rk = hr - head * k;
          wt[u] = in ? w.w[(((size_t)m * H + head) * w.max_T + wt0 + t_local) * k + rk] * invH : 0.f;
          tl_[u] = t_local;
        } else {
          wt[u] = in ? wrow[tr] : 0.f;
        }
        const float4* rr = resid + (size_t)(in ? t_local : 0) * dv4;
        const float4* vr = reinterpret_cast<const float4*>(Vm + (size_t)(hd && okslot ? slot : 0) * dm.dv);
#pragma unroll
        for (int c = 0; c < VPL; ++c) {
          const int e4 = lane + 32 * c;
          R[u][c] = (in && e4 < dv4) ? ld_row4<COHERENT>(rr + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
          Vh[u][c] = (hd && okslot && e4 < dv4) ? ld_row4<COHERENT>(vr + e4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      // ---- accumulate in list order; a segment is stored at its last pair ----
#pragma unroll
      for (int u = 0; u < WB; ++u) {
        const int l = b0 + u;
        if (l >= lim) break;
        if ((hm >> l) & 1u) {
          const int slot = (int)(__shfl_sync(0xffffffffu, key, l) >> 32);
          if (slot < 0 || (long long)slot >= dm.N) {
            if (lane == 0) raise_status(w.status, w.hstat, DEV_BAD_SLOT);
            cur = -2;
          } else {
            cur = slot;
#pragma unroll
            for (int c = 0; c < VPL; ++c) {
              cv[c] = Vh[u][c];
              acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            nr = 0;
            last_t = -1;
          }
        }
        if (cur >= 0) {
          const float a = wt[u];
#pragma unroll
          for (int c = 0; c < VPL; ++c) {
            acc[c].x = fmaf(a, R[u][c].x, acc[c].x); acc[c].y = fmaf(a, R[u][c].y, acc[c].y);
            acc[c].z = fmaf(a, R[u][c].z, acc[c].z); acc[c].w = fmaf(a, R[u][c].w, acc[c].w);
          }
          if (!HEADS) {
            ++nr;
          } else if (tl_[u] != last_t) {
            ++nr;
            last_t = tl_[u];
          }
        }
        // the segment ends at this pair if the next position starts another one or the list
        // ends; at the window's last position the next head is only known in the next window
        const int nx = pos0 + l + 1;
        const bool ends = nx >= P || (l < 31 && ((hm >> (l + 1)) & 1u));
        if (ends && cur != -1) {
          if (cur >= 0) store_row<VPL>(Vm, cur, dm, cv, acc, nr, lane);
          cur = -1;
        }
      }
    }
    if (lim < 32) break;  // a peer's head (or the list's end) was reached in this window
  }
}

template <int VPL, int WB, bool HEADS>
__global__ void __launch_bounds__(WR_WARPS * 32)
write_batched_kernel(Dims dm, Work w, float* __restrict__ V, int wt0, int warps_per_mem) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * WR_WARPS + warp;
  const int m = gw / warps_per_mem, wi = gw - m * warps_per_mem;  // m: the value table (sequence)
  if (m >= dm.B) return;
  write_warp<VPL, WB, HEADS, false>(dm, w, V, wt0, m, wi, warps_per_mem, lane);
}

// ---------------------------------------------------------------------------
// Persistent value loop (frozen keys).  With the slot lists of a run of chunks already
// made, one launch takes every chunk of the run through its read (gather_token, all tables)
// and its write (write_warp, all tables) on every SM: no launch, ramp or drain per kernel.
// Two grid-wide arrivals order the phases: the write of chunk c starts when every
// residual of c is stored, the read of c+1 when every row of c's write is stored.  Rows
// and residuals made inside the launch are read through L2 (COHERENT loads).  The grid is
// launched cooperatively and never exceeds the CTAs that fit on the GPU, so each CTA it
// waits for is resident; each wait is still bounded (VL_TIMEOUT_NS), after which the CTA
// latches FWPKM_ERR_TIMEOUT and returns, leaving the counters for fwpkm_sync to clear.
// The arithmetic is that of the per-chunk kernels, in the same order: the bits agree.
// ---------------------------------------------------------------------------
constexpr uint64_t VL_TIMEOUT_NS = 200ull * 1000 * 1000;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t vl_clock() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Arrive on the grid counter and wait until `target` CTAs have arrived in total.  False:
// this CTA gave up (the counter did not reach the target in time).
__device__ __forceinline__ bool grid_arrive_wait(unsigned* cnt, unsigned target, const Work& w, int* s_abort) {
  __syncthreads();  // this CTA's stores of the phase are issued
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(cnt, 1u);
    const uint64_t deadline = vl_clock() + VL_TIMEOUT_NS;
    uint32_t spins = 0;
    while (ld_acquire_u32(cnt) < target) {
      __nanosleep(32);
      if ((++spins & 15u) == 0 && vl_clock() > deadline) {
        raise_status(w.status, w.hstat, DEV_TIMEOUT);
        *s_abort = 1;
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return *s_abort == 0;
}

template <int VPL>
struct VlOcc {  // CTAs per SM the loop is compiled for (the write holds up to ~176 registers)
  static constexpr int value = VPL <= 4 ? 2 : 1;
};

template <typename VT, int VPL, int WB, bool HEADS, bool SPLIT>
__global__ void __launch_bounds__(VAL_WARPS * 32, VlOcc<VPL>::value)
value_loop_kernel(Dims dm, Work w, float* __restrict__ V, const VT* __restrict__ v, const float* __restrict__ g,
                  int T, int c0, int c1, float* __restrict__ o, int warps_per_mem, int stall) {
  __shared__ float4 s_part[GATHER_TOK][VPL][32];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tpc = SPLIT ? GATHER_TOK : VAL_WARPS;  // tokens per CTA per iteration
  const int tl = SPLIT ? warp >> 1 : warp, half = SPLIT ? warp & 1 : 0;
  if (threadIdx.x == 0) s_abort = 0;
  unsigned* arrivals = w.vl_cnt;
  unsigned* exits = w.vl_cnt + 1;
  const unsigned G = gridDim.x;
  // test hook: the first wait's target is one no launch reaches
  unsigned target = stall ? 0x40000000u : 0u;
  const int C = dm.C, dv = dm.dv;
  for (int c = c0; c < c1; ++c) {
    const int t0 = c * C, len = T - t0 < C ? T - t0 : C;
    const VT* vc = v + (long long)t0 * dv;
    const VT* vn = (t0 + len < T) ? v + (long long)(t0 + len) * dv : nullptr;
    if (c > c0) {  // the previous chunk's rows are written
      target += G;
      if (!grid_arrive_wait(arrivals, target, w, &s_abort)) return;
    }
    const int ntok = dm.B * len;
    for (int base = blockIdx.x * tpc; base < ntok; base += G * tpc) {
      const int j = base + tl;
      const bool active = j < ntok;
      const int m = active ? j / len : 0, i = active ? j - m * len : 0;
      gather_token<VT, VPL, HEADS, true, SPLIT>(dm, w, V, vc, g + t0, T, t0, len, o + (long long)t0 * dv, 1, vn, m,
                                                i, active, half, lane, s_part[SPLIT ? tl : 0]);
      if (SPLIT) __syncthreads();  // s_part is refilled by the next token
    }
    target += G;
    if (!grid_arrive_wait(arrivals, target, w, &s_abort)) return;  // every residual of chunk c is stored
    const int nvw = dm.B * warps_per_mem;
    for (int vw = blockIdx.x * VAL_WARPS + warp; vw < nvw; vw += G * VAL_WARPS) {
      const int m = vw / warps_per_mem;
      write_warp<VPL, WB, HEADS, true>(dm, w, V, t0, m, vw - m * warps_per_mem, warps_per_mem, lane);
    }
  }
  // the last CTA out (every CTA has passed every wait) zeroes the counters for the next launch
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(exits, 1u) == G - 1) {
      *arrivals = 0;
      *exits = 0;
      __threadfence();
    }
  }
}

// ---- launchers ----
static int vpl_of(int dv) {
  int v = (dv / 4 + 31) / 32;
  return v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : 8;
}

#define FWPKM_VPL_DISPATCH(VPLV, ...)            \
  switch (VPLV) {                                \
    case 1: { constexpr int VPL = 1; __VA_ARGS__; } break; \
    case 2: { constexpr int VPL = 2; __VA_ARGS__; } break; \
    case 4: { constexpr int VPL = 4; __VA_ARGS__; } break; \
    default: { constexpr int VPL = 8; __VA_ARGS__; } break; \
  }

int launch_gather(const Dims& d, const Work& w, const float* V, const void* v, const float* g,
                  long long stride, int wt0, int len, float* o, bool fuse_resid, const void* v_next,
                  cudaStream_t s) {
  if (len <= 0) return 0;
  const bool split = gather_split(d);
  const int tpc = split ? GATHER_TOK : VAL_WARPS;
  dim3 grid((len + tpc - 1) / tpc, d.B);
  const bool heads = d.H > 1;
#define FWPKM_GATHER_GO(VTT)                                                                                    \
  FWPKM_VPL_DISPATCH(vpl_of(d.dv),                                                                              \
      launch_k(heads ? (split ? gather_kernel<VTT, VPL, true, true> : gather_kernel<VTT, VPL, true, false>)     \
                     : (split ? gather_kernel<VTT, VPL, false, true> : gather_kernel<VTT, VPL, false, false>),  \
               grid, VAL_WARPS * 32, 0, s, d, w, V, (const VTT*)v, g, stride, wt0, len, o, fuse_resid ? 1 : 0, \
               (const VTT*)v_next))
  if (d.qv_bf16) {
    FWPKM_GATHER_GO(__nv_bfloat16);
  } else {
    FWPKM_GATHER_GO(float);
  }
#undef FWPKM_GATHER_GO
  return 1;
}

int launch_resid(const Dims& d, const Work& w, const void* v, const float* g, long long stride, int len,
                 const void* v_next, cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + VAL_WARPS - 1) / VAL_WARPS, d.B);
  if (d.qv_bf16) {
    FWPKM_VPL_DISPATCH(vpl_of(d.dv), launch_k(resid_kernel<__nv_bfloat16, VPL>, grid, VAL_WARPS * 32, 0, s, 
        d, w, (const __nv_bfloat16*)v, g, stride, len, (const __nv_bfloat16*)v_next));
  } else {
    FWPKM_VPL_DISPATCH(vpl_of(d.dv), launch_k(resid_kernel<float, VPL>, grid, VAL_WARPS * 32, 0, s, 
        d, w, (const float*)v, g, stride, len, (const float*)v_next));
  }
  return 1;
}

// Token-at-a-time inference: copy rows of up to three inputs into the staging buffers
// (grid z = 0..2), and with `qn_src` the staged queries' half norms (grid z = 3, one warp
// per token, read from the source rows).
struct StageJobs {
  StageJob j[3];
  int r0, len;
  const __nv_bfloat16* qn_src;
  long long qn_stride;
};

__global__ void __launch_bounds__(256) stage_kernel(StageJobs jobs, Dims dm, Work w) {
  pdl_wait();  // the previous chunk's write may still read the staging rows
  pdl_trigger();
  if (blockIdx.z == 3) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, m = blockIdx.y;
    for (int i = blockIdx.x * 8 + warp; i < jobs.len; i += gridDim.x * 8)
      qnorm_row(dm, w, jobs.qn_src + ((long long)m * jobs.qn_stride + i) * dm.d, m, (long long)jobs.r0 + i, lane);
    return;
  }
  const StageJob& J = jobs.j[blockIdx.z];
  if (J.src == nullptr) return;
  const int m = blockIdx.y;
  const uint32_t* src = reinterpret_cast<const uint32_t*>(J.src) + (long long)m * J.src_stride * J.words;
  uint32_t* dst = reinterpret_cast<uint32_t*>(J.dst) + ((long long)m * J.dst_stride + jobs.r0) * J.words;
  const long long total = (long long)jobs.len * J.words;  // rows are contiguous on both sides
  for (long long i = (long long)blockIdx.x * 256 + threadIdx.x; i < total; i += (long long)gridDim.x * 256)
    dst[i] = src[i];
}

int launch_stage(const Dims& d, const StageJob (&jobs)[3], int r0, int len, cudaStream_t s, const Work* w,
                 const void* qn_src, long long qn_stride) {
  if (len <= 0) return 0;
  StageJobs J;
  int words = 1;
  for (int i = 0; i < 3; ++i) {
    J.j[i] = jobs[i];
    if (jobs[i].src && jobs[i].words > words) words = jobs[i].words;
  }
  J.r0 = r0;
  J.len = len;
  const bool norms = w != nullptr && qn_src != nullptr;
  J.qn_src = norms ? (const __nv_bfloat16*)qn_src : nullptr;
  J.qn_stride = qn_stride;
  long long bx = ((long long)len * words + 255) / 256;
  if (bx > 64) bx = 64;
  launch_k(stage_kernel, dim3((unsigned)bx, d.M, norms ? 4 : 3), 256, 0, s, J, d, norms ? *w : Work{});
  return 1;
}

// CTAs of one kernel that fit on the GPU at once (cached per kernel).
static int resident_ctas(const void* kern, int threads) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  static const void* keys[8];
  static int vals[8];
  static int used = 0;
  for (int i = 0; i < used; ++i)
    if (keys[i] == kern) return vals[i];
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  const int v = sms * per_sm;
  if (used < 8) {
    keys[used] = kern;
    vals[used++] = v;
  }
  return v;
}

// The per-position write (FWPKM_WRITE_V1=1): each warp walks whole segments from G list
// positions with a dependent load per pair; kept to measure against the batched write.
static int launch_write_v1(const Dims& d, const Work& w, float* V, int wt0, cudaStream_t s) {
  const int vpl = vpl_of(d.dv);
  const int G = vpl <= 2 ? 4 : vpl == 4 ? 2 : 1;
  const int need = (d.C * d.k + VAL_WARPS * G - 1) / (VAL_WARPS * G);
  auto grid_for = [&](int resident) {
    const int per_mem = (resident / 2 + d.M - 1) / d.M;
    return dim3(need < per_mem ? need : (per_mem < 1 ? 1 : per_mem), d.M);
  };
  switch (vpl) {
    case 1: launch_k(write_kernel<1, 4>, grid_for(resident_ctas((const void*)write_kernel<1, 4>, VAL_WARPS * 32)), VAL_WARPS * 32, 0, s, d, w, V, wt0); break;
    case 2: launch_k(write_kernel<2, 4>, grid_for(resident_ctas((const void*)write_kernel<2, 4>, VAL_WARPS * 32)), VAL_WARPS * 32, 0, s, d, w, V, wt0); break;
    case 4: launch_k(write_kernel<4, 2>, grid_for(resident_ctas((const void*)write_kernel<4, 2>, VAL_WARPS * 32)), VAL_WARPS * 32, 0, s, d, w, V, wt0); break;
    default: launch_k(write_kernel<8, 1>, grid_for(resident_ctas((const void*)write_kernel<8, 1>, VAL_WARPS * 32)), VAL_WARPS * 32, 0, s, d, w, V, wt0); break;
  }
  return 1;
}

// The fewest list positions a write warp is given (FWPKM_WRITE_MINPOS, default 32): a
// chunk's list is split over at most P / this many warps per table.
static int write_min_positions() {
  static const int v = [] {
    const char* e = getenv("FWPKM_WRITE_MINPOS");
    const int x = e ? atoi(e) : 32;
    return x < 4 ? 4 : x > 256 ? 256 : x;
  }();
  return v;
}

int launch_write(const Dims& d, const Work& w, float* V, int wt0, cudaStream_t s) {
  static const bool v1 = [] {
    const char* e = getenv("FWPKM_WRITE_V1");
    return e && e[0] == '1';
  }();
  if (v1 && d.H == 1) return launch_write_v1(d, w, V, wt0, s);
  const int vpl = vpl_of(d.dv);
  // one warp per ~32 positions of a memory's list at most, and no more warps than fit on the
  // GPU at once (FWPKM_WRITE_SHARE percent of them, default 100)
  static const int share = [] {
    const char* e = getenv("FWPKM_WRITE_SHARE");
    const int v = e ? atoi(e) : 100;
    return v < 5 ? 5 : v > 100 ? 100 : v;
  }();
  auto go = [&](const void* kern, auto kfn) {
    const int resident_warps = resident_ctas(kern, WR_WARPS * 32) * WR_WARPS;
    int per_mem = (int)((long long)resident_warps * share / 100 / d.B);
    const int most = (d.C * d.k * d.H + write_min_positions() - 1) / write_min_positions();
    if (per_mem > most) per_mem = most;
    if (per_mem < 1) per_mem = 1;
    const int blocks = (d.B * per_mem + WR_WARPS - 1) / WR_WARPS;
    launch_k(kfn, dim3((unsigned)blocks), WR_WARPS * 32, 0, s, d, w, V, wt0, per_mem);
  };
#define FWPKM_WRITE_GO(VPLV, WBV)                                                                      \
  (d.H > 1 ? go((const void*)write_batched_kernel<VPLV, WBV, true>, write_batched_kernel<VPLV, WBV, true>) \
           : go((const void*)write_batched_kernel<VPLV, WBV, false>, write_batched_kernel<VPLV, WBV, false>))
  switch (vpl) {
    case 1: FWPKM_WRITE_GO(1, 8); break;
    case 2: FWPKM_WRITE_GO(2, 4); break;
    case 4: FWPKM_WRITE_GO(4, 2); break;
    default: FWPKM_WRITE_GO(8, 1); break;
  }
#undef FWPKM_WRITE_GO
  return 1;
}

// The same for the write phase of the persistent loop (FWPKM_LOOP_MINPOS, default 8): there
// the grid's warps are resident anyway, and shorter ranges mean fewer dependent batches.
static int loop_min_positions() {
  static const int v = [] {
    const char* e = getenv("FWPKM_LOOP_MINPOS");
    const int x = e ? atoi(e) : 8;
    return x < 4 ? 4 : x > 256 ? 256 : x;
  }();
  return v;
}

bool value_loop_enabled() {
  static const bool on = [] {
    const char* e = getenv("FWPKM_VALUE_LOOP");
    if (e && e[0] == '0') return false;
    int dev = 0, coop = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    return coop != 0;
  }();
  return on;
}

int launch_value_loop(const Dims& d, const Work& w, float* V, const void* v, const float* g, int T, int c0, int c1,
                      float* o, cudaStream_t s) {
  if (c1 <= c0) return 0;
  if (!value_loop_enabled() || w.vl_cnt == nullptr) return 0;
  const int stall = take_test_stall();
  auto go = [&](auto kfn, auto vt) -> int {
    using VT = decltype(vt);
    const int resident = resident_ctas((const void*)kfn, VAL_WARPS * 32);
    // write warps per table: one per loop_min_positions() list positions, at most the grid's warps
    int per_mem = (d.C * d.k * d.H + loop_min_positions() - 1) / loop_min_positions();
    if ((long long)per_mem * d.B > (long long)resident * VAL_WARPS) per_mem = resident * VAL_WARPS / d.B;
    if (per_mem < 1) per_mem = 1;
    const int tpc = gather_split(d) ? GATHER_TOK : VAL_WARPS;
    const int gather_ctas = (d.B * d.C + tpc - 1) / tpc;
    const int write_ctas = (d.B * per_mem + VAL_WARPS - 1) / VAL_WARPS;
    int grid = gather_ctas > write_ctas ? gather_ctas : write_ctas;
    if (grid > resident) grid = resident;
    const cudaError_t e = launch_coop(kfn, dim3((unsigned)grid), dim3(VAL_WARPS * 32), 0, s, d, w, V,
                                      (const VT*)v, g, T, c0, c1, o, per_mem, stall);
    return e == cudaSuccess ? 1 : -1;
  };
  const bool split = gather_split(d);
#define FWPKM_VLOOP_GO(VTT, VPLV, WBV)                                                                   \
  (d.H > 1 ? (split ? go(value_loop_kernel<VTT, VPLV, WBV, true, true>, VTT())                           \
                    : go(value_loop_kernel<VTT, VPLV, WBV, true, false>, VTT()))                         \
           : (split ? go(value_loop_kernel<VTT, VPLV, WBV, false, true>, VTT())                          \
                    : go(value_loop_kernel<VTT, VPLV, WBV, false, false>, VTT())))
  const int vpl = vpl_of(d.dv);
  int r;
  if (d.qv_bf16) {
    switch (vpl) {
      case 1: r = FWPKM_VLOOP_GO(__nv_bfloat16, 1, 8); break;
      case 2: r = FWPKM_VLOOP_GO(__nv_bfloat16, 2, 4); break;
      case 4: r = FWPKM_VLOOP_GO(__nv_bfloat16, 4, 2); break;
      default: r = FWPKM_VLOOP_GO(__nv_bfloat16, 8, 1); break;
    }
  } else {
    switch (vpl) {
      case 1: r = FWPKM_VLOOP_GO(float, 1, 8); break;
      case 2: r = FWPKM_VLOOP_GO(float, 2, 4); break;
      case 4: r = FWPKM_VLOOP_GO(float, 4, 2); break;
      default: r = FWPKM_VLOOP_GO(float, 8, 1); break;
    }
  }
#undef FWPKM_VLOOP_GO
  return r;
}

}  // namespace fwpkm
