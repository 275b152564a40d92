// tc_path.cu -- kernels around the tensor-core contractions (bf16 queries, d/2 in {64, 128}).
//
// Scoring (Fast-weight Product Key Memory (paperlayer summary) §2.2, §A.2): the GEMM in
// tc_gemm.cu writes the squared distances of a chunk's tokens to every sub-key; the
// per-half top-k is taken here from those rows.
// Entropy key step ((rainbus summary) method step 5; (paperlayer summary) §3.4): with
// w = 1/(eps + D), Z_t = sum_a w, P = w / Z_t, pbar = mean_t P, lp = log pbar,
// L_t = sum_a P lp, W[t][b] = (1/len) P[t][b] (lp[b] - L_t) w[t][b]; the key-step GEMM
// then forms sum_t W[t][b] q_t and updates the keys in its epilogue.
#include "bitonic.cuh"
#include "fwpkm_internal.cuh"
#include "sm100.cuh"

namespace fwpkm {

constexpr int TP_THREADS = 256;

__device__ __forceinline__ void split3_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  float r = x - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r);
  lo = __float2bfloat16_rn(r - __bfloat162float(mid));
}

// ||q_half||^2 per (memory, half, token): one warp per token, both halves.
__global__ void __launch_bounds__(TP_THREADS)
qnorm_kernel(Dims dm, Work w, const __nv_bfloat16* __restrict__ q, long long q_stride, int wt0, int len) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (TP_THREADS / 32) + warp;
  const int m = blockIdx.y;
  if (i >= len) return;
  qnorm_row(dm, w, q + ((long long)m * q_stride + i) * dm.d, m, (long long)wt0 + i, lane);
}

// bf16 pieces and squared norm of every key: four threads per (problem, sub-key), thread g
// taking features [32 g, 32 g + 32) in order (adjacent threads read adjacent 128-byte
// pieces of the row).  The squared norm is the four 32-feature partial sums combined in
// order, exactly as the key-step epilogues form it, so both give the same bits.
__global__ void __launch_bounds__(TP_THREADS)
keyprep_kernel(Dims dm, Work w, const float* __restrict__ K1, const float* __restrict__ K2) {
  pdl_wait();
  pdl_trigger();
  const int P = dm.M * 2;
  const long long gid = (long long)blockIdx.x * TP_THREADS + threadIdx.x;
  const long long idx = gid >> 2;  // (problem, sub-key)
  const int g = (int)(gid & 3);
  const bool row_ok = idx < (long long)P * dm.n;
  const int p = row_ok ? (int)(idx / dm.n) : 0, b = row_ok ? (int)(idx - (long long)p * dm.n) : 0;
  const int m = p >> 1, j = p & 1, h = dm.h;
  float part = 0.f;
  if (row_ok && 32 * g < h) {
    const float* K = (j == 0 ? K1 : K2) + ((size_t)m * dm.n + b) * h + 32 * g;
    const size_t pstride = (size_t)w.P_all * dm.n * h;
    __nv_bfloat16* pc = w.Kpc + ((size_t)p * dm.n + b) * h + 32 * g;
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
      float4 k0 = *reinterpret_cast<const float4*>(K + e);
      float4 k1 = *reinterpret_cast<const float4*>(K + e + 4);
      float kin[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
      __align__(16) __nv_bfloat16 hi[8], mid[8], lo[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        part += kin[u] * kin[u];
        split3_bf16(kin[u], hi[u], mid[u], lo[u]);
      }
      *reinterpret_cast<uint4*>(pc + e) = *reinterpret_cast<uint4*>(hi);
      *reinterpret_cast<uint4*>(pc + pstride + e) = *reinterpret_cast<uint4*>(mid);
      *reinterpret_cast<uint4*>(pc + 2 * pstride + e) = *reinterpret_cast<uint4*>(lo);
    }
  }
  // the row's four partials sit in lanes 4r .. 4r + 3 of the warp
  const int lane = threadIdx.x & 31, base = lane & ~3;
  const float p0 = __shfl_sync(0xffffffffu, part, base), p1 = __shfl_sync(0xffffffffu, part, base + 1);
  const float p2 = __shfl_sync(0xffffffffu, part, base + 2), p3 = __shfl_sync(0xffffffffu, part, base + 3);
  if (row_ok && g == 0) w.kn[(size_t)p * dm.n + b] = ((p0 + p1) + p2) + p3;
}

// Partial column sums sum_t w[t][a] / Z_t over one token slice; also Z_t itself.  The
// last of the slice blocks of a column block to finish (arrival counter, reset by
// that block) adds the slices in slice order and writes lp = log(pbar).
__global__ void __launch_bounds__(TP_THREADS)
tc_pbar_kernel(Dims dm, Work w, int len) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_invz[1024 / 8 + 1];  // tokens of one slice (at least 8 slices)
  __shared__ int s_last;
  const int p = blockIdx.y, sl = blockIdx.z;
  const int ns = gridDim.z;
  const int t0 = (sl * len) / ns, t1 = ((sl + 1) * len) / ns;
  const int nt = (dm.n + 127) / 128 * 4;  // 4 column groups per 128-column tile
  for (int t = t0 + threadIdx.x; t < t1; t += TP_THREADS) {
    // Z_t from the scoring epilogue's nt partial sums (a multiple of 4, 16-byte aligned):
    // all loads issued together, summed in order
    const float4* zp = reinterpret_cast<const float4*>(w.zpart + ((size_t)p * dm.C + t) * nt);
    float z = 0.f;
    for (int u0 = 0; u0 < nt / 4; u0 += 8) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = u0 + u < nt / 4 ? zp[u0 + u] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) z = (((z + x[u].x) + x[u].y) + x[u].z) + x[u].w;
    }
    s_invz[t - t0] = 1.f / z;
    if (blockIdx.x == 0) w.Z[(size_t)p * dm.C + t] = z;
  }
  __syncthreads();
  const int a = blockIdx.x * TP_THREADS + threadIdx.x;
  const bool av = a < dm.n;
  if (av) {
    const float* D = w.Dfull + (size_t)p * w.drows * dm.n;
    float s = 0.f;
#pragma unroll 16
    for (int t = t0; t < t1; ++t) s += __fdividef(1.f, dm.eps_idw + D[(size_t)t * dm.n + a]) * s_invz[t - t0];
    w.ppart[((size_t)p * ns + sl) * dm.n + a] = s;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int* c = w.pbar_cnt + (size_t)p * gridDim.x + blockIdx.x;
    const int prev = atomicAdd(c, 1);
    s_last = prev == ns - 1;
    if (s_last) *c = 0;  // every slice has arrived: ready for the next launch
  }
  __syncthreads();
  if (s_last && av) {
    __threadfence();
    float s = 0.f;
    for (int k = 0; k < ns; ++k) s += __ldcg(w.ppart + ((size_t)p * ns + k) * dm.n + a);
    w.lp[(size_t)p * dm.n + a] = logf(s / (float)len);
  }
}

// W for a block of WB_T tokens and every sub-key, written sub-key major as two bf16
// pieces (the A operand of the key-step GEMM), plus the block's per-sub-key sum of W.
// First L_t = sum_a P[t][a] lp[a] = (sum_a lp[a] w[t][a]) / Z_t for the block's tokens (one
// warp per token, a row's loads all in flight), then W[t][b] = (1/len) (w/Z_t) (lp[b] -
// L_t) w for WB_SUB sub-keys per thread (the block's rows re-read, all loads in flight).
constexpr int WB_T = 16;  // tokens per CTA (one wave of CTAs at the paper-scale shapes)
constexpr int WB_G = 8;   // tokens per pass of the W phase (one 16-byte store per piece)
constexpr int WB_SUB = 4; // sub-keys per thread per pass: 256 threads x 4 = 1024
__global__ void __launch_bounds__(TP_THREADS, 3)
tc_wbuild_kernel(Dims dm, Work w, int len, int cpad) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_invz[WB_T], s_L[WB_T];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.y, t0 = blockIdx.x * WB_T;
  const int n = dm.n;
  const float* D = w.Dfull + (size_t)p * w.drows * n;
  const float* lp = w.lp + (size_t)p * n;
  // two tokens per warp, their row loads and the shared log-marginal loads in flight together
  static_assert(WB_T == 2 * (TP_THREADS / 32), "two tokens per warp");
  {
    const int ta = t0 + 2 * warp, tb = ta + 1;
    const bool va = ta < len, vb = tb < len;
    const float* Da = D + (size_t)(va ? ta : 0) * n;
    const float* Db = D + (size_t)(vb ? tb : 0) * n;
    float sa = 0.f, sb = 0.f;
    for (int a0 = 0; a0 < n; a0 += 32 * 16) {
      float da[16], db[16], ll[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int a = a0 + lane + 32 * u;
        ll[u] = a < n ? lp[a] : 0.f;
        da[u] = (va && a < n) ? Da[a] : 0.f;
        db[u] = (vb && a < n) ? Db[a] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        sa += __fdividef(ll[u], dm.eps_idw + da[u]);
        sb += __fdividef(ll[u], dm.eps_idw + db[u]);
      }
    }
    sa = warp_sum(sa);
    sb = warp_sum(sb);
    if (lane == 0) {
      const float za = va ? w.Z[(size_t)p * dm.C + ta] : 1.f, zb = vb ? w.Z[(size_t)p * dm.C + tb] : 1.f;
      s_L[2 * warp] = va ? sa / za : 0.f;
      s_invz[2 * warp] = va ? 1.f / za : 0.f;
      s_L[2 * warp + 1] = vb ? sb / zb : 0.f;
      s_invz[2 * warp + 1] = vb ? 1.f / zb : 0.f;
    }
  }
  __syncthreads();
  const float inv_len = 1.f / (float)len;
  const size_t pstride = (size_t)w.P_all * n * cpad;
  const int ntb = gridDim.x;
  for (int b0 = threadIdx.x; b0 < n; b0 += TP_THREADS * WB_SUB) {
    float wsum[WB_SUB];
#pragma unroll
    for (int q = 0; q < WB_SUB; ++q) wsum[q] = 0.f;
    for (int g0 = 0; g0 < WB_T; g0 += WB_G) {
      const int tg = t0 + g0;
      if (tg >= len) break;
      float dd[WB_SUB][WB_G], lpb[WB_SUB];
#pragma unroll
      for (int q = 0; q < WB_SUB; ++q) {
        const int b = b0 + q * TP_THREADS;
        lpb[q] = b < n ? lp[b] : 0.f;
#pragma unroll
        for (int tl = 0; tl < WB_G; ++tl) dd[q][tl] = (b < n && tg + tl < len) ? D[(size_t)(tg + tl) * n + b] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < WB_SUB; ++q) {
        const int b = b0 + q * TP_THREADS;
        if (b >= n) continue;
        __align__(16) __nv_bfloat16 hi[WB_G], lo[WB_G];
#pragma unroll
        for (int tl = 0; tl < WB_G; ++tl) {
          float W = 0.f;
          if (tg + tl < len) {
            const float wv = __fdividef(1.f, dm.eps_idw + dd[q][tl]);
            const float P_ = wv * s_invz[g0 + tl];
            W = inv_len * P_ * (lpb[q] - s_L[g0 + tl]) * wv;
          }
          wsum[q] += W;
          // two bf16 pieces (~16 significant bits): W only scales the key step, whose
          // error this leaves at ~1e-5 of the step
          hi[tl] = __float2bfloat16_rn(W);
          lo[tl] = __float2bfloat16_rn(W - __bfloat162float(hi[tl]));
        }
        __nv_bfloat16* dst = w.Wt + ((size_t)p * n + b) * cpad + tg;
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(hi);
        *reinterpret_cast<uint4*>(dst + pstride) = *reinterpret_cast<uint4*>(lo);
      }
    }
#pragma unroll
    for (int q = 0; q < WB_SUB; ++q) {
      const int b = b0 + q * TP_THREADS;
      if (b < n) w.wsum_part[((size_t)p * ntb + blockIdx.x) * n + b] = wsum[q];
    }
  }
}

// Feature-major copy of the half-queries of `len` tokens: Qt[p][e][qt0 + t].  One CTA
// per (64-token tile, problem); 16-byte loads and stores through a shared-memory tile.
// Token columns past `len` in the last tile are written as zeros (finite values, since the
// key-step GEMM multiplies them by zero-filled weights).
__global__ void __launch_bounds__(TP_THREADS)
qtrans_kernel(Dims dm, Work w, const __nv_bfloat16* __restrict__ q, long long q_stride, int qt0, int len) {
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) __nv_bfloat16 s_q[64][128 + 8];
  const int p = blockIdx.y, m = p >> 1, j = p & 1;
  const int t0 = blockIdx.x * 64, h = dm.h, h8 = h / 8;
  for (int idx = threadIdx.x; idx < 64 * h8; idx += TP_THREADS) {
    const int tl = idx / h8, e8 = idx - tl * h8;
    const int t = t0 + tl;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (t < len) val = *reinterpret_cast<const uint4*>(q + ((long long)m * q_stride + t) * dm.d + (long long)j * h + e8 * 8);
    *reinterpret_cast<uint4*>(&s_q[tl][e8 * 8]) = val;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < h * 8; idx += TP_THREADS) {
    const int e = idx >> 3, c8 = idx & 7;
    __align__(16) __nv_bfloat16 v8[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v8[u] = s_q[c8 * 8 + u][e];
    *reinterpret_cast<uint4*>(w.Qt + ((size_t)p * h + e) * w.qt_T + qt0 + t0 + c8 * 8) = *reinterpret_cast<uint4*>(v8);
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
int launch_qnorm(const Dims& d, const Work& w, const void* q, long long q_stride, int wt0, int len, cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + 7) / 8, d.M);
  launch_k(qnorm_kernel, grid, TP_THREADS, 0, s, d, w, (const __nv_bfloat16*)q, q_stride, wt0, len);
  return 1;
}

int launch_keyprep(const Dims& d, const Work& w, const float* K1, const float* K2, cudaStream_t s) {
  const long long threads = (long long)d.M * 2 * d.n * 4;
  launch_k(keyprep_kernel, (unsigned)((threads + TP_THREADS - 1) / TP_THREADS), TP_THREADS, 0, s, d, w, K1, K2);
  return 1;
}

int launch_tc_score(const Dims& d, const Work& w, const void* q_base, long long q_stride, int q_extent, int q_row0,
                    int wt0, int len, bool key_update, cudaStream_t s) {
  if (len <= 0) return 0;
  const int P = d.M * 2;
  CUtensorMap A, B;
  if (!make_tmap_bf16_3d(&A, q_base, d.d, q_extent, d.M, (uint64_t)d.d * 2, (uint64_t)q_stride * d.d * 2)) return -1;
  // pieces of problem p sit at z = p, p + P_all, p + 2 P_all
  if (!make_tmap_bf16_3d(&B, w.Kpc, d.h, d.n, 2 * w.P_all + P, (uint64_t)d.h * 2, (uint64_t)d.n * d.h * 2))
    return -1;
  TcGemm g = {};
  g.P = P;
  g.k_blocks = d.h / 64;
  g.n_tiles = (d.n + 127) / 128;
  g.tiles_per_cta = 2;
  g.a_pieces = 1; g.b_pieces = 3;
  g.a_div = 2; g.a_xoff = d.h; g.a_y0 = q_row0; g.a_zpiece = 0; g.b_zpiece = w.P_all;
  g.m_valid = len; g.n_valid = d.n;
  g.epi = TC_EPI_DIST;
  g.out = w.Dfull; g.out_pstride = (long long)w.drows * d.n; g.out_ld = d.n;
  g.rowv = w.qn; g.rowv_pstride = w.max_T; g.rowv_off = wt0;
  g.colv = w.kn; g.colv_pstride = d.n;
  g.zpart = key_update ? w.zpart : nullptr; g.zpart_pstride = d.C; g.eps = d.eps_idw;
  g.status = w.status;
  g.hstat = w.hstat;
  g.stall = take_test_stall();
  return launch_tc_gemm(A, B, g, (len + 127) / 128, s);
}

int launch_qtrans(const Dims& d, const Work& w, const void* q, long long q_stride, int qt0, int len, cudaStream_t s) {
  if (len <= 0) return 0;
  launch_k(qtrans_kernel, dim3((len + 63) / 64, d.M * 2), TP_THREADS, 0, s, d, w, (const __nv_bfloat16*)q, q_stride, qt0,
                                                                       len);
  return 1;
}

int launch_tc_pbar(const Dims& d, const Work& w, int len, cudaStream_t s) {
  if (len <= 0) return 0;
  launch_k(tc_pbar_kernel, dim3((d.n + TP_THREADS - 1) / TP_THREADS, d.M * 2, pbar_slices()), TP_THREADS, 0, s, d, w,
           len);
  return 1;
}

int launch_tc_wbuild(const Dims& d, const Work& w, int len, cudaStream_t s) {
  if (len <= 0) return 0;
  const int cpad = (d.C + 63) / 64 * 64;
  launch_k(tc_wbuild_kernel, dim3((len + WB_T - 1) / WB_T, d.M * 2), TP_THREADS, 0, s, d, w, len, cpad);
  return 1;
}

int launch_tc_keystep(const Dims& d, const Work& w, float* K1, float* K2, const void* q, long long q_stride, int len,
                      int qt_t0, cudaStream_t s) {
  if (len <= 0) return 0;
  const int P = d.M * 2;
  const int cpad = (d.C + 63) / 64 * 64;
  const int ntt = (len + 63) / 64;
  const int ntb = (len + WB_T - 1) / WB_T;
  int launched = 1;
  if (qt_t0 < 0) {
    launch_qtrans(d, w, q, q_stride, 0, len, s);
    qt_t0 = 0;
    ++launched;
  }
  CUtensorMap A, B;
  if (!make_tmap_bf16_3d(&A, w.Wt, len, d.n, w.P_all + P, (uint64_t)cpad * 2, (uint64_t)d.n * cpad * 2))
    return -1;
  if (!make_tmap_bf16_3d(&B, w.Qt, w.qt_T, d.h, P, (uint64_t)w.qt_T * 2, (uint64_t)d.h * w.qt_T * 2)) return -1;
  TcGemm g = {};
  g.P = P;
  g.k_blocks = ntt;
  g.n_tiles = 1;
  g.tiles_per_cta = 1;
  g.a_pieces = 2; g.b_pieces = 1;
  g.a_div = 1; g.a_xoff = 0; g.a_y0 = 0; g.a_zpiece = w.P_all; g.b_zpiece = 0; g.b_x0 = qt_t0;
  g.m_valid = d.n; g.n_valid = d.h;
  g.epi = TC_EPI_KEYSTEP;
  g.K1 = K1; g.K2 = K2; g.Kpc = w.Kpc; g.kn = w.kn; g.piece_P = w.P_all;
  g.wsum_part = w.wsum_part; g.wsum_tiles = ntb; g.lr = d.lr_key;
  g.status = w.status;
  g.hstat = w.hstat;
  g.stall = take_test_stall();
  if (launch_tc_gemm(A, B, g, (d.n + 127) / 128, s) < 0) return -1;
  return launched;
}

}  // namespace fwpkm
