// tc_gemm.cu -- the dense contractions of the hot path on the 5th-generation tensor
// cores (tcgen05.mma, TMEM accumulators, TMA-fed 128-byte-swizzled tiles).
//
//  * scoring (Fast-weight Product Key Memory (paperlayer summary) §2.2, §A.2):
//      D[t][a] = ||q_t||^2 + ||K[a]||^2 - 2 q_t . K[a]   for every token of a chunk and
//      every sub-key of a half; epilogue writes the distance rows (clamped at 0) and the
//      per-tile partial sums of 1/(eps + D) used by the entropy step.
//  * entropy key step ((rainbus summary) method step 5; (paperlayer summary) §3.4):
//      G[b][e] = sum_t W[t][b] q_t[e]; epilogue applies K[b] -= lr * 2 (G[b] - Wsum[b] K[b])
//      and refreshes the bf16 pieces and squared norms of the new keys.
//  * slow-weight projections ((rainbus summary) method steps 1 and 3, see layer.cu):
//      y[r][c] = (1/rms_r) sum_e x[r][e] W'[c][e] + b[c]; the epilogue applies the
//      per-row scale and the bias and writes fp32 or bf16.
//
// Precision: q and v are bf16 (exact); the keys enter as three bf16 pieces hi + mid + lo
// (~24 significant bits), each piece pair accumulating into one fp32 TMEM accumulator, so
// the distances match fp32 arithmetic to ~1e-7 relative; the key-step weights W enter as
// two pieces (~16 bits: the step they scale is then exact to ~1e-5 of itself).
//
// CTA = 18 warps: warp 0 issues TMA loads, warp 1 owns TMEM and issues the MMAs (one
// thread), warps 2-17 drain TMEM: warp w reads TMEM lanes 32*(w%4)..+31 (tile rows) and
// the 32 columns of column group (w-2)/4, so four warps share every lane quarter.
// Accumulators are double-buffered (2 x 128 columns) so the epilogue of tile j overlaps
// the MMAs of tile j+1.  Every wait is bounded (globaltimer); on timeout the CTA raises a
// shared abort flag, drains its own in-flight copies and MMAs, frees TMEM and reports
// DEV_TIMEOUT through the status word.
#include <cstdio>

#include "fwpkm_internal.cuh"
#include "sm100.cuh"

namespace fwpkm {

using namespace sm100;

constexpr int TC_BM = 128, TC_BN = 128, TC_BK = 64;
constexpr int TC_TILE_BYTES = TC_BM * TC_BK * 2;  // 16 KiB, also the B tile (TC_BN == TC_BM)
// Pipeline depth: two stages (up to four were measured slower: the larger shared-memory
// carve-out leaves the epilogue's loads and stores less L1).
constexpr int TC_MAX_STAGES = 2;
constexpr int TC_EPI_WARPS = 16;
constexpr int TC_THREADS = (2 + TC_EPI_WARPS) * 32;
constexpr uint32_t TC_TMEM_COLS = 256;
constexpr uint64_t TC_TIMEOUT_NS = 200ull * 1000 * 1000;  // every wait of the main loop
constexpr uint64_t TC_DRAIN_NS = 200ull * 1000 * 1000;    // draining in-flight copies/MMAs on abort

int tc_stages(int npieces, int kblocks_per_cta) {
  int st = (200 * 1024) / (npieces * TC_TILE_BYTES);
  if (st > TC_MAX_STAGES) st = TC_MAX_STAGES;
  if (st > kblocks_per_cta) st = kblocks_per_cta;
  return st < 1 ? 1 : st;
}

size_t tc_smem_bytes(int npieces, int stages) {
  return 1024 + (size_t)stages * npieces * TC_TILE_BYTES + 256;  // tiles + barriers and flags
}

__device__ __forceinline__ bool wait_deadline(uint64_t* bar, uint32_t parity, uint64_t deadline) {
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() > deadline) return false;
  return true;
}

__device__ __forceinline__ void split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  float r = x - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r);
  lo = __float2bfloat16_rn(r - __bfloat162float(mid));
}

__global__ void __launch_bounds__(TC_THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcGemm g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int npc = g.a_pieces + g.b_pieces;
  uint8_t* tiles = smem;
  const int S = g.stages;
  uint64_t* full = (uint64_t*)(tiles + (size_t)S * npc * TC_TILE_BYTES);
  uint64_t* empty = full + TC_MAX_STAGES;
  uint64_t* accf = empty + TC_MAX_STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint64_t* normbar = drain + 1;
  uint64_t* stallbar = normbar + 1;  // test hook: a barrier that nothing completes
  uint32_t* tmem_slot = (uint32_t*)(stallbar + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  __shared__ float s_norm[4][TC_BM];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.z, mt = blockIdx.y;
  const int nt0 = blockIdx.x * g.tiles_per_cta;
  const int ntiles = min(g.n_tiles, nt0 + g.tiles_per_cta) - nt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], TC_EPI_WARPS);
    }
    mbar_init(drain, 1);
    mbar_init(normbar, TC_EPI_WARPS);
    mbar_init(stallbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TC_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // barriers and TMEM are set up; from here on the CTA reads what earlier kernels wrote
  pdl_wait();
  pdl_trigger();
  const uint64_t deadline = globaltimer() + TC_TIMEOUT_NS;
  int issued = 0;  // producer: loads issued

  if (ntiles > 0 && warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    const int a_z = p / g.a_div, a_x0 = (p % g.a_div) * g.a_xoff;
    for (int j = 0; j < ntiles && !*abort_flag; ++j) {
      const int nt = nt0 + j;
      bool ok = true;
      for (int kb = 0; kb < g.k_blocks; ++kb) {
        const int s = issued % S;
        const uint32_t ph = (issued / S) & 1;
        if (issued >= S && !mbar_wait(&empty[s], ph ^ 1, abort_flag, deadline)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&full[s], (uint32_t)(npc * TC_TILE_BYTES));
        uint8_t* st = tiles + (size_t)s * npc * TC_TILE_BYTES;
        for (int pa = 0; pa < g.a_pieces; ++pa)
          tma_load_3d(st + pa * TC_TILE_BYTES, &tmA, &full[s], a_x0 + kb * TC_BK, g.a_y0 + mt * TC_BM,
                      a_z + pa * g.a_zpiece);
        for (int pb = 0; pb < g.b_pieces; ++pb)
          tma_load_3d(st + (g.a_pieces + pb) * TC_TILE_BYTES, &tmB, &full[s], g.b_x0 + kb * TC_BK, nt * TC_BN,
                      p + pb * g.b_zpiece);
        ++issued;
      }
      if (!ok) break;
    }
  } else if (ntiles > 0 && warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(TC_BM, TC_BN);
    int it = 0;
    // test hook of the timeout path: wait on a barrier that nothing completes; the bounded
    // wait runs out and raises the abort flag, and every role unwinds as on a real timeout
    const bool stalled = g.stall && !mbar_wait(stallbar, 0, abort_flag, deadline);
    for (int j = 0; j < ntiles && !stalled; ++j) {
      const int b = j & 1;
      const uint32_t aph = (j >> 1) & 1;
      if (j >= 2 && !mbar_wait(&acce[b], aph ^ 1, abort_flag, deadline)) break;
      tc_fence_after();
      const uint32_t dt = tmem + (uint32_t)(b * TC_BN);
      bool ok = true;
      for (int kb = 0; kb < g.k_blocks; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        if (!mbar_wait(&full[s], ph, abort_flag, deadline)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(tiles + (size_t)s * npc * TC_TILE_BYTES);
        for (int pa = 0; pa < g.a_pieces; ++pa)
          for (int pb = 0; pb < g.b_pieces; ++pb)
#pragma unroll
            for (int kk = 0; kk < TC_BK / 16; ++kk) {
              const uint64_t ad = sdesc_k_sw128(st + pa * TC_TILE_BYTES + kk * 32);
              const uint64_t bd = sdesc_k_sw128(st + (g.a_pieces + pb) * TC_TILE_BYTES + kk * 32);
              umma_bf16(dt, ad, bd, idesc, (kb | pa | pb | kk) != 0 ? 1u : 0u);
            }
        umma_commit(&empty[s]);
      }
      if (!ok) break;
      umma_commit(&accf[b]);
    }
    umma_commit(drain);  // completes once every MMA issued above has finished
    wait_deadline(drain, 0, deadline + TC_DRAIN_NS);
  } else if (ntiles > 0 && warp >= 2) {
    // ---------------- epilogue: 16 warps; warp w reads TMEM lane quarter w%4 (tile rows
    // 32*(w%4)..+31, one per thread) and column group (w-2)/4 (32 columns) ----------------
    const int q = warp & 3;
    const int cg = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int m = p >> 1, jh = p & 1;
    for (int j = 0; j < ntiles; ++j) {
      const int b = j & 1;
      const uint32_t aph = (j >> 1) & 1;
      const int nt = nt0 + j;
      const int r = mt * TC_BM + row;
      const bool rv = r < g.m_valid;
      // operands of the epilogue that do not depend on the accumulator are loaded while
      // the MMAs run: DIST the row norm and 32 column norms, KEYSTEP sum_t W and the key
      float pre_s = 0.f, pre[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) pre[i] = 0.f;
      if (g.epi == TC_EPI_DIST) {
        const int c0 = nt * TC_BN + cg * 32;
        pre_s = rv ? g.rowv[(size_t)p * g.rowv_pstride + g.rowv_off + r] : 0.f;
        const float* kn = g.colv + (size_t)p * g.colv_pstride;
        if (c0 + 32 <= g.n_valid) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(kn + c0 + i);
            pre[i] = k4.x; pre[i + 1] = k4.y; pre[i + 2] = k4.z; pre[i + 3] = k4.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pre[i] = c0 + i < g.n_valid ? kn[c0 + i] : 0.f;
        }
      } else if (g.epi == TC_EPI_KEYSTEP) {
        const int h = g.n_valid, n = g.m_valid, e0 = cg * 32;
        if (rv && e0 < h) {
          // the partial sums are independent loads: four interleaved accumulators keep
          // them in flight, combined in a fixed order
          const float* wp = g.wsum_part + (size_t)p * g.wsum_tiles * n + r;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
          int tt = 0;
          for (; tt + 4 <= g.wsum_tiles; tt += 4) {
            a0 += wp[(size_t)tt * n];
            a1 += wp[(size_t)(tt + 1) * n];
            a2 += wp[(size_t)(tt + 2) * n];
            a3 += wp[(size_t)(tt + 3) * n];
          }
          for (; tt < g.wsum_tiles; ++tt) a0 += wp[(size_t)tt * n];
          pre_s = (a0 + a1) + (a2 + a3);
          const float* K = (jh == 0 ? g.K1 : g.K2) + ((size_t)m * n + r) * h + e0;
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(K + i);
            pre[i] = k4.x; pre[i + 1] = k4.y; pre[i + 2] = k4.z; pre[i + 3] = k4.w;
          }
        }
      }
      // one lane waits; the verdict is shared so the warp stays converged for tcgen05.ld
      int ok = lane == 0 ? (mbar_wait(&accf[b], aph, abort_flag, deadline) ? 1 : 0) : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(lane_base + (uint32_t)(b * TC_BN + cg * 32), v);
      tmem_wait_ld();
      // accumulator drained: hand the buffer back before the (longer) epilogue math
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      if (g.epi == TC_EPI_DIST) {
        const int c0 = nt * TC_BN + cg * 32;
        const float rq = pre_s;
        float* out = g.out + ((size_t)p * g.out_pstride + (size_t)r * g.out_ld);
        float dv[32];
        float zacc = 0.f;
        if (c0 + 32 <= g.n_valid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            dv[i] = fmaxf((rq + pre[i]) - 2.f * __uint_as_float(v[i]), 0.f);
            zacc += __fdividef(1.f, g.eps + dv[i]);
          }
          if (rv) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(out + c0 + i) = make_float4(dv[i], dv[i + 1], dv[i + 2], dv[i + 3]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = c0 + i;
            dv[i] = fmaxf((rq + pre[i]) - 2.f * __uint_as_float(v[i]), 0.f);
            if (c < g.n_valid) {
              zacc += __fdividef(1.f, g.eps + dv[i]);
              if (rv) out[c] = dv[i];
            }
          }
        }
        if (rv && g.zpart)
          g.zpart[(((size_t)p * g.zpart_pstride + r) * g.n_tiles + nt) * 4 + cg] = zacc;
      } else if (g.epi == TC_EPI_PROJ) {
        const int c0 = nt * TC_BN + cg * 32;
        if (rv && c0 < g.n_valid) {
          const float rs = g.rowscale[r];
          float y[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] = __uint_as_float(v[i]) * rs + (g.bias ? g.bias[c0 + i] : 0.f);
          const bool first = c0 < g.split;
          const size_t off = first ? (size_t)r * g.ld0 + c0 : (size_t)r * g.ld1 + (c0 - g.split);
          if (g.out_bf16) {
            __nv_bfloat16* dst = (__nv_bfloat16*)(first ? g.pout0 : g.pout1) + off;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              __align__(16) __nv_bfloat16 yb[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) yb[u] = __float2bfloat16_rn(y[i + u]);
              *reinterpret_cast<uint4*>(dst + i) = *reinterpret_cast<uint4*>(yb);
            }
          } else {
            float* dst = (float*)(first ? g.pout0 : g.pout1) + off;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
          }
        }
      } else {  // TC_EPI_KEYSTEP: row = sub-key b, columns = features e (one tile covers h)
        const int h = g.n_valid;
        const int n = g.m_valid;
        const int e0 = cg * 32;
        float ss = 0.f;
        if (rv && e0 < h) {
          const float wsum = pre_s;
          float* K = (jh == 0 ? g.K1 : g.K2) + ((size_t)m * n + r) * h;
          const size_t pstride = (size_t)g.piece_P * n * h;
          __nv_bfloat16* pc = g.Kpc + ((size_t)p * n + r) * h;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const int e = e0 + i;
            float kin[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) kin[u] = pre[i + u];
            float kout[8];
            __align__(16) __nv_bfloat16 hi[8], mid[8], lo[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float grad = 2.f * (__uint_as_float(v[i + u]) - wsum * kin[u]);
              kout[u] = kin[u] - g.lr * grad;
              ss += kout[u] * kout[u];
              split3(kout[u], hi[u], mid[u], lo[u]);
            }
            *reinterpret_cast<float4*>(K + e) = make_float4(kout[0], kout[1], kout[2], kout[3]);
            *reinterpret_cast<float4*>(K + e + 4) = make_float4(kout[4], kout[5], kout[6], kout[7]);
            *reinterpret_cast<uint4*>(pc + e) = *reinterpret_cast<uint4*>(hi);
            *reinterpret_cast<uint4*>(pc + pstride + e) = *reinterpret_cast<uint4*>(mid);
            *reinterpret_cast<uint4*>(pc + 2 * pstride + e) = *reinterpret_cast<uint4*>(lo);
          }
        }
        // squared norm of the new key: the four column groups' partials, summed in order
        // by the column-group-0 warp once all 16 warps have published theirs (one tile per
        // CTA in this mode, so the barrier has a single phase; the wait is bounded)
        s_norm[cg][row] = ss;
        __syncwarp();
        if (lane == 0) mbar_arrive(normbar);
        if (cg == 0) {
          int okn = lane == 0 ? (mbar_wait(normbar, 0, abort_flag, deadline) ? 1 : 0) : 0;
          okn = __shfl_sync(0xffffffffu, okn, 0);
          if (okn && rv)
            g.kn[(size_t)p * n + r] = ((s_norm[0][row] + s_norm[1][row]) + s_norm[2][row]) + s_norm[3][row];
        }
      }
    }
  }

  // ---------------- teardown ----------------
  __syncwarp();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let the copies this CTA issued land before its shared memory goes away
    for (int i = issued - S < 0 ? 0 : issued - S; i < issued; ++i)
      wait_deadline(&full[i % S], (i / S) & 1, deadline + TC_DRAIN_NS);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) raise_status(g.status, g.hstat, DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// host side: tensor maps (driver entry point, no link-time dependency on libcuda)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// bf16 tensor [z][y][x] with row pitch `pitch_y` and plane pitch `pitch_z` (bytes);
// box 64 x 128 x 1, 128-byte swizzle, zero fill outside the extents.
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint64_t pitch_y,
                       uint64_t pitch_z) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {x, y, z};
  cuuint64_t strides[2] = {pitch_y, pitch_z};
  cuuint32_t box[3] = {TC_BK, TC_BM, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) fprintf(stderr, "fwpkm: cuTensorMapEncodeTiled failed (%d)\n", (int)r);
  return r == CUDA_SUCCESS;
}

// fp32 tensor [z][y][x] (pitches in bytes), box box_x x box_y x 1, no swizzle: the
// shared-memory side of a copy is the dense box, row-major.
bool make_tmap_f32_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint64_t pitch_y,
                      uint64_t pitch_z, uint32_t box_x, uint32_t box_y) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {x, y, z};
  cuuint64_t strides[2] = {pitch_y, pitch_z};
  cuuint32_t box[3] = {box_x, box_y, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) fprintf(stderr, "fwpkm: cuTensorMapEncodeTiled (fp32) failed (%d)\n", (int)r);
  return r == CUDA_SUCCESS;
}

int launch_tc_gemm(const CUtensorMap& A, const CUtensorMap& B, const TcGemm& g0, int m_tiles, cudaStream_t s) {
  TcGemm g = g0;
  const int npc = g.a_pieces + g.b_pieces;
  g.stages = tc_stages(npc, g.k_blocks * g.tiles_per_cta);
  const size_t smem = tc_smem_bytes(npc, g.stages);
  // The kernel's dynamic shared-memory limit is one attribute of the function, while its
  // launches need different amounts (scoring 129 KiB, key step 97 KiB, ...): it is only
  // ever raised, so that no captured launch is above it (a replay that launches graph
  // nodes one by one checks each node against the function's current limit).
  if (!raise_smem_limit((const void*)tc_gemm_kernel, smem)) return -1;
  dim3 grid((g.n_tiles + g.tiles_per_cta - 1) / g.tiles_per_cta, m_tiles, g.P);
  launch_k(tc_gemm_kernel, grid, TC_THREADS, smem, s, A, B, g);
  return 1;
}

}  // namespace fwpkm
