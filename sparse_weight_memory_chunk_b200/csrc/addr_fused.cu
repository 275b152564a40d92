// addr_fused.cu -- the whole addressing step of one chunk in one launch (key update on,
// tensor-core path): sub-key distances, their rows for the selection, the usage
// marginals and the entropy gradient step on the keys.
//
// Fast-weight Product Key Memory (paperlayer summary) §2.2, §A.2 (scoring: squared
// Euclidean distance of each half-query to every sub-key, inverse-distance weights) and
// §3.4 ((rainbus summary) method step 5): with w[t][b] = 1/(eps + D[t][b]),
// Z_t = sum_b w, P = w / Z_t, pbar_b = (1/len) sum_t P, lp = log pbar,
// L_t = sum_b P lp, W[t][b] = (1/len) P (lp_b - L_t) w and
// K_b -= lr * 2 (sum_t W[t][b] q_t - (sum_t W[t][b]) K_b)   (the gradient of
// L_addr = -H(pbar) for this half, taken at the keys the chunk was read with).
//
// Layout: problem p = (memory, half) is handled by n/128 CTAs; CTA c owns sub-keys
// [128c, 128c + 128) and every token of the chunk, so
//   * the distance tile D^T[b][t] (128 sub-keys x len tokens, fp32) comes out of the
//     scoring MMA (A = the keys' three bf16 pieces, B = the chunk's half-queries) into
//     tensor memory; the first epilogue pass stages it in shared memory for one TMA store
//     into the rows the selection reads, and puts w = 1/(eps + D) back in the same
//     tensor-memory columns for the later passes;
//   * pbar, log pbar, W, sum_t W and the key update are local to the CTA (its sub-keys
//     over all tokens); only Z_t and L_t are sums over all n sub-keys: each CTA reduces its
//     128 across TMEM lanes (warp butterflies, then the four lane quarters in order),
//     publishes the partial vector to global memory, and after the problem's CTAs have all
//     arrived (an arrival counter, bounded wait) every CTA adds the partials in CTA order;
//   * W is written by the epilogue warps straight into shared memory as the key-step
//     MMA's A operand (two bf16 pieces, 128-byte swizzle), next to the half-queries in
//     feature-major order (B), and the key-step accumulator G[b][e] = sum_t W[t][b] q_t[e]
//     lands in tensor memory beside w.
// The distance rows go to global memory once (the selection reads them); apart from two
// small partial vectors per CTA nothing else of the step leaves the chip except the new
// keys, their bf16 pieces and squared norms, staged in shared memory and written by
// per-row bulk copies.
//
// Roles: warp 0 issues TMA loads, warp 1 owns tensor memory and issues the MMAs (one
// thread), warps 2-17 are the epilogue: warp w reads TMEM lane quarter w % 4 (sub-keys
// 32 (w % 4) .. +31 of the CTA) and the 32-column groups g = (w - 2) / 4 (mod 4).
// Every wait (mbarriers and the arrival counters) is bounded by a deadline; on timeout the
// CTA raises its abort flag, skips its remaining work but still arrives on the counters,
// in-flight copies and MMAs are drained, tensor memory is freed and DEV_TIMEOUT is
// latched.  A CTA waits on its peers only while they are certain to run: the grid is at
// most one CTA per SM and its CTAs depend on nothing launched after them.
#include "fwpkm_internal.cuh"
#include "sm100.cuh"

namespace fwpkm {

using namespace sm100;

constexpr int AF_EPI_WARPS = 16;
constexpr int AF_EPI_THREADS = AF_EPI_WARPS * 32;
constexpr int AF_THREADS = (2 + AF_EPI_WARPS) * 32;
constexpr int AF_TILE = 128 * 64 * 2;  // one 128-row x 64-element bf16 tile (16 KiB)
constexpr int AF_MAX_C = 256;          // tokens per chunk (MMA N <= 256)
constexpr uint64_t AF_TIMEOUT_NS = 200ull * 1000 * 1000;
constexpr uint64_t AF_DRAIN_NS = 200ull * 1000 * 1000;

struct AddrFused {
  int n, h, len, npad;    // npad: scoring MMA N = len rounded up to 16
  int hk;                 // 64-feature k-blocks of the scoring (h / 64)
  int nbox;               // 128-row boxes of one half-query tile (ceil(npad / 128))
  int kbw;                // 64-token k-blocks of the key step (ceil(len / 64))
  int q_y0;               // first row of the chunk in the half-query map
  int qt_x0;              // first token column of the chunk in the feature-major map
  int P_all;              // problems between consecutive key pieces (z of the key map)
  int score_only;         // 1: distances only (no key step)
  const float* qn; long long qn_pstride; int qn_off;  // squared half-query norms
  float* kn;              // [P][n] squared key norms (read, then rewritten)
  float* K1; float* K2;   // [M][n][h]
  __nv_bfloat16* Kpc;     // [3][P_all][n][h] key pieces (read by TMA, rewritten)
  float* Dfull; long long d_pstride;  // distance rows [P][rows][n]
  float* part;            // [P][n/128][2][AF_MAX_C] partial Z and L of every CTA
  int* cnt;               // [P][2] arrival counters (zero between launches)
  float eps, lr;
  int off_q, off_qt, off_small;       // shared-memory layout (bytes)
  uint32_t tmem_cols, tmem_g;         // allocated TMEM columns; first column of G
  int* status; int* hstat; int stall;
};

// Named barrier of the epilogue warps only.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(AF_EPI_THREADS) : "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Column sums of a 32 x 32 block held one row per lane (x[i] = column i of this lane's
// row): after the butterfly, lane i returns the sum over the 32 rows of column i.  The
// order of the additions is fixed, so the result is deterministic.
__device__ __forceinline__ float col_sums32(float (&x)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = up ? x[i] : x[i + s];
      const float keep = up ? x[i + s] : x[i];
      x[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return x[0];
}

__device__ __forceinline__ void split3(float x, __nv_bfloat16& hi, __nv_bfloat16& mid, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  const float r = x - __bfloat162float(hi);
  mid = __float2bfloat16_rn(r);
  lo = __float2bfloat16_rn(r - __bfloat162float(mid));
}

// Publish this CTA's partial vector (written by the epilogue threads to `mine` before the
// call), then wait until all `ncl` CTAs of the problem have arrived `phase` times; thread
// 0 of the epilogue polls (bounded).  Returns with the peers' partials readable.
__device__ __forceinline__ void arrive_and_wait(int* cnt, int target, int et, volatile int* abort_flag,
                                                uint64_t deadline) {
  epi_sync();  // every partial of this CTA is written
  if (et == 0) {
    __threadfence();
    atomicAdd(cnt, 1);
    uint32_t spins = 0;
    while (ld_acquire(cnt) < target) {
      __nanosleep(64);
      if ((++spins & 15u) == 0 && (*abort_flag || globaltimer() > deadline)) {
        *abort_flag = 1;
        break;
      }
    }
    __threadfence();
  }
  epi_sync();
}

__global__ void __launch_bounds__(AF_THREADS, 1)
addr_fused_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmD, AddrFused a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  float* s_part = (float*)(smem + a.off_small);   // [4][AF_MAX_C] per-lane-quarter column sums
  float* s_iz = s_part + 4 * AF_MAX_C;           // [AF_MAX_C] 1 / Z_t (0 past len)
  float* s_c = s_iz + AF_MAX_C;                  // [AF_MAX_C] 1 / (len Z_t)
  float* s_L = s_c + AF_MAX_C;                   // [AF_MAX_C] L_t
  float* s_qn = s_L + AF_MAX_C;                  // [AF_MAX_C] squared half-query norms of the chunk
  float* s_pb = s_qn + AF_MAX_C;                 // [4][128] partial column sums (pbar)
  float* s_ws = s_pb + 512;                      // [4][128] partial sum_t W
  float* s_kn = s_ws + 512;                      // [4][128] squared-norm partials of the new keys
  uint64_t* bars = (uint64_t*)(s_kn + 512);
  uint64_t* fullA = bars + 0;   // keys + half-queries landed
  uint64_t* rfree = bars + 1;   // scoring MMAs done: their operand region may be overwritten
  uint64_t* fullQt = bars + 2;  // feature-major half-queries landed
  uint64_t* accf = bars + 3;    // scoring accumulator ready
  uint64_t* wready = bars + 4;  // W written (epilogue warps)
  uint64_t* accg = bars + 5;    // key-step accumulator ready
  uint64_t* drain = bars + 6;   // every MMA issued has completed
  uint64_t* stallb = bars + 7;  // test hook: a barrier that nothing completes
  uint32_t* tmem_slot = (uint32_t*)(bars + 8);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;            // sub-key tile of this CTA
  const int ncl = gridDim.x;           // CTAs of the problem
  const int p = blockIdx.y, m = p >> 1, jh = p & 1;
  const int n = a.n, h = a.h, len = a.len;

  if (threadIdx.x == 0) {
    mbar_init(fullA, 1);
    mbar_init(rfree, 1);
    mbar_init(fullQt, 1);
    mbar_init(accf, 1);
    mbar_init(wready, AF_EPI_WARPS);
    mbar_init(accg, 1);
    mbar_init(drain, 1);
    mbar_init(stallb, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  const uint64_t deadline = globaltimer() + AF_TIMEOUT_NS;
  int issuedA = 0, issuedQt = 0;  // producer: copies in flight to drain on abort

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch(&tmK);
      tma_prefetch(&tmQ);
      mbar_expect_tx(fullA, (uint32_t)((3 * a.hk + a.hk * a.nbox) * AF_TILE));
      for (int pc = 0; pc < 3; ++pc)
        for (int kb = 0; kb < a.hk; ++kb)
          tma_load_3d(smem + (pc * a.hk + kb) * AF_TILE, &tmK, fullA, 64 * kb, 128 * c, p + pc * a.P_all);
      for (int kb = 0; kb < a.hk; ++kb)
        for (int bx = 0; bx < a.nbox; ++bx)
          tma_load_3d(smem + a.off_q + (kb * a.nbox + bx) * AF_TILE, &tmQ, fullA, jh * h + 64 * kb,
                      a.q_y0 + 128 * bx, m);
      issuedA = 1;
      // the feature-major half-queries overwrite the scoring operands once those are consumed
      if (!a.score_only && mbar_wait(rfree, 0, abort_flag, deadline)) {
        tma_prefetch(&tmQt);
        mbar_expect_tx(fullQt, (uint32_t)(a.kbw * AF_TILE));
        for (int kb = 0; kb < a.kbw; ++kb)
          tma_load_3d(smem + a.off_qt + kb * AF_TILE, &tmQt, fullQt, a.qt_x0 + 64 * kb, 0, p);
        issuedQt = 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const bool stalled = a.stall && !mbar_wait(stallb, 0, abort_flag, deadline);
      if (!stalled && mbar_wait(fullA, 0, abort_flag, deadline)) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, a.npad);
        const uint32_t base = smem_u32(smem);
        for (int kb = 0; kb < a.hk; ++kb)
          for (int pc = 0; pc < 3; ++pc)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_k_sw128(base + (pc * a.hk + kb) * AF_TILE + kk * 32);
              const uint64_t bd = sdesc_k_sw128(base + a.off_q + kb * a.nbox * AF_TILE + kk * 32);
              umma_bf16(tmem, ad, bd, idesc, (kb | pc | kk) != 0 ? 1u : 0u);
            }
        umma_commit(accf);
        umma_commit(rfree);
      }
      if (!a.score_only && !*abort_flag && mbar_wait(wready, 0, abort_flag, deadline) &&
          mbar_wait(fullQt, 0, abort_flag, deadline)) {
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, h);
        const uint32_t base = smem_u32(smem);
        for (int kb = 0; kb < a.kbw; ++kb)
          for (int pc = 0; pc < 2; ++pc)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = sdesc_k_sw128(base + (pc * a.kbw + kb) * AF_TILE + kk * 32);
              const uint64_t bd = sdesc_k_sw128(base + a.off_qt + kb * AF_TILE + kk * 32);
              umma_bf16(tmem + a.tmem_g, ad, bd, idesc, (kb | pc | kk) != 0 ? 1u : 0u);
            }
        umma_commit(accg);
      }
      umma_commit(drain);  // completes once every MMA issued above has finished
      uint32_t spins = 0;
      while (!mbar_try_wait(drain, 0))
        if ((++spins & 255u) == 0 && globaltimer() > deadline + AF_DRAIN_NS) break;
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: 16 warps ----------------
    const int q = warp & 3, cq = (warp - 2) >> 2;
    const int bl = q * 32 + lane;                     // sub-key of this CTA (TMEM lane)
    const int b = 128 * c + bl;
    const int et = threadIdx.x - 64;                  // 0 .. AF_EPI_THREADS - 1
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int ngroups = (a.npad + 31) / 32;           // 32-column groups of the distance tile
    const float eps = a.eps;
    float* part = a.part + ((size_t)p * ncl + c) * 2 * AF_MAX_C;
    const float* part_p = a.part + (size_t)p * ncl * 2 * AF_MAX_C;
    int* cnt = a.cnt + 2 * p;
    // stage the chunk's squared half-query norms, and this sub-key's squared norm
    for (int t = et; t < AF_MAX_C; t += AF_EPI_THREADS)
      s_qn[t] = t < len ? a.qn[(size_t)p * a.qn_pstride + a.qn_off + t] : 0.f;
    const float knb = a.kn[(size_t)p * n + b];
    epi_sync();
    int ok = lane == 0 ? (mbar_wait(accf, 0, abort_flag, deadline) ? 1 : 0) : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) tc_fence_after();
    // the distance tile [npad][128] fp32, row-major, over the consumed scoring operands;
    // one TMA store writes it to the rows the selection reads
    float* sD = reinterpret_cast<float*>(smem);

    // pass 1: distances (rows for the selection), w back into tensor memory (0 past len),
    // and the CTA's partial Z_t
    for (int g = cq; g < ngroups; g += 4) {
      float x[32];
      if (ok) {
        uint32_t v[32];
        tmem_ld32(lane_base + (uint32_t)(32 * g), v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int t = 32 * g + i;
          const float D = fmaxf((s_qn[t] + knb) - 2.f * __uint_as_float(v[i]), 0.f);
          if (t < a.npad) sD[t * 128 + bl] = D;
          x[i] = t < len ? __fdividef(1.f, eps + D) : 0.f;
          v[i] = __float_as_uint(x[i]);
        }
        if (!a.score_only) {
          tmem_st32(lane_base + (uint32_t)(32 * g), v);
          tmem_wait_st();
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.f;
      }
      if (!a.score_only) s_part[q * AF_MAX_C + 32 * g + lane] = col_sums32(x, lane);
    }
    fence_async_smem();
    epi_sync();
    if (et == 0 && ok) {
      tma_store_3d(&tmD, sD, 128 * c, 0, p);
      bulk_commit();
    }
    if (!a.score_only) {
      for (int t = et; t < a.npad; t += AF_EPI_THREADS)
        part[t] = ((s_part[t] + s_part[AF_MAX_C + t]) + s_part[2 * AF_MAX_C + t]) + s_part[3 * AF_MAX_C + t];
      arrive_and_wait(cnt, ncl, et, abort_flag, deadline);  // every CTA's partial Z is published
      const float inv_len = 1.f / (float)len;
      for (int t = et; t < AF_MAX_C; t += AF_EPI_THREADS) {
        float z = 0.f;
        if (t < len)
          for (int r = 0; r < ncl; ++r) z += __ldcg(part_p + (size_t)r * 2 * AF_MAX_C + t);
        const float iz = t < len ? 1.f / z : 0.f;
        s_iz[t] = iz;
        s_c[t] = iz * inv_len;
      }
      epi_sync();
      // pass 2: pbar of this sub-key (its row sum over the chunk, in four column quarters)
      float sp = 0.f;
      for (int g = cq; g < ngroups && ok; g += 4) {
        uint32_t v[32];
        tmem_ld32(lane_base + (uint32_t)(32 * g), v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) sp = fmaf(__uint_as_float(v[i]), s_iz[32 * g + i], sp);
      }
      s_pb[cq * 128 + bl] = sp;
      epi_sync();
      const float lpb = logf((((s_pb[bl] + s_pb[128 + bl]) + s_pb[256 + bl]) + s_pb[384 + bl]) * inv_len);
      // pass 3: partial sum_b w lp_b of the CTA
      for (int g = cq; g < ngroups; g += 4) {
        float x[32];
        if (ok) {
          uint32_t v[32];
          tmem_ld32(lane_base + (uint32_t)(32 * g), v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]) * lpb;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = 0.f;
        }
        s_part[q * AF_MAX_C + 32 * g + lane] = col_sums32(x, lane);
      }
      epi_sync();
      for (int t = et; t < a.npad; t += AF_EPI_THREADS)
        part[AF_MAX_C + t] =
            ((s_part[t] + s_part[AF_MAX_C + t]) + s_part[2 * AF_MAX_C + t]) + s_part[3 * AF_MAX_C + t];
      arrive_and_wait(cnt + 1, ncl, et, abort_flag, deadline);  // every CTA's partial L is published
      for (int t = et; t < AF_MAX_C; t += AF_EPI_THREADS) {
        float l = 0.f;
        if (t < len)
          for (int r = 0; r < ncl; ++r) l += __ldcg(part_p + (size_t)r * 2 * AF_MAX_C + AF_MAX_C + t);
        s_L[t] = l * s_iz[t];
      }
      if (et == 0) bulk_wait_read();  // the distance tile has been read: pass 4 writes over it
      epi_sync();
      // the problem's counters are read by every CTA before it arrives here: the last CTA
      // to arrive resets them for the next launch
      if (et == 0) {
        __threadfence();
        const int prev = atomicAdd(cnt + 1, 1);
        if (prev == 2 * ncl - 1) {
          cnt[0] = 0;
          cnt[1] = 0;
        }
      }
      // pass 4: W (two bf16 pieces) into the key step's A operand, and sum_t W
      float ws = 0.f;
      for (int g = cq; g < 2 * a.kbw; g += 4) {
        float W[32];
        if (ok && g < ngroups) {
          uint32_t v[32];
          tmem_ld32(lane_base + (uint32_t)(32 * g), v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int t = 32 * g + i;
            const float wv = __uint_as_float(v[i]);
            W[i] = (wv * wv) * s_c[t] * (lpb - s_L[t]);
            ws += W[i];
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) W[i] = 0.f;
        }
        // 128-byte-swizzled K-major tile of 64 tokens: row bl holds eight 16-byte chunks of
        // 8 tokens, chunk j stored at position j ^ (bl % 8)
        const int kb = g >> 1;
        uint8_t* thi = smem + kb * AF_TILE;
        uint8_t* tlo = smem + (a.kbw + kb) * AF_TILE;
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          __align__(16) __nv_bfloat16 hi[8], lo[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            hi[u] = __float2bfloat16_rn(W[8 * j4 + u]);
            lo[u] = __float2bfloat16_rn(W[8 * j4 + u] - __bfloat162float(hi[u]));
          }
          const int j = (g & 1) * 4 + j4;
          const int off = bl * 128 + ((j ^ (bl & 7)) << 4);
          *reinterpret_cast<uint4*>(thi + off) = *reinterpret_cast<const uint4*>(hi);
          *reinterpret_cast<uint4*>(tlo + off) = *reinterpret_cast<const uint4*>(lo);
        }
      }
      s_ws[cq * 128 + bl] = ws;
      fence_proxy_async_smem();
      epi_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(wready);
      // pass 5: K_b -= lr * 2 (G_b - sum_t W K_b) for the 32-feature group cq (groups past h
      // idle), and the squared norm of the new key as four 32-feature partials combined in
      // group order (as the key preparation forms it).  The new keys and their bf16 pieces
      // are staged in shared memory (the key step's operands are consumed by then) and
      // written out row-contiguous.
      const bool fgo = 32 * cq < h;
      const int e0 = 32 * cq;
      float* Kr = (jh == 0 ? a.K1 : a.K2) + ((size_t)m * n + b) * h + e0;
      float kin[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (fgo) k4 = *reinterpret_cast<const float4*>(Kr + i);
        kin[i] = k4.x; kin[i + 1] = k4.y; kin[i + 2] = k4.z; kin[i + 3] = k4.w;
      }
      const float wsum = ((s_ws[bl] + s_ws[128 + bl]) + s_ws[256 + bl]) + s_ws[384 + bl];
      int okg = lane == 0 ? ((ok && mbar_wait(accg, 0, abort_flag, deadline)) ? 1 : 0) : 0;
      okg = __shfl_sync(0xffffffffu, okg, 0);
      // staging rows: fp32 keys [128][h + 4], then three bf16 pieces [128][h + 8] each (the
      // padding spreads consecutive rows over the banks)
      const int kstr = h + 4, pstr = h + 8;
      float* sK = reinterpret_cast<float*>(smem);
      __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem + (size_t)128 * kstr * 4);
      float ss = 0.f;
      if (okg && fgo) {
        tc_fence_after();
        uint32_t v[32];
        tmem_ld32(lane_base + a.tmem_g + (uint32_t)e0, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          float kout[8];
          __align__(16) __nv_bfloat16 hi[8], mid[8], lo[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float kv = kin[i + u];
            const float grad = 2.f * (__uint_as_float(v[i + u]) - wsum * kv);
            kout[u] = kv - a.lr * grad;
            ss += kout[u] * kout[u];
            split3(kout[u], hi[u], mid[u], lo[u]);
          }
          float* dk = sK + (size_t)bl * kstr + e0 + i;
          *reinterpret_cast<float4*>(dk) = make_float4(kout[0], kout[1], kout[2], kout[3]);
          *reinterpret_cast<float4*>(dk + 4) = make_float4(kout[4], kout[5], kout[6], kout[7]);
          __nv_bfloat16* dp = sP + (size_t)bl * pstr + e0 + i;
          *reinterpret_cast<uint4*>(dp) = *reinterpret_cast<uint4*>(hi);
          *reinterpret_cast<uint4*>(dp + (size_t)128 * pstr) = *reinterpret_cast<uint4*>(mid);
          *reinterpret_cast<uint4*>(dp + (size_t)256 * pstr) = *reinterpret_cast<uint4*>(lo);
        }
      }
      s_kn[cq * 128 + bl] = ss;
      fence_async_smem();
      epi_sync();
      if (okg) {
        // the CTA's 128 rows of K (h fp32 each) and of each bf16 piece (h each): one bulk
        // copy per row, one row per epilogue thread
        const int arr = et >> 7, r = et & 127;
        if (arr == 0) {
          float* Kt = (jh == 0 ? a.K1 : a.K2) + ((size_t)m * n + 128 * c + r) * h;
          bulk_store(Kt, sK + (size_t)r * kstr, (uint32_t)(h * 4));
        } else {
          const size_t pstride = (size_t)a.P_all * n * h;
          __nv_bfloat16* Pt = a.Kpc + (arr - 1) * pstride + ((size_t)p * n + 128 * c + r) * h;
          bulk_store(Pt, sP + (size_t)((arr - 1) * 128 + r) * pstr, (uint32_t)(h * 2));
        }
        bulk_commit();
        if (cq == 0) a.kn[(size_t)p * n + b] = ((s_kn[bl] + s_kn[128 + bl]) + s_kn[256 + bl]) + s_kn[384 + bl];
      }
    }
    bulk_wait_read();  // this thread's bulk stores have read shared memory (no-op if none)
  }

  // ---------------- teardown ----------------
  __syncwarp();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // let the copies this CTA issued land before its shared memory goes away
    uint32_t spins = 0;
    if (issuedA)
      while (!mbar_try_wait(fullA, 0))
        if ((++spins & 255u) == 0 && globaltimer() > deadline + AF_DRAIN_NS) break;
    if (issuedQt)
      while (!mbar_try_wait(fullQt, 0))
        if ((++spins & 255u) == 0 && globaltimer() > deadline + AF_DRAIN_NS) break;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, a.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort_flag) raise_status(a.status, a.hstat, DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
bool use_fused_addressing(const Dims& d) {
  static const bool off = [] {
    const char* e = getenv("FWPKM_FUSED_ADDR");
    return e && e[0] == '0';
  }();
  // one CTA per SM: all the CTAs of a launch (2 M n / 128) must fit on the GPU at once, so
  // that each can wait for its problem's peers
  static const int sms = [] {
    int dev = 0, v = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  return !off && d.qv_bf16 && (d.h == 64 || d.h == 128) && d.n % 128 == 0 && d.C <= AF_MAX_C && d.C % 16 == 0 &&
         2LL * d.M * (d.n / 128) <= sms;
}

static size_t af_smem_bytes(const Dims& d, AddrFused* a) {
  const int hk = d.h / 64, nbox = (d.C + 127) / 128, kbw = (d.C + 63) / 64;
  const int off_q = 3 * hk * AF_TILE;
  const int score_end = off_q + hk * nbox * AF_TILE;
  const int off_qt = 2 * kbw * AF_TILE;
  const int key_end = off_qt + kbw * AF_TILE;
  // the new keys and their pieces are staged over the same region once the MMAs are done
  const int stage = 128 * (d.h + 4) * 4 + 3 * 128 * (d.h + 8) * 2;
  int off_small = score_end > key_end ? score_end : key_end;
  if (off_small < stage) off_small = (stage + 1023) / 1024 * 1024;
  // small: 8 vectors of AF_MAX_C floats and 12 of 128, 8 barriers, the TMEM slot and a flag
  const int small = (8 * AF_MAX_C + 12 * 128) * 4 + 8 * 8 + 16;
  if (a) {
    a->hk = hk;
    a->off_q = off_q;
    a->off_qt = off_qt;
    a->off_small = off_small;
  }
  return 1024 + (size_t)off_small + small;
}

size_t addr_fused_part_floats(const Dims& d) { return (size_t)2 * d.M * (d.n / 128) * 2 * AF_MAX_C; }

int launch_addr_fused(const Dims& d, const Work& w, float* K1, float* K2, const void* q_base, long long q_stride,
                      int q_extent, int q_row0, int wt0, int len, int qt_x0, bool score_only, cudaStream_t s) {
  if (len <= 0) return 0;
  const int P = d.M * 2;
  CUtensorMap tK, tQ, tQt;
  // key pieces: problem p's piece pc at z = p + pc * P_all
  if (!make_tmap_bf16_3d(&tK, w.Kpc, d.h, d.n, 2 * w.P_all + P, (uint64_t)d.h * 2, (uint64_t)d.n * d.h * 2))
    return -1;
  // half-queries: x = feature (half j at x = j h), y = token, z = memory
  if (!make_tmap_bf16_3d(&tQ, q_base, d.d, q_extent, d.M, (uint64_t)d.d * 2, (uint64_t)q_stride * d.d * 2))
    return -1;
  if (!score_only) {
    if (!make_tmap_bf16_3d(&tQt, w.Qt, w.qt_T, d.h, P, (uint64_t)w.qt_T * 2, (uint64_t)d.h * w.qt_T * 2)) return -1;
  } else {
    tQt = tQ;  // unused
  }
  // distance rows [P][drows][n] fp32: each CTA stores a box of 128 sub-keys x npad tokens
  const int npad = (len + 15) / 16 * 16;
  CUtensorMap tD;
  if (!make_tmap_f32_3d(&tD, w.Dfull, d.n, w.drows, P, (uint64_t)d.n * 4, (uint64_t)w.drows * d.n * 4, 128,
                        (uint32_t)npad))
    return -1;
  AddrFused a = {};
  a.n = d.n; a.h = d.h; a.len = len;
  a.npad = (len + 15) / 16 * 16;
  const size_t smem = af_smem_bytes(d, &a);
  a.nbox = (a.npad + 127) / 128;
  a.kbw = (len + 63) / 64;
  a.q_y0 = q_row0;
  a.qt_x0 = qt_x0;
  a.P_all = w.P_all;
  a.score_only = score_only ? 1 : 0;
  a.qn = w.qn; a.qn_pstride = w.max_T; a.qn_off = wt0;
  a.kn = w.kn;
  a.K1 = K1; a.K2 = K2;
  a.Kpc = w.Kpc;
  a.Dfull = w.Dfull; a.d_pstride = (long long)w.drows * d.n;
  a.part = w.af_part; a.cnt = w.af_cnt;
  a.eps = d.eps_idw; a.lr = d.lr_key;
  // w takes 128 or 256 columns (every 32-column group the epilogue reads); G (h <= 128
  // columns) starts right after it
  const uint32_t dcols = a.npad <= 128 ? 128u : 256u;
  a.tmem_g = dcols;
  a.tmem_cols = score_only ? dcols : 2 * dcols;
  a.status = w.status; a.hstat = w.hstat;
  a.stall = take_test_stall();
  if (!raise_smem_limit((const void*)addr_fused_kernel, smem)) return -1;
  launch_k(addr_fused_kernel, dim3((unsigned)(d.n / 128), (unsigned)P, 1), AF_THREADS, smem, s, tK, tQ, tQt, tD, a);
  return 1;
}

}  // namespace fwpkm
