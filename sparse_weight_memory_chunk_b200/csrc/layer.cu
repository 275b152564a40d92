// layer.cu -- the slow-weight projections around the memory ("快速权重积键值记忆
// Fast-weight Product Key Memory" (rainbus summary), method steps 1 and 3):
//   q = Linear_q(RMSNorm_q(h)), v = Linear_v(RMSNorm_v(h)), g = sigmoid(Linear_g(RMSNorm_g(h))),
//   o' = Linear_o(RMSNorm_o(o)),  RMSNorm(x) = x / sqrt(mean(x^2) + eps) * gamma.
//
// Because RMSNorm is a per-row scale times a per-feature weight,
//   Linear(RMSNorm(x)) = (1/rms(x)) * (x (gamma . W)^T) + b,
// so gamma is folded into W once (fp32 product, kept as bf16 pieces) and 1/rms
// scales the tensor-core accumulator in the GEMM epilogue.  The input side is one
// row-statistics pass over h (1/rms and the gate's dot product; the gate is a single
// output column, so it never reaches the tensor cores) and one GEMM whose epilogue writes
// q and v.  The output side splits o (fp32) into two bf16 pieces while it forms 1/rms,
// then one GEMM writes o' in bf16.
#include <cstdio>
#include <new>

#include "fwpkm_internal.cuh"

using namespace fwpkm;

struct fwpkm_layer {
  fwpkm_layer_config cfg;
  __nv_bfloat16* Wqv;   // [3][d + d_v][d_model]  folded q and v weights, bf16 pieces
  float* wg;            // [d_model]              folded gate weights (fp32)
  float* bqv;           // [d + d_v]              q and v biases
  __nv_bfloat16* Wo;    // [3][d_model][d_v]      folded output weights, bf16 pieces
  float* bo;            // [d_model]              output bias
  float* inv_rms;       // [max_rows]             per-row 1/rms scratch
  __nv_bfloat16* opc;   // [2][max_rows][d_v]     bf16 pieces of o
  int* status;          // device status word (GEMM wait timeouts)
  int* hstat;           // its host copy (pinned, mapped), written by the kernel that latches
  int* hstat_dev;       // device view of hstat
  float b_g;
  int qv_pieces, o_pieces;  // 1 when the norm weight is absent (folded weights exact in bf16)
  int have_params;
};

namespace {

constexpr size_t LALIGN = 256;
size_t lalign(size_t x) { return (x + LALIGN - 1) & ~(LALIGN - 1); }
constexpr int LAYER_THREADS = 256;

size_t layer_carve(const fwpkm_layer_config& c, fwpkm_layer* L, char* base) {
  const size_t D = c.d_model, nqv = (size_t)c.d + c.d_v, dv = c.d_v, R = c.max_rows;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = lalign(off + bytes);
    return p;
  };
  int* status = (int*)take(sizeof(int));
  __nv_bfloat16* Wqv = (__nv_bfloat16*)take(2 * 3 * nqv * D);
  float* wg = (float*)take(4 * D);
  float* bqv = (float*)take(4 * nqv);
  __nv_bfloat16* Wo = (__nv_bfloat16*)take(2 * 3 * D * dv);
  float* bo = (float*)take(4 * D);
  float* inv = (float*)take(4 * R);
  __nv_bfloat16* opc = (__nv_bfloat16*)take(2 * 2 * R * dv);
  if (L) {
    L->Wqv = Wqv; L->wg = wg; L->bqv = bqv; L->Wo = Wo; L->bo = bo; L->inv_rms = inv; L->opc = opc;
    L->status = status;
  }
  return off;
}

fwpkm_status check_layer_cfg(const fwpkm_layer_config* c) {
  if (!c || c->d_model <= 0 || c->d <= 0 || c->d_v <= 0 || c->max_rows < 1 || !(c->eps_rms >= 0.f))
    return FWPKM_ERR_INVALID_ARG;
  if (c->qv_dtype != FWPKM_F32 && c->qv_dtype != FWPKM_BF16) return FWPKM_ERR_INVALID_ARG;
  if (c->d_model % 64 != 0 || c->d_model < 64 || c->d_model > 16384 || c->d % 32 != 0 || c->d_v % 64 != 0 ||
      c->d < 32 || c->d > 1024 || c->d_v > 1024)
    return FWPKM_ERR_UNSUPPORTED;
  return FWPKM_OK;
}

bool al(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

fwpkm_status cuda_status() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "fwpkm: CUDA error: %s\n", cudaGetErrorString(e));
    return FWPKM_ERR_CUDA;
  }
  return FWPKM_OK;
}

// A device error already latched in the handle's host copy (read without waiting).
fwpkm_status layer_peek(const fwpkm_layer* L) {
  const int h = L->hstat ? *(volatile int*)L->hstat : DEV_OK;
  return h != DEV_OK ? status_of_device(h) : cuda_status();
}

}  // namespace

namespace fwpkm {

// W' = gamma[e] * W[j][e] in fp32, stored as `pieces` bf16 pieces at dst[piece][row0 + j][e]:
// hi = bf16(W'), then mid = bf16(W' - hi), lo = bf16(W' - hi - mid) (~24 significant bits).
__global__ void __launch_bounds__(LAYER_THREADS)
fold_weights_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ gamma, int rows, int cols,
                    __nv_bfloat16* __restrict__ dst, long long piece_stride, int row0, int pieces) {
  const long long i = (long long)blockIdx.x * LAYER_THREADS + threadIdx.x;
  if (i >= (long long)rows * cols) return;
  const int j = (int)(i / cols), e = (int)(i - (long long)j * cols);
  const float w = __bfloat162float(W[i]) * (gamma ? gamma[e] : 1.f);
  const __nv_bfloat16 hi = __float2bfloat16_rn(w);
  const size_t o = (size_t)(row0 + j) * cols + e;
  dst[o] = hi;
  if (pieces >= 2) {
    const float r = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r);
    dst[piece_stride + o] = mid;
    if (pieces >= 3) dst[2 * piece_stride + o] = __float2bfloat16_rn(r - __bfloat162float(mid));
  }
}

__global__ void __launch_bounds__(LAYER_THREADS)
fold_gate_kernel(const __nv_bfloat16* __restrict__ w, const float* __restrict__ gamma, int D, float* __restrict__ out) {
  const int e = blockIdx.x * LAYER_THREADS + threadIdx.x;
  if (e < D) out[e] = __bfloat162float(w[e]) * (gamma ? gamma[e] : 1.f);
}

__global__ void __launch_bounds__(LAYER_THREADS)
copy_bias_kernel(const float* __restrict__ b, int n, float* __restrict__ out) {
  const int i = blockIdx.x * LAYER_THREADS + threadIdx.x;
  if (i < n) out[i] = b ? b[i] : 0.f;
}

// One warp per row of h: 1/rms = 1/sqrt(mean h^2 + eps) and g = sigmoid(dot(h, w_g') / rms + b_g).
__global__ void __launch_bounds__(LAYER_THREADS)
rms_gate_kernel(const __nv_bfloat16* __restrict__ h, int rows, int D, float eps, const float* __restrict__ wg,
                float b_g, float* __restrict__ inv_rms, float* __restrict__ g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (LAYER_THREADS / 32) + warp;
  if (r >= rows) return;
  const __nv_bfloat16* x = h + (size_t)r * D;
  float ss = 0.f, dot = 0.f;
  for (int e = lane * 8; e < D; e += 256) {
    const uint4 u = *reinterpret_cast<const uint4*>(x + e);
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&u);
    const float4 w0 = *reinterpret_cast<const float4*>(wg + e);
    const float4 w1 = *reinterpret_cast<const float4*>(wg + e + 4);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int u8 = 0; u8 < 8; ++u8) {
      const float xv = __bfloat162float(xb[u8]);
      ss = fmaf(xv, xv, ss);
      dot = fmaf(xv, wv[u8], dot);
    }
  }
  ss = warp_sum(ss);
  dot = warp_sum(dot);
  if (lane == 0) {
    const float inv = 1.f / sqrtf(ss / (float)D + eps);
    inv_rms[r] = inv;
    g[r] = 1.f / (1.f + expf(-(dot * inv + b_g)));
  }
}

// One warp per row of o: 1/rms, and o as bf16 pieces hi, lo (o - hi) at opc[piece][r][e].
__global__ void __launch_bounds__(LAYER_THREADS)
rms_split_kernel(const float* __restrict__ o, int rows, int dv, float eps, float* __restrict__ inv_rms,
                 __nv_bfloat16* __restrict__ opc, long long piece_stride) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (LAYER_THREADS / 32) + warp;
  if (r >= rows) return;
  const float* x = o + (size_t)r * dv;
  __nv_bfloat16* hi = opc + (size_t)r * dv;
  float ss = 0.f;
  for (int e = lane * 4; e < dv; e += 128) {
    const float4 u = *reinterpret_cast<const float4*>(x + e);
    const float xv[4] = {u.x, u.y, u.z, u.w};
    __align__(8) __nv_bfloat16 h4[4], l4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ss = fmaf(xv[i], xv[i], ss);
      h4[i] = __float2bfloat16_rn(xv[i]);
      l4[i] = __float2bfloat16_rn(xv[i] - __bfloat162float(h4[i]));
    }
    *reinterpret_cast<uint2*>(hi + e) = *reinterpret_cast<uint2*>(h4);
    *reinterpret_cast<uint2*>(hi + piece_stride + e) = *reinterpret_cast<uint2*>(l4);
  }
  ss = warp_sum(ss);
  if (lane == 0) inv_rms[r] = 1.f / sqrtf(ss / (float)dv + eps);
}

}  // namespace fwpkm

namespace fwpkm {
const fwpkm_layer_config* layer_config(const fwpkm_layer* L) { return L ? &L->cfg : nullptr; }
}  // namespace fwpkm

extern "C" {

fwpkm_status fwpkm_layer_workspace_size(const fwpkm_layer_config* cfg, size_t* bytes) {
  fwpkm_status s = check_layer_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!bytes) return FWPKM_ERR_INVALID_ARG;
  *bytes = layer_carve(*cfg, nullptr, nullptr);
  return FWPKM_OK;
}

fwpkm_status fwpkm_layer_init(const fwpkm_layer_config* cfg, void* workspace, size_t ws_bytes, fwpkm_layer** out) {
  fwpkm_status s = check_layer_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!out || !workspace || !al(workspace, LALIGN)) return FWPKM_ERR_INVALID_ARG;
  if (ws_bytes < layer_carve(*cfg, nullptr, nullptr)) return FWPKM_ERR_WORKSPACE;
  fwpkm_layer* L = new (std::nothrow) fwpkm_layer();
  if (!L) return FWPKM_ERR_INVALID_ARG;
  L->cfg = *cfg;
  layer_carve(*cfg, L, (char*)workspace);
  L->hstat = L->hstat_dev = nullptr;
  if (cudaHostAlloc((void**)&L->hstat, sizeof(int), cudaHostAllocMapped) != cudaSuccess ||
      cudaHostGetDevicePointer((void**)&L->hstat_dev, L->hstat, 0) != cudaSuccess ||
      cudaMemset(L->status, 0, sizeof(int)) != cudaSuccess) {
    cuda_status();
    fwpkm_layer_destroy(L);
    return FWPKM_ERR_CUDA;
  }
  *(volatile int*)L->hstat = DEV_OK;
  *out = L;
  return FWPKM_OK;
}

fwpkm_status fwpkm_layer_sync(fwpkm_layer* L, void* stream) {
  if (!L) return FWPKM_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    cuda_status();
    return FWPKM_ERR_CUDA;
  }
  int h = 0;
  if (cudaMemcpy(&h, L->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return cuda_status();
  if (h == DEV_OK && L->hstat) h = *(volatile int*)L->hstat;
  if (h != DEV_OK) {
    if (cudaMemset(L->status, 0, sizeof(int)) != cudaSuccess) return cuda_status();
    if (L->hstat) *(volatile int*)L->hstat = DEV_OK;
    return status_of_device(h);
  }
  return cuda_status();
}

void fwpkm_layer_destroy(fwpkm_layer* L) {
  if (!L) return;
  if (L->hstat) cudaFreeHost(L->hstat);
  delete L;
}

fwpkm_status fwpkm_layer_set_params(fwpkm_layer* L, const fwpkm_layer_params* p, void* stream) {
  NvtxRange nvtx_range("fwpkm_layer_set_params");
  if (!L || !p || !p->W_q || !p->W_v || !p->w_g || !p->W_o) return FWPKM_ERR_INVALID_ARG;
  const fwpkm_layer_config& c = L->cfg;
  cudaStream_t s = (cudaStream_t)stream;
  const int D = c.d_model, nqv = c.d + c.d_v;
  // one piece suffices when no norm weight is folded in (W is exact in bf16); else three
  // pieces carry the fp32 product.  The q and v weights share one GEMM and its piece
  // count; the output GEMM's result is rounded to bf16, so two pieces are enough there.
  L->qv_pieces = (p->gamma_q || p->gamma_v) ? 3 : 1;
  L->o_pieces = p->gamma_o ? 2 : 1;
  const long long qv_ps = (long long)nqv * D, o_ps = (long long)D * c.d_v;
  auto blocks = [](long long n) { return (unsigned)((n + LAYER_THREADS - 1) / LAYER_THREADS); };
  fold_weights_kernel<<<blocks((long long)c.d * D), LAYER_THREADS, 0, s>>>(
      (const __nv_bfloat16*)p->W_q, p->gamma_q, c.d, D, L->Wqv, qv_ps, 0, L->qv_pieces);
  fold_weights_kernel<<<blocks((long long)c.d_v * D), LAYER_THREADS, 0, s>>>(
      (const __nv_bfloat16*)p->W_v, p->gamma_v, c.d_v, D, L->Wqv, qv_ps, c.d, L->qv_pieces);
  fold_gate_kernel<<<blocks(D), LAYER_THREADS, 0, s>>>((const __nv_bfloat16*)p->w_g, p->gamma_g, D, L->wg);
  copy_bias_kernel<<<blocks(c.d), LAYER_THREADS, 0, s>>>(p->b_q, c.d, L->bqv);
  copy_bias_kernel<<<blocks(c.d_v), LAYER_THREADS, 0, s>>>(p->b_v, c.d_v, L->bqv + c.d);
  fold_weights_kernel<<<blocks((long long)D * c.d_v), LAYER_THREADS, 0, s>>>(
      (const __nv_bfloat16*)p->W_o, p->gamma_o, D, c.d_v, L->Wo, o_ps, 0, L->o_pieces);
  copy_bias_kernel<<<blocks(D), LAYER_THREADS, 0, s>>>(p->b_o, D, L->bo);
  count_launches(7);
  L->b_g = p->b_g;
  L->have_params = 1;
  return cuda_status();
}

fwpkm_status fwpkm_layer_in(fwpkm_layer* L, const void* h, int rows, void* q, void* v, float* g, void* stream) {
  NvtxRange nvtx_range("fwpkm_layer_in");
  if (!L) return FWPKM_ERR_INVALID_ARG;
  if (rows == 0) return FWPKM_OK;
  const fwpkm_layer_config& c = L->cfg;
  if (!h || !q || !v || !g || rows < 0 || rows > c.max_rows) return FWPKM_ERR_INVALID_ARG;
  if (!al(h, 16) || !al(q, 16) || !al(v, 16) || !al(g, 4)) return FWPKM_ERR_INVALID_ARG;
  if (!L->have_params) return FWPKM_ERR_STATE;
  {
    const fwpkm_status ps = layer_peek(L);
    if (ps != FWPKM_OK) return ps;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int D = c.d_model, nqv = c.d + c.d_v;
  rms_gate_kernel<<<(rows + 7) / 8, LAYER_THREADS, 0, s>>>((const __nv_bfloat16*)h, rows, D, c.eps_rms, L->wg,
                                                           L->b_g, L->inv_rms, g);
  CUtensorMap A, B;
  if (!make_tmap_bf16_3d(&A, h, D, rows, 1, (uint64_t)D * 2, (uint64_t)rows * D * 2)) return FWPKM_ERR_CUDA;
  if (!make_tmap_bf16_3d(&B, L->Wqv, D, nqv, 3, (uint64_t)D * 2, (uint64_t)nqv * D * 2)) return FWPKM_ERR_CUDA;
  TcGemm t = {};
  t.P = 1; t.k_blocks = D / 64; t.n_tiles = (nqv + 127) / 128; t.tiles_per_cta = 2;
  t.a_pieces = 1; t.b_pieces = L->qv_pieces;
  t.a_div = 1; t.a_xoff = 0; t.a_y0 = 0; t.a_zpiece = 0; t.b_zpiece = 1; t.b_x0 = 0;
  t.m_valid = rows; t.n_valid = nqv;
  t.epi = TC_EPI_PROJ;
  t.rowscale = L->inv_rms; t.bias = L->bqv;
  t.pout0 = q; t.ld0 = c.d; t.pout1 = v; t.ld1 = c.d_v; t.split = c.d;
  t.out_bf16 = c.qv_dtype == FWPKM_BF16;
  t.status = L->status;
  t.hstat = L->hstat_dev;
  t.stall = take_test_stall();
  if (launch_tc_gemm(A, B, t, (rows + 127) / 128, s) < 0) return FWPKM_ERR_CUDA;
  count_launches(2);
  return cuda_status();
}

fwpkm_status fwpkm_layer_out(fwpkm_layer* L, const float* o, int rows, void* o_out, void* stream) {
  NvtxRange nvtx_range("fwpkm_layer_out");
  if (!L) return FWPKM_ERR_INVALID_ARG;
  if (rows == 0) return FWPKM_OK;
  const fwpkm_layer_config& c = L->cfg;
  if (!o || !o_out || rows < 0 || rows > c.max_rows) return FWPKM_ERR_INVALID_ARG;
  if (!al(o, 16) || !al(o_out, 16)) return FWPKM_ERR_INVALID_ARG;
  if (!L->have_params) return FWPKM_ERR_STATE;
  {
    const fwpkm_status ps = layer_peek(L);
    if (ps != FWPKM_OK) return ps;
  }
  cudaStream_t s = (cudaStream_t)stream;
  const int D = c.d_model, dv = c.d_v;
  const long long ops = (long long)c.max_rows * dv;
  rms_split_kernel<<<(rows + 7) / 8, LAYER_THREADS, 0, s>>>(o, rows, dv, c.eps_rms, L->inv_rms, L->opc, ops);
  CUtensorMap A, B;
  if (!make_tmap_bf16_3d(&A, L->opc, dv, rows, 2, (uint64_t)dv * 2, (uint64_t)ops * 2)) return FWPKM_ERR_CUDA;
  if (!make_tmap_bf16_3d(&B, L->Wo, dv, D, 3, (uint64_t)dv * 2, (uint64_t)D * dv * 2)) return FWPKM_ERR_CUDA;
  TcGemm t = {};
  t.P = 1; t.k_blocks = dv / 64; t.n_tiles = (D + 127) / 128; t.tiles_per_cta = 4;
  t.a_pieces = 2; t.b_pieces = L->o_pieces;
  t.a_div = 1; t.a_xoff = 0; t.a_y0 = 0; t.a_zpiece = 1; t.b_zpiece = 1; t.b_x0 = 0;
  t.m_valid = rows; t.n_valid = D;
  t.epi = TC_EPI_PROJ;
  t.rowscale = L->inv_rms; t.bias = L->bo;
  t.pout0 = o_out; t.ld0 = D; t.pout1 = nullptr; t.ld1 = 0; t.split = D;
  t.out_bf16 = 1;
  t.status = L->status;
  t.hstat = L->hstat_dev;
  t.stall = take_test_stall();
  if (launch_tc_gemm(A, B, t, (rows + 127) / 128, s) < 0) return FWPKM_ERR_CUDA;
  count_launches(2);
  return cuda_status();
}

}  // extern "C"
