// noalloc.cu -- fwpkm_chunk_step_noalloc: one whole chunk step (read, write and key
// step) whose scratch lives in a fixed device array inside this library, for callers
// that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is unavailable or forbidden -- a
// real-time or embedded loop with a no-allocation rule, a plugin whose host process
// owns the device allocator, or a caller in the middle of building a larger program
// that must not change the device memory map.  Every other entry point takes its
// scratch from a caller-provided workspace; this one takes nothing but its inputs,
// outputs and the state.  It makes CUDA runtime calls and launches kernels, so it must
// not be called from a CUDA host function (a stream callback or cudaLaunchHostFunc),
// where CUDA calls are not allowed.
//
// It runs the CUDA-core kernels of the chunk step (never the tensor-core ones), so its
// scratch is sized for those alone.
//
// The scratch is the file-scope array g_scratch below (FWPKM_NOALLOC_SCRATCH_BYTES).
// Every GPU that loads the library keeps it allocated until the process exits.
// Host code cannot use the array's name as a device address: the name in host code
// is only a host-side shadow.  The first call on each device, with that device
// current, looks up the real device address with cudaGetSymbolAddress and caches
// it; make that first call before any stream capture.  All calls share the one
// array, so calls whose work overlaps on the GPU (different streams, or different
// host threads on the same device) race on it and must be serialised by the caller.
#include <cstdio>

#include "fwpkm_internal.cuh"

using namespace fwpkm;

#define FWPKM_NOALLOC_SCRATCH_BYTES (16u << 20)
#define FWPKM_NOALLOC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char g_scratch[FWPKM_NOALLOC_SCRATCH_BYTES];

static void* g_scratch_dev[FWPKM_NOALLOC_MAX_DEVICES];

static fwpkm_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= FWPKM_NOALLOC_MAX_DEVICES) {
    cudaGetLastError();
    return FWPKM_ERR_CUDA;
  }
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      fprintf(stderr, "fwpkm: cudaGetSymbolAddress(g_scratch) failed: %s\n", cudaGetErrorString(e));
      cudaGetLastError();
      return FWPKM_ERR_CUDA;
    }
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return FWPKM_OK;
}

extern "C" fwpkm_status fwpkm_chunk_step_noalloc(const fwpkm_config* cfg, float* K1, float* K2, float* V,
                                                 const void* q, const void* v, const float* g,
                                                 const void* v_next, int c_len, int seq_stride, float* o,
                                                 void* stream) {
  NvtxRange nvtx_range("fwpkm_chunk_step_noalloc");
  if (!cfg || !K1 || !K2 || !V || !q || !v || !g || !o) return FWPKM_ERR_INVALID_ARG;
  size_t need = 0;
  fwpkm_status s = fwpkm_workspace_size(cfg, cfg->chunk, &need);  // validates cfg
  if (s != FWPKM_OK) return s;
  Dims d;
  d.n = cfg->n; d.h = cfg->d / 2; d.d = cfg->d; d.dv = cfg->d_v; d.k = cfg->k; d.C = cfg->chunk;
  d.M = cfg->num_mem; d.N = (long long)cfg->n * cfg->n; d.qv_bf16 = cfg->qv_dtype == FWPKM_BF16;
  d.eps_idw = cfg->eps_idw; d.eps_norm = cfg->eps_norm; d.lr_key = cfg->lr_key; d.flags = cfg->flags;
  d.H = 1; d.B = d.M;
  if (cfg->v_heads > 1) return FWPKM_ERR_UNSUPPORTED;  // independent memories only
  // no token-at-a-time staging and no tensor-core buffers: only what the kernels below use
  need = workspace_bytes(d, cfg->chunk, nullptr, nullptr, false, false);
  if (need > FWPKM_NOALLOC_SCRATCH_BYTES) {
    fprintf(stderr, "fwpkm_chunk_step_noalloc: this shape needs %zu bytes of scratch; the built-in "
                    "array holds %u\n", need, FWPKM_NOALLOC_SCRATCH_BYTES);
    return FWPKM_ERR_UNSUPPORTED;
  }
  if (c_len < 1 || c_len > cfg->chunk || seq_stride < c_len) return FWPKM_ERR_INVALID_ARG;
  const uintptr_t a16 = 15;
  if (((uintptr_t)K1 | (uintptr_t)K2 | (uintptr_t)V | (uintptr_t)q | (uintptr_t)v | (uintptr_t)o) & a16)
    return FWPKM_ERR_INVALID_ARG;
  if (((uintptr_t)g & 3) || ((uintptr_t)v_next & 3)) return FWPKM_ERR_INVALID_ARG;
  void* base = nullptr;
  s = scratch_address(&base);
  if (s != FWPKM_OK) return s;

  Work w;
  workspace_bytes(d, cfg->chunk, &w, (char*)base, false, false);

  cudaStream_t st = (cudaStream_t)stream;
  // The array keeps the previous call's contents.  Every buffer the kernels below read is
  // written earlier in the same call, so nothing needs clearing (the status word a
  // skipped bad slot would set is not read by this entry point).
  const bool ku = (d.flags & FWPKM_KEY_UPDATE) != 0;
  const bool last_has_target = (v_next != nullptr) || !(d.flags & FWPKM_LOOKAHEAD);
  bool ok = launch_score_topk(d, w, K1, K2, q, seq_stride, 0, c_len, ku, st) >= 0;
  ok = ok && launch_cartesian(d, w, 0, c_len, nullptr, nullptr, st) >= 0;
  ok = ok && launch_gather(d, w, V, v, g, seq_stride, 0, c_len, o, true, v_next, st) >= 0;
  ok = ok && launch_sort_pairs(d, w, 0, c_len, last_has_target, st) >= 0;
  ok = ok && launch_write(d, w, V, 0, st) >= 0;
  if (ok && ku) ok = launch_address(d, w, K1, K2, q, seq_stride, c_len, st) >= 0;
  cudaError_t e = cudaGetLastError();
  if (!ok && e == cudaSuccess) return FWPKM_ERR_CUDA;
  if (e != cudaSuccess) {
    fprintf(stderr, "fwpkm_chunk_step_noalloc: %s\n", cudaGetErrorString(e));
    return FWPKM_ERR_CUDA;
  }
  return FWPKM_OK;
}
