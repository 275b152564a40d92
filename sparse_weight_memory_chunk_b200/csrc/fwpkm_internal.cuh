// fwpkm_internal.cuh -- shared declarations of the B200 FwPKM library (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fwpkm.h"

namespace fwpkm {

// Device status word values (latched by kernels, read by fwpkm_sync).
enum : int { DEV_OK = 0, DEV_BAD_SLOT = 1, DEV_TIMEOUT = 2 };

// Kernel kinds for the launch counter / per-kernel timing.
enum KernelKind : int { KK_NONE = 0, KK_GATHER = 1, KK_WRITE = 2, KK_SCORE = 3, KK_CART = 4,
                        KK_SORT = 5, KK_ADDR = 6, KK_OTHER = 7 };

struct Dims {
  int n, h, d, dv, k, C, M;
  long long N;
  int qv_bf16;
  float eps_idw, eps_norm, lr_key;
  unsigned flags;
};

// Per-memory workspace carve (all device pointers into the caller's workspace).
struct Work {
  int max_T;
  int max_chunks;
  int32_t* A;        // [M][2][max_T][k]   per-half survivors (sub-key index), rank order
  float* Dsv;        // [M][2][max_T][k]   their squared distances
  int32_t* idx;      // [M][max_T][k]      final slots, rank order
  float* w;          // [M][max_T][k]      softmax weights
  uint32_t* pair_tr; // [M][max_T*k]       sorted pairs: t_local*k + r, per chunk region of C*k
  int32_t* seg_start;// [M][max_chunks][C*k + 1]
  int32_t* seg_slot; // [M][max_chunks][C*k]
  int32_t* nseg;     // [M][max_chunks]
  float* resid;      // [M][C][dv]         vhat, then r_t = g_t (vhat_t - tau_t)
  float* Dfull;      // [M][2][C][n]       key update: all sub-key distances of the chunk
  float* Z;          // [M][2][C]          key update: sum_a 1/(eps + D)
  float* lp;         // [M][2][n]          key update: log pbar
  float* Lt;         // [M][2][C]          key update: sum_a P log pbar
  int* status;       // device status word
};

size_t workspace_bytes(const Dims& d, int max_T, Work* carve, char* base);

// ---- launchers (each enqueues on `s` and returns the number of kernels launched) ----
// Tokens are addressed two ways: user buffers are passed already offset to the first
// token of the range, with `stride` = tokens between consecutive memories; workspace
// arrays indexed by token use `wt0` = the workspace token of the range's first token.
//
// Sub-key distances + per-half top-k for `len` tokens.  With key_update (len <= C,
// one chunk) the full distance rows and sum_a 1/(eps + D) are kept for the key step.
int launch_score_topk(const Dims& d, const Work& w, const float* K1, const float* K2,
                      const void* q, long long q_stride, int wt0, int len, bool key_update,
                      cudaStream_t s);
// Restricted Cartesian top-k + softmax for `len` tokens: writes idx, w and the
// optional user copies idx_out/w_out ([M][len][k]).
int launch_cartesian(const Dims& d, const Work& w, int wt0, int len, int32_t* idx_out, float* w_out,
                     cudaStream_t s);
// Sort the (slot, token) pairs of the chunks covering workspace tokens
// [wt0, wt0 + total_len) (wt0 a multiple of C) and build their segments.  Every token
// reads with a target except the range's last one when !last_has_target.
int launch_sort_pairs(const Dims& d, const Work& w, int wt0, int total_len, bool last_has_target,
                      cudaStream_t s);
// Gather + gated output for the `len` tokens of one chunk.  fuse_resid: also form the
// residual r_t (lookahead of the last token = v_next, NULL = none); else store vhat.
int launch_gather(const Dims& d, const Work& w, const float* V, const void* v, const float* g,
                  long long stride, int wt0, int len, float* o, bool fuse_resid,
                  const void* v_next, cudaStream_t s);
// Streaming write path: turn the stored vhat of a chunk into residuals.
int launch_resid(const Dims& d, const Work& w, const void* v, const float* g, long long stride,
                 int len, const void* v_next, cudaStream_t s);
// One read-modify-write per touched row of the chunk starting at workspace token wt0.
int launch_write(const Dims& d, const Work& w, float* V, int wt0, cudaStream_t s);
// Entropy key step for the chunk whose distances are in Dfull/Z (`len` tokens).
int launch_address(const Dims& d, const Work& w, float* K1, float* K2, const void* q,
                   long long q_stride, int len, cudaStream_t s);

// ---- small device helpers ----
__device__ __forceinline__ float load_qv(const float* p, long long i) { return p[i]; }
__device__ __forceinline__ float load_qv(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}

// Total order on floats (NaN largest) as an unsigned key.
__device__ __forceinline__ uint32_t orderable(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long warp_min_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y < x ? y : x;
  }
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

}  // namespace fwpkm
