// fwpkm_internal.cuh -- shared declarations of the B200 FwPKM library (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "fwpkm.h"

namespace fwpkm {

// Device status word values (latched by kernels, read by fwpkm_sync).
enum : int { DEV_OK = 0, DEV_BAD_SLOT = 1, DEV_TIMEOUT = 2 };

// Latch a device-detected error: the device status word (read by the sync calls) and,
// when the handle has one, its host-visible copy in mapped pinned host memory, which the
// next host call reads without waiting for the GPU.
__device__ __forceinline__ void raise_status(int* dev, int* host, int code) {
  atomicExch(dev, code);
  if (host) {
    *reinterpret_cast<volatile int*>(host) = code;
    __threadfence_system();
  }
}

// Status of a device word value as returned by the C ABI.
inline fwpkm_status status_of_device(int h) {
  return h == DEV_OK ? FWPKM_OK : h == DEV_TIMEOUT ? FWPKM_ERR_TIMEOUT
                              : h == DEV_BAD_SLOT ? FWPKM_ERR_BAD_SLOT : FWPKM_ERR_CUDA;
}

// Test hook of the timeout path (fwpkm_test_stall_waits): launches of the kernels with
// bounded waits that should wait once on something nothing completes.  Returns 1 (and
// counts one down) while any remain.
int take_test_stall();
bool test_stalls_pending();

// Kernel kinds for the launch counter / per-kernel timing.
enum KernelKind : int { KK_NONE = 0, KK_GATHER = 1, KK_WRITE = 2, KK_SCORE = 3, KK_CART = 4,
                        KK_SORT = 5, KK_ADDR = 6, KK_OTHER = 7, KK_TOPK = 8, KK_PREP = 9, KK_PBAR = 10,
                        KK_WBUILD = 11, KK_FUSED = 12, KK_VLOOP = 13, KK_LAST = 13 };

struct Dims {
  int n, h, d, dv, k, C, M;
  int H, B;  // heads per value table (1: independent memories) and value tables (M / H)
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
  unsigned long long* sk; // [M][max_chunks][C*k] read pairs (slot << 32 | t_local*k + r), each
                          // slot's pairs contiguous and in token order
  int32_t* npairs;   // [M][max_chunks]    pairs in the chunk's list
  float* resid;      // [M][C][dv]         vhat, then r_t = g_t (vhat_t - tau_t)
  float* Dfull;      // [M][2][C][n]       key update: all sub-key distances of the chunk
  float* Z;          // [M][2][C]          key update: sum_a 1/(eps + D)
  float* lp;         // [M][2][n]          key update: log pbar
  float* Lt;         // [M][2][C]          key update: sum_a P log pbar
  int* status;       // device status word
  int* hstat;        // device view of the handle's mapped host copy of it (nullptr: none)
  // tensor-core path (bf16 q, d/2 in {64, 128})
  int tc;            // 1 if the tensor-core path is used
  int drows;         // rows of Dfull per problem (C with the key step, else the addressing window)
  __nv_bfloat16* Kpc;// [3][M*2][n][h]     bf16 pieces hi/mid/lo of the keys
  float* kn;         // [M*2][n]           squared key norms
  float* qn;         // [M*2][max_T]       squared half-query norms
  float* zpart;      // [M*2][C][n/128][4] per-32-column partial sums of 1/(eps + D)
  float* ppart;      // [M*2][PBAR_SLICES][n] partial column sums for pbar
  __nv_bfloat16* Wt; // [2][M*2][n][Cpad]  key-step weights, sub-key major, bf16 pieces hi, lo
  __nv_bfloat16* Qt; // [M*2][h][qt_T]     half-queries, feature major (operand B of the key step)
  int qt_T;          // token columns of Qt (a multiple of 64)
  float* wsum_part;  // [M*2][Cpad/16][n]  per-16-token-block sums of W
  int* pbar_cnt;     // [M*2][ceil(n/256)] arrival counters of the pbar column blocks (zero between launches)
  float* af_part;    // [M*2][n/128][2][256] one-launch addressing: every CTA's partial Z_t and L_t
  int* af_cnt;       // [M*2][2]           its arrival counters (zero between launches)
  unsigned* vl_cnt;  // [M][2]             persistent value loop: arrivals, exits (zero between launches)
  // Every array above is memory-major except the bf16 pieces (Kpc, Wt), whose piece
  // stride is P_all problems; a Work for a group of memories is the same carve with its
  // pointers advanced to the group's first memory (see group_work).
  int P_all;         // problems between consecutive bf16 pieces of Kpc / Wt (2 * all memories)
  long long dfull_buf; // elements between the two distance-row buffers
  // token-at-a-time inference: the pending chunk's inputs (nullptr when not carved)
  void* stage_q;     // [M][C][d]     q of the pending chunk (qv dtype)
  void* stage_v;     // [M][C+1][dv]  v of the pending chunk; row C: the lookahead token's v
  float* stage_g;    // [M][C+1]      g of the pending chunk
};

enum : int { TC_EPI_DIST = 0, TC_EPI_KEYSTEP = 1, TC_EPI_PROJ = 2 };

// Token slices of the usage-marginal pass (pbar): each column's sum is formed in up to
// this many partial sums, one per CTA slice (8 by default; FWPKM_PBAR_SLICES=16 for 16).
constexpr int PBAR_SLICES = 16;
int pbar_slices();

// One batched tensor-core contraction (see tc_gemm.cu).  Problem p (blockIdx.z) owns
// A tiles at (x = (p % a_div) * a_xoff + 64 kb, y = a_y0 + 128 mt, z = p / a_div + pa * a_zpiece)
// and B tiles at (x = b_x0 + 64 kb, y = 128 nt, z = p + pb * b_zpiece).
struct TcGemm {
  int P, k_blocks, n_tiles, tiles_per_cta;
  int stages;  // pipeline stages (set by launch_tc_gemm)
  int a_pieces, b_pieces;
  int a_div, a_xoff, a_y0, a_zpiece, b_zpiece, b_x0;
  int m_valid, n_valid;
  int epi;
  // TC_EPI_DIST
  float* out; long long out_pstride; int out_ld;
  const float* rowv; long long rowv_pstride; int rowv_off;
  const float* colv; long long colv_pstride;
  float* zpart; long long zpart_pstride; float eps;
  // TC_EPI_KEYSTEP
  float* K1; float* K2; __nv_bfloat16* Kpc; float* kn; int piece_P;
  const float* wsum_part; int wsum_tiles; float lr;
  // TC_EPI_PROJ: y[r][c] = acc * rowscale[r] + bias[c] (n_valid and split multiples of 32)
  // into pout0[r][c] (c < split) or pout1[r][c - split], fp32 or (out_bf16) bf16
  const float* rowscale; const float* bias;
  void* pout0; void* pout1; int split, ld0, ld1, out_bf16;
  int* status;
  int* hstat;  // mapped host copy of the status word (nullptr: none)
  int stall;   // test hook: the MMA issuer first waits on a barrier that nothing completes
};

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint64_t pitch_y,
                       uint64_t pitch_z);
bool make_tmap_f32_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint64_t pitch_y,
                      uint64_t pitch_z, uint32_t box_x, uint32_t box_y);
int launch_tc_gemm(const CUtensorMap& A, const CUtensorMap& B, const TcGemm& g, int m_tiles, cudaStream_t s);

// stream_stage: also carve the staging rows of token-at-a-time inference (at the end).
// allow_tc: false carves only what the CUDA-core kernels use (no tensor-core buffers).
size_t workspace_bytes(const Dims& d, int max_T, Work* carve, char* base, bool stream_stage = true,
                       bool allow_tc = true);
// The carve `w` of all memories seen from memory m0 on (kernels index it from 0).
Work group_work(const Dims& d, const Work& w, int m0);

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
// Token-at-a-time inference: copy `len` tokens (rows of `words` 32-bit words, per memory
// `src_stride` rows apart) of up to three inputs into staging rows r0.. (`dst_stride` rows
// per memory).  A job with a null source is skipped.
struct StageJob {
  const void* src;
  void* dst;
  long long src_stride, dst_stride;
  int words;
};
// With `qn_src` (bf16 queries of the staged tokens, per memory `qn_stride` rows apart), the
// same launch also writes their squared half norms to w.qn at tokens r0.. (qnorm_row).
int launch_stage(const Dims& d, const StageJob (&jobs)[3], int r0, int len, cudaStream_t s,
                 const Work* w = nullptr, const void* qn_src = nullptr, long long qn_stride = 0);
// Streaming write path: turn the stored vhat of a chunk into residuals.
int launch_resid(const Dims& d, const Work& w, const void* v, const float* g, long long stride,
                 int len, const void* v_next, cudaStream_t s);
// One read-modify-write per touched row of the chunk starting at workspace token wt0.
int launch_write(const Dims& d, const Work& w, float* V, int wt0, cudaStream_t s);
// Frozen keys: the read and write of chunks [c0, c1) of every table in one persistent
// launch (v, g, o of stride T per table, as for launch_gather with the lookahead target).
// Returns 0 (nothing launched) when the loop is switched off (FWPKM_VALUE_LOOP=0) or
// the GPU cannot hold the grid; the caller then launches the chunks one by one.
int launch_value_loop(const Dims& d, const Work& w, float* V, const void* v, const float* g, int T, int c0, int c1,
                      float* o, cudaStream_t s);
bool value_loop_enabled();
// The read path's backward (dq, dv, dg from dL/do) for `len` tokens of every memory.
int launch_read_backward(const Dims& d, const float* K1, const float* K2, const float* V, const void* q,
                         const void* v, const float* g, const int32_t* idx, const float* d_o, int len,
                         long long stride, float* dq, float* dv, float* dg, cudaStream_t s);
// Entropy key step for the chunk whose distances are in Dfull/Z (`len` tokens).
int launch_address(const Dims& d, const Work& w, float* K1, float* K2, const void* q,
                   long long q_stride, int len, cudaStream_t s);

// ---- tensor-core path ----
// Squared norms of both halves of q for `len` tokens (workspace tokens wt0..).
int launch_qnorm(const Dims& d, const Work& w, const void* q, long long q_stride, int wt0, int len, cudaStream_t s);
// bf16 pieces + squared norms of the current keys.
int launch_keyprep(const Dims& d, const Work& w, const float* K1, const float* K2, cudaStream_t s);
// Distances of `len` tokens (workspace tokens wt0.., user q pointer at the range start,
// q extent T_ext tokens per memory) into Dfull rows 0..len-1, plus zpart if key_update.
int launch_tc_score(const Dims& d, const Work& w, const void* q_base, long long q_stride, int q_extent, int q_row0,
                    int wt0, int len, bool key_update, cudaStream_t s);
// Fused per-half top-k + Cartesian search + softmax from Dfull rows 0..len-1 (workspace
// tokens wt0..): writes idx, w and the optional user copies; A/Dsv are not written.
int launch_select(const Dims& d, const Work& w, int wt0, int len, int32_t* idx_out, float* w_out, cudaStream_t s);
// Feature-major copy of both half-queries of `len` tokens into Qt columns qt0.. (the key
// step's B operand).
int launch_qtrans(const Dims& d, const Work& w, const void* q, long long q_stride, int qt0, int len, cudaStream_t s);
// Entropy key step from Dfull/zpart (tensor-core path), in three launches: pbar (Z,
// column sums, lp), wbuild (L_t and the bf16 pieces of W), keystep (the GEMM and the key
// update).  The chunk's half-queries are read from Qt columns qt_t0..; qt_t0 < 0:
// keystep transposes them first into columns 0.. .
int launch_tc_pbar(const Dims& d, const Work& w, int len, cudaStream_t s);
int launch_tc_wbuild(const Dims& d, const Work& w, int len, cudaStream_t s);
int launch_tc_keystep(const Dims& d, const Work& w, float* K1, float* K2, const void* q, long long q_stride, int len,
                      int qt_t0, cudaStream_t s);

// ---- fused addressing (addr_fused.cu) ----
// Whether the key-update path takes the one-launch addressing step of a chunk (bf16 q,
// d/2 in {64, 128}, n a multiple of 128, C <= 256 and a multiple of 16, and the launch's
// 2 M n / 128 CTAs no more than the GPU's SMs; FWPKM_FUSED_ADDR=0 turns it off).
bool use_fused_addressing(const Dims& d);
// Distances of `len` tokens (workspace tokens wt0.., half-query rows q_row0.. of a map over
// q_base with q_extent rows per memory, q_stride tokens apart) into Dfull rows 0..len-1,
// then (unless score_only) the whole entropy key step of those tokens: K1, K2, their bf16
// pieces and squared norms updated in place.  The chunk's feature-major half-queries are
// read from Qt columns qt_x0.. .  One launch of n/128 CTAs per problem (one per SM).
int launch_addr_fused(const Dims& d, const Work& w, float* K1, float* K2, const void* q_base, long long q_stride,
                      int q_extent, int q_row0, int wt0, int len, int qt_x0, bool score_only, cudaStream_t s);
// Floats of the partial-sum buffer (af_part) for the memories of `d`.
size_t addr_fused_part_floats(const Dims& d);

// ---- launches ----
// Whether kernels are launched with programmatic dependent launch.  Off by default for the
// chunk schedule (on the paper-scale step the early-resident dependents held SM slots that
// the other chains' kernels needed: 1.53 ms per step against 1.42 ms without); on inside a
// PdlScope, which the token-at-a-time calls on the tensor-core path open (their reads are
// chains of small dependent launches on one stream: 26.8 us per token against 34.1 us at
// one token per call).  FWPKM_PDL=1 turns it on everywhere, FWPKM_PDL=0 off everywhere.
bool pdl_enabled();
extern thread_local bool pdl_scope;
struct PdlScope {
  bool prev;
  explicit PdlScope(bool on) : prev(pdl_scope) { pdl_scope = prev || on; }
  ~PdlScope() { pdl_scope = prev; }
  PdlScope(const PdlScope&) = delete;
  PdlScope& operator=(const PdlScope&) = delete;
};
// With FWPKM_CARVEOUT=1, give `kern` the largest shared-memory carveout once per process,
// so that an SM never has to drain to switch its L1/shared split before a CTA of another
// kernel can start beside the running ones.  Off by default: the smaller L1 it leaves
// cost more than the switches (2.02 ms per paper-scale step against 1.73 ms without).
void set_carveout(const void* kern);
// Raise `kern`'s dynamic shared-memory limit to at least `bytes` (never lowered, so that a
// launch captured earlier with more never finds the function's limit below its own need).
// Returns false if the attribute cannot be set.
bool raise_smem_limit(const void* kern, size_t bytes);

// Launch `kern` on `s`, allowing it to start while the previous kernel of the same stream
// finishes (programmatic stream serialization).  Every kernel launched this way calls
// pdl_wait() before it touches memory that an earlier kernel writes, so the overlap
// covers only its launch and set-up.
// An NVTX range named after the C-ABI call that opens it, for the Nsight tools' timelines
// (a no-op when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// The configuration a layer handle was created with (nullptr for a null handle).
const fwpkm_layer_config* layer_config(const fwpkm_layer* L);

// Adds kernel launches made outside a state's schedule (layer projections, metrics) to
// the count fwpkm_launch_count() reports.
void count_launches(int n);

// Scheduling priority given to the kernels launched by this host thread (set around a
// launcher call by the schedule; `launch_priority_set` false: the stream's own).
extern thread_local int launch_priority;
extern thread_local bool launch_priority_set;

template <typename... KArgs, typename... Args>
inline void launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  if (pdl_enabled()) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na++].val.programmaticStreamSerializationAllowed = 1;
  }
  if (launch_priority_set) {
    attr[na].id = cudaLaunchAttributePriority;
    attr[na++].val.priority = launch_priority;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  set_carveout((const void*)kern);
  cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// A cooperative launch: every CTA of the grid is resident at once, which a kernel whose
// CTAs wait for one another needs (no programmatic dependency: it starts after the
// stream's previous kernel has completed).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_coop(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               Args... args) {
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeCooperative;
  attr[na++].val.cooperative = 1;
  if (launch_priority_set) {
    attr[na].id = cudaLaunchAttributePriority;
    attr[na++].val.priority = launch_priority;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  set_carveout((const void*)kern);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Device side of programmatic dependent launch: wait until the preceding kernel of the
// stream has completed and its writes are visible (a no-op without a programmatic
// dependency), then let the next kernel of the stream begin its launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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

// ||q_half||^2 of one bf16 query row (both halves) by one warp into w.qn[m][half][t]: each
// lane sums its strided features in order, then a warp sum.  The chunk path's query-norm
// kernel and the token-at-a-time staging kernel both use it, so their norms have the same
// bits.
__device__ __forceinline__ void qnorm_row(const Dims& dm, const Work& w, const __nv_bfloat16* __restrict__ row,
                                          int m, long long t, int lane) {
  for (int j = 0; j < 2; ++j) {
    float s = 0.f;
    for (int e = lane; e < dm.h; e += 32) {
      float x = __bfloat162float(row[j * dm.h + e]);
      s += x * x;
    }
    s = warp_sum(s);
    if (lane == 0) w.qn[((size_t)m * 2 + j) * w.max_T + t] = s;
  }
}

}  // namespace fwpkm
