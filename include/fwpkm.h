/*
 * fwpkm.h -- C ABI of the B200 FwPKM retrieve + chunk-write library (libfwpkm.so).
 *
 * Fast-weight Product Key Memory keeps, per independent memory (one per sequence
 * and head), a value table V of N = n*n rows and two sub-key codebooks K1, K2 of n
 * keys each.  For every token of a chunk it reads the memory (product-key top-k
 * with inverse-distance scores, softmax weights, weighted sum of k value rows,
 * gated residual output); after the chunk it writes the memory (one gradient step
 * of the gated lookahead reconstruction loss, averaged per row by its read count)
 * and, optionally, takes an entropy gradient step on K1 and K2.
 *
 * Sources (page title, section):
 *   "快速权重积键值记忆 Fast-weight Product Key Memory" (rainbus summary), method
 *     steps 1-5 and the PKM prerequisite;
 *   "Fast-weight Product Key Memory" (paperlayer summary of arXiv 2601.00671v2),
 *     §2.2, §3.1-§3.5, §A.1-§A.5 and App. B.
 *
 * Conventions shared by every call:
 *   - Every device buffer is allocated and owned by the caller.  The library never
 *     allocates device memory; its scratch lives in the caller's workspace.
 *   - Memories are independent and laid out memory-major: m = b*H + head.
 *     Sequence inputs are [M][T][width] row-major; q's first d/2 entries are
 *     half 1.  V is [M][n*n][d_v] fp32 with slot i = a*n + b (a: half-1 sub-key,
 *     b: half-2 sub-key); K1, K2 are [M][n][d/2] fp32.
 *   - q and v are fp32 or bf16 (cfg.qv_dtype); g, o and the state are fp32.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only
 *     enqueues work on it and returns; results are ready when the stream is.
 *   - Calls return a status and never throw.  Argument checks run synchronously
 *     before anything is enqueued (then nothing is enqueued).  Errors detected on
 *     the device (FWPKM_ERR_TIMEOUT, FWPKM_ERR_BAD_SLOT) are latched in a device
 *     status word and in a copy of it in pinned host memory that the kernel writes
 *     when it detects the error.  fwpkm_sync() waits for the stream and returns the
 *     latched error, clearing it.  Every other call on the same handle first reads
 *     the host copy without waiting: once the error has reached it, the call returns
 *     that error and enqueues nothing, until fwpkm_sync() clears it.  (A call made
 *     while the failing kernel is still running cannot know yet: it returns OK.)
 *   - Results are deterministic: the same inputs give bit-identical outputs.
 */
#ifndef FWPKM_H
#define FWPKM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FWPKM_OK = 0,
  FWPKM_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned buffer            */
  FWPKM_ERR_UNSUPPORTED = -2, /* valid but outside the supported shape limits          */
  FWPKM_ERR_WORKSPACE = -3,   /* workspace smaller than fwpkm_workspace_size()         */
  FWPKM_ERR_CUDA = -4,        /* a CUDA runtime call failed                            */
  FWPKM_ERR_TIMEOUT = -5,     /* a bounded device-side wait gave up                    */
  FWPKM_ERR_STATE = -6,      /* call out of order (write_chunk without forward_chunk) */
  FWPKM_ERR_BAD_SLOT = -7     /* the write met a slot index outside [0, n*n); that row was skipped */
} fwpkm_status;

typedef enum { FWPKM_F32 = 0, FWPKM_BF16 = 1 } fwpkm_dtype;

/* cfg.flags */
enum {
  FWPKM_KEY_UPDATE = 1,  /* entropy step on K1, K2 after each chunk (rainbus step 5; paperlayer §3.4) */
  FWPKM_TARGET_NORM = 2, /* z-score the reconstruction target per token (paperlayer §A.3)            */
  FWPKM_LOOKAHEAD = 4,   /* target of token t is v_{t+1} (paperlayer §A.1); off: v_t (rainbus step 4) */
  FWPKM_GATE_WEIGHT = 8  /* weight each token's loss by g_t (paperlayer §A.5)                        */
};
#define FWPKM_DEFAULT_FLAGS (FWPKM_TARGET_NORM | FWPKM_LOOKAHEAD | FWPKM_GATE_WEIGHT)

/* Shape and hyper-parameters of M memories (heads).
 * Supported limits (else FWPKM_ERR_UNSUPPORTED):
 *   1 <= k <= 32, k <= n <= 4096, d even with 8 <= d <= 512, d_v % 4 == 0 with
 *   4 <= d_v <= 1024, 1 <= chunk <= 1024 with chunk*k*H <= 16384, num_mem >= 1;
 *   with v_heads = H > 1: num_mem % H == 0 and k*H <= 64.
 *
 * Heads sharing one value table (v_heads = H > 1; "Fast-weight Product Key Memory"
 * (paperlayer summary) §D.1 ablates the head count with the slot count, §D.3 notes that
 * more heads raise the collision rate): the memories m = b*H + h (h < H) of sequence b
 * have their own codebooks K1, K2 and queries q and select their own k slots, but read
 * and write one table V_b.  The read is the mean of the heads' reads,
 *   vhat_t = (1/H) sum_h sum_{i in I^h_t} s'^h_{t,i} V_b[i],
 * the write is the gradient of the gated reconstruction loss on the shared rows divided
 * by the number of the chunk's tokens that read a row through any head, and each head's
 * codebooks take their own addressing step.  Then V is [M/H][n*n][d_v] and v, g, o are
 * per sequence ([M/H][T][...]); q, K1, K2, idx_out, w_out stay per head.  Token-at-a-time
 * inference, the allocation-free step and fwpkm_run_layer take v_heads <= 1 only. */
typedef struct {
  int n;         /* sub-keys per codebook; the memory has N = n*n slots              */
  int d;         /* query width (two halves of d/2)                                  */
  int d_v;       /* value width                                                      */
  int k;         /* per-half top-k and final top-k                                   */
  int chunk;     /* C, tokens per fast-weight update                                 */
  int num_mem;   /* M independent memories                                           */
  int qv_dtype;  /* fwpkm_dtype of q and v                                           */
  float eps_idw; /* IDW score sigma = -log(eps_idw + ||q_j - K_j[a]||^2)              */
  float eps_norm;/* z-score: (u - mean) / sqrt(var + eps_norm)                       */
  float lr_key;  /* step size of the key update                                      */
  unsigned flags;/* FWPKM_* flags                                                    */
  int v_heads;   /* heads per value table (0 or 1: every memory has its own V)      */
} fwpkm_config;

/* Opaque host-side handle.  It records the caller's state pointers and the carved
 * workspace; it owns no device memory (only CUDA streams/events/graphs and one word of
 * pinned host memory, the host copy of the status word). */
typedef struct fwpkm_state fwpkm_state;

/* Bytes of device workspace needed for sequences of up to max_T tokens.
 * Returns FWPKM_ERR_INVALID_ARG / FWPKM_ERR_UNSUPPORTED for a bad config. */
fwpkm_status fwpkm_workspace_size(const fwpkm_config* cfg, int max_T, size_t* bytes);

/* Validate cfg, record the caller-owned state (K1, K2 [M][n][d/2] fp32 and
 * V [M][n*n][d_v] fp32, all device pointers, 16-byte aligned) and carve the
 * workspace (device, >= fwpkm_workspace_size(cfg, max_T), 256-byte aligned).
 * The state tensors are read and written in place by later calls; the caller
 * keeps them and the workspace alive until fwpkm_destroy_state().  Nothing is
 * enqueued.  (Host-only; the state's memory can persist across sequences, which
 * is how memory carries over sequence boundaries, paperlayer §E.1.) */
fwpkm_status fwpkm_init_state(const fwpkm_config* cfg, float* K1, float* K2, float* V, int max_T,
                              void* workspace, size_t ws_bytes, fwpkm_state** out);

/* Read phase of one chunk for all M memories (rainbus steps 2-3; paperlayer §2.2,
 * §3.2, §A.2): per-half IDW top-k, restricted Cartesian top-k, softmax weights,
 * vhat_t = sum_i s'_{t,i} V_i and o_t = g_t vhat_t + (1 - g_t) v_t, all against
 * the state left by the previous chunk (paperlayer §3.1 causality).
 *   q  device, element (m, t, e) at q[(m*seq_stride + t)*d + e]   (qv_dtype)
 *   v  device, element (m, t, e) at v[(m*seq_stride + t)*d_v + e] (qv_dtype)
 *   g  device fp32, (m, t) at g[m*seq_stride + t]
 *   c_len tokens in this chunk, 1 <= c_len <= cfg.chunk; seq_stride >= c_len
 *   o  device fp32 output, (m, t, e) at o[(m*seq_stride + t)*d_v + e]
 *   idx_out [M][c_len][k] int32 and w_out [M][c_len][k] fp32 (device, nullable):
 *      selected slots in rank order (score desc, slot asc) and their weights.
 * q, v, g must stay valid until the matching fwpkm_write_chunk() has run. */
fwpkm_status fwpkm_forward_chunk(fwpkm_state* st, const void* q, const void* v, const float* g,
                                 int c_len, int seq_stride, float* o, int32_t* idx_out,
                                 float* w_out, void* stream);

/* Write phase of the chunk last passed to fwpkm_forward_chunk (rainbus steps 4-5;
 * paperlayer §3.3, §3.4, §A.1-§A.5): for every slot i read by a token that has a
 * target, V_i -= (sum_t s'_{t,i} g_t (vhat_t - z(u_t))) / N_read,i with u_t the
 * lookahead value; then, if FWPKM_KEY_UPDATE, K_j -= lr_key * dL_addr/dK_j with
 * L_addr = -H(pbar_1) - H(pbar_2) taken at the keys the chunk was read with.
 *   v_next  device, value of the token after the chunk for each memory, element
 *           (m, e) at v_next[m*seq_stride*d_v + e] (same seq_stride as the forward
 *           call), or NULL when the chunk ends the sequence: its last token then has
 *           no lookahead target and is left out of the write and of N_read.
 * Returns FWPKM_ERR_STATE if no forward_chunk is pending. */
fwpkm_status fwpkm_write_chunk(fwpkm_state* st, const void* v_next, void* stream);

/* The whole chunk-sequential loop over a sequence of T tokens (1 <= T <= max_T)
 * for all M memories, repeated n_iter >= 1 times over the same input with the
 * state carried across chunks and passes (paperlayer §3.1, §4.3 iterative
 * reading).  Equivalent to forward_chunk/write_chunk over consecutive chunks with
 * v_next = the following token (NULL for the last chunk), but scheduled as one
 * stream-ordered program (addressing, which never depends on V, runs ahead of the
 * value loop).  q, v, g, o use the forward_chunk layout with seq_stride = T;
 * o receives the final pass.  T = 0 is a no-op. */
fwpkm_status fwpkm_run_sequence(fwpkm_state* st, const void* q, const void* v, const float* g,
                                int T, int n_iter, float* o, void* stream);

/* fwpkm_run_sequence from host memory (no counterpart in the paper: the end-to-end call).
 * q, v, g, o are HOST buffers in the fwpkm_run_sequence layout (seq_stride = T), and
 * must be page-locked (cudaHostAlloc, or cudaHostRegister'd): anything else returns
 * FWPKM_ERR_INVALID_ARG.  The call copies chunk c's inputs to device scratch while
 * earlier chunks compute (cudaMemcpy2DAsync on an internal stream), starts each chunk's
 * kernels when its inputs (and the lookahead row after it) have landed, and copies each
 * chunk's final-pass o back as soon as it is written, so the copies overlap the compute.  Everything is enqueued on
 * `stream` (captured once into the state's cached graph, like fwpkm_run_sequence); the
 * host buffers must stay valid, and o unread, until the stream passes the call.
 *   scratch  device, 256-byte aligned, >= fwpkm_run_sequence_host_scratch_size(cfg, T)
 *            bytes (device copies of q, v, g and o, each on a 256-byte boundary); too
 *            small: FWPKM_ERR_WORKSPACE.
 * Results are bit-identical to fwpkm_run_sequence on the same inputs. */
fwpkm_status fwpkm_run_sequence_host_scratch_size(const fwpkm_config* cfg, int T, size_t* bytes);
fwpkm_status fwpkm_run_sequence_host(fwpkm_state* st, const void* q, const void* v, const float* g,
                                     int T, int n_iter, float* o, void* scratch, size_t scratch_bytes,
                                     void* stream);

/* The read path's backward: the gradient that reaches the slow weights' outputs q, v, g
 * from an upstream dL/do ("Fast-weight Product Key Memory" (paperlayer summary) §2 /
 * Figure 1: slow weights learn during training; §3.1-§3.2: the read o = g vhat + (1-g) v,
 * vhat = sum_i s'_i V_i, s' = softmax over the selected slots of sigma_1 + sigma_2,
 * sigma = -log(eps_idw + ||q_j - K_j||^2)).  The fast weights V, K1, K2 as they were when
 * the tokens were read are constants (they learn only from their own chunk-local losses),
 * and the discrete selection passes no gradient.  Per token with slots I (rank order):
 *   dg = <dL/do, vhat - v>, dv = (1 - g) dL/do,
 *   dq_j = sum_r dS_r (-2 / (eps_idw + D_j,r)) (q_j - K_j[row of slot r]),
 *   dS = s' (ds - <s', ds>), ds_r = <g dL/do, V_{I_r}>;
 * the distances and weights are recomputed from q, K1, K2 (direct form).  Stateless: no
 * handle, no workspace.  cfg.v_heads > 1: FWPKM_ERR_UNSUPPORTED.
 *   K1, K2, V   device fp32, the state the tokens were read with ([M][n][d/2], [M][n*n][d_v])
 *   q, v, g     device, the forward_chunk layout (seq_stride >= len)
 *   idx         device int32 [M][len][k]: the slots the forward read (forward_chunk's idx_out);
 *               slots outside [0, N) contribute nothing
 *   d_o         device fp32, (m, t, e) at d_o[(m*seq_stride + t)*d_v + e]
 *   dq, dv, dg  device fp32 outputs in the q, v, g layouts (seq_stride)
 * V, d_o and dv must be 16-byte aligned.  len = 0 is a no-op. */
fwpkm_status fwpkm_read_backward(const fwpkm_config* cfg, const float* K1, const float* K2, const float* V,
                                 const void* q, const void* v, const float* g, const int32_t* idx,
                                 const float* d_o, int len, int seq_stride, float* dq, float* dv, float* dg,
                                 void* stream);

/* Token-at-a-time inference ("Fast-weight Product Key Memory" (paperlayer summary),
 * §A.1: at inference the memory accumulates (q_t, v_{t+1}) pairs and writes once a
 * chunk's worth is ready).  Each call reads n_tok >= 1 new tokens of every memory at once,
 * in order, against the state left by the last write, and writes o for them; the tokens
 * are staged in the workspace.  A chunk of cfg.chunk pending tokens is written as soon as
 * the token after it arrives (that token's v is the lookahead target of the chunk's last
 * token), before that token is read; fwpkm_stream_flush() writes a partial or full
 * pending chunk with no lookahead (end of the sequence).  The tokens of a sequence fed in
 * any grouping followed by a flush give the outputs and final state of
 * fwpkm_run_sequence over the same tokens (n_iter = 1).
 *   q, v, g, o  device, element (m, t, e) of the call's tokens at q[(m*seq_stride + t)*d + e]
 *               etc., as in fwpkm_forward_chunk (seq_stride >= n_tok); read/written by work
 *               enqueued on `stream` (keep them until the stream passes the call).
 * The state must have been initialised with max_T >= cfg.chunk (else
 * FWPKM_ERR_UNSUPPORTED).  While tokens are pending, fwpkm_forward_chunk and
 * fwpkm_run_sequence return FWPKM_ERR_STATE, and the caller must not change K1, K2, V
 * (between chunks it may: the keys are re-read at the start of every chunk).  With the
 * key update, a chunk's write recomputes its distance rows from the staged queries. */
fwpkm_status fwpkm_stream_tokens(fwpkm_state* st, const void* q, const void* v, const float* g, int n_tok,
                                 int seq_stride, float* o, void* stream);

/* End of a token-at-a-time sequence: write the pending tokens (if any) with no lookahead
 * target for the last one.  No-op when nothing is pending. */
fwpkm_status fwpkm_stream_flush(fwpkm_state* st, void* stream);

/* Tokens read by fwpkm_stream_tokens and not yet written (0 .. cfg.chunk), host-only.
 * Checkpoint/resume of a token-at-a-time sequence: save K1, K2, V (the caller's tensors)
 * after the last write together with the inputs of the pending tokens; on resume, feed
 * those tokens again -- the reads depend only on the saved state, so the outputs and the
 * staged chunk come back bit for bit. */
fwpkm_status fwpkm_stream_pending(const fwpkm_state* st, int* n_pending);

/* One whole chunk step -- the read of fwpkm_forward_chunk followed by the write (and
 * key step) of fwpkm_write_chunk -- that allocates nothing and needs no workspace.
 * The paper has no counterpart: this exists for callers that cannot allocate device
 * memory (loops under a no-allocation rule, plugins whose host owns the allocator, code
 * that must not change the device memory map).  It makes CUDA calls and launches
 * kernels, so it must not be called from a CUDA host function (stream callback).
 * Arguments mean what they mean in fwpkm_forward_chunk / fwpkm_write_chunk (K1, K2, V
 * are the caller's state, updated in place; v_next NULL = the chunk ends the sequence).
 * It runs the CUDA-core kernels of the chunk step, whatever the shape.
 * Scratch is a fixed 16 MiB array inside the library that every GPU loading the
 * library keeps until exit; shapes whose scratch for one chunk on the CUDA-core kernels
 * (the workspace of one chunk without the tensor-core buffers and the staging rows of
 * token-at-a-time inference) exceeds it are rejected with FWPKM_ERR_UNSUPPORTED.  The
 * first call on a device looks up that array's device address (make it before any
 * stream capture).  All calls share the array: calls that overlap on the GPU race and
 * must be serialised by the caller.  Device-side errors are not reported by this entry
 * point. */
fwpkm_status fwpkm_chunk_step_noalloc(const fwpkm_config* cfg, float* K1, float* K2, float* V,
                                      const void* q, const void* v, const float* g, const void* v_next,
                                      int c_len, int seq_stride, float* o, void* stream);

/* ---------------------------------------------------------------------------
 * Slow-weight projections around the memory ("快速权重积键值记忆 Fast-weight Product
 * Key Memory" (rainbus summary), method steps 1 and 3):
 *   q_t = Linear_q(RMSNorm_q(h_t)), v_t = Linear_v(RMSNorm_v(h_t)),
 *   g_t = sigmoid(Linear_g(RMSNorm_g(h_t))), o'_t = Linear_o(RMSNorm_o(o_t)),
 * with RMSNorm(x) = x / sqrt(mean(x^2) + eps_rms) * gamma and Linear(x) = x W^T + b.
 * The rows (tokens) of h, q, v, g, o and o' are [rows][width] row-major; with one
 * head per sequence the memory index is the sequence, so q, v, g and o are exactly
 * the [M][T][width] inputs and output of the memory calls above.
 * Precision: h and the weights W are bf16; the norm weights, biases, g and o fp32;
 * q and v fp32 or bf16 (fwpkm_layer_config.qv_dtype); o' bf16.  gamma is folded into
 * W in fp32 (three bf16 pieces for the input GEMM, two for the output GEMM; one when
 * gamma is NULL, as W is then exact); o enters the output GEMM as two bf16 pieces;
 * accumulation is fp32 on the tensor cores and 1/rms scales the accumulator.
 * ------------------------------------------------------------------------- */
typedef struct fwpkm_layer fwpkm_layer;  /* opaque host handle */

/* Supported limits (else FWPKM_ERR_UNSUPPORTED): d_model % 64 == 0 with
 * 64 <= d_model <= 16384; d % 32 == 0, d_v % 64 == 0, 32 <= d, d_v <= 1024;
 * max_rows >= 1. */
typedef struct {
  int d_model;   /* width of h and o'                                   */
  int d;         /* query width                                         */
  int d_v;       /* value width                                         */
  int max_rows;  /* most rows (tokens) of one layer_in / layer_out call */
  float eps_rms; /* RMSNorm epsilon                                     */
  int qv_dtype;  /* fwpkm_dtype of the q and v that fwpkm_layer_in writes */
} fwpkm_layer_config;

/* Parameters (device pointers, read only during fwpkm_layer_set_params).  W_* are
 * bf16 [out][in]: W_q [d][d_model], W_v [d_v][d_model], w_g [d_model],
 * W_o [d_model][d_v].  gamma_* are fp32 [in] (NULL = ones); b_* fp32 [out]
 * (NULL = zeros); b_g is the gate's scalar bias. */
typedef struct {
  const void* W_q; const float* gamma_q; const float* b_q;
  const void* W_v; const float* gamma_v; const float* b_v;
  const void* w_g; const float* gamma_g; float b_g;
  const void* W_o; const float* gamma_o; const float* b_o;
} fwpkm_layer_params;

/* Bytes of device workspace (folded weights, biases and the output call's per-row
 * scratch) for `cfg`.  The workspace must be 256-byte aligned. */
fwpkm_status fwpkm_layer_workspace_size(const fwpkm_layer_config* cfg, size_t* bytes);

/* Create a handle over the caller's workspace.  Nothing is enqueued. */
fwpkm_status fwpkm_layer_init(const fwpkm_layer_config* cfg, void* workspace, size_t ws_bytes,
                              fwpkm_layer** out);

/* Fold the norm weights into the linear weights (fp32 product, split into bf16
 * pieces) and copy the biases into the workspace.  Enqueued on `stream`; the
 * parameters may be freed once the stream has passed this point. */
fwpkm_status fwpkm_layer_set_params(fwpkm_layer* L, const fwpkm_layer_params* p, void* stream);

/* Method step 1 for rows <= max_rows tokens: h bf16 [rows][d_model] (16-byte
 * aligned) -> q [rows][d], v [rows][d_v] (cfg.qv_dtype: fp32, or bf16 rounded to
 * nearest from the fp32 result; 16-byte aligned) and g fp32 [rows].  rows == 0 is a no-op.  One row-statistics kernel (1/rms and the gate)
 * and one tensor-core GEMM with both outputs in its epilogue.  Uses the workspace's
 * per-row scratch, so calls on one handle must not overlap on the GPU. */
fwpkm_status fwpkm_layer_in(fwpkm_layer* L, const void* h, int rows, void* q, void* v, float* g,
                            void* stream);

/* Method step 3, output side, for rows <= max_rows tokens: o fp32 [rows][d_v] ->
 * o' bf16 [rows][d_model] (both 16-byte aligned).  Uses the workspace's per-row
 * scratch, so calls on one handle must not overlap on the GPU. */
fwpkm_status fwpkm_layer_out(fwpkm_layer* L, const float* o, int rows, void* o_out, void* stream);

/* Wait for `stream` and return the handle's latched device status (a GEMM wait
 * that timed out gives FWPKM_ERR_TIMEOUT), clearing it.  As for fwpkm_state, the other
 * calls on the handle return a latched error once its host copy shows it. */
fwpkm_status fwpkm_layer_sync(fwpkm_layer* L, void* stream);

/* Release the handle (the workspace is the caller's). */
void fwpkm_layer_destroy(fwpkm_layer* L);

/* The whole FwPKM layer ("快速权重积键值记忆 Fast-weight Product Key Memory" (rainbus
 * summary), method steps 1-5) for M = cfg.num_mem sequences of one head each: method
 * step 1 (fwpkm_layer_in on the M*T rows of h), the chunk-sequential memory loop over
 * T tokens with n_iter passes (fwpkm_run_sequence), then the output projection of method
 * step 3 (fwpkm_layer_out) on the final pass's o.  One call, stream-ordered.
 *   L, st    the projections and the memory state; they must agree on d, d_v and the q/v
 *            dtype, with M*T <= the layer's max_rows and T <= the state's max_T
 *            (else FWPKM_ERR_INVALID_ARG).
 *   h        device bf16 [M][T][d_model] (16-byte aligned); o_out device bf16
 *            [M][T][d_model] (16-byte aligned).
 *   scratch  device, 256-byte aligned, scratch_bytes >= fwpkm_run_layer_scratch_size()
 *            (else FWPKM_ERR_WORKSPACE).  It receives, in this order, each part starting
 *            on a 256-byte boundary: q [M][T][d] and v [M][T][d_v] (q/v dtype), g [M][T]
 *            fp32 and o [M][T][d_v] fp32 -- the memory's inputs and output, readable once
 *            the stream has passed the call.
 * T = 0 is a no-op.  Errors are those of the three calls it makes (the first failing
 * one is returned; nothing after it is enqueued). */
fwpkm_status fwpkm_run_layer_scratch_size(const fwpkm_config* cfg, int T, size_t* bytes);
fwpkm_status fwpkm_run_layer(fwpkm_layer* L, fwpkm_state* st, const void* h, int T, int n_iter, void* scratch,
                             size_t scratch_bytes, void* o_out, void* stream);

/* Copy the slot indices and softmax weights that the most recent call computed for
 * tokens [0, T) of every memory (final pass of fwpkm_run_sequence, the chunk of
 * fwpkm_forward_chunk with T <= c_len, or -- after fwpkm_stream_tokens -- the positions
 * 0..T-1 of the current or last written chunk) into idx_out [M][T][k] int32 and
 * w_out [M][T][k] fp32 (device, either nullable).  Enqueued on `stream`.  Used for
 * inspection and for comparing selections against a reference. */
fwpkm_status fwpkm_last_addressing(fwpkm_state* st, int T, int32_t* idx_out, float* w_out, void* stream);

/* ---------------------------------------------------------------------------
 * Addressing metrics ("Fast-weight Product Key Memory" (paperlayer summary), §D.3
 * Addressing Metrics): slot-use balance of the reads over windows of tokens.
 * The row contribution c_i of slot i is how many accesses it receives in a window,
 * an access being one (token, selected slot) pair; windows are consecutive blocks of
 * `window` tokens of each memory (the paper uses 32768; the last window may be
 * shorter).  Per (memory, window):
 *   coverage  = #{i : c_i > 0} / N
 *   collision = (accesses whose slot receives >= 2 accesses in the window) / (accesses)
 *   KLD       = sum_i p_i log(p_i N), p_i = c_i / sum c   (KL to uniform, natural log)
 * (all three 0 for a window without accesses).  Entries outside [0, N) are not
 * accesses and are counted apart.
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace that lets fwpkm_addressing_metrics histogram up to 32
 * windows at once (4 * N bytes plus 8 KiB per window).  Any workspace that holds
 * one window works; a smaller one only processes fewer windows at a time. */
fwpkm_status fwpkm_metrics_workspace_size(int num_mem, int T, int N, int window, size_t* bytes);

/* Metrics of every (memory, window) of the selections idx.
 *   idx      device int32 [num_mem][T][k] (4-byte aligned): selected slots, as written by
 *            fwpkm_forward_chunk (idx_out) or fwpkm_last_addressing; read only.
 *   N        slots per memory (n*n); window >= 1 tokens; k >= 1.
 *   workspace device, 256-byte aligned, ws_bytes >= the one-window size (else
 *            FWPKM_ERR_WORKSPACE); scratch, contents need not be initialised.
 *   metrics  device fp64 [num_mem][W][3] (coverage, collision, KLD), W = ceil(T/window).
 *   counts   device int64 [num_mem][W][4] or NULL: rows accessed, accesses, competitive
 *            accesses, invalid entries -- exact integers.
 * Coverage and collision are exact ratios of those integers (fp64 division); KLD is
 * (sum_i c_i log c_i) / S + log(N / S) in fp64 with a fixed summation order, so the
 * call is deterministic.  T == 0 is a no-op.  Enqueued on `stream`; the workspace must
 * not be shared with a concurrent call. */
fwpkm_status fwpkm_addressing_metrics(const int32_t* idx, int num_mem, int T, int k, int N, int window,
                                      void* workspace, size_t ws_bytes, double* metrics, int64_t* counts,
                                      void* stream);

/* Wait for `stream` and return the latched device status (FWPKM_OK,
 * FWPKM_ERR_TIMEOUT, FWPKM_ERR_BAD_SLOT), clearing it (device word and host copy). */
fwpkm_status fwpkm_sync(fwpkm_state* st, void* stream);

/* Test hook of the timeout path (no counterpart in the paper).  Each of the next
 * `n_launches` launches made by this process of a kernel with a bounded wait (the
 * tensor-core scoring, key step and projections; the one-launch addressing step; the
 * persistent value loop of fwpkm_run_sequence with frozen keys) first waits on
 * something that nothing completes: an mbarrier for the MMA-issuing thread, or an
 * arrival count that no launch reaches for the value loop.  That wait is bounded like
 * every other wait in those kernels (0.2 s): it runs out, the kernel takes its abort
 * path (in-flight copies drained, tensor memory freed, no further work) and latches
 * FWPKM_ERR_TIMEOUT in the handle's status word.  Nothing faults and the context stays
 * usable.  n_launches = 0 cancels.  While a stall is pending fwpkm_run_sequence enqueues
 * its launches directly instead of through its cached CUDA graph. */
void fwpkm_test_stall_waits(int n_launches);

/* Release the handle (streams, events, graphs).  Caller buffers are untouched. */
void fwpkm_destroy_state(fwpkm_state* st);

/* Static description of a status code. */
const char* fwpkm_status_string(fwpkm_status s);

/* Number of kernels this library has launched in this process (graph replays count
 * every kernel node).  Used to report how many launches a timed region made. */
uint64_t fwpkm_launch_count(void);

/* Per-kernel timing with CUDA events recorded on the launching stream around every
 * launch of the given kernel kind (0 = none).  Kinds: 1 gather, 2 write, 3 score,
 * 4 cartesian, 5 sort, 6 key-step GEMM (or the whole key step on the SIMT path),
 * 7 residual, 8 per-half top-k (on the tensor-core path fused with the Cartesian
 * search), 9 query/key prep, 10 usage marginals (pbar, log pbar),
 * 11 key-step weights W, 12 the one-launch addressing step of a chunk (distances and,
 * with the key update, the whole entropy step).  fwpkm_kernel_time() waits for the events and
 * returns the summed duration (ms) and the number of timed launches since the last
 * reset, then resets.  Graph replays overwrite their own events, so after graph
 * replays it covers the last replay. */
#define FWPKM_PROFILE_ALL 100 /* fwpkm_profile_kernel kind: time every launch */
fwpkm_status fwpkm_profile_kernel(fwpkm_state* st, int kind);
fwpkm_status fwpkm_kernel_time(fwpkm_state* st, double* total_ms, int* launches);

/* The timed launches of the last call (in enqueue order, at most `max`): kind, start and
 * end in ms from the earliest start.  *n receives the number of timed launches.  Waits
 * for the events.  A diagnostic of the schedule (events themselves add some latency). */
fwpkm_status fwpkm_kernel_timeline(fwpkm_state* st, int max, int* kinds, float* start_ms, float* end_ms,
                                   int* n);

#ifdef __cplusplus
}
#endif
#endif /* FWPKM_H */
