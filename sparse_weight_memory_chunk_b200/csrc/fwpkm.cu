// fwpkm.cu -- the C ABI of libfwpkm.so: validation, workspace carve-up and the
// chunk-sequential schedule (Fast-weight Product Key Memory (paperlayer summary)
// §3.1: reads in a chunk use the fast weights left by earlier chunks; the write
// follows the chunk; App. B: forward, then memorization, then addressing).
//
// Scheduling observation used by fwpkm_run_sequence: the addressing (scores,
// top-k, Cartesian search, the pair sort) depends on q and the keys only, never on
// V.  With the key update off the keys are constant, so the addressing of every
// chunk and every pass is computed once, up front, in a few large launches, and only
// the value loop (gather, write) stays chunk-sequential.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "fwpkm_internal.cuh"

using namespace fwpkm;

static std::atomic<uint64_t> g_launches{0};

struct SeqKey {
  const void *q, *v, *g, *o;
  const void *hq, *hv, *hg, *ho;  // host buffers of fwpkm_run_sequence_host (else null)
  int T, n_iter, prof_kind;
  bool operator==(const SeqKey& x) const {
    return q == x.q && v == x.v && g == x.g && o == x.o && hq == x.hq && hv == x.hv && hg == x.hg && ho == x.ho &&
           T == x.T && n_iter == x.n_iter && prof_kind == x.prof_kind;
  }
};

// Host inputs and output of fwpkm_run_sequence_host: page-locked buffers laid out like the
// device ones, copied chunk by chunk beside the compute.
struct HostIO {
  const void* q;
  const void* v;
  const float* g;
  float* o;
};

struct fwpkm_state {
  fwpkm_config cfg;
  Dims dm;
  Work wk;
  float *K1, *K2, *V;
  // streaming (forward_chunk -> write_chunk)
  int pending;
  const void *q, *v;
  const float* g;
  int len;
  long long stride;
  // token-at-a-time inference: tokens of the pending chunk read so far (staged in the
  // workspace); its write waits for the next token (the lookahead) or a flush
  int spos;
  // per-kernel timing
  int prof_kind;  // kernel kind timed with events; FWPKM_PROFILE_ALL: every kind
  std::vector<int> ev_kind;  // kind of each timed launch (event pair)
  std::vector<cudaEvent_t> ev;
  int ev_used;
  int host_error;  // a launch could not be set up (e.g. tensor map encoding failed)
  // host copy of the device status word (pinned, mapped: kernels that latch an error
  // store it here too, so a later call sees it without waiting for the GPU)
  int* hstat;
  int* hstat_dev;
  // run_sequence schedule: internal streams, dependency events and the cached graph
  // Memories are split into `groups` contiguous groups; each group runs its own three
  // chains, so one group's latency-bound kernels overlap another's.
  static constexpr int MAX_GROUPS = 8;
  int groups;
  cudaStream_t sK[MAX_GROUPS], sS[MAX_GROUPS], sV[MAX_GROUPS], sCap;
  // host-buffer calls: input copies, the query preparation of each chunk, output copies
  cudaStream_t sH[MAX_GROUPS], sP[MAX_GROUPS], sD[MAX_GROUPS];
  // scheduling priorities of the kernels of the three chains (the addressing chain is the
  // critical path: highest); use_prio = 0 (FWPKM_PRIO=0) leaves them all at the default
  int use_prio, prio_K, prio_S, prio_V;
  std::vector<cudaEvent_t> sync_ev;
  size_t ev_next;
  int no_graph;
  int serial;  // diagnostics: all three chains on one stream (per-kernel timing without overlap)
  // two cached graphs (e.g. the plain step and the same step with timing events),
  // least recently used replaced
  static constexpr int NGRAPH = 2;
  cudaGraphExec_t graph_exec[NGRAPH];
  SeqKey graph_key[NGRAPH];
  uint64_t graph_kernels[NGRAPH];
  int graph_ev_used[NGRAPH];
  uint64_t graph_used[NGRAPH];
  uint64_t graph_clock;
};

namespace {

constexpr size_t ALIGN = 256;

size_t align_up(size_t x) { return (x + ALIGN - 1) & ~(ALIGN - 1); }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

fwpkm_status check_cfg(const fwpkm_config* c) {
  if (!c) return FWPKM_ERR_INVALID_ARG;
  if (c->n <= 0 || c->d <= 0 || c->d_v <= 0 || c->k <= 0 || c->chunk <= 0 || c->num_mem <= 0)
    return FWPKM_ERR_INVALID_ARG;
  if (c->qv_dtype != FWPKM_F32 && c->qv_dtype != FWPKM_BF16) return FWPKM_ERR_INVALID_ARG;
  if (!(c->eps_idw >= 0.f) || !(c->eps_norm >= 0.f)) return FWPKM_ERR_INVALID_ARG;
  if (c->d % 2 != 0 || c->d_v % 4 != 0) return FWPKM_ERR_INVALID_ARG;
  if (c->k > c->n) return FWPKM_ERR_INVALID_ARG;
  if (c->v_heads < 0) return FWPKM_ERR_INVALID_ARG;
  const int H = c->v_heads > 1 ? c->v_heads : 1;
  if (c->num_mem % H != 0) return FWPKM_ERR_INVALID_ARG;
  if (c->k > 32 || c->n > 4096 || c->d < 8 || c->d > 512 || c->d_v > 1024 || c->chunk > 1024 ||
      (long long)c->chunk * c->k * H > 16384 || c->k * H > 64)
    return FWPKM_ERR_UNSUPPORTED;
  return FWPKM_OK;
}

Dims make_dims(const fwpkm_config* c) {
  Dims d;
  d.n = c->n; d.h = c->d / 2; d.d = c->d; d.dv = c->d_v; d.k = c->k; d.C = c->chunk; d.M = c->num_mem;
  d.N = (long long)c->n * c->n;
  d.H = c->v_heads > 1 ? c->v_heads : 1;
  d.B = d.M / d.H;
  d.qv_bf16 = c->qv_dtype == FWPKM_BF16;
  d.eps_idw = c->eps_idw; d.eps_norm = c->eps_norm; d.lr_key = c->lr_key; d.flags = c->flags;
  return d;
}

size_t qv_size(const Dims& d) { return d.qv_bf16 ? 2 : 4; }

const void* offs(const void* p, long long elems, size_t esize) {
  return p ? (const void*)((const char*)p + elems * (long long)esize) : nullptr;
}

fwpkm_status last_cuda() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "fwpkm: CUDA error: %s\n", cudaGetErrorString(e));
    return FWPKM_ERR_CUDA;
  }
  return FWPKM_OK;
}

int stream_priority(const fwpkm_state* st, cudaStream_t s) {
  for (int gi = 0; gi < st->groups; ++gi) {
    if (s == st->sK[gi]) return st->prio_K;
    if (s == st->sS[gi]) return st->prio_S;
    if (s == st->sV[gi]) return st->prio_V;
  }
  return st->prio_V;
}

template <class F>
void run(fwpkm_state* st, int kind, cudaStream_t s, F&& f) {
  launch_priority_set = st->use_prio != 0 && !st->serial;
  launch_priority = launch_priority_set ? stream_priority(st, s) : 0;
  const bool prof = (st->prof_kind == kind || st->prof_kind == FWPKM_PROFILE_ALL) &&
                    st->ev_used + 2 <= (int)st->ev.size();
  // Under stream capture a plain record is only a dependency marker; timing events must
  // become event-record nodes of the graph.
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (prof) cudaStreamIsCapturing(s, &cs);
  const unsigned rec_flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (prof) cudaEventRecordWithFlags(st->ev[st->ev_used], s, rec_flags);
  int nl = f();
  launch_priority_set = false;
  if (prof) {
    cudaEventRecordWithFlags(st->ev[st->ev_used + 1], s, rec_flags);
    st->ev_kind[st->ev_used / 2] = kind;
    st->ev_used += 2;
  }
  if (nl < 0) st->host_error = 1;
  else g_launches += (uint64_t)nl;
}

cudaEvent_t next_event(fwpkm_state* st) {
  if (st->ev_next == st->sync_ev.size()) {
    cudaEvent_t e = nullptr;
    cudaEventCreateWithFlags(&e, cudaEventDisableTiming);
    st->sync_ev.push_back(e);
  }
  return st->sync_ev[st->ev_next++];
}

}  // namespace

namespace fwpkm {

void set_carveout(const void* kern) {
  static std::mutex mu;
  static std::vector<const void*> done;
  static const bool on = [] {
    const char* e = getenv("FWPKM_CARVEOUT");
    return e && e[0] == '1';
  }();
  if (!on) return;
  std::lock_guard<std::mutex> lock(mu);
  for (const void* k : done)
    if (k == kern) return;
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  done.push_back(kern);
}

bool raise_smem_limit(const void* kern, size_t bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, size_t>> lim;
  std::lock_guard<std::mutex> lock(mu);
  for (auto& e : lim)
    if (e.first == kern) {
      if (bytes <= e.second) return true;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
      e.second = bytes;
      return true;
    }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) return false;
  lim.emplace_back(kern, bytes);
  return true;
}

void count_launches(int n) { g_launches += (uint64_t)n; }

thread_local int launch_priority = 0;
thread_local bool launch_priority_set = false;

static std::atomic<int> g_test_stalls{0};

bool test_stalls_pending() { return g_test_stalls.load() > 0; }

int take_test_stall() {
  int n = g_test_stalls.load();
  while (n > 0)
    if (g_test_stalls.compare_exchange_weak(n, n - 1)) return 1;
  return 0;
}

int pbar_slices() {
  static const int v = [] {
    const char* e = getenv("FWPKM_PBAR_SLICES");
    return (e && atoi(e) == 16) ? 16 : 8;  // 8 measured faster (1.597 against 1.625 ms per step)
  }();
  return v;
}

thread_local bool pdl_scope = false;

bool pdl_enabled() {
  static const int env = [] {  // 1: on everywhere, 0: off everywhere, -1: by scope
    const char* e = getenv("FWPKM_PDL");
    return (e && e[0] == '1') ? 1 : (e && e[0] == '0') ? 0 : -1;
  }();
  return env < 0 ? pdl_scope : env == 1;
}

// The tensor-core path needs bf16 queries (exact tcgen05 operands) and half widths that
// are whole 64-element swizzle atoms no wider than one 128-column accumulator tile.
bool use_tensor_cores(const Dims& d) {
  return d.qv_bf16 && (d.h == 64 || d.h == 128) && d.n % 8 == 0 && d.n >= 64;
}

// Tokens addressed per batch when the keys are frozen: the distance rows of a batch are
// kept (up to ~64 MiB) so that the per-half top-k can read them back.
int addressing_window(const Dims& d, int max_T) {
  const size_t per_tok = (size_t)d.M * 2 * d.n * 4;
  size_t wtok = ((size_t)64 << 20) / per_tok / 128 * 128;
  if (wtok < 128) wtok = 128;
  const size_t need = ((size_t)max_T + 127) / 128 * 128;
  if (wtok > need) wtok = need;
  wtok = wtok / d.C * d.C;  // whole chunks, so a window's pairs can be sorted on their own
  if (wtok < (size_t)d.C) wtok = d.C;
  return (int)wtok;
}

size_t workspace_bytes(const Dims& d, int max_T, Work* w, char* base, bool stream_stage, bool allow_tc) {
  const size_t M = d.M, k = d.k, C = d.C, n = d.n, dv = d.dv;
  const size_t T = max_T;
  const size_t nch = (T + C - 1) / C;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  Work x;
  x.max_T = max_T;
  x.max_chunks = (int)nch;
  x.status = (int*)take(sizeof(int));
  x.hstat = nullptr;  // set by the handle that owns the carve
  x.A = (int32_t*)take(4 * M * 2 * T * k);
  x.Dsv = (float*)take(4 * M * 2 * T * k);
  x.idx = (int32_t*)take(4 * M * T * k);
  x.w = (float*)take(4 * M * T * k);
  x.sk = (unsigned long long*)take(8 * M * nch * C * k);
  x.npairs = (int32_t*)take(4 * M * nch);
  x.resid = (float*)take(4 * M * C * dv);
  const bool ku = (d.flags & FWPKM_KEY_UPDATE) != 0;
  x.tc = (allow_tc && use_tensor_cores(d)) ? 1 : 0;
  x.drows = ku ? (int)C : (x.tc ? addressing_window(d, max_T) : 0);
  // with the key step the tensor-core path keeps two chunks of distance rows in flight
  const size_t dbufs = (ku && x.tc) ? 2 : 1;
  x.Dfull = x.drows ? (float*)take(4 * dbufs * M * 2 * (size_t)x.drows * n) : nullptr;
  if (ku) {
    x.Z = (float*)take(4 * M * 2 * C);
    x.lp = (float*)take(4 * M * 2 * n);
    x.Lt = (float*)take(4 * M * 2 * C);
  } else {
    x.Z = nullptr; x.lp = nullptr; x.Lt = nullptr;
  }
  x.Kpc = nullptr; x.kn = nullptr; x.qn = nullptr; x.zpart = nullptr; x.ppart = nullptr;
  x.Wt = nullptr; x.Qt = nullptr; x.wsum_part = nullptr; x.pbar_cnt = nullptr; x.qt_T = 0;
  x.af_part = nullptr; x.af_cnt = nullptr;
  // frozen keys: the persistent value loop's counters (one pair per memory, so that each
  // group of memories has its own)
  x.vl_cnt = ku ? nullptr : (unsigned*)take(4 * M * 2);
  if (x.tc) {
    const size_t P = 2 * M, h = d.h, cpad = (C + 63) / 64 * 64, nt = (n + 127) / 128;
    x.Kpc = (__nv_bfloat16*)take(2 * 3 * P * n * h);
    x.kn = (float*)take(4 * P * n);
    x.qn = (float*)take(4 * P * T);
    if (ku) {
      x.zpart = (float*)take(4 * P * C * nt * 4);
      x.ppart = (float*)take(4 * P * PBAR_SLICES * n);
      x.Wt = (__nv_bfloat16*)take(2 * 2 * P * n * cpad);
      x.qt_T = (int)((T > C ? T : C) + 63) / 64 * 64;
      x.Qt = (__nv_bfloat16*)take(2 * P * h * (size_t)x.qt_T);
      x.wsum_part = (float*)take(4 * P * (cpad / 16) * n);
      x.pbar_cnt = (int*)take(4 * P * ((n + 255) / 256));
      if (n % 128 == 0) {
        x.af_part = (float*)take(4 * addr_fused_part_floats(d));
        x.af_cnt = (int*)take(4 * P * 2);
      }
    }
  }
  x.P_all = (int)(2 * M);
  x.dfull_buf = (long long)(M * 2 * (size_t)x.drows * n);
  x.stage_q = x.stage_v = nullptr;
  x.stage_g = nullptr;
  if (stream_stage) {
    const size_t es = d.qv_bf16 ? 2 : 4;
    x.stage_q = take(es * M * C * d.d);
    x.stage_v = take(es * M * (C + 1) * dv);
    x.stage_g = (float*)take(4 * M * (C + 1));
  }
  if (w) *w = x;
  return off;
}

Work group_work(const Dims& d, const Work& w, int m0) {
  Work x = w;
  const size_t M0 = m0, T = w.max_T, k = d.k, C = d.C, n = d.n, h = d.h, dv = d.dv, nch = w.max_chunks;
  const size_t cpad = (C + 63) / 64 * 64, nt = (n + 127) / 128;
  x.A += M0 * 2 * T * k;
  x.Dsv += M0 * 2 * T * k;
  x.idx += M0 * T * k;
  x.w += M0 * T * k;
  x.sk += M0 * nch * C * k;
  x.npairs += M0 * nch;
  x.resid += M0 * C * dv;
  if (x.Dfull) x.Dfull += M0 * 2 * (size_t)w.drows * n;
  if (x.Z) x.Z += M0 * 2 * C;
  if (x.lp) x.lp += M0 * 2 * n;
  if (x.Lt) x.Lt += M0 * 2 * C;
  if (x.Kpc) x.Kpc += M0 * 2 * n * h;
  if (x.kn) x.kn += M0 * 2 * n;
  if (x.qn) x.qn += M0 * 2 * T;
  if (x.zpart) x.zpart += M0 * 2 * C * nt * 4;
  if (x.ppart) x.ppart += M0 * 2 * PBAR_SLICES * n;
  if (x.Wt) x.Wt += M0 * 2 * n * cpad;
  if (x.Qt) x.Qt += M0 * 2 * h * (size_t)w.qt_T;
  if (x.wsum_part) x.wsum_part += M0 * 2 * (cpad / 16) * n;
  if (x.pbar_cnt) x.pbar_cnt += M0 * 2 * ((n + 255) / 256);
  if (x.af_part) x.af_part += M0 * 2 * (n / 128) * 2 * 256;
  if (x.af_cnt) x.af_cnt += M0 * 2 * 2;
  if (x.vl_cnt) x.vl_cnt += M0 * 2;
  return x;
}

}  // namespace fwpkm

extern "C" {

const char* fwpkm_status_string(fwpkm_status s) {
  switch (s) {
    case FWPKM_OK: return "ok";
    case FWPKM_ERR_INVALID_ARG: return "invalid argument";
    case FWPKM_ERR_UNSUPPORTED: return "unsupported shape";
    case FWPKM_ERR_WORKSPACE: return "workspace too small";
    case FWPKM_ERR_CUDA: return "CUDA error";
    case FWPKM_ERR_TIMEOUT: return "device wait timed out";
    case FWPKM_ERR_STATE: return "call out of order";
    case FWPKM_ERR_BAD_SLOT: return "slot index out of range in the write";
  }
  return "unknown status";
}

uint64_t fwpkm_launch_count(void) { return g_launches.load(); }

void fwpkm_test_stall_waits(int n_launches) { g_test_stalls.store(n_launches > 0 ? n_launches : 0); }

fwpkm_status fwpkm_workspace_size(const fwpkm_config* cfg, int max_T, size_t* bytes) {
  fwpkm_status s = check_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!bytes || max_T < 1) return FWPKM_ERR_INVALID_ARG;
  *bytes = workspace_bytes(make_dims(cfg), max_T, nullptr, nullptr);
  return FWPKM_OK;
}

fwpkm_status fwpkm_init_state(const fwpkm_config* cfg, float* K1, float* K2, float* V, int max_T,
                              void* workspace, size_t ws_bytes, fwpkm_state** out) {
  fwpkm_status s = check_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!out || !K1 || !K2 || !V || !workspace || max_T < 1) return FWPKM_ERR_INVALID_ARG;
  if (!aligned(K1, 16) || !aligned(K2, 16) || !aligned(V, 16) || !aligned(workspace, ALIGN))
    return FWPKM_ERR_INVALID_ARG;
  Dims dm = make_dims(cfg);
  if (ws_bytes < workspace_bytes(dm, max_T, nullptr, nullptr)) return FWPKM_ERR_WORKSPACE;
  fwpkm_state* st = new (std::nothrow) fwpkm_state();
  if (!st) return FWPKM_ERR_INVALID_ARG;
  st->cfg = *cfg;
  st->dm = dm;
  workspace_bytes(dm, max_T, &st->wk, (char*)workspace);
  st->K1 = K1; st->K2 = K2; st->V = V;
  st->pending = 0;
  st->spos = 0;
  st->prof_kind = 0;
  st->ev_used = 0;
  st->host_error = 0;
  st->ev_next = 0;
  st->hstat = nullptr;
  st->hstat_dev = nullptr;
  for (int i = 0; i < fwpkm_state::NGRAPH; ++i) {
    st->graph_exec[i] = nullptr;
    st->graph_kernels[i] = 0;
    st->graph_ev_used[i] = 0;
    st->graph_used[i] = 0;
  }
  st->graph_clock = 0;
  {
    const char* e = getenv("FWPKM_NO_GRAPH");
    st->no_graph = (e && e[0] == '1') ? 1 : 0;
    const char* sv = getenv("FWPKM_SERIAL");
    st->serial = (sv && sv[0] == '1') ? 1 : 0;
  }
  {
    // default one group: on the paper-scale workload more groups were slower (every
    // kernel keeps a fixed cost of several microseconds however little work it has,
    // and the chains of one group already overlap), so the split is opt-in
    int gr = 1;
    const char* e = getenv("FWPKM_GROUPS");
    if (e && atoi(e) > 0) gr = atoi(e);
    if (gr > dm.M) gr = dm.M;
    if (gr > fwpkm_state::MAX_GROUPS) gr = fwpkm_state::MAX_GROUPS;
    if (dm.H > 1) gr = 1;  // the memories of a sequence share V: keep them in one group
    st->groups = gr < 1 ? 1 : gr;
  }
  {
    const char* e = getenv("FWPKM_PRIO");
    st->use_prio = (e && e[0] == '0') ? 0 : 1;
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    st->prio_K = greatest;
    st->prio_S = (least + greatest) / 2;
    st->prio_V = least;
  }
  bool ok = cudaHostAlloc((void**)&st->hstat, sizeof(int), cudaHostAllocMapped) == cudaSuccess &&
            cudaHostGetDevicePointer((void**)&st->hstat_dev, st->hstat, 0) == cudaSuccess;
  if (ok) {
    *(volatile int*)st->hstat = DEV_OK;
    st->wk.hstat = st->hstat_dev;
  }
  st->sCap = nullptr;
  ok = ok && cudaStreamCreateWithFlags(&st->sCap, cudaStreamNonBlocking) == cudaSuccess;
  for (int gi = 0; gi < fwpkm_state::MAX_GROUPS; ++gi)
    st->sK[gi] = st->sS[gi] = st->sV[gi] = st->sH[gi] = st->sP[gi] = st->sD[gi] = nullptr;
  for (int gi = 0; gi < st->groups && ok; ++gi)
    ok = cudaStreamCreateWithFlags(&st->sK[gi], cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&st->sS[gi], cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&st->sV[gi], cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&st->sH[gi], cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&st->sP[gi], cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&st->sD[gi], cudaStreamNonBlocking) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    fwpkm_destroy_state(st);
    return FWPKM_ERR_CUDA;
  }
  if (cudaMemset(st->wk.status, 0, sizeof(int)) != cudaSuccess ||
      (st->wk.pbar_cnt &&
       cudaMemset(st->wk.pbar_cnt, 0, sizeof(int) * 2 * (size_t)dm.M * ((dm.n + 255) / 256)) != cudaSuccess) ||
      (st->wk.af_cnt && cudaMemset(st->wk.af_cnt, 0, sizeof(int) * 4 * (size_t)dm.M) != cudaSuccess) ||
      (st->wk.vl_cnt && cudaMemset(st->wk.vl_cnt, 0, sizeof(unsigned) * 2 * (size_t)dm.M) != cudaSuccess)) {
    cudaGetLastError();
    fwpkm_destroy_state(st);
    return FWPKM_ERR_CUDA;
  }
  *out = st;
  return FWPKM_OK;
}

void fwpkm_destroy_state(fwpkm_state* st) {
  if (!st) return;
  for (int i = 0; i < fwpkm_state::NGRAPH; ++i)
    if (st->graph_exec[i]) cudaGraphExecDestroy(st->graph_exec[i]);
  for (cudaEvent_t e : st->sync_ev) cudaEventDestroy(e);
  for (int gi = 0; gi < fwpkm_state::MAX_GROUPS; ++gi) {
    if (st->sK[gi]) cudaStreamDestroy(st->sK[gi]);
    if (st->sS[gi]) cudaStreamDestroy(st->sS[gi]);
    if (st->sV[gi]) cudaStreamDestroy(st->sV[gi]);
    if (st->sH[gi]) cudaStreamDestroy(st->sH[gi]);
    if (st->sP[gi]) cudaStreamDestroy(st->sP[gi]);
    if (st->sD[gi]) cudaStreamDestroy(st->sD[gi]);
  }
  if (st->sCap) cudaStreamDestroy(st->sCap);
  for (cudaEvent_t e : st->ev) cudaEventDestroy(e);
  if (st->hstat) cudaFreeHost(st->hstat);
  delete st;
}

// Before enqueueing anything: a device error that a kernel has already latched (its host
// copy, read without waiting) is returned until fwpkm_sync clears it; then any pending
// CUDA error of this thread.
static fwpkm_status peek_status(fwpkm_state* st) {
  const int h = st->hstat ? *(volatile int*)st->hstat : DEV_OK;
  if (h != DEV_OK) return status_of_device(h);
  return last_cuda();
}

fwpkm_status fwpkm_forward_chunk(fwpkm_state* st, const void* q, const void* v, const float* g, int c_len,
                                 int seq_stride, float* o, int32_t* idx_out, float* w_out, void* stream) {
  NvtxRange nvtx_range("fwpkm_forward_chunk");
  if (!st || !q || !v || !g || !o) return FWPKM_ERR_INVALID_ARG;
  const Dims& d = st->dm;
  if (c_len < 1 || c_len > d.C || c_len > st->wk.max_T || seq_stride < c_len) return FWPKM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(g, 4)) return FWPKM_ERR_INVALID_ARG;
  if (st->spos) return FWPKM_ERR_STATE;  // token-at-a-time chunk pending
  fwpkm_status ps = peek_status(st);
  if (ps != FWPKM_OK) return ps;
  cudaStream_t s = (cudaStream_t)stream;
  const bool ku = (d.flags & FWPKM_KEY_UPDATE) != 0;
  st->host_error = 0;
  if (st->wk.tc && ku && use_fused_addressing(d)) {
    // the chunk's whole addressing step in one launch: distances for the selection, then
    // the entropy step on K1, K2 (it needs only this chunk's queries and the keys they
    // were read with, so it is taken here; write_chunk then writes V)
    run(st, KK_PREP, s, [&] { return launch_qnorm(d, st->wk, q, seq_stride, 0, c_len, s); });
    run(st, KK_PREP, s, [&] { return launch_keyprep(d, st->wk, st->K1, st->K2, s); });
    run(st, KK_PREP, s, [&] { return launch_qtrans(d, st->wk, q, seq_stride, 0, c_len, s); });
    run(st, KK_FUSED, s, [&] {
      return launch_addr_fused(d, st->wk, st->K1, st->K2, q, seq_stride, c_len, 0, 0, c_len, 0, false, s);
    });
    run(st, KK_TOPK, s, [&] { return launch_select(d, st->wk, 0, c_len, idx_out, w_out, s); });
  } else if (st->wk.tc) {
    run(st, KK_PREP, s, [&] { return launch_qnorm(d, st->wk, q, seq_stride, 0, c_len, s); });
    run(st, KK_PREP, s, [&] { return launch_keyprep(d, st->wk, st->K1, st->K2, s); });
    run(st, KK_SCORE, s, [&] { return launch_tc_score(d, st->wk, q, seq_stride, c_len, 0, 0, c_len, ku, s); });
    run(st, KK_TOPK, s, [&] { return launch_select(d, st->wk, 0, c_len, idx_out, w_out, s); });
  } else {
    run(st, KK_SCORE, s, [&] { return launch_score_topk(d, st->wk, st->K1, st->K2, q, seq_stride, 0, c_len, ku, s); });
    run(st, KK_CART, s, [&] { return launch_cartesian(d, st->wk, 0, c_len, idx_out, w_out, s); });
  }
  run(st, KK_GATHER, s, [&] {
    return launch_gather(d, st->wk, st->V, v, g, seq_stride, 0, c_len, o, false, nullptr, s);
  });
  st->pending = 1;
  st->q = q; st->v = v; st->g = g; st->len = c_len; st->stride = seq_stride;
  if (st->host_error) return FWPKM_ERR_CUDA;
  return last_cuda();
}

fwpkm_status fwpkm_write_chunk(fwpkm_state* st, const void* v_next, void* stream) {
  NvtxRange nvtx_range("fwpkm_write_chunk");
  if (!st) return FWPKM_ERR_INVALID_ARG;
  if (!st->pending) return FWPKM_ERR_STATE;
  if (v_next && !aligned(v_next, 4)) return FWPKM_ERR_INVALID_ARG;
  {
    fwpkm_status ps = peek_status(st);
    if (ps != FWPKM_OK) return ps;
  }
  const Dims& d = st->dm;
  cudaStream_t s = (cudaStream_t)stream;
  const bool last_has_target = (v_next != nullptr) || !(d.flags & FWPKM_LOOKAHEAD);
  st->host_error = 0;
  run(st, KK_OTHER, s, [&] { return launch_resid(d, st->wk, st->v, st->g, st->stride, st->len, v_next, s); });
  run(st, KK_SORT, s, [&] { return launch_sort_pairs(d, st->wk, 0, st->len, last_has_target, s); });
  run(st, KK_WRITE, s, [&] { return launch_write(d, st->wk, st->V, 0, s); });
  if ((d.flags & FWPKM_KEY_UPDATE) && st->wk.tc && use_fused_addressing(d)) {
    // the key step was taken with the chunk's distances in fwpkm_forward_chunk
  } else if ((d.flags & FWPKM_KEY_UPDATE) && st->wk.tc) {
    run(st, KK_PBAR, s, [&] { return launch_tc_pbar(d, st->wk, st->len, s); });
    run(st, KK_WBUILD, s, [&] { return launch_tc_wbuild(d, st->wk, st->len, s); });
    run(st, KK_ADDR, s, [&] {
      return launch_tc_keystep(d, st->wk, st->K1, st->K2, st->q, st->stride, st->len, -1, s);
    });
  } else if (d.flags & FWPKM_KEY_UPDATE) {
    run(st, KK_ADDR, s, [&] { return launch_address(d, st->wk, st->K1, st->K2, st->q, st->stride, st->len, s); });
  }
  st->pending = 0;
  if (st->host_error) return FWPKM_ERR_CUDA;
  return last_cuda();
}

// ---- token-at-a-time inference ----
// The pending chunk's q, v, g are staged in the workspace as they arrive (chunk-local
// rows 0..spos-1), and each arriving group of tokens is read at once against the state
// left by the last write: the reads are per token, so reading a chunk in pieces gives
// the bits of reading it whole.  The chunk is written when the token after it arrives
// (its v is the lookahead target of the chunk's last token) or at a flush (no target).
// The key step needs every token's distance row, so the write recomputes the chunk's
// distances from the staged queries with the same kernel (the keys have not changed
// since the reads).

// Read tokens [spos, spos + len) of the pending chunk (already staged); v, g, o are the
// caller's rows of those tokens.
static void stream_read(fwpkm_state* st, const void* v, const float* g, long long stride, int len, float* o,
                        cudaStream_t s) {
  const Dims& d = st->dm;
  const Work& wk = st->wk;
  const size_t es = qv_size(d);
  const int p = st->spos;
  const void* qs = offs(wk.stage_q, (long long)p * d.d, es);
  if (wk.tc) {
    // with the fused key step the reads take their distances from the same kernel (scoring
    // only), so a token read here gets the bits it gets inside a whole chunk; the staging
    // launch has already written these tokens' query norms
    const bool fused = (d.flags & FWPKM_KEY_UPDATE) && use_fused_addressing(d);
    if (fused)
      run(st, KK_FUSED, s, [&] {
        return launch_addr_fused(d, wk, st->K1, st->K2, wk.stage_q, d.C, d.C, p, p, len, 0, true, s);
      });
    else
      run(st, KK_SCORE, s, [&] { return launch_tc_score(d, wk, wk.stage_q, d.C, d.C, p, p, len, false, s); });
    run(st, KK_TOPK, s, [&] { return launch_select(d, wk, p, len, nullptr, nullptr, s); });
  } else {
    run(st, KK_SCORE, s, [&] { return launch_score_topk(d, wk, st->K1, st->K2, qs, d.C, p, len, false, s); });
    run(st, KK_CART, s, [&] { return launch_cartesian(d, wk, p, len, nullptr, nullptr, s); });
  }
  run(st, KK_GATHER, s, [&] { return launch_gather(d, wk, st->V, v, g, stride, p, len, o, false, nullptr, s); });
}

// Write the pending chunk (spos tokens); has_next: staged row C holds the lookahead v.
static void stream_write(fwpkm_state* st, bool has_next, cudaStream_t s) {
  const Dims& d = st->dm;
  const Work& wk = st->wk;
  const size_t es = qv_size(d);
  const int len = st->spos;
  const void* vn = has_next ? offs(wk.stage_v, (long long)d.C * d.dv, es) : nullptr;
  const bool last_has_target = has_next || !(d.flags & FWPKM_LOOKAHEAD);
  run(st, KK_OTHER, s, [&] { return launch_resid(d, wk, wk.stage_v, wk.stage_g, d.C + 1, len, vn, s); });
  run(st, KK_SORT, s, [&] { return launch_sort_pairs(d, wk, 0, len, last_has_target, s); });
  run(st, KK_WRITE, s, [&] { return launch_write(d, wk, st->V, 0, s); });
  if (d.flags & FWPKM_KEY_UPDATE) {
    if (wk.tc && use_fused_addressing(d)) {
      // distances recomputed from the staged queries and the key step, in one launch (it
      // also leaves the new keys' bf16 pieces for the next chunk's reads)
      run(st, KK_PREP, s, [&] { return launch_qtrans(d, wk, wk.stage_q, d.C, 0, len, s); });
      run(st, KK_FUSED, s, [&] {
        return launch_addr_fused(d, wk, st->K1, st->K2, wk.stage_q, d.C, d.C, 0, 0, len, 0, false, s);
      });
    } else if (wk.tc) {
      run(st, KK_SCORE, s, [&] { return launch_tc_score(d, wk, wk.stage_q, d.C, d.C, 0, 0, len, true, s); });
      run(st, KK_PBAR, s, [&] { return launch_tc_pbar(d, wk, len, s); });
      run(st, KK_WBUILD, s, [&] { return launch_tc_wbuild(d, wk, len, s); });
      run(st, KK_ADDR, s, [&] { return launch_tc_keystep(d, wk, st->K1, st->K2, wk.stage_q, d.C, len, -1, s); });
      run(st, KK_PREP, s, [&] { return launch_keyprep(d, wk, st->K1, st->K2, s); });
    } else {
      run(st, KK_SCORE, s, [&] {
        return launch_score_topk(d, wk, st->K1, st->K2, wk.stage_q, d.C, 0, len, true, s);
      });
      run(st, KK_ADDR, s, [&] { return launch_address(d, wk, st->K1, st->K2, wk.stage_q, d.C, len, s); });
    }
  }
  st->spos = 0;
}

fwpkm_status fwpkm_stream_tokens(fwpkm_state* st, const void* q, const void* v, const float* g, int n_tok,
                                 int seq_stride, float* o, void* stream) {
  NvtxRange nvtx_range("fwpkm_stream_tokens");
  if (!st || !q || !v || !g || !o) return FWPKM_ERR_INVALID_ARG;
  const Dims& d = st->dm;
  if (n_tok < 1 || seq_stride < n_tok) return FWPKM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(g, 4)) return FWPKM_ERR_INVALID_ARG;
  if (st->pending) return FWPKM_ERR_STATE;
  if (st->wk.max_T < d.C || !st->wk.stage_q || d.H > 1) return FWPKM_ERR_UNSUPPORTED;
  fwpkm_status ps = peek_status(st);
  if (ps != FWPKM_OK) return ps;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t es = qv_size(d);
  const Work& wk = st->wk;
  st->host_error = 0;
  // every kernel of the tensor-core path's reads and writes waits for its predecessor's
  // results (griddepcontrol.wait) before it touches memory, so its launch may overlap
  // the predecessor's tail
  const PdlScope pdl(wk.tc);
  // bf16 pieces of the keys for the scoring GEMM: made at the start of every chunk (the
  // caller may change the keys between chunks, never inside one) and after a key step
  if (wk.tc && st->spos == 0) run(st, KK_PREP, s, [&] { return launch_keyprep(d, wk, st->K1, st->K2, s); });
  int j = 0;
  while (j < n_tok) {
    if (st->spos == d.C) {
      // token j completes the pending chunk's last pair: stage its v as the lookahead, write
      const StageJob la[3] = {{nullptr, nullptr, 0, 0, 0},
                              {offs(v, (long long)j * d.dv, es), wk.stage_v, seq_stride, d.C + 1,
                               (int)(d.dv * es / 4)},
                              {nullptr, nullptr, 0, 0, 0}};
      run(st, KK_PREP, s, [&] { return launch_stage(d, la, d.C, 1, s); });
      stream_write(st, true, s);
    }
    const int len = std::min(d.C - st->spos, n_tok - j);
    const StageJob in[3] = {
        {offs(q, (long long)j * d.d, es), wk.stage_q, seq_stride, d.C, (int)(d.d * es / 4)},
        {offs(v, (long long)j * d.dv, es), wk.stage_v, seq_stride, d.C + 1, (int)(d.dv * es / 4)},
        {g + j, wk.stage_g, seq_stride, d.C + 1, 1}};
    // on the tensor-core path the same launch writes the tokens' query norms
    run(st, KK_PREP, s, [&] {
      return wk.tc ? launch_stage(d, in, st->spos, len, s, &wk, offs(q, (long long)j * d.d, es), seq_stride)
                   : launch_stage(d, in, st->spos, len, s);
    });
    stream_read(st, offs(v, (long long)j * d.dv, es), g + j, seq_stride, len, o + (long long)j * d.dv, s);
    st->spos += len;
    j += len;
  }
  if (st->host_error) return FWPKM_ERR_CUDA;
  return last_cuda();
}

fwpkm_status fwpkm_stream_pending(const fwpkm_state* st, int* n_pending) {
  if (!st || !n_pending) return FWPKM_ERR_INVALID_ARG;
  *n_pending = st->spos;
  return FWPKM_OK;
}

fwpkm_status fwpkm_stream_flush(fwpkm_state* st, void* stream) {
  NvtxRange nvtx_range("fwpkm_stream_flush");
  if (!st) return FWPKM_ERR_INVALID_ARG;
  if (st->pending) return FWPKM_ERR_STATE;
  fwpkm_status ps = peek_status(st);
  if (ps != FWPKM_OK) return ps;
  if (st->spos == 0) return FWPKM_OK;
  st->host_error = 0;
  const PdlScope pdl(st->wk.tc);
  stream_write(st, false, (cudaStream_t)stream);
  if (st->host_error) return FWPKM_ERR_CUDA;
  return last_cuda();
}

// Enqueue a whole sequence as three stream-ordered chains that fork from and join back
// to `origin`:
//   sK  addressing: q norms, key pieces, scoring GEMM, entropy key step (K-chain)
//   sS  selection: per-half top-k, Cartesian search, pair sort
//   sV  values: gather + gated output, sorted write
// Addressing never reads V, so sK/sS run ahead of sV; sV only waits for the selection
// of the chunk it is about to read.  The scoring GEMM writes its distance rows into one
// of two buffers, so sK may start chunk c+1 while sS still reads chunk c's rows.  Across
// passes, chunk c's selection waits for the previous pass's write of chunk c (its slot
// lists and weights are overwritten).
static void enqueue_group(fwpkm_state* st, int gi, const Dims& d, const Work& wk, float* K1, float* K2, float* V,
                          const void* q, const void* v, const float* g, int T, int n_iter, float* o,
                          const HostIO* hio, cudaStream_t origin) {
  const size_t es = qv_size(d);
  const int C = d.C;
  const bool ku = (d.flags & FWPKM_KEY_UPDATE) != 0;
  const bool la = (d.flags & FWPKM_LOOKAHEAD) != 0;
  const bool tc = wk.tc != 0;
  const int nch = (T + C - 1) / C;
  // the key step reads every chunk's half-queries from one feature-major copy made up front
  // (its TMA x offset, the chunk start, must be a multiple of 8 tokens)
  const bool qt_whole = tc && ku && C % 8 == 0;
  // one launch per chunk for the whole addressing step (its half-queries need the
  // feature-major copy: C % 16 == 0 keeps qt_whole)
  const bool fused = tc && ku && use_fused_addressing(d);
  cudaStream_t sK = st->serial ? st->sK[0] : st->sK[gi];
  cudaStream_t sS = st->serial ? sK : st->sS[gi], sV = st->serial ? sK : st->sV[gi];
  auto dep = [&](cudaStream_t from, cudaStream_t to) {
    cudaEvent_t e = next_event(st);
    cudaEventRecord(e, from);
    cudaStreamWaitEvent(to, e, 0);
  };
  auto mark = [&](cudaStream_t s) {
    cudaEvent_t e = next_event(st);
    cudaEventRecord(e, s);
    return e;
  };
  dep(origin, sK);
  dep(origin, sS);
  dep(origin, sV);

  // Host buffers: chunk c's inputs are copied to the device on sH, in chunk order (copies
  // only, so they run ahead of the compute), and in_ready[c] marks them; each consumer
  // waits only for the chunks it reads.  On the tensor-core path the chunk's query norms and
  // feature-major half-queries are made from the copy (see host_prep).  o goes back on sD
  // as soon as the last pass's value work of a chunk (or window) has ended.
  std::vector<cudaEvent_t> in_ready;
  cudaStream_t sH = nullptr, sP = nullptr, sD = nullptr;
  // where the query preparation of host-buffer calls runs (FWPKM_HOST_PREP): 'a' (default)
  // with the one-launch addressing step: chunk c+1's on its own stream once chunk c's
  // addressing kernel has finished, so it runs beside chunk c's selection (else as 'k');
  // 'k' per chunk on the addressing stream just before the chunk's addressing (on the
  // critical chain: 1.58 ms per paper-scale call); 'p' per chunk on its own stream as soon as
  // the chunk's copies land (its small kernels then take SMs the addressing kernel waits
  // for: 1.93 ms); 'w' once for the whole call after the last copy (2.25 ms)
  static const char host_prep = [] {
    const char* e = getenv("FWPKM_HOST_PREP");
    return (e && (e[0] == 'p' || e[0] == 'w' || e[0] == 'k')) ? e[0] : 'a';
  }();
  const bool prep_after = hio && tc && host_prep == 'a' && fused;
  if (hio) {
    sH = st->serial ? sK : st->sH[gi];
    sP = st->serial ? sK : st->sP[gi];
    sD = st->serial ? sK : st->sD[gi];
    dep(origin, sH);
    dep(origin, sP);
    dep(origin, sD);
    in_ready.resize(nch);
    auto h2d = [&](const void* dst, const void* src, size_t row_bytes, size_t width, int rows) {
      if (cudaMemcpy2DAsync(const_cast<void*>(dst), row_bytes, src, row_bytes, width, rows, cudaMemcpyHostToDevice,
                            sH) != cudaSuccess)
        st->host_error = 1;
    };
    for (int c = 0; c < nch; ++c) {
      const int t0 = c * C, len = T - t0 < C ? T - t0 : C;
      h2d(offs(q, (long long)t0 * d.d, es), offs(hio->q, (long long)t0 * d.d, es), (size_t)T * d.d * es,
          (size_t)len * d.d * es, d.M);
      h2d(offs(v, (long long)t0 * d.dv, es), offs(hio->v, (long long)t0 * d.dv, es), (size_t)T * d.dv * es,
          (size_t)len * d.dv * es, d.B);
      h2d(g + t0, hio->g + t0, (size_t)T * 4, (size_t)len * 4, d.B);
      in_ready[c] = mark(sH);
      if (prep_after && c == 0) {  // the first chunk's preparation follows its copies
        cudaStreamWaitEvent(sP, in_ready[0], 0);
        const void* qc = offs(q, 0, es);
        run(st, KK_PREP, sP, [&] { return launch_qnorm(d, wk, qc, T, 0, len, sP); });
        if (qt_whole) run(st, KK_PREP, sP, [&] { return launch_qtrans(d, wk, qc, T, 0, len, sP); });
        in_ready[0] = mark(sP);
      }
      if (tc && host_prep == 'p') {
        cudaStreamWaitEvent(sP, in_ready[c], 0);
        const void* qc = offs(q, (long long)t0 * d.d, es);
        run(st, KK_PREP, sP, [&] { return launch_qnorm(d, wk, qc, T, t0, len, sP); });
        if (qt_whole) run(st, KK_PREP, sP, [&] { return launch_qtrans(d, wk, qc, T, t0, len, sP); });
        in_ready[c] = mark(sP);
      }
    }
    if (tc && host_prep == 'w') {  // one preparation over the whole call once every copy has landed
      cudaStreamWaitEvent(sP, in_ready[nch - 1], 0);
      run(st, KK_PREP, sP, [&] { return launch_qnorm(d, wk, q, T, 0, T, sP); });
      if (qt_whole) run(st, KK_PREP, sP, [&] { return launch_qtrans(d, wk, q, T, 0, T, sP); });
      const cudaEvent_t e = mark(sP);
      for (int c = 0; c < nch; ++c) in_ready[c] = e;
    }
  }
  // the query preparation of tokens [t0, t0 + len) on stream s (host buffers, 'k' mode)
  auto prep_on = [&](cudaStream_t s, int t0, int len) {
    if (!(hio && tc && (host_prep == 'k' || (host_prep == 'a' && !prep_after)))) return;
    const void* qc = offs(q, (long long)t0 * d.d, es);
    run(st, KK_PREP, s, [&] { return launch_qnorm(d, wk, qc, T, t0, len, s); });
    if (qt_whole) run(st, KK_PREP, s, [&] { return launch_qtrans(d, wk, qc, T, t0, len, s); });
  };
  auto wait_in = [&](cudaStream_t s, int c) {  // inputs of chunks <= c are on the device
    if (hio) cudaStreamWaitEvent(s, in_ready[c < nch ? c : nch - 1], 0);
  };
  auto copy_out = [&](cudaStream_t from, int c0, int c1) {  // o of chunks [c0, c1) to the host
    if (!hio) return;
    cudaStreamWaitEvent(sD, mark(from), 0);
    const long long t0 = (long long)c0 * C, t1 = (long long)c1 * C < T ? (long long)c1 * C : T;
    const size_t pitch = (size_t)T * d.dv * 4;
    if (cudaMemcpy2DAsync(hio->o + t0 * d.dv, pitch, o + t0 * d.dv, pitch, (size_t)(t1 - t0) * d.dv * 4, d.B,
                          cudaMemcpyDeviceToHost, sD) != cudaSuccess)
      st->host_error = 1;
  };

  // before_write: an event the write (not the gather) waits for (the pair sort), or null
  auto value_chunk = [&](int c, cudaEvent_t before_write = nullptr) {
    const int t0 = c * C, len = T - t0 < C ? T - t0 : C;
    const void* vc = offs(v, (long long)t0 * d.dv, es);
    const void* vn = (t0 + len < T) ? offs(v, (long long)(t0 + len) * d.dv, es) : nullptr;
    run(st, KK_GATHER, sV, [&] {
      return launch_gather(d, wk, V, vc, g + t0, T, t0, len, o + (long long)t0 * d.dv, true, vn, sV);
    });
    if (before_write) cudaStreamWaitEvent(sV, before_write, 0);
    run(st, KK_WRITE, sV, [&] { return launch_write(d, wk, V, t0, sV); });
  };

  if (tc && !hio) {
    // the three per-call preparations are independent: query norms (selection stream),
    // query transpose (values stream) and key pieces (addressing stream) run side by side
    run(st, KK_PREP, sS, [&] { return launch_qnorm(d, wk, q, T, 0, T, sS); });
    const cudaEvent_t qn_done = mark(sS);
    if (qt_whole) run(st, KK_PREP, sV, [&] { return launch_qtrans(d, wk, q, T, 0, T, sV); });
    const cudaEvent_t qt_done = mark(sV);
    run(st, KK_PREP, sK, [&] { return launch_keyprep(d, wk, K1, K2, sK); });
    cudaStreamWaitEvent(sK, qn_done, 0);
    cudaStreamWaitEvent(sK, qt_done, 0);
  } else if (tc) {
    run(st, KK_PREP, sK, [&] { return launch_keyprep(d, wk, K1, K2, sK); });
  }
  if (!ku) {
    // frozen keys: address window by window on sK; the value loop of a window starts as
    // soon as its chunks are sorted.  The addressing serves every pass.
    const int wtok = tc ? wk.drows : T;
    std::vector<cudaEvent_t> ready;
    for (int w0 = 0; w0 < T; w0 += wtok) {
      const int wl = T - w0 < wtok ? T - w0 : wtok;
      wait_in(sK, (w0 + wl - 1) / C);
      prep_on(sK, w0, wl);
      if (tc) {
        run(st, KK_SCORE, sK, [&] { return launch_tc_score(d, wk, q, T, T, w0, w0, wl, false, sK); });
        run(st, KK_TOPK, sK, [&] { return launch_select(d, wk, w0, wl, nullptr, nullptr, sK); });
      } else {
        run(st, KK_SCORE, sK, [&] {
          return launch_score_topk(d, wk, K1, K2, offs(q, (long long)w0 * d.d, es), T, w0, wl, false, sK);
        });
        run(st, KK_CART, sK, [&] { return launch_cartesian(d, wk, w0, wl, nullptr, nullptr, sK); });
      }
      run(st, KK_SORT, sK, [&] { return launch_sort_pairs(d, wk, w0, wl, !la || (w0 + wl < T), sK); });
      ready.push_back(mark(sK));
    }
    // the value loop: one persistent launch per addressing window in the first pass and
    // one for all chunks in each later pass, else the chunks one by one
    const bool vloop = value_loop_enabled() && wk.vl_cnt != nullptr;
    const int wch = wtok >= T ? nch : wtok / C;  // chunks per window (wtok < T is whole chunks)
    for (int pass = 0; pass < n_iter; ++pass)
      for (int c = 0; c < nch; c += (pass == 0 ? wch : nch)) {
        if (pass == 0) cudaStreamWaitEvent(sV, ready[c / wch], 0);
        const int c1 = pass > 0 ? nch : (c + wch < nch ? c + wch : nch);
        if (pass == 0) wait_in(sV, c1);  // the window's v, g and the lookahead row after it
        if (vloop) {
          run(st, KK_VLOOP, sV, [&] { return launch_value_loop(d, wk, V, v, g, T, c, c1, o, sV); });
        } else {
          for (int cc = c; cc < c1; ++cc) value_chunk(cc);
        }
        if (pass == n_iter - 1) copy_out(sV, c, c1);
      }
  } else {
    const size_t dbuf = (size_t)wk.dfull_buf;
    std::vector<cudaEvent_t> topk_done(2, nullptr), sel_done(nch, nullptr), val_done(nch, nullptr);
    // The addressing of chunk c+1 also waits for the selection of chunk c, so the selection
    // runs beside the value kernels rather than beside the addressing, which occupies most
    // SMs (paper-scale step 1.453 against 1.555 ms); FWPKM_SEL_FIRST=0 lets them overlap.
    static const bool sel_first = [] {
      const char* e = getenv("FWPKM_SEL_FIRST");
      return !(e && e[0] == '0');
    }();
    // FWPKM_SEL_ON_SK=1 (with selection first and the one-launch addressing step) runs the
    // selection on the addressing stream itself, so that addressing(c) -> selection(c) ->
    // addressing(c+1) is stream order.  Measured slower (1.486 against 1.44 ms per step at
    // the paper scale: the selection then meets the next chunk's gather), so off.
    static const bool sel_on_k = [] {
      const char* e = getenv("FWPKM_SEL_ON_SK");
      return e && e[0] == '1';
    }();
    const bool selk = sel_first && sel_on_k && fused;
    cudaStream_t sSel = selk ? sK : sS;
    cudaEvent_t last_topk = nullptr;
    int cnt = 0;
    for (int pass = 0; pass < n_iter; ++pass) {
      for (int c = 0; c < nch; ++c, ++cnt) {
        const int t0 = c * C, len = T - t0 < C ? T - t0 : C;
        const void* qc = offs(q, (long long)t0 * d.d, es);
        Work wb = wk;
        if (tc) wb.Dfull = wk.Dfull + (size_t)(cnt & 1) * dbuf;
        if (sel_done[c]) cudaStreamWaitEvent(sK, sel_done[c], 0);    // previous pass read A/Dsv
        if (topk_done[cnt & 1]) cudaStreamWaitEvent(sK, topk_done[cnt & 1], 0);  // buffer reuse
        if (sel_first && last_topk) cudaStreamWaitEvent(sK, last_topk, 0);
        if (pass == 0) {
          wait_in(sK, c);
          prep_on(sK, t0, len);
        }
        if (fused) {
          // the chunk's whole addressing step in one launch; the selection needs its rows
          run(st, KK_FUSED, sK, [&] {
            return launch_addr_fused(d, wb, K1, K2, q, T, T, t0, t0, len, t0, false, sK);
          });
          const cudaEvent_t addr_done = mark(sK);
          cudaStreamWaitEvent(sS, addr_done, 0);
          if (prep_after && pass == 0 && c + 1 < nch) {
            // the next chunk's query preparation beside this chunk's selection
            const int tn = t0 + C, ln = T - tn < C ? T - tn : C;
            const void* qn = offs(q, (long long)tn * d.d, es);
            cudaStreamWaitEvent(sP, in_ready[c + 1], 0);
            cudaStreamWaitEvent(sP, addr_done, 0);
            run(st, KK_PREP, sP, [&] { return launch_qnorm(d, wk, qn, T, tn, ln, sP); });
            if (qt_whole) run(st, KK_PREP, sP, [&] { return launch_qtrans(d, wk, qn, T, tn, ln, sP); });
            in_ready[c + 1] = mark(sP);
          }
        } else if (tc) {
          run(st, KK_SCORE, sK, [&] { return launch_tc_score(d, wb, q, T, T, t0, t0, len, true, sK); });
          // the selection needs the distance rows; it also waits for the usage marginals, so
          // that pbar (on the critical addressing chain) does not share the GPU with it
          // (1.606 against 1.628 ms per step)
          run(st, KK_PBAR, sK, [&] { return launch_tc_pbar(d, wb, len, sK); });
          cudaStreamWaitEvent(sS, mark(sK), 0);
          run(st, KK_WBUILD, sK, [&] { return launch_tc_wbuild(d, wb, len, sK); });
          run(st, KK_ADDR, sK, [&] { return launch_tc_keystep(d, wb, K1, K2, qc, T, len, qt_whole ? t0 : -1, sK); });
        } else {
          run(st, KK_SCORE, sK, [&] { return launch_score_topk(d, wb, K1, K2, qc, T, t0, len, true, sK); });
          cudaStreamWaitEvent(sS, mark(sK), 0);
          run(st, KK_ADDR, sK, [&] { return launch_address(d, wb, K1, K2, qc, T, len, sK); });
        }
        if (val_done[c]) cudaStreamWaitEvent(sSel, val_done[c], 0);   // previous pass wrote chunk c
        if (tc) {
          run(st, KK_TOPK, sSel, [&] { return launch_select(d, wb, t0, len, nullptr, nullptr, sSel); });
          topk_done[cnt & 1] = mark(sSel);
          last_topk = selk ? nullptr : topk_done[cnt & 1];  // on sK the order is the stream's
          if (selk) cudaStreamWaitEvent(sS, topk_done[cnt & 1], 0);
        } else {
          run(st, KK_CART, sS, [&] { return launch_cartesian(d, wb, t0, len, nullptr, nullptr, sS); });
        }
        run(st, KK_SORT, sS, [&] { return launch_sort_pairs(d, wb, t0, len, !la || (t0 + len < T), sS); });
        sel_done[c] = mark(sS);
        // The gather of a chunk needs its slots and weights (the selection); only its write
        // needs the pair sort, which then runs beside the gather (paper scale: 1.45 against
        // 1.48 ms per step; FWPKM_GATHER_EARLY=0 waits for the sort, which with the
        // four-kernel addressing chain had been the faster order, 1.62 against 1.82 ms).
        static const bool gather_early = [] {
          const char* e = getenv("FWPKM_GATHER_EARLY");
          return !(e && e[0] == '0');
        }();
        const bool early = gather_early && tc && topk_done[cnt & 1];
        cudaStreamWaitEvent(sV, early ? topk_done[cnt & 1] : sel_done[c], 0);
        if (pass == 0) wait_in(sV, c + 1);  // v, g of the chunk and its lookahead row
        value_chunk(c, early ? sel_done[c] : nullptr);
        val_done[c] = mark(sV);
        if (pass == n_iter - 1) copy_out(sV, c, c + 1);
      }
    }
  }
  dep(sK, origin);
  dep(sS, origin);
  dep(sV, origin);
  if (hio) {
    dep(sH, origin);
    dep(sP, origin);
    dep(sD, origin);
  }
}

// Split the memories into st->groups contiguous groups and enqueue each as its own set of
// chains (all of them fork from and join back to `origin`).
static void enqueue_sequence(fwpkm_state* st, const void* q, const void* v, const float* g, int T, int n_iter,
                             float* o, const HostIO* hio, cudaStream_t origin) {
  const Dims& d = st->dm;
  const size_t es = qv_size(d);
  st->ev_next = 0;
  const int G = st->groups;
  for (int gi = 0; gi < G; ++gi) {
    const int m0 = (int)((long long)gi * d.M / G), m1 = (int)((long long)(gi + 1) * d.M / G);
    Dims dg = d;
    dg.M = m1 - m0;
    dg.B = dg.M / dg.H;  // one group when heads share V (dg.M = d.M)
    const Work wg = G == 1 ? st->wk : group_work(d, st->wk, m0);
    const size_t kh = (size_t)m0 * d.n * d.h;
    HostIO hg;
    if (hio) {
      hg.q = offs(hio->q, (long long)m0 * T * d.d, es);
      hg.v = offs(hio->v, (long long)m0 * T * d.dv, es);
      hg.g = hio->g + (size_t)m0 * T;
      hg.o = hio->o + (size_t)m0 * T * d.dv;
    }
    enqueue_group(st, gi, dg, wg, st->K1 + kh, st->K2 + kh, st->V + (size_t)m0 * d.N * d.dv,
                  offs(q, (long long)m0 * T * d.d, es), offs(v, (long long)m0 * T * d.dv, es), g + (size_t)m0 * T,
                  T, n_iter, o + (size_t)m0 * T * d.dv, hio ? &hg : nullptr, origin);
  }
}

// The schedule of fwpkm_run_sequence (hio = nullptr) and fwpkm_run_sequence_host, captured
// into a cached graph.  Arguments are checked by the callers.
static fwpkm_status run_sequence_impl(fwpkm_state* st, const void* q, const void* v, const float* g, int T,
                                      int n_iter, float* o, const HostIO* hio, void* stream) {
  if (st->spos) return FWPKM_ERR_STATE;  // token-at-a-time chunk pending
  fwpkm_status ps = peek_status(st);
  if (ps != FWPKM_OK) return ps;
  st->pending = 0;
  st->host_error = 0;
  cudaStream_t user = (cudaStream_t)stream;
  // a pending test stall is taken at launch time, so such a call is not captured (the
  // stall would stay in a cached graph)
  if (st->no_graph || test_stalls_pending()) {
    enqueue_sequence(st, q, v, g, T, n_iter, o, hio, user);
    if (st->host_error) return FWPKM_ERR_CUDA;
    return last_cuda();
  }
  // One CUDA graph per distinct call (arguments and timing kind), replayed while they stay
  // the same; the last two are kept.
  const SeqKey key = {q, v, g, o, hio ? hio->q : nullptr, hio ? hio->v : nullptr, hio ? (const void*)hio->g : nullptr,
                      hio ? (const void*)hio->o : nullptr, T, n_iter, st->prof_kind};
  int slot = -1;
  for (int i = 0; i < fwpkm_state::NGRAPH; ++i)
    if (st->graph_exec[i] && st->graph_key[i] == key) slot = i;
  if (slot < 0) {
    slot = 0;
    for (int i = 1; i < fwpkm_state::NGRAPH; ++i)
      if (st->graph_used[i] < st->graph_used[slot]) slot = i;
    if (st->graph_exec[slot]) {
      cudaGraphExecDestroy(st->graph_exec[slot]);
      st->graph_exec[slot] = nullptr;
    }
    const uint64_t before = g_launches.load();
    if (cudaStreamBeginCapture(st->sCap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) return last_cuda();
    enqueue_sequence(st, q, v, g, T, n_iter, o, hio, st->sCap);
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamEndCapture(st->sCap, &graph);
    st->graph_kernels[slot] = g_launches.load() - before;
    g_launches -= st->graph_kernels[slot];  // counted per replay below
    if (e != cudaSuccess || st->host_error) {
      if (graph) cudaGraphDestroy(graph);
      last_cuda();
      return FWPKM_ERR_CUDA;
    }
    e = cudaGraphInstantiate(&st->graph_exec[slot], graph, 0);
    cudaGraphDestroy(graph);
    if (e != cudaSuccess) {
      st->graph_exec[slot] = nullptr;
      last_cuda();
      return FWPKM_ERR_CUDA;
    }
    st->graph_key[slot] = key;
    st->graph_ev_used[slot] = st->ev_used;
  }
  st->graph_used[slot] = ++st->graph_clock;
  if (cudaGraphLaunch(st->graph_exec[slot], user) != cudaSuccess) return last_cuda();
  g_launches += st->graph_kernels[slot];
  st->ev_used = st->graph_ev_used[slot];
  return last_cuda();
}

fwpkm_status fwpkm_run_sequence(fwpkm_state* st, const void* q, const void* v, const float* g, int T,
                                int n_iter, float* o, void* stream) {
  NvtxRange nvtx_range("fwpkm_run_sequence");
  if (!st) return FWPKM_ERR_INVALID_ARG;
  if (T == 0) return FWPKM_OK;
  if (!q || !v || !g || !o || T < 0 || T > st->wk.max_T || n_iter < 1) return FWPKM_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(g, 4)) return FWPKM_ERR_INVALID_ARG;
  return run_sequence_impl(st, q, v, g, T, n_iter, o, nullptr, stream);
}

// ---- the read path's backward ----
fwpkm_status fwpkm_read_backward(const fwpkm_config* cfg, const float* K1, const float* K2, const float* V,
                                 const void* q, const void* v, const float* g, const int32_t* idx,
                                 const float* d_o, int len, int seq_stride, float* dq, float* dv, float* dg,
                                 void* stream) {
  NvtxRange nvtx_range("fwpkm_read_backward");
  fwpkm_status cs = check_cfg(cfg);
  if (cs != FWPKM_OK) return cs;
  if (cfg->v_heads > 1) return FWPKM_ERR_UNSUPPORTED;
  if (len == 0) return FWPKM_OK;
  if (len < 0 || seq_stride < len || !K1 || !K2 || !V || !q || !v || !g || !idx || !d_o || !dq || !dv || !dg)
    return FWPKM_ERR_INVALID_ARG;
  if (!aligned(V, 16) || !aligned(d_o, 16) || !aligned(dv, 16)) return FWPKM_ERR_INVALID_ARG;
  const Dims d = make_dims(cfg);
  cudaGetLastError();
  const int nl = launch_read_backward(d, K1, K2, V, q, v, g, idx, d_o, len, seq_stride, dq, dv, dg,
                                      (cudaStream_t)stream);
  count_launches(nl);
  return last_cuda();
}

// ---- host buffers: device copies of q, v, g, o in caller scratch ----
static size_t host_io_carve(const Dims& d, int T, char* base, void** q, void** v, float** g, float** o) {
  const size_t es = qv_size(d);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  void* pq = take(es * (size_t)d.M * T * d.d);
  void* pv = take(es * (size_t)d.B * T * d.dv);
  float* pg = (float*)take(4 * (size_t)d.B * T);
  float* po = (float*)take(4 * (size_t)d.B * T * d.dv);
  if (q) { *q = pq; *v = pv; *g = pg; *o = po; }
  return off;
}

static bool host_pinned(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

fwpkm_status fwpkm_run_sequence_host_scratch_size(const fwpkm_config* cfg, int T, size_t* bytes) {
  fwpkm_status s = check_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!bytes || T < 0) return FWPKM_ERR_INVALID_ARG;
  *bytes = host_io_carve(make_dims(cfg), T, nullptr, nullptr, nullptr, nullptr, nullptr);
  return FWPKM_OK;
}

fwpkm_status fwpkm_run_sequence_host(fwpkm_state* st, const void* q, const void* v, const float* g, int T,
                                     int n_iter, float* o, void* scratch, size_t scratch_bytes, void* stream) {
  NvtxRange nvtx_range("fwpkm_run_sequence_host");
  if (!st) return FWPKM_ERR_INVALID_ARG;
  if (T == 0) return FWPKM_OK;
  if (!q || !v || !g || !o || !scratch || T < 0 || T > st->wk.max_T || n_iter < 1) return FWPKM_ERR_INVALID_ARG;
  if (!aligned(scratch, ALIGN)) return FWPKM_ERR_INVALID_ARG;
  if (!host_pinned(q) || !host_pinned(v) || !host_pinned(g) || !host_pinned(o)) return FWPKM_ERR_INVALID_ARG;
  const Dims& d = st->dm;
  if (scratch_bytes < host_io_carve(d, T, nullptr, nullptr, nullptr, nullptr, nullptr)) return FWPKM_ERR_WORKSPACE;
  void *dq, *dv;
  float *dg, *dout;
  host_io_carve(d, T, (char*)scratch, &dq, &dv, &dg, &dout);
  const HostIO hio = {q, v, g, o};
  return run_sequence_impl(st, dq, dv, dg, T, n_iter, dout, &hio, stream);
}

// ---- the whole layer: projections in, the memory loop, projection out ----
// Scratch parts: q, v (q/v dtype), g, o, each starting on a 256-byte boundary.
static size_t run_layer_carve(const Dims& d, int T, char* base, void** q, void** v, float** g, float** o) {
  const size_t rows = (size_t)d.M * T, es = qv_size(d);
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return p;
  };
  void* pq = take(es * rows * d.d);
  void* pv = take(es * rows * d.dv);
  float* pg = (float*)take(4 * rows);
  float* po = (float*)take(4 * rows * d.dv);
  if (q) { *q = pq; *v = pv; *g = pg; *o = po; }
  return off;
}

fwpkm_status fwpkm_run_layer_scratch_size(const fwpkm_config* cfg, int T, size_t* bytes) {
  fwpkm_status s = check_cfg(cfg);
  if (s != FWPKM_OK) return s;
  if (!bytes || T < 0) return FWPKM_ERR_INVALID_ARG;
  *bytes = run_layer_carve(make_dims(cfg), T, nullptr, nullptr, nullptr, nullptr, nullptr);
  return FWPKM_OK;
}

fwpkm_status fwpkm_run_layer(fwpkm_layer* L, fwpkm_state* st, const void* h, int T, int n_iter, void* scratch,
                             size_t scratch_bytes, void* o_out, void* stream) {
  NvtxRange nvtx_range("fwpkm_run_layer");
  const fwpkm_layer_config* lc = layer_config(L);
  if (!lc || !st) return FWPKM_ERR_INVALID_ARG;
  if (T == 0) return FWPKM_OK;
  const Dims& d = st->dm;
  if (!h || !scratch || !o_out || T < 0 || n_iter < 1 || T > st->wk.max_T) return FWPKM_ERR_INVALID_ARG;
  if (d.H > 1) return FWPKM_ERR_UNSUPPORTED;
  if (lc->d != d.d || lc->d_v != d.dv || lc->qv_dtype != st->cfg.qv_dtype ||
      (long long)d.M * T > (long long)lc->max_rows)
    return FWPKM_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(o_out, 16) || !aligned(scratch, ALIGN)) return FWPKM_ERR_INVALID_ARG;
  if (scratch_bytes < run_layer_carve(d, T, nullptr, nullptr, nullptr, nullptr, nullptr)) return FWPKM_ERR_WORKSPACE;
  void *q, *v;
  float *g, *o;
  run_layer_carve(d, T, (char*)scratch, &q, &v, &g, &o);
  const int rows = d.M * T;
  fwpkm_status s = fwpkm_layer_in(L, h, rows, q, v, g, stream);
  if (s != FWPKM_OK) return s;
  s = fwpkm_run_sequence(st, q, v, g, T, n_iter, o, stream);
  if (s != FWPKM_OK) return s;
  return fwpkm_layer_out(L, o, rows, o_out, stream);
}

fwpkm_status fwpkm_last_addressing(fwpkm_state* st, int T, int32_t* idx_out, float* w_out, void* stream) {
  if (!st || T < 1 || T > st->wk.max_T) return FWPKM_ERR_INVALID_ARG;
  {
    fwpkm_status ps = peek_status(st);
    if (ps != FWPKM_OK) return ps;
  }
  const Dims& d = st->dm;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t row = (size_t)T * d.k, src_pitch = (size_t)st->wk.max_T * d.k;
  for (int m = 0; m < d.M; ++m) {
    if (idx_out && cudaMemcpyAsync(idx_out + m * row, st->wk.idx + m * src_pitch, row * 4,
                                   cudaMemcpyDeviceToDevice, s) != cudaSuccess) return last_cuda();
    if (w_out && cudaMemcpyAsync(w_out + m * row, st->wk.w + m * src_pitch, row * 4,
                                 cudaMemcpyDeviceToDevice, s) != cudaSuccess) return last_cuda();
  }
  return FWPKM_OK;
}

fwpkm_status fwpkm_sync(fwpkm_state* st, void* stream) {
  NvtxRange nvtx_range("fwpkm_sync");
  if (!st) return FWPKM_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    last_cuda();
    return FWPKM_ERR_CUDA;
  }
  int h = 0;
  if (cudaMemcpy(&h, st->wk.status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return last_cuda();
  const int hh = st->hstat ? *(volatile int*)st->hstat : DEV_OK;
  if (h == DEV_OK) h = hh;
  if (h != DEV_OK) {
    // the word is cleared before the host copy, so a kernel still running on another
    // stream can only leave both set again
    if (cudaMemset(st->wk.status, 0, sizeof(int)) != cudaSuccess) return last_cuda();
    // a kernel that gave up may have left arrival counters between launches non-zero
    if (h == DEV_TIMEOUT && st->wk.af_cnt &&
        cudaMemset(st->wk.af_cnt, 0, sizeof(int) * 4 * (size_t)st->dm.M) != cudaSuccess)
      return last_cuda();
    if (h == DEV_TIMEOUT && st->wk.vl_cnt &&
        cudaMemset(st->wk.vl_cnt, 0, sizeof(unsigned) * 2 * (size_t)st->dm.M) != cudaSuccess)
      return last_cuda();
    if (st->hstat) *(volatile int*)st->hstat = DEV_OK;
    return status_of_device(h);
  }
  return last_cuda();
}

fwpkm_status fwpkm_profile_kernel(fwpkm_state* st, int kind) {
  if (!st || ((kind < 0 || kind > KK_LAST) && kind != FWPKM_PROFILE_ALL)) return FWPKM_ERR_INVALID_ARG;
  if (kind != 0 && st->ev.empty()) {
    st->ev.resize(4096);
    st->ev_kind.assign(2048, 0);
    for (auto& e : st->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return FWPKM_ERR_CUDA;
  }
  st->prof_kind = kind;
  st->ev_used = 0;
  return FWPKM_OK;
}

fwpkm_status fwpkm_kernel_timeline(fwpkm_state* st, int max, int* kinds, float* start_ms, float* end_ms,
                                   int* n) {
  if (!st || !n || max < 0 || (max > 0 && (!kinds || !start_ms || !end_ms))) return FWPKM_ERR_INVALID_ARG;
  const int pairs = st->ev_used / 2;
  *n = pairs;
  if (pairs == 0) return FWPKM_OK;
  if (cudaEventSynchronize(st->ev[st->ev_used - 1]) != cudaSuccess) return FWPKM_ERR_CUDA;
  // the earliest start is the origin
  int first = 0;
  for (int i = 1; i < pairs; ++i) {
    float d = 0.f;
    if (cudaEventElapsedTime(&d, st->ev[2 * first], st->ev[2 * i]) != cudaSuccess) return FWPKM_ERR_CUDA;
    if (d < 0.f) first = i;
  }
  for (int i = 0; i < pairs && i < max; ++i) {
    float a = 0.f, b = 0.f;
    if (cudaEventElapsedTime(&a, st->ev[2 * first], st->ev[2 * i]) != cudaSuccess ||
        cudaEventElapsedTime(&b, st->ev[2 * first], st->ev[2 * i + 1]) != cudaSuccess)
      return FWPKM_ERR_CUDA;
    kinds[i] = st->ev_kind[i];
    start_ms[i] = a;
    end_ms[i] = b;
  }
  return FWPKM_OK;
}

fwpkm_status fwpkm_kernel_time(fwpkm_state* st, double* total_ms, int* launches) {
  if (!st || !total_ms || !launches) return FWPKM_ERR_INVALID_ARG;
  double tot = 0.0;
  for (int i = 0; i + 1 < st->ev_used; i += 2) {
    if (cudaEventSynchronize(st->ev[i + 1]) != cudaSuccess) return FWPKM_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, st->ev[i], st->ev[i + 1]) != cudaSuccess) return FWPKM_ERR_CUDA;
    tot += ms;
  }
  *total_ms = tot;
  *launches = st->ev_used / 2;
  st->ev_used = 0;
  return FWPKM_OK;
}

}  // extern "C"
