// metrics.cu -- addressing metrics: how evenly the reads use the memory's slots.
//
// Fast-weight Product Key Memory (paperlayer summary of arXiv 2601.00671v2), §D.3
// Addressing Metrics: the row contribution c_i of value row i is the number of accesses
// it receives within a window of tokens; coverage = share of the N slots with c_i > 0,
// collision rate = share of the accesses that are competitive, KLD = divergence of the
// slot-use distribution p_i = c_i / sum c from the uniform one.  Readings: an access is
// one (token, selected slot) pair; windows are consecutive blocks of `window` tokens of
// one memory (the last one may be shorter); an access is competitive when its row
// receives at least two accesses in the window; KLD = sum_i p_i log(p_i N), natural log;
// entries outside [0, N) are counted apart and are not accesses.
//
// Per window: a dense histogram of N 32-bit counters (integer atomics, so the counts
// are exact and independent of the order of arrival), then one pass over the counters
// that forms rows / accesses / competitive accesses exactly in 64-bit integers and
// sum c log c (c >= 2) in fp64 over a fixed partition with a fixed reduction tree, so
// the result is deterministic.  Counts below 256 are tallied per CTA in shared memory
// (integer atomics) and their c log c taken once per count value, so the scan evaluates
// no logarithm per row (a divergent fp64 log per row was most of the pass's time).  KLD = (sum c log c) / S + log(N / S) with S = sum c.
// Several windows are histogrammed at once (up to MT_MAX_BATCH, as the workspace
// allows); the counters of a batch are zeroed while they are read when another batch
// follows, so the whole call zero-fills them only once.  Launches: one zero-fill, then
// per batch a histogram pass and a reduction pass whose last CTA per window finishes it.
#include "fwpkm_internal.cuh"

namespace fwpkm {
namespace {

constexpr int MT_THREADS = 256;
constexpr int MT_RED_BLOCKS = 256;  // reduction CTAs per window (fixes the fp64 summation order)
constexpr int MT_MAX_BATCH = 32;    // windows histogrammed together at most
constexpr int MT_HIST = 256;        // counts below this are tallied per CTA (one log per count value)
static_assert(MT_HIST == MT_THREADS, "one thread per tallied count value");

struct MetricPart {
  unsigned long long rows, acc, comp;
  double clogc;
};

long long padded_slots(long long N) { return (N + 3) / 4 * 4; }  // uint4 rows of counters

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace of a batch of B windows: counters [B][Np] u32 | parts [B][MT_RED_BLOCKS] |
// invalid entries [B] u64 | reduction CTAs arrived [B] u32.
size_t metrics_carve(long long N, int B, char* base, uint32_t** cnt, MetricPart** part,
                     unsigned long long** bad, unsigned** arrive) {
  const size_t c_bytes = al256((size_t)B * padded_slots(N) * 4);
  const size_t p_bytes = al256((size_t)B * MT_RED_BLOCKS * sizeof(MetricPart));
  const size_t b_bytes = al256((size_t)B * 8);
  const size_t a_bytes = al256((size_t)B * 4);
  if (base) {
    *cnt = (uint32_t*)base;
    *part = (MetricPart*)(base + c_bytes);
    *bad = (unsigned long long*)(base + c_bytes + p_bytes);
    *arrive = (unsigned*)(base + c_bytes + p_bytes + b_bytes);
  }
  return c_bytes + p_bytes + b_bytes + a_bytes;
}

__global__ void __launch_bounds__(MT_THREADS)
metric_zero_kernel(uint4* __restrict__ cnt, long long n_vec, unsigned long long* __restrict__ bad,
                   unsigned* __restrict__ arrive, int nb) {
  const long long stride = (long long)gridDim.x * MT_THREADS;
  for (long long i = (long long)blockIdx.x * MT_THREADS + threadIdx.x; i < n_vec; i += stride)
    cnt[i] = make_uint4(0u, 0u, 0u, 0u);
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b < nb; b += MT_THREADS) {
      bad[b] = 0ull;
      arrive[b] = 0u;
    }
}

// Histogram of the accesses of window (w0 + blockIdx.y): the window's indices are one
// contiguous run of the [M][T][k] array, read once with streaming loads.
__global__ void __launch_bounds__(MT_THREADS)
metric_count_kernel(const int32_t* __restrict__ idx, long long T, int k, long long N, long long window, long long W,
                    long long w0, uint32_t* __restrict__ cnt, long long np_, unsigned long long* __restrict__ bad) {
  const long long gw = w0 + blockIdx.y;
  const long long m = gw / W, w = gw % W;
  const long long t0 = w * window;
  const long long t1 = t0 + window < T ? t0 + window : T;
  const int32_t* src = idx + (m * T + t0) * k;
  const long long len = (t1 - t0) * k;
  uint32_t* c = cnt + (long long)blockIdx.y * np_;
  unsigned nbad = 0;
  const long long stride = (long long)gridDim.x * MT_THREADS;
  for (long long i = (long long)blockIdx.x * MT_THREADS + threadIdx.x; i < len; i += stride) {
    const int s = __ldcs(src + i);
    if (s >= 0 && (long long)s < N) atomicAdd(c + s, 1u);
    else ++nbad;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nbad += __shfl_xor_sync(0xffffffffu, nbad, o);
  if ((threadIdx.x & 31) == 0 && nbad) atomicAdd(bad + blockIdx.y, (unsigned long long)nbad);
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ double warp_sum_f64(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Partial statistics of the counters of window blockIdx.y over a fixed slice pattern; the
// last CTA of the window to finish (arrival counter, after a fence) sums the partials --
// each lane a fixed stride, then a fixed butterfly, so the bits never depend on which CTA
// is last -- and writes the window's metrics.
__global__ void __launch_bounds__(MT_THREADS)
metric_reduce_kernel(uint32_t* __restrict__ cnt, long long np_, int rezero, MetricPart* __restrict__ part,
                     unsigned long long* __restrict__ bad, unsigned* __restrict__ arrive, long long w0, long long N,
                     double* __restrict__ out, long long* __restrict__ counts) {
  __shared__ MetricPart s_part[MT_THREADS / 32];
  __shared__ unsigned s_hist[MT_HIST];  // rows of this CTA's slice with count c (2 <= c < MT_HIST)
  __shared__ bool s_last;
  s_hist[threadIdx.x] = 0u;
  __syncthreads();
  uint4* c = reinterpret_cast<uint4*>(cnt + (long long)blockIdx.y * np_);
  const long long nv = np_ / 4;
  unsigned long long rows = 0, acc = 0, comp = 0;
  double clogc = 0.0;
  for (long long i = (long long)blockIdx.x * MT_THREADS + threadIdx.x; i < nv; i += (long long)MT_RED_BLOCKS * MT_THREADS) {
    const uint4 v = c[i];
    if (rezero) c[i] = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rows += x[e] != 0u;
      acc += x[e];
      if (x[e] >= 2u) {
        comp += x[e];
        if (x[e] < (uint32_t)MT_HIST) atomicAdd(&s_hist[x[e]], 1u);  // exact integer tally
        else clogc += (double)x[e] * log((double)x[e]);
      }
    }
  }
  __syncthreads();
  {  // c log c of the tallied rows: thread c takes count value c (a fixed assignment)
    const unsigned hc = s_hist[threadIdx.x];
    if (hc != 0u) clogc += (double)hc * ((double)threadIdx.x * log((double)threadIdx.x));
  }
  rows = warp_sum_u64(rows);
  acc = warp_sum_u64(acc);
  comp = warp_sum_u64(comp);
  clogc = warp_sum_f64(clogc);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_part[warp] = MetricPart{rows, acc, comp, clogc};
  __syncthreads();
  MetricPart* wpart = part + (long long)blockIdx.y * MT_RED_BLOCKS;
  if (threadIdx.x == 0) {
    MetricPart t = s_part[0];
    for (int i = 1; i < MT_THREADS / 32; ++i) {
      t.rows += s_part[i].rows; t.acc += s_part[i].acc; t.comp += s_part[i].comp; t.clogc += s_part[i].clogc;
    }
    wpart[blockIdx.x] = t;
    __threadfence();
    s_last = atomicAdd(arrive + blockIdx.y, 1u) == MT_RED_BLOCKS - 1;
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  MetricPart t{0ull, 0ull, 0ull, 0.0};
  for (int i = lane; i < MT_RED_BLOCKS; i += 32) {
    t.rows += __ldcg(&wpart[i].rows);
    t.acc += __ldcg(&wpart[i].acc);
    t.comp += __ldcg(&wpart[i].comp);
    t.clogc += __ldcg(&wpart[i].clogc);
  }
  t.rows = warp_sum_u64(t.rows);
  t.acc = warp_sum_u64(t.acc);
  t.comp = warp_sum_u64(t.comp);
  t.clogc = warp_sum_f64(t.clogc);
  if (lane != 0) return;
  const int b = blockIdx.y;
  const unsigned long long nbad = __ldcg(bad + b);
  bad[b] = 0ull;     // ready for the next batch
  arrive[b] = 0u;
  double cov = 0.0, col = 0.0, kld = 0.0;
  if (t.acc > 0) {
    const double S = (double)t.acc;
    cov = (double)t.rows / (double)N;
    col = (double)t.comp / S;
    kld = t.clogc / S + log((double)N / S);
  }
  const long long gw = w0 + b;
  out[gw * 3 + 0] = cov;
  out[gw * 3 + 1] = col;
  out[gw * 3 + 2] = kld;
  if (counts) {
    counts[gw * 4 + 0] = (long long)t.rows;
    counts[gw * 4 + 1] = (long long)t.acc;
    counts[gw * 4 + 2] = (long long)t.comp;
    counts[gw * 4 + 3] = (long long)nbad;
  }
}

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace
}  // namespace fwpkm

using namespace fwpkm;

extern "C" {

fwpkm_status fwpkm_metrics_workspace_size(int num_mem, int T, int N, int window, size_t* bytes) {
  if (!bytes || num_mem < 1 || T < 0 || N < 1 || window < 1) return FWPKM_ERR_INVALID_ARG;
  const long long total = (long long)num_mem * (((long long)T + window - 1) / window);
  const int B = (int)(total < 1 ? 1 : (total < MT_MAX_BATCH ? total : MT_MAX_BATCH));
  *bytes = metrics_carve(N, B, nullptr, nullptr, nullptr, nullptr, nullptr);
  return FWPKM_OK;
}

fwpkm_status fwpkm_addressing_metrics(const int32_t* idx, int num_mem, int T, int k, int N, int window,
                                      void* workspace, size_t ws_bytes, double* metrics, int64_t* counts,
                                      void* stream) {
  NvtxRange nvtx_range("fwpkm_addressing_metrics");
  if (num_mem < 1 || T < 0 || k < 1 || N < 1 || window < 1) return FWPKM_ERR_INVALID_ARG;
  if (T == 0) return FWPKM_OK;
  if (!idx || !workspace || !metrics) return FWPKM_ERR_INVALID_ARG;
  if (!is_aligned(idx, 4) || !is_aligned(workspace, 256) || !is_aligned(metrics, 8) ||
      (counts && !is_aligned(counts, 8)))
    return FWPKM_ERR_INVALID_ARG;
  const long long W = ((long long)T + window - 1) / window;
  const long long total = (long long)num_mem * W;
  int B = (int)(total < MT_MAX_BATCH ? total : MT_MAX_BATCH);
  while (B > 1 && metrics_carve(N, B, nullptr, nullptr, nullptr, nullptr, nullptr) > ws_bytes) --B;
  if (metrics_carve(N, B, nullptr, nullptr, nullptr, nullptr, nullptr) > ws_bytes) return FWPKM_ERR_WORKSPACE;
  uint32_t* cnt;
  MetricPart* part;
  unsigned long long* bad;
  unsigned* arrive;
  metrics_carve(N, B, (char*)workspace, &cnt, &part, &bad, &arrive);
  cudaStream_t s = (cudaStream_t)stream;
  const long long np_ = padded_slots(N);
  const long long n_vec = (long long)B * np_ / 4;
  const long long zb = (n_vec + MT_THREADS - 1) / MT_THREADS;
  metric_zero_kernel<<<(unsigned)(zb < 1184 ? (zb < 1 ? 1 : zb) : 1184), MT_THREADS, 0, s>>>(
      reinterpret_cast<uint4*>(cnt), n_vec, bad, arrive, B);
  int launches = 1;
  const long long max_len = (window < T ? (long long)window : (long long)T) * k;
  for (long long w0 = 0; w0 < total; w0 += B) {
    const int nb = (int)(total - w0 < B ? total - w0 : B);
    // about two resident waves (148 SMs x 8 CTAs of 256 threads) across the batch
    long long gx = (max_len + MT_THREADS * 4 - 1) / (MT_THREADS * 4);
    const long long cap = (2 * 148 * 8 + nb - 1) / nb;
    if (gx > cap) gx = cap;
    if (gx < 1) gx = 1;
    metric_count_kernel<<<dim3((unsigned)gx, (unsigned)nb), MT_THREADS, 0, s>>>(idx, T, k, N, window, W, w0, cnt,
                                                                                  np_, bad);
    const int rezero = w0 + nb < total ? 1 : 0;
    metric_reduce_kernel<<<dim3(MT_RED_BLOCKS, (unsigned)nb), MT_THREADS, 0, s>>>(
        cnt, np_, rezero, part, bad, arrive, w0, N, metrics, (long long*)counts);
    launches += 2;
  }
  count_launches(launches);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FWPKM_OK : FWPKM_ERR_CUDA;
}

}  // extern "C"
