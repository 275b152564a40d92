// topk.cu -- per-half top-k over the distance rows written by the scoring GEMM (the row
// routine is in topk.cuh).
#include "topk.cuh"

namespace fwpkm {

constexpr int TK_THREADS = 256;

template <int NPL>
__global__ void __launch_bounds__(TK_THREADS, 3)
topk_rows_kernel(Dims dm, Work w, int wt0, int len) {
  pdl_wait();
  pdl_trigger();
  __shared__ u64 s_cand[TK_THREADS / 32][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x * (TK_THREADS / 32) + warp;
  const int p = blockIdx.y;
  if (i >= len) return;
  const float* row = w.Dfull + ((size_t)p * w.drows + i) * dm.n;
  const size_t obase = ((size_t)p * w.max_T + wt0 + i) * dm.k;
  row_topk<NPL>(row, dm.n, dm.k, lane, s_cand[warp], w.A + obase, w.Dsv + obase);
}

int launch_topk_rows(const Dims& d, const Work& w, int wt0, int len, cudaStream_t s) {
  if (len <= 0) return 0;
  dim3 grid((len + 7) / 8, d.M * 2);
  const int npl = (d.n + 31) / 32;
  if (npl <= 2) launch_k(topk_rows_kernel<2>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else if (npl <= 4) launch_k(topk_rows_kernel<4>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else if (npl <= 8) launch_k(topk_rows_kernel<8>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else if (npl <= 16) launch_k(topk_rows_kernel<16>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else if (npl <= 32) launch_k(topk_rows_kernel<32>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else if (npl <= 64) launch_k(topk_rows_kernel<64>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  else launch_k(topk_rows_kernel<128>, grid, TK_THREADS, 0, s, d, w, wt0, len);
  return 1;
}

}  // namespace fwpkm
