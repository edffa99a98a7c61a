// select.cu - the selection kernel of the launch chain: one CTA per (token, expert) pair runs
// the pair's selection (select_pair.cuh: top-K radix select or threshold, kept-set mask, the
// expert's union of kept neurons and its compaction by the expert's last pair).
#include "kernels.h"
#include "select_pair.cuh"

namespace moe {
namespace {

// NT threads per pair: 256, or 1024 for intermediate sizes of 4096 and more.  The kernel is
// latency-bound (dependent shared-memory and warp-level steps), so a large pair gets more warps
// to hide the latencies and fewer keys per thread in each pass.
template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(FwdParams p) {
  extern __shared__ uint32_t sm[];
  __shared__ SelShared<NT> ss;
  pdl_trigger();
  trace_point(p.trace, 2, 0);
  pdl_wait();
  trace_point(p.trace, 2, 1);
  const int n_pairs = ld_cg(&p.meta[kMetaPairs]);
  bool nan_seen = false;
  auto bar = []() { __syncthreads(); };
  for (int q = blockIdx.x; q < n_pairs; q += gridDim.x) {
    int j;
    const bool first = q == (int)blockIdx.x;
    auto mark = [&](int i) {
      if (first) trace_point(p.trace, 2, i);
    };
    select_pair<NT, false>(p, q, (int)threadIdx.x, sm, ss, bar, nan_seen, &j, mark);
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
  trace_point(p.trace, 2, 7);
}

}  // namespace

size_t select_smem_bytes(int imax) { return sel_key_bytes(imax); }

// 1024 threads per pair from this intermediate size on
constexpr int kWideSelect = 4096;

cudaError_t launch_select(const FwdParams& p, const LaunchShape& ls, cudaStream_t st, bool pdl) {
  const int pairs = p.B * (p.k + p.S);
  const int grid = pairs < ls.grid_select ? pairs : ls.grid_select;
  if (p.Imax >= kWideSelect)
    return launch_pdl(select_kernel<1024>, dim3(grid), dim3(1024), select_smem_bytes(p.Imax), st,
                      pdl, p);
  return launch_pdl(select_kernel<256>, dim3(grid), dim3(256), select_smem_bytes(p.Imax), st,
                    pdl, p);
}

cudaError_t configure_select(int imax, int budget, int* occupancy) {
  const size_t smem = select_smem_bytes(imax);
  cudaError_t e = allow_max_smem(select_kernel<256>, budget);
  if (e == cudaSuccess) e = allow_max_smem(select_kernel<1024>, budget);
  if (e != cudaSuccess) return e;
  return imax >= kWideSelect
             ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, select_kernel<1024>, 1024,
                                                             smem)
             : cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, select_kernel<256>, 256,
                                                             smem);
}

}  // namespace moe
