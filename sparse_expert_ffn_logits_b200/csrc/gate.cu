// gate.cu - dense gate projection + SiLU of every evaluated (token, expert) pair.
//
// The gate is the part of an expert that cannot be skipped: it is what scores the neurons
// ("Uncovering Intra-expert Activation Sparsity ...", technical summary, Methodology: the gate
// projection runs densely to determine the activation scores).  Every evaluated expert's gate
// block [I][H] is read from HBM once per token tile.
//
// Persistent grid over work items (slot, row group of 16 neurons, token tile of 8 pairs),
// row group outer so that the token tiles of one row group run at the same time and share the
// rows through L2.  In an item the 8 warps split H; their partial 16x8 fragments are summed in
// shared memory and warp 0 writes act[q][n] = SiLU(g) in fp32.
#include "kernels.h"
#include "tile.cuh"

namespace moe {
namespace {

constexpr int kMaxSlots = kMaxRouted + kMaxShared;

template <typename T>
__global__ void __launch_bounds__(kThreads) gate_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ Slot s_slot[kMaxSlots];
  __shared__ int s_item0[kMaxSlots];
  __shared__ const T* s_x[kTileTok];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, Imax = p.Imax;
  const int n_slots = ld_cg(&p.meta[kMetaSlots]);
  const int n_items = ld_cg(&p.meta[kMetaGateItems]);
  for (int j = threadIdx.x; j < n_slots; j += blockDim.x) {
    s_slot[j] = p.slots[j];
    s_item0[j] = p.slots[j].item0;
  }
  __syncthreads();
  const T* x = static_cast<const T*>(p.x);
  bool nan_seen = false;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int j = find_slot(s_item0, n_slots, item);
    const Slot s = s_slot[j];
    const int local = item - s.item0;
    const int ntt = (s.T + kTileTok - 1) / kTileTok;
    const int rg = local / ntt, tt = local % ntt;
    const int n0 = rg * kTileRows;
    if (threadIdx.x < kTileTok) {
      const int ti = tt * kTileTok + threadIdx.x;
      s_x[threadIdx.x] = ti < s.T ? x + (size_t)p.pair_token[s.q0 + ti] * H : nullptr;
    }
    __syncthreads();
    const T* base = s.kind == 0
                        ? static_cast<const T*>(p.gate_r) + (size_t)s.expert * p.I * H
                        : static_cast<const T*>(p.gate_s) + (size_t)s.expert * p.Ish * H;
    const T* rowA = base + (size_t)(n0 + g) * H;
    const T* rowB = base + (size_t)(n0 + g + 8) * H;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    tile_dot<4>(rowA, rowB, s_x, warp, kWarps, H / 32, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
    __syncthreads();
    if (warp == 0) {
      reduce_fragments(red, d);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int ti = tt * kTileTok + 2 * t + (c & 1);
        if (ti < s.T) {
          const int n = n0 + g + (c >> 1) * 8;
          const float a = silu(d[c]);
          nan_seen |= isnan(a);
          p.act[(size_t)(s.q0 + ti) * Imax + n] = a;
        }
      }
    }
    __syncthreads();
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
}

}  // namespace

cudaError_t launch_gate(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st) {
  if (dtype == 0)
    return launch_pdl(gate_kernel<__nv_bfloat16>, dim3(ls.grid_gate), dim3(kThreads), 0, st, true,
                      p);
  return launch_pdl(gate_kernel<float>, dim3(ls.grid_gate), dim3(kThreads), 0, st, true, p);
}

int gate_occupancy(int dtype) {
  int n = 0;
  if (dtype == 0)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gate_kernel<__nv_bfloat16>, kThreads, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gate_kernel<float>, kThreads, 0);
  return n;
}

}  // namespace moe
