// updown.cu - fused sparse up/down projection over the kept neurons, weighted into the output.
//
// Only the weights of active neurons are read ("Uncovering Intra-expert Activation Sparsity
// ...", technical summary, Methodology: fused up-down projection).  The packed layout keeps a
// neuron's W_up row and W_down column side by side ([I][2][H]), so the rows of the expert's
// kept-neuron union are gathered as contiguous 2*H*elt chunks and a dropped neuron costs no
// bytes.  Each row is read once per token tile of its expert; tokens of the tile whose own
// kept set lacks the neuron get coefficient 0.
//
// Work item = (slot, 16 union rows, token tile of 8 pairs), row group outer.  Per item:
//   1. u[r][c] = W_up[n_r] . x_c           tensor cores, the 8 warps split H (tile_dot)
//   2. hc[r][c] = mask * SiLU(g) * u        fp32, rounded to bf16 for the tensor cores
//   3. y[h][c] += sum_r W_down[h][n_r] hc   tensor cores, 64 h per warp step (tile_down)
//   4. out_acc[token][h] += w_c * y         fp32 vector reductions in L2
#include "kernels.h"
#include "tile.cuh"

namespace moe {
namespace {

constexpr int kMaxSlots = kMaxRouted + kMaxShared;

template <typename T>
__global__ void __launch_bounds__(kThreads) updown_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ Slot s_slot[kMaxSlots];
  __shared__ int s_item0[kMaxSlots + 1];
  __shared__ int scratch[33];
  __shared__ const T* s_x[kTileTok];
  __shared__ const T* s_up[kTileRows];
  __shared__ const T* s_dn[kTileRows];
  __shared__ int s_n[kTileRows];
  __shared__ int s_rvalid[kTileRows];
  __shared__ int s_q[kTileTok];
  __shared__ int s_tok[kTileTok];
  __shared__ float s_w[kTileTok];
  __shared__ float s_coef[kTileRows][kTileTok];
  __shared__ float s_hcf[kTileRows][kTileTok];               // fp32 variant
  __shared__ __align__(16) uint32_t s_hcw[kTileTok][kTileRows / 2];  // bf16 pairs, token-major
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, Imax = p.Imax, Wmax = p.Imax / 32;
  const int n_slots = ld_cg(&p.meta[kMetaSlots]);
  // items per slot = row groups of the kept-neuron union x token tiles
  {
    const int per = (n_slots + blockDim.x - 1) / blockDim.x;
    const int b0 = min(n_slots, (int)threadIdx.x * per), b1 = min(n_slots, b0 + per);
    int c = 0;
    for (int j = b0; j < b1; ++j) {
      const Slot s = p.slots[j];
      s_slot[j] = s;
      const int rows = ld_cg(&p.ucnt[j]);
      const int v = ((rows + kTileRows - 1) / kTileRows) * ((s.T + kTileTok - 1) / kTileTok);
      s_item0[j] = v;
      c += v;
    }
    int total;
    int run = block_exclusive_scan(c, scratch, &total);
    for (int j = b0; j < b1; ++j) {
      const int v = s_item0[j];
      s_item0[j] = run;
      run += v;
    }
    if (threadIdx.x == 0) s_item0[n_slots] = total;
    __syncthreads();
  }
  const int n_items = s_item0[n_slots];
  const T* x = static_cast<const T*>(p.x);
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int j = find_slot(s_item0, n_slots, item);
    const Slot s = s_slot[j];
    const int local = item - s_item0[j];
    const int ntt = (s.T + kTileTok - 1) / kTileTok;
    const int rg = local / ntt, tt = local % ntt;
    const int rows = ld_cg(&p.ucnt[j]);
    const T* ud = s.kind == 0
                      ? static_cast<const T*>(p.updown_r) + (size_t)s.expert * p.I * 2 * H
                      : static_cast<const T*>(p.updown_s) + (size_t)s.expert * p.Ish * 2 * H;
    if (threadIdx.x < kTileRows) {
      const int r = threadIdx.x;
      const int idx = rg * kTileRows + r;
      const bool valid = idx < rows;
      const int n = p.ulist[(size_t)j * Imax + (valid ? idx : rg * kTileRows)];
      s_n[r] = n;
      s_rvalid[r] = valid;
      s_up[r] = ud + (size_t)n * 2 * H;
      s_dn[r] = ud + (size_t)n * 2 * H + H;
    } else if (threadIdx.x >= 32 && threadIdx.x < 32 + kTileTok) {
      const int c = threadIdx.x - 32;
      const int ti = tt * kTileTok + c;
      if (ti < s.T) {
        const int q = s.q0 + ti;
        const int tok = p.pair_token[q];
        s_q[c] = q;
        s_tok[c] = tok;
        s_w[c] = p.pair_w[q];
        s_x[c] = x + (size_t)tok * H;
      } else {
        s_q[c] = -1;
        s_tok[c] = -1;
        s_w[c] = 0.f;
        s_x[c] = nullptr;
      }
    }
    __syncthreads();
    if (threadIdx.x < kTileRows * kTileTok) {
      const int r = threadIdx.x >> 3, c = threadIdx.x & 7;
      const int q = s_q[c], n = s_n[r];
      float coef = 0.f;
      if (q >= 0 && s_rvalid[r] && ((p.maskbits[(size_t)q * Wmax + (n >> 5)] >> (n & 31)) & 1u))
        coef = p.act[(size_t)q * Imax + n];
      s_coef[r][c] = coef;
    }
    // 1. up projection
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    tile_dot<4>(s_up[g], s_up[g + 8], s_x, warp, kWarps, H / 32, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
    __syncthreads();
    // 2. coefficients
    if (warp == 0) {
      reduce_fragments(red, d);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = g + (c >> 1) * 8, tok = 2 * t + (c & 1);
        const float hc = s_coef[r][tok] * d[c];
        s_hcf[r][tok] = hc;
        reinterpret_cast<__nv_bfloat16*>(&s_hcw[tok][0])[r] = __float2bfloat16_rn(hc);
      }
    }
    __syncthreads();
    // 3-4. down projection and weighted reduction into out_acc
    const uint32_t b0 = s_hcw[g][t], b1 = s_hcw[g][4 + t];
    const int tok0 = s_tok[2 * t], tok1 = s_tok[2 * t + 1];
    const float w0 = s_w[2 * t], w1 = s_w[2 * t + 1];
    for (int ch = warp; ch < H / 64; ch += kWarps) {
      const int h0 = ch * 64;
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
      tile_down(s_dn, h0, b0, b1, s_hcf, acc);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int h = h0 + 8 * g + 2 * i;
        if (tok0 >= 0) red_add_v2(p.out_acc + (size_t)tok0 * H + h, w0 * acc[i][0], w0 * acc[i][2]);
        if (tok1 >= 0) red_add_v2(p.out_acc + (size_t)tok1 * H + h, w1 * acc[i][1], w1 * acc[i][3]);
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_updown(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st) {
  if (dtype == 0)
    return launch_pdl(updown_kernel<__nv_bfloat16>, dim3(ls.grid_updown), dim3(kThreads), 0, st,
                      true, p);
  return launch_pdl(updown_kernel<float>, dim3(ls.grid_updown), dim3(kThreads), 0, st, true, p);
}

int updown_occupancy(int dtype) {
  int n = 0;
  if (dtype == 0)
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, updown_kernel<__nv_bfloat16>, kThreads, 0);
  else
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, updown_kernel<float>, kThreads, 0);
  return n;
}

}  // namespace moe
