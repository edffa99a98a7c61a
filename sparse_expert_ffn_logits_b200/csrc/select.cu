// select.cu - per-(token, expert) neuron selection and the per-expert union of kept neurons.
//
// Inside a pair the lowest-scoring neuron activations are dropped ("Uncovering Intra-expert
// Activation Sparsity ...", technical summary, Methodology: activation masking).  The score of
// neuron n is |SiLU(g_n)|, an fp32 value whose bit pattern (sign cleared) orders like the value.
//   top-K mode: an MSB-first radix select (four 8-bit digits, shared-memory histograms) finds
//     the K-th largest key tau and how many keys equal to tau are kept; the kept set is every
//     key > tau plus the lowest-indexed keys == tau.  No sort.
//   threshold mode: one pass, keep key > t (the page's single-pass threshold mask).
// The kept set is written as an ascending index list + count (for export), as a bitmask row,
// and OR-ed into the expert's union bitmask.  The last pair of an expert to finish (atomic
// ticket, no waiting) compacts the union into an ascending row list for the up/down kernel and
// clears the bitmask for the next call.
#include "kernels.h"

namespace moe {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

__global__ void __launch_bounds__(kSelThreads) select_kernel(FwdParams p) {
  extern __shared__ uint32_t sm[];
  __shared__ int hist[256];
  __shared__ int scratch[33];
  __shared__ int wtot[kSelWarps];
  __shared__ int s_digit, s_above, s_last;
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Imax = p.Imax, Wmax = p.Imax / 32;
  uint32_t* key = sm;                                               // [Imax]
  unsigned char* keep = reinterpret_cast<unsigned char*>(sm + Imax);  // [Imax]
  const int n_pairs = ld_cg(&p.meta[kMetaPairs]);
  bool nan_seen = false;
  for (int q = blockIdx.x; q < n_pairs; q += gridDim.x) {
    const int j = p.pair_slot[q];
    const Slot s = p.slots[j];
    const int I = s.I, kind = s.kind;
    const float* a = p.act + (size_t)q * Imax;
    for (int n = threadIdx.x; n < I; n += blockDim.x) {
      const float f = a[n];
      uint32_t u = __float_as_uint(fabsf(f));
      if (isnan(f)) {
        nan_seen = true;
        u = 0;
      }
      key[n] = u;
    }
    __syncthreads();
    const int mode = p.sel_mode[kind];
    const int K = min(p.sel_K[kind], I);
    const float thr = p.sel_t[kind];
    uint32_t tau = 0;
    int need = 0;
    if (mode == 0 && K > 0 && K < I) {
      uint32_t prefix = 0, pmask = 0;
      int krem = K;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int n = threadIdx.x; n < I; n += blockDim.x) {
          const uint32_t u = key[n];
          if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
        }
        __syncthreads();
        if (warp == 0) {
          // lane l owns digits 255-8l .. 248-8l (descending); find the digit holding the
          // krem-th largest key
          int c[8], sum = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            c[i] = hist[255 - 8 * lane - i];
            sum += c[i];
          }
          int incl = sum;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          int above = incl - sum;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (above < krem && above + c[i] >= krem) {
              s_digit = 255 - 8 * lane - i;
              s_above = above;
            }
            above += c[i];
          }
        }
        __syncthreads();
        krem -= s_above;
        prefix |= (uint32_t)s_digit << shift;
        pmask |= 255u << shift;
        __syncthreads();
      }
      tau = prefix;
      need = krem;
    }
    // warp-contiguous segments of the neuron range, walked 32 at a time (ordered ballots)
    const int seg = ((I + 32 * kSelWarps - 1) / (32 * kSelWarps)) * 32;
    const int sb = warp * seg, se = min(I, sb + seg);
    int tie_base = 0;
    if (mode == 0 && K > 0 && K < I) {
      int ties = 0;
      for (int n0 = sb; n0 < se; n0 += 32) {
        const int n = n0 + lane;
        ties += __popc(__ballot_sync(0xffffffffu, n < se && key[n] == tau));
      }
      if (lane == 0) wtot[warp] = ties;
      __syncthreads();
      for (int w = 0; w < warp; ++w) tie_base += wtot[w];
      __syncthreads();
    }
    int kept = 0;
    {
      int run = tie_base;
      for (int n0 = sb; n0 < se; n0 += 32) {
        const int n = n0 + lane;
        bool k_n = false;
        if (n < se) {
          const uint32_t u = key[n];
          if (mode == 1) {
            k_n = __uint_as_float(u) > thr;
          } else if (K >= I) {
            k_n = true;
          } else if (K > 0) {
            k_n = u > tau;
          }
        }
        if (mode == 0 && K > 0 && K < I) {
          const bool eq = n < se && key[n] == tau;
          const unsigned be = __ballot_sync(0xffffffffu, eq);
          const int rank = run + __popc(be & lanemask_lt());
          if (eq && rank < need) k_n = true;
          run += __popc(be);
        }
        if (n < se) keep[n] = k_n ? 1 : 0;
        kept += __popc(__ballot_sync(0xffffffffu, k_n));
      }
    }
    if (lane == 0) wtot[warp] = kept;
    __syncthreads();
    int pos = 0, total = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      if (w < warp) pos += wtot[w];
      total += wtot[w];
    }
    int* list = p.lists + (size_t)q * Imax;
    uint32_t* mrow = p.maskbits + (size_t)q * Wmax;
    uint32_t* urow = p.ubits + (size_t)j * Wmax;
    for (int n0 = sb; n0 < se; n0 += 32) {
      const int n = n0 + lane;
      const bool k_n = n < se && keep[n];
      const unsigned b = __ballot_sync(0xffffffffu, k_n);
      if (k_n) list[pos + __popc(b & lanemask_lt())] = n;
      pos += __popc(b);
      if (lane == 0) {
        mrow[n0 >> 5] = b;
        if (b) atomicOr(&urow[n0 >> 5], b);
      }
    }
    if (threadIdx.x == 0) p.cnt[q] = total;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned ticket = atomicAdd(&p.slot_ticket[j], 1u);
      s_last = ticket == (unsigned)s.T - 1u;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      // compact the expert's union bitmask into an ascending row list, then clear it
      const int W = I / 32;
      const int per = (W + blockDim.x - 1) / blockDim.x;
      const int wb = min(W, (int)threadIdx.x * per), we = min(W, wb + per);
      uint32_t words[4];
      int c = 0;
      for (int w = wb; w < we; ++w) {
        words[w - wb] = ld_cg(&urow[w]);
        c += __popc(words[w - wb]);
      }
      int utotal;
      int upos = block_exclusive_scan(c, scratch, &utotal);
      int* ul = p.ulist + (size_t)j * Imax;
      for (int w = wb; w < we; ++w) {
        uint32_t b = words[w - wb];
        while (b) {
          const int bit = __ffs(b) - 1;
          ul[upos++] = w * 32 + bit;
          b &= b - 1;
        }
        urow[w] = 0;
      }
      if (threadIdx.x == 0) {
        p.ucnt[j] = utotal;
        p.slot_ticket[j] = 0;
      }
    }
    __syncthreads();
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
}

}  // namespace

size_t select_smem_bytes(int imax) { return (size_t)imax * 5 + 16; }

cudaError_t launch_select(const FwdParams& p, const LaunchShape& ls, cudaStream_t st) {
  const int pairs = p.B * (p.k + p.S);
  const int grid = pairs < ls.grid_select ? pairs : ls.grid_select;
  return launch_pdl(select_kernel, dim3(grid), dim3(kSelThreads), select_smem_bytes(p.Imax), st,
                    true, p);
}

cudaError_t configure_select(int imax, int* occupancy) {
  const size_t smem = select_smem_bytes(imax);
  cudaError_t e =
      cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, select_kernel, kSelThreads, smem);
}

}  // namespace moe
