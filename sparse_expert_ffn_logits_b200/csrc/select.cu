// select.cu - per-(token, expert) neuron selection and the per-expert union of kept neurons.
//
// Inside a pair the lowest-scoring neuron activations are dropped ("Uncovering Intra-expert
// Activation Sparsity ...", technical summary, Methodology: activation masking).  The score of
// neuron n is |SiLU(g_n)|, an fp32 value whose bit pattern (sign cleared) orders like the value.
//   top-K mode: an MSB-first radix select (eight 4-bit digits) finds the K-th largest key tau
//     and how many keys equal to tau are kept; the kept set is every key > tau plus the
//     lowest-indexed keys == tau.  No sort.
//   threshold mode: one pass, keep key > t (the page's single-pass threshold mask).
// One CTA per pair: its keys sit in shared memory; each radix pass counts digits in registers
// (packed 16-bit bins) and merges them with warp reductions, with no atomics.  The kept set is
// written as an ascending index list + count (for export), as a bitmask row, and
// OR-ed into the expert's union bitmask.  The last pair of an expert to finish (atomic ticket,
// no waiting) compacts the union into an ascending row list for the up/down kernel and clears
// the bitmask.
#include "kernels.h"

namespace moe {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;

__global__ void __launch_bounds__(kSelThreads) select_kernel(FwdParams p) {
  extern __shared__ uint32_t sm[];
  __shared__ int hist[2048];
  __shared__ int scratch[33];
  __shared__ int wtot[kSelWarps];
  __shared__ int s_digit, s_above, s_last;
  pdl_trigger();
  trace_point(p.trace, 2, 0);
  pdl_wait();
  trace_point(p.trace, 2, 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Imax = p.Imax, Wmax = p.Imax / 32;
  uint32_t* key = sm;                                                 // [Imax]
  unsigned char* keep = reinterpret_cast<unsigned char*>(sm + Imax);  // [Imax]
  const int n_pairs = ld_cg(&p.meta[kMetaPairs]);
  bool nan_seen = false;
  for (int q = blockIdx.x; q < n_pairs; q += gridDim.x) {
    const int j = __ldcg(&p.pair_slot[q]);
    const Slot s = load_slot(&p.slots[j]);
    const int I = s.I, kind = s.kind;
    {
      const float4* a4 = reinterpret_cast<const float4*>(p.act + (size_t)q * Imax);
      for (int v0 = threadIdx.x; v0 < I / 4; v0 += 4 * kSelThreads) {
        float4 f[4];  // four 16-byte loads in flight per thread
#pragma unroll
        for (int u = 0; u < 4; ++u)
          f[u] = v0 + u * kSelThreads < I / 4 ? __ldcg(a4 + v0 + u * kSelThreads)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = v0 + u * kSelThreads;
          if (v < I / 4) {
            const float fv[4] = {f[u].x, f[u].y, f[u].z, f[u].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t k4 = __float_as_uint(fabsf(fv[c]));
              if (isnan(fv[c])) {
                nan_seen = true;
                k4 = 0;
              }
              key[v * 4 + c] = k4;
            }
          }
        }
      }
    }
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 2);
    const int mode = p.sel_mode[kind];
    const int K = min(p.sel_K[kind], I);
    const float thr = p.sel_t[kind];
    const bool radix = mode == 0 && K > 0 && K < I;
    uint32_t tau = 0;
    int need = 0;
    if (radix) {
      // eight 4-bit digits, most significant first.  Each thread counts its keys per digit in
      // packed 16-bit fields (bins 2i, 2i+1 in c[i]), a warp sum merges them, and warp 0 reads
      // the eight warps' sums to pick the digit: no atomics, two barriers per digit.
      uint32_t prefix = 0, pmask = 0;
      int krem = K;
#pragma unroll 1
      for (int shift = 28; shift >= 0; shift -= 4) {
        uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int n = threadIdx.x; n < I; n += blockDim.x) {
          const uint32_t u = key[n];
          if ((u & pmask) == prefix) {
            const uint32_t d = (u >> shift) & 15u;
            const uint32_t inc = 1u << ((d & 1u) * 16);
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] += (d >> 1) == (uint32_t)i ? inc : 0u;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) c[i] = __reduce_add_sync(0xffffffffu, c[i]);
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) hist[warp * 8 + i] = (int)c[i];
        }
        __syncthreads();
        if (warp == 0) {
          // lane l < 16 holds digit 15 - l; a suffix scan over the lanes finds the digit
          int cnt = 0;
          if (lane < 16) {
            const int d = 15 - lane;
#pragma unroll
            for (int w = 0; w < kSelWarps; ++w)
              cnt += (int)(((uint32_t)hist[w * 8 + (d >> 1)] >> ((d & 1) * 16)) & 0xFFFFu);
          }
          int incl = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const int above = incl - cnt;
          const unsigned hit = __ballot_sync(0xffffffffu, lane < 16 && above < krem && incl >= krem);
          const int src = __ffs(hit) - 1;
          if (lane == src) {
            s_digit = 15 - lane;
            s_above = above;
          }
        }
        __syncthreads();
        krem -= s_above;
        prefix |= (uint32_t)s_digit << shift;
        pmask |= 15u << shift;
      }
      tau = prefix;
      need = krem;
    }
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 3);
    // warp-contiguous segments of the neuron range, walked 32 at a time (ordered ballots)
    const int seg = ((I + 32 * kSelWarps - 1) / (32 * kSelWarps)) * 32;
    const int sb = warp * seg, se = min(I, sb + seg);
    int tie_base = 0;
    if (radix) {
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
        const uint32_t u = n < se ? key[n] : 0u;
        bool k_n;
        if (mode == 1) {
          k_n = __uint_as_float(u) > thr;
        } else if (K >= I) {
          k_n = true;
        } else if (K == 0) {
          k_n = false;
        } else {
          const bool eq = n < se && u == tau;
          const unsigned be = __ballot_sync(0xffffffffu, eq);
          k_n = u > tau || (eq && run + __popc(be & lanemask_lt()) < need);
          run += __popc(be);
        }
        k_n = k_n && n < se;
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
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 4);
    __threadfence();
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 5);
    if (threadIdx.x == 0) {
      const unsigned ticket = atomicAdd(&p.slot_ticket[j], 1u);
      s_last = ticket == (unsigned)s.T - 1u;
    }
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 6);
    if (s_last) {
      // last pair of this expert: compact the union bitmask into a row list, clear it
      __threadfence();
      const int W = I / 32;
      const int per = (W + blockDim.x - 1) / blockDim.x;
      const int wb = min(W, (int)threadIdx.x * per), we = min(W, wb + per);
      uint32_t words[2];
      int c = 0;
      for (int w = wb; w < we; ++w) {
        words[w - wb] = __ldcg(&urow[w]);
        c += __popc(words[w - wb]);
      }
      int utotal;
      int upos = block_exclusive_scan(c, scratch, &utotal);
      int* ul = p.ulist + (size_t)j * Imax;
      for (int w = wb; w < we; ++w) {
        uint32_t b = words[w - wb];
        while (b) {
          ul[upos++] = w * 32 + __ffs(b) - 1;
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
  trace_point(p.trace, 2, 7);
}

}  // namespace

size_t select_smem_bytes(int imax) { return (size_t)imax * 5 + 16; }

cudaError_t launch_select(const FwdParams& p, const LaunchShape& ls, cudaStream_t st, bool pdl) {
  const int pairs = p.B * (p.k + p.S);
  const int grid = pairs < ls.grid_select ? pairs : ls.grid_select;
  return launch_pdl(select_kernel, dim3(grid), dim3(kSelThreads), select_smem_bytes(p.Imax), st,
                    pdl, p);
}

cudaError_t configure_select(int imax, int budget, int* occupancy) {
  const size_t smem = select_smem_bytes(imax);
  cudaError_t e = allow_max_smem(select_kernel, budget);
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(occupancy, select_kernel, kSelThreads, smem);
}

}  // namespace moe
