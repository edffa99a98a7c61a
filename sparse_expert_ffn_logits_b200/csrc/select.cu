// select.cu - per-(token, expert) neuron selection and the per-expert union of kept neurons.
//
// Inside a pair the lowest-scoring neuron activations are dropped ("Uncovering Intra-expert
// Activation Sparsity ...", technical summary, Methodology: activation masking).  The score of
// neuron n is |SiLU(g_n)|, an fp32 value whose bit pattern (sign cleared) orders like the value.
//   top-K mode: an MSB-first radix select (4-bit digits) finds the K-th largest key tau and
//     how many keys equal to tau are kept; the kept set is every key > tau plus the
//     lowest-indexed keys == tau.  No sort.  Once at most 32 keys share the decided prefix,
//     one warp ranks those directly.
//   threshold mode: one pass, keep key > t (the page's single-pass threshold mask).
// One CTA per pair: its keys sit in shared memory; each radix pass counts digits in registers
// (packed 16-bit bins), merges them with warp reductions and one barrier.  The kept set is
// written as the pair's bitmask row and OR-ed into the expert's union bitmask; the last pair
// of an expert to finish (atomic ticket, no waiting) compacts the union into the ascending row
// list that the up/down kernel reads, and clears it.  (Ascending index lists and counts of the
// pairs, for export only, are derived from the mask rows on request.)
#include "kernels.h"

namespace moe {
namespace {

// NT threads per pair: 256, or 1024 for intermediate sizes of 4096 and more.  The kernel is
// latency-bound (dependent shared-memory and warp-level steps), so a large pair gets more warps
// to hide the latencies and fewer keys per thread in each pass.
template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(FwdParams p) {
  constexpr int kSelThreads = NT, kSelWarps = NT / 32;
  constexpr int kBpt = kHistBins / NT;  // histogram bins per thread (8 or 2)
  static_assert(kBpt == 8 || kBpt == 2, "histogram bins per thread");
  extern __shared__ uint32_t sm[];
  __shared__ int hist[2 * kSelWarps * 8];
  __shared__ uint32_t cbuf[32];
  __shared__ int s_ncand, s_need, s_eqtot, s_last;
  __shared__ uint32_t s_tau;
  pdl_trigger();
  trace_point(p.trace, 2, 0);
  pdl_wait();
  trace_point(p.trace, 2, 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Imax = p.Imax, Wmax = p.Imax / 32;
  uint32_t* key = sm;  // [Imax]
  const int n_pairs = ld_cg(&p.meta[kMetaPairs]);
  bool nan_seen = false;
  for (int q = blockIdx.x; q < n_pairs; q += gridDim.x) {
    // The first activations are requested before the pair's slot is known (the row is Imax
    // long whatever the expert's I): one round trip instead of three dependent ones.
    const float4* a4 = reinterpret_cast<const float4*>(p.act + (size_t)q * Imax);
    constexpr int kKeyLoads = 8;  // 16-byte loads in flight per thread (I <= 8192 in one round)
    float4 f[kKeyLoads];
#pragma unroll
    for (int u = 0; u < kKeyLoads; ++u) {
      const int v = threadIdx.x + u * kSelThreads;
      f[u] = v < Imax / 4 ? __ldcg(a4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // routed pairs come first (B * k of them), then the shared experts' pairs
    const int kind = q >= p.B * p.k ? 1 : 0;
    const int I = kind ? p.Ish : p.I;
    // the pair's score histogram (top-K pairs) is requested together with its activations:
    // thread r holds the kBpt bins counted from the top, [kBpt (NT - 1 - r), kBpt (NT - r))
    const bool hist_on = uses_hist(p, kind);
    unsigned hb[kBpt];
    unsigned* hrow = p.hist + (size_t)q * kHistBins;
    const int hb0 = kBpt * (kSelThreads - 1 - threadIdx.x);
    if constexpr (kBpt == 8) {
      uint4 h0 = make_uint4(0, 0, 0, 0), h1 = make_uint4(0, 0, 0, 0);
      if (hist_on) {
        h0 = __ldcg(reinterpret_cast<const uint4*>(hrow + hb0));
        h1 = __ldcg(reinterpret_cast<const uint4*>(hrow + hb0 + 4));
      }
      hb[0] = h0.x; hb[1] = h0.y; hb[2] = h0.z; hb[3] = h0.w;
      hb[4] = h1.x; hb[5] = h1.y; hb[6] = h1.z; hb[7] = h1.w;
    } else {
      uint2 h0 = make_uint2(0, 0);
      if (hist_on) h0 = __ldcg(reinterpret_cast<const uint2*>(hrow + hb0));
      hb[0] = h0.x; hb[1] = h0.y;
    }
    const int j = __ldcg(&p.pair_slot[q]);  // the expert's slot, for its union row
    if (j < 0) continue;  // an expert another handle evaluates (the same for the whole CTA)
    if (threadIdx.x == 0) s_ncand = 0;
    for (int v0 = threadIdx.x;; v0 += kKeyLoads * kSelThreads) {
#pragma unroll
      for (int u = 0; u < kKeyLoads; ++u) {
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
      if (v0 + kKeyLoads * kSelThreads >= I / 4) break;
#pragma unroll
      for (int u = 0; u < kKeyLoads; ++u) {  // the next 16-byte loads per thread
        const int v = v0 + kKeyLoads * kSelThreads + u * kSelThreads;
        f[u] = v < I / 4 ? __ldcg(a4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 2);
    const int mode = p.sel_mode[kind];
    const int K = min(p.sel_K[kind], I);
    const float thr = p.sel_t[kind];
    const bool radix = mode == 0 && K > 0 && K < I;
    uint32_t tau = 0;
    int need = 0, eqtot = 0;  // keys equal to tau, and how many of them are kept
    if (radix) {
      // MSB-first radix select of the K-th largest key, 4-bit digits.  Each thread counts its
      // keys per digit in packed 16-bit fields, a warp sum merges them, and after one barrier
      // every warp reads the eight warps' sums and finds the digit itself (the histogram is
      // double-buffered, so the next pass can write while a slow warp still reads).  Once at
      // most 32 keys share the prefix, one warp ranks them directly.
      uint32_t prefix = 0, pmask = 0;
      int krem = K, cand = I, shift = 28, pass = 0;
      if (hist_on) {
        // The gate counted this pair's keys by their top 12 bits.  An exclusive scan of the
        // threads' bin sums in thread order gives the keys in the bins above each thread's
        // bins, and the thread whose bins hold the K-th largest key names its bin.  The row is
        // cleared for the next call.
        const int b0 = hb0;
#pragma unroll
        for (int i = 0; i < kBpt; ++i) hrow[b0 + i] = 0;
        int mine = 0;
#pragma unroll
        for (int i = 0; i < kBpt; ++i) mine += (int)hb[i];
        int above = block_exclusive_scan(mine, reinterpret_cast<int*>(hist), nullptr);
        if (above < K && above + mine >= K) {
#pragma unroll
          for (int i = kBpt - 1; i >= 0; --i) {
            const int c = (int)hb[i];
            if (above < K && above + c >= K) {
              s_tau = (uint32_t)(b0 + i);
              s_need = K - above;
              s_eqtot = c;
            }
            above += c;
          }
        }
        __syncthreads();
        prefix = s_tau << kHistShift;
        pmask = ~0u << kHistShift;
        krem = s_need;
        cand = s_eqtot;
        shift = kHistShift - 4;
        __syncthreads();  // s_tau and friends are written again below
      }
#pragma unroll 1
      for (; shift >= 0 && cand > 32; shift -= 4, ++pass) {
        uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int n = threadIdx.x; n < I; n += kSelThreads) {
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
        int* hb = hist + (pass & 1) * (kSelWarps * 8);
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) hb[warp * 8 + i] = (int)c[i];
        }
        __syncthreads();
        // lane l < 16 holds digit 15 - l; a scan over the lanes finds the digit of the K-th key
        int cnt = 0;
        if (lane < 16) {
          const int d = 15 - lane;
#pragma unroll
          for (int w = 0; w < kSelWarps; ++w)
            cnt += (int)(((uint32_t)hb[w * 8 + (d >> 1)] >> ((d & 1) * 16)) & 0xFFFFu);
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int above = incl - cnt;
        const unsigned hit = __ballot_sync(0xffffffffu, lane < 16 && above < krem && incl >= krem);
        const int src = __ffs(hit) - 1;
        krem -= __shfl_sync(0xffffffffu, above, src);
        cand = __shfl_sync(0xffffffffu, cnt, src);
        prefix |= (uint32_t)(15 - src) << shift;
        pmask |= 15u << shift;
      }
      if (shift < 0) {
        tau = prefix;  // every bit decided: the krem largest keys equal to prefix are kept
        need = krem;
        eqtot = cand;
      } else {
        // at most 32 keys carry the prefix: gather them (any order) and rank them in warp 0
        for (int n = threadIdx.x; n < I; n += kSelThreads) {
          const uint32_t u = key[n];
          if ((u & pmask) == prefix) {
            const int slot = atomicAdd(&s_ncand, 1);  // < cand <= 32 by construction
            if (slot < 32) cbuf[slot] = u;
          }
        }
        __syncthreads();
        if (warp == 0) {
          const bool valid = lane < cand;
          const uint32_t mine = valid ? cbuf[lane] : 0u;
          int gt = 0, ge = 0;
          for (int j = 0; j < cand; ++j) {
            const uint32_t o = __shfl_sync(0xffffffffu, mine, j);
            gt += o > mine;
            ge += o >= mine;
          }
          const unsigned hit = __ballot_sync(0xffffffffu, valid && gt < krem && ge >= krem);
          const int src = __ffs(hit) - 1;
          if (lane == src) {
            s_tau = mine;
            s_need = krem - gt;
            s_eqtot = ge - gt;
          }
        }
        __syncthreads();
        tau = s_tau;
        need = s_need;
        eqtot = s_eqtot;
      }
    }
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 3);
    // Kept set, one ballot per 32-neuron chunk c (neurons 32c .. 32c + 31), gathered in shared
    // memory, then written by all threads at once as the pair's mask row and OR-ed into the
    // expert's union row.  When every key equal to the cut is kept (the usual case) the mask is
    // simply key >= tau.  Otherwise ties are kept lowest index first: warp 0 scans the chunks'
    // tie counts in order and trims each chunk's ties.
    const int nch = I / 32;
    uint32_t* mrow = p.maskbits + (size_t)q * Wmax;
    uint32_t* urow = p.ubits + (size_t)j * Wmax;
    uint32_t* s_km = key + Imax;        // [Imax / 32] above-cut masks, then the kept masks
    uint32_t* s_em = s_km + Imax / 32;  // [Imax / 32] tie masks
    if (!radix || eqtot == need) {
      for (int c = warp; c < nch; c += kSelWarps) {
        const uint32_t u = key[32 * c + lane];
        bool k_n;
        if (radix) k_n = u >= tau;
        else if (mode == 1) k_n = __uint_as_float(u) > thr;
        else k_n = K >= I;
        const unsigned km = __ballot_sync(0xffffffffu, k_n);
        if (lane == 0) s_km[c] = km;
      }
    } else {
      for (int c = warp; c < nch; c += kSelWarps) {
        const uint32_t u = key[32 * c + lane];
        const unsigned gm = __ballot_sync(0xffffffffu, u > tau);
        const unsigned em = __ballot_sync(0xffffffffu, u == tau);
        if (lane == 0) {
          s_km[c] = gm;
          s_em[c] = em;
        }
      }
      __syncthreads();
      if (warp == 0) {
        const int cpl = (nch + 31) / 32;  // lane l owns chunks [l * cpl, (l + 1) * cpl)
        const int c0 = min(nch, lane * cpl), c1 = min(nch, c0 + cpl);
        int ties = 0;
        for (int c = c0; c < c1; ++c) ties += __popc(s_em[c]);
        int tincl = ties;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, tincl, o);
          if (lane >= o) tincl += y;
        }
        int tb = tincl - ties;  // ties before this lane's block
        for (int c = c0; c < c1; ++c) {
          uint32_t em = s_em[c];
          const int ne = __popc(em);
          const int take = max(0, min(ne, need - tb));
          for (int d = ne - take; d > 0; --d) em ^= 1u << (31 - __clz(em));  // drop the highest
          s_km[c] |= em;
          tb += ne;
        }
      }
    }
    __syncthreads();
    for (int c = threadIdx.x; c < nch; c += kSelThreads) {
      const uint32_t km = s_km[c];
      mrow[c] = km;
      if (km) red_or(&urow[c], km);
    }
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 4);
    // the last pair of an expert to finish compacts the expert's union (atomic ticket, no
    // waiting): every pair's union bits are published before its ticket
    __threadfence();
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 5);
    if (threadIdx.x == 0) {
      const unsigned ticket = atomicAdd(&p.slot_ticket[j], 1u);
      s_last = ticket == (unsigned)__ldcg(&p.slots[j].T) - 1u;
    }
    __syncthreads();
    if (q == (int)blockIdx.x) trace_point(p.trace, 2, 6);
    if (s_last) {
      // The whole CTA compacts the union bitmask into the ascending row list and clears it:
      // thread t owns the words [t wpt, (t + 1) wpt), a block scan of their bit counts gives
      // each word's first list position, and then each warp writes one word per step, lane l
      // placing bit l at its rank among the word's set bits.
      __threadfence();
      const int W = I / 32, wpt = (W + kSelThreads - 1) / kSelThreads;
      uint32_t* s_word = key;               // [W] union words (the keys are no longer needed)
      int* s_base = reinterpret_cast<int*>(key + Imax / 2);  // [W] first position of each word
      const int wb = min(W, (int)threadIdx.x * wpt), we = min(W, wb + wpt);
      int c = 0;
      for (int w = wb; w < we; ++w) {
        const uint32_t b = __ldcg(&urow[w]);
        urow[w] = 0;
        s_word[w] = b;
        c += __popc(b);
      }
      int total;
      int base = block_exclusive_scan(c, reinterpret_cast<int*>(hist), &total);
      for (int w = wb; w < we; ++w) {
        s_base[w] = base;
        base += __popc(s_word[w]);
      }
      __syncthreads();
      int* ul = p.ulist + (size_t)j * Imax;
      for (int w = warp; w < W; w += kSelWarps) {
        const uint32_t b = s_word[w];
        if ((b >> lane) & 1u) ul[s_base[w] + __popc(b & lanemask_lt())] = w * 32 + lane;
      }
      if (threadIdx.x == 0) {
        p.ucnt[j] = total;
        p.slot_ticket[j] = 0;
      }
    }
    __syncthreads();  // the next pair reuses the key and chunk buffers
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
  trace_point(p.trace, 2, 7);
}

}  // namespace

// keys [Imax] | kept masks, tie masks [Imax / 32] each
size_t select_smem_bytes(int imax) { return (size_t)imax * 4 + (size_t)(imax / 32) * 8 + 16; }

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
