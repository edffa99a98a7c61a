// select_pair.cuh - the kept set of one (token, expert) pair and its part of the expert's union,
// as a device function for NT cooperating threads (the select kernel's CTA, or the consumer
// warps of the fused layer kernel).
//
// Inside a pair the lowest-scoring neuron activations are dropped ("Uncovering Intra-expert
// Activation Sparsity ...", technical summary, Methodology: activation masking).  The score of
// neuron n is |SiLU(g_n)|, an fp32 value whose bit pattern (sign cleared) orders like the value.
//   top-K mode: an MSB-first radix select (4-bit digits) finds the K-th largest key tau and
//     how many keys equal to tau are kept; the kept set is every key > tau plus the
//     lowest-indexed keys == tau.  No sort.  Once at most 32 keys share the decided prefix,
//     one warp ranks those directly.  The gate's score histogram of the pair decides the top
//     12 bits before the first pass.
//   threshold mode: one pass, keep key > t (the page's single-pass threshold mask).
// The kept set is written as the pair's bitmask row and OR-ed into the expert's union bitmask;
// the last pair of an expert to finish (atomic ticket, no waiting) compacts the union into the
// ascending row list that the up/down step reads, and clears it.
#pragma once

#include "common.cuh"

namespace moe {

// Shared memory of one selection besides the key buffer.
template <int NT>
struct SelShared {
  static constexpr int kW = NT / 32;
  int hist[2 * kW * 8];
  uint32_t cbuf[32];
  int scan[33];
  uint32_t cset[NT];  // the keys left after the histogram, when they fit one per thread
  int ncand, need, eqtot, last, nset;
  uint32_t tau;
};

// Exclusive prefix sum over the NT threads (tid 0 .. NT-1) of the selection, with `bar` as
// the barrier among them; *total gets the sum.
template <int NT, typename Bar>
__device__ __forceinline__ int sel_scan(int v, int* scratch, int* total, int tid, Bar bar) {
  constexpr int nw = NT / 32;
  const int lane = tid & 31, warp = tid >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  bar();
  if (warp == 0) {
    const int s = lane < nw ? scratch[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    if (lane < nw) scratch[lane] = si - s;
    if (lane == 31) scratch[32] = si;
  }
  bar();
  const int res = scratch[warp] + incl - v;
  if (total) *total = scratch[32];
  bar();
  return res;
}

// Bytes of the key buffer of a selection: keys [Imax] | kept masks, tie masks [Imax / 32] each.
__host__ __device__ constexpr size_t sel_key_bytes(int imax) {
  return (size_t)imax * 4 + (size_t)(imax / 32) * 8 + 16;
}

// Selects pair q.  tid in [0, NT); key: the key buffer (sel_key_bytes(Imax)); bar: the barrier
// of the NT threads.  kStaged = false: the pair's activations are read with 16-byte loads through
// L2; kStaged = true: the key buffer already holds them (fp32, the expert's I values) and they
// are turned into keys in place.  Returns the slot j of the pair in *slot_out, and the union size
// when this call compacted the slot's union (the slot's last pair), else -1.  A pair of no slot
// (another handle's expert) does nothing and returns -1 with *slot_out = -1.
struct NoMark {
  __device__ __forceinline__ void operator()(int) const {}
};

// mark(i) is called by every thread at the phase boundaries i = 2 (keys in place), 3 (cut
// found), 4 (kept masks stored), 5 (union bits fenced), 6 (ticket taken), for tracing.
template <int NT, bool kStaged, typename Bar, typename Mark = NoMark>
__device__ int select_pair(const FwdParams& p, int q, int tid, uint32_t* key, SelShared<NT>& ss,
                           Bar bar, bool& nan_seen, int* slot_out, Mark mark = Mark{}) {
  constexpr int kSelThreads = NT, kSelWarps = NT / 32;
  constexpr int kBpt = kHistBins / NT;  // histogram bins per thread (8 or 2)
  static_assert(kBpt == 8 || kBpt == 2, "histogram bins per thread");
  const int lane = tid & 31, warp = tid >> 5;
  const int Imax = p.Imax, Wmax = p.Imax / 32;
  // The first activations are requested before the pair's slot is known (the row is Imax long
  // whatever the expert's I): one round trip instead of three dependent ones.
  const float4* a4 = reinterpret_cast<const float4*>(p.act + (size_t)q * Imax);
  // routed pairs come first (B * k of them), then the shared experts' pairs
  const int kind = q >= p.B * p.k ? 1 : 0;
  const int I = kind ? p.Ish : p.I;
  // top-K with K = 0 or K >= I keeps nothing or everything: the scores are not read (the gate
  // epilogues already flag NaN activations)
  const bool need_keys = p.sel_mode[kind] == 1 || (p.sel_K[kind] > 0 && p.sel_K[kind] < I);
  constexpr int kKeyLoads = 8;  // 16-byte loads in flight per thread
  float4 f[kKeyLoads];
#pragma unroll
  for (int u = 0; u < kKeyLoads; ++u) {
    const int v = tid + u * kSelThreads;
    f[u] = !kStaged && need_keys && v < Imax / 4 ? __ldcg(a4 + v)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // the pair's score histogram (top-K pairs) is requested together with its activations:
  // thread r holds the kBpt bins counted from the top, [kBpt (NT - 1 - r), kBpt (NT - r))
  const bool hist_on = uses_hist(p, kind);
  unsigned hb[kBpt];
  unsigned* hrow = p.hist + (size_t)q * kHistBins;
  const int hb0 = kBpt * (kSelThreads - 1 - tid);
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
  *slot_out = j;
  if (j < 0) return -1;  // an expert another handle evaluates (the same for all NT threads)
  // A slot with one pair: the pair's kept set is the union, compacted straight from the masks in
  // shared memory (no union bitmask, no fence, no ticket).  A slot on the tensor-core path needs
  // no union at all: its GEMMs read the mask rows.
  const int Tj = __ldcg(&p.slots[j].T);
  const bool single = Tj == 1, no_union = Tj >= p.dense_min;
  if (tid == 0) ss.ncand = 0;
  if (!need_keys) {
  } else if constexpr (kStaged) {
    for (int n = tid; n < I; n += kSelThreads) {
      const float a = __uint_as_float(key[n]);
      if (isnan(a)) nan_seen = true;
      key[n] = score_key(a);
    }
  } else {
    for (int v0 = tid;; v0 += kKeyLoads * kSelThreads) {
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
  }
  bar();
  mark(2);
  const int mode = p.sel_mode[kind];
  const int K = min(p.sel_K[kind], I);
  const float thr = p.sel_t[kind];
  const bool radix = mode == 0 && K > 0 && K < I;
  uint32_t tau = 0;
  int need = 0, eqtot = 0;  // keys equal to tau, and how many of them are kept
  if (radix) {
    // MSB-first radix select of the K-th largest key, 4-bit digits.  Each thread counts its
    // keys per digit in packed 16-bit fields, a warp sum merges them, and after one barrier
    // every warp reads the warps' sums and finds the digit itself (the histogram is double
    // buffered, so the next pass can write while a slow warp still reads).  Once at most 32
    // keys share the prefix, one warp ranks them directly.
    uint32_t prefix = 0, pmask = 0;
    int krem = K, cand = I, shift = 28, pass = 0;
    if (hist_on) {
      // The gate counted this pair's keys by their top 12 bits.  An exclusive scan of the
      // threads' bin sums in thread order gives the keys in the bins above each thread's
      // bins, and the thread whose bins hold the K-th largest key names its bin.  The row is
      // cleared for the next call.
#pragma unroll
      for (int i = 0; i < kBpt; ++i) hrow[hb0 + i] = 0;
      int mine = 0;
#pragma unroll
      for (int i = 0; i < kBpt; ++i) mine += (int)hb[i];
      int above = sel_scan<NT>(mine, ss.scan, nullptr, tid, bar);
      if (above < K && above + mine >= K) {
#pragma unroll
        for (int i = kBpt - 1; i >= 0; --i) {
          const int c = (int)hb[i];
          if (above < K && above + c >= K) {
            ss.tau = (uint32_t)(hb0 + i);
            ss.need = K - above;
            ss.eqtot = c;
          }
          above += c;
        }
      }
      bar();
      prefix = ss.tau << kHistShift;
      pmask = ~0u << kHistShift;
      krem = ss.need;
      cand = ss.eqtot;
      shift = kHistShift - 4;
      bar();  // ss.tau and friends are written again below
    }
    // When the histogram leaves at most NT keys (the usual case: a bin of the 2048 holds a few
    // hundred keys at most), they are gathered once, one per thread, and the radix passes below
    // count those instead of scanning every key of the pair again.
    const bool gathered = hist_on && shift >= 0 && cand > 32 && cand <= kSelThreads;
    uint32_t mine_key = 0;
    bool mine_ok = false;
    if (gathered) {
      if (tid == 0) ss.nset = 0;
      bar();
      // each warp counts its hits over its chunks, reserves its range with one atomic, then
      // writes the keys in chunk order (the keys are read twice from shared memory)
      int whits = 0;
      for (int n0 = warp * 32; n0 < I; n0 += kSelThreads) {
        const int n = n0 + lane;
        whits += __popc(__ballot_sync(0xffffffffu, n < I && (key[n] & pmask) == prefix));
      }
      int base = 0;
      if (lane == 0 && whits) base = atomicAdd(&ss.nset, whits);
      base = __shfl_sync(0xffffffffu, base, 0);
      for (int n0 = warp * 32; n0 < I && whits; n0 += kSelThreads) {
        const int n = n0 + lane;
        const uint32_t u = n < I ? key[n] : 0u;
        const bool hit = n < I && (u & pmask) == prefix;
        const unsigned hm = __ballot_sync(0xffffffffu, hit);
        const int at = base + __popc(hm & lanemask_lt());
        if (hit && at < kSelThreads) ss.cset[at] = u;  // at < cand <= NT by construction
        base += __popc(hm);
      }
      bar();
      mine_ok = tid < cand && tid < ss.nset;  // cand == ss.nset by construction
      mine_key = mine_ok ? ss.cset[tid] : 0u;
    }
#pragma unroll 1
    for (; shift >= 0 && cand > 32; shift -= 4, ++pass) {
      uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      auto count = [&](uint32_t u) {
        if ((u & pmask) == prefix) {
          const uint32_t d = (u >> shift) & 15u;
          const uint32_t inc = 1u << ((d & 1u) * 16);
#pragma unroll
          for (int i = 0; i < 8; ++i) c[i] += (d >> 1) == (uint32_t)i ? inc : 0u;
        }
      };
      if (gathered) {
        if (mine_ok) count(mine_key);
      } else {
        for (int n = tid; n < I; n += kSelThreads) count(key[n]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = __reduce_add_sync(0xffffffffu, c[i]);
      int* hbuf = ss.hist + (pass & 1) * (kSelWarps * 8);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) hbuf[warp * 8 + i] = (int)c[i];
      }
      bar();
      // lane l < 16 holds digit 15 - l; a scan over the lanes finds the digit of the K-th key
      int cnt = 0;
      if (lane < 16) {
        const int d = 15 - lane;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w)
          cnt += (int)(((uint32_t)hbuf[w * 8 + (d >> 1)] >> ((d & 1) * 16)) & 0xFFFFu);
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
      auto take = [&](uint32_t u) {
        if ((u & pmask) == prefix) {
          const int slot = atomicAdd(&ss.ncand, 1);  // < cand <= 32 by construction
          if (slot < 32) ss.cbuf[slot] = u;
        }
      };
      if (gathered) {
        if (mine_ok) take(mine_key);
      } else {
        for (int n = tid; n < I; n += kSelThreads) take(key[n]);
      }
      bar();
      if (warp == 0) {
        const bool valid = lane < cand;
        const uint32_t mine = valid ? ss.cbuf[lane] : 0u;
        int gt = 0, ge = 0;
        for (int i = 0; i < cand; ++i) {
          const uint32_t o = __shfl_sync(0xffffffffu, mine, i);
          gt += o > mine;
          ge += o >= mine;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, valid && gt < krem && ge >= krem);
        const int src = __ffs(hit) - 1;
        if (lane == src) {
          ss.tau = mine;
          ss.need = krem - gt;
          ss.eqtot = ge - gt;
        }
      }
      bar();
      tau = ss.tau;
      need = ss.need;
      eqtot = ss.eqtot;
    }
  }
  mark(3);
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
      const uint32_t u = need_keys ? key[32 * c + lane] : 0u;
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
    bar();
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
  bar();
  for (int c = tid; c < nch; c += kSelThreads) {
    const uint32_t km = s_km[c];
    mrow[c] = km;
    if (km && !single && !no_union) red_or(&urow[c], km);
  }
  mark(4);
  if (no_union) {
    bar();  // the next pair reuses the key and chunk buffers
    return -1;
  }
  if (!single) {
    // the last pair of an expert to finish compacts the expert's union (atomic ticket, no
    // waiting): every pair's union bits are published before its ticket
    __threadfence();
    bar();
    mark(5);
    if (tid == 0) {
      const unsigned ticket = atomicAdd(&p.slot_ticket[j], 1u);
      ss.last = ticket == (unsigned)__ldcg(&p.slots[j].T) - 1u;
    }
  } else if (tid == 0) {
    ss.last = 1;
  }
  bar();
  mark(6);
  int result = -1;
  if (ss.last) {
    // All NT threads compact the union bitmask into the ascending row list and clear it:
    // thread t owns the words [t wpt, (t + 1) wpt), a scan of their bit counts gives each
    // word's first list position, and then each warp writes one word per step, lane l placing
    // bit l at its rank among the word's set bits.
    if (!single) __threadfence();
    const int W = I / 32, wpt = (W + kSelThreads - 1) / kSelThreads;
    uint32_t* s_word = key;                                // [W] union words (keys are done)
    int* s_base = reinterpret_cast<int*>(key + Imax / 2);  // [W] first position of each word
    const int wb = min(W, tid * wpt), we = min(W, wb + wpt);
    int c = 0;
    for (int w = wb; w < we; ++w) {
      uint32_t b;
      if (single) {
        b = s_km[w];
      } else {
        b = __ldcg(&urow[w]);
        urow[w] = 0;
      }
      s_word[w] = b;
      c += __popc(b);
    }
    int total;
    int base = sel_scan<NT>(c, ss.scan, &total, tid, bar);
    for (int w = wb; w < we; ++w) {
      s_base[w] = base;
      base += __popc(s_word[w]);
    }
    bar();
    int* ul = p.ulist + (size_t)j * Imax;
    for (int w = warp; w < W; w += kSelWarps) {
      const uint32_t b = s_word[w];
      if ((b >> lane) & 1u) ul[s_base[w] + __popc(b & lanemask_lt())] = w * 32 + lane;
    }
    if (tid == 0) {
      p.ucnt[j] = total;
      if (!single) p.slot_ticket[j] = 0;
    }
    result = total;
  }
  bar();  // the next pair reuses the key and chunk buffers
  return result;
}

}  // namespace moe
