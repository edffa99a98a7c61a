// gate.cu - dense gate projection + SiLU of every evaluated (token, expert) pair.
//
// The gate is the part of an expert that cannot be skipped: it is what scores the neurons
// ("Uncovering Intra-expert Activation Sparsity ...", technical summary, Methodology: the gate
// projection runs densely to determine the activation scores).  Every evaluated expert's gate
// block [I][H] is read from HBM once per tile of 8 of its tokens.
//
// Work item = (slot, token tile of 8 pairs, group of 16 neurons), ordered slot, token tile,
// neuron group; each CTA takes a contiguous range of items.  Output act[q][n] = SiLU(g) in fp32.
//
// bf16: one persistent CTA per SM with three roles.
//   meta warp    walks the items ahead of the others (at most kMetaRing): resolves each item's
//                rows and tokens into a small shared-memory ring;
//   copier warp  streams the item's 16 gate rows, kc columns at a time, into a ring of
//                shared-memory stages (one bulk asynchronous copy per row piece, completed on an
//                mbarrier);
//   8 consumer warps  split each stage's columns, multiply on the tensor cores against the
//                token tile, and sum their partial 16x8 tiles at the end of the item.
// Consumers issue no global load except their token fragments when the token tile changes.
// Template <NK, BPW>: the row is NK stages of kc = H/NK columns and warp w always takes the
// column blocks w, w+8, ... (at most BPW per stage), so its token fragments stay in registers and
// the whole shared memory goes to the ring.  NK = 0 is the generic variant for other H: the token
// tile is bulk-copied into (double-buffered) shared memory by the meta warp.
// Bulk copies of a few kilobytes per row piece reach the HBM copy rate; 1 KB copies reach about
// half of it, which is why the pieces are as wide as shared memory allows.
// fp32: a plain CUDA-core variant (register loads, same fragment layout).
#include "kernels.h"
#include "tile.cuh"
#include "tma.cuh"

namespace moe {
namespace {

constexpr int kRingThreads = kThreads + 64;  // 8 consumer warps, copier, meta
constexpr int kCopier = kWarps, kMetaWarp = kWarps + 1;

struct GateMeta {
  const __nv_bfloat16* rows;  // first of the item's 16 consecutive gate rows
  int q0;                     // pair index of the tile's first token
  int nt;                     // valid tokens in the tile (1..8)
  int n0;                     // first neuron
  int key;                    // token tile id (slot * 1024 + tile)
  int xb, xpar, xlast;        // generic variant: token tile buffer, fill phase, last user
  int end;                    // 1: no more items (the CTA's loops end here)
  int tok[kTileTok];          // register variant: token of each tile column (-1 past the end)
};

constexpr int kGateChunk = 2;  // items claimed at a time from the work counter

template <int NK, int BPW>
__global__ void __launch_bounds__(kRingThreads, 1) gate_tma_kernel(FwdParams p, Ring rc) {
  constexpr bool kReg = NK > 0;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int4 s_tab[kMaxSlots];
  __shared__ GateMeta s_meta[kMetaRing];
  __shared__ int s_abort;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + rc.ns;
  uint64_t* mfull = empty + rc.ns;
  uint64_t* mempty = mfull + kMetaRing;
  uint64_t* xfull = mempty + kMetaRing;
  uint64_t* xempty = xfull + 2;
  uint64_t* mrows = xempty + 2;  // the record's row pointer is written (all the copier needs)
  float(*red)[kWarps][4][32] = reinterpret_cast<float(*)[kWarps][4][32]>(smem + kBarBytes);
  unsigned char* xbuf = smem + kBarBytes + kRedBytes;
  unsigned char* ring = xbuf + rc.nxb * rc.xs_bytes;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  trace_point(p.trace, 1, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < rc.ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    for (int i = 0; i < kMetaRing; ++i) {
      mbar_init(&mfull[i], 1);
      mbar_init(&mempty[i], kWarps + 1);
      mbar_init(&mrows[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], kWarps);
    }
    s_abort = 0;
    mbar_init_fence();
  }
  for (int i = threadIdx.x; i < kMetaRing * (int)(sizeof(GateMeta) / 4); i += blockDim.x)
    reinterpret_cast<int*>(s_meta)[i] = 0;  // pointers become null, tokens 0
  pdl_trigger();
  __syncthreads();
  const int H = p.H;
  volatile int* abort = &s_abort;

  if (warp == kMetaWarp) {
    // ---------------- meta: claims items and publishes their records: the row pointer for the
    // copier (mrows), then the tokens for the consumers (mfull); it also fills the token tiles
    // of the generic variant.  A record with end = 1 closes the stream.
    // Items come in two spaces.  First the shared experts' items, which need no routing (shared
    // expert s evaluates every token: token t is pair B k + s B + t), claimed a few at a time
    // from a counter while the router may still run.  Then, after the wait for the router, the
    // routed items: a contiguous share of 7/8 of them per CTA (token tiles stay together), the
    // rest from a second counter in small chunks, so that fast CTAs take more of the tail.
    // Only this warp reads what the router wrote, so only it waits.
    int xuse[2] = {0, 0};
    const int Bt = (p.B + kTileTok - 1) / kTileTok;
    const int sh_groups = p.Ish / kTileRows;
    const bool sh_sparse = p.S > 0 && p.B < p.dense_min;
    const int n_pre = sh_sparse ? __popc(p.shared_mask) * sh_groups * Bt : 0;
    int n_slots = 0, n_items = n_pre, share = 0, dyn0 = 0;
    bool routed_known = false;
    int cb = 0, ce = 0;
    auto learn_routing = [&]() {
      pdl_wait();
      if (p.trace && lane == 0 && blockIdx.x < kTraceCtas)
        const_cast<unsigned long long*>(p.trace)[((size_t)1 * kTraceCtas + blockIdx.x) *
                                                     kTracePoints + 1] = globaltimer();
      // the slot count and every slot entry that can exist (E + S) in one round trip; entries
      // at n_slots and beyond are stale and never searched
      n_slots = ld_cg(&p.meta[kMetaSlots]);
      const int n_routed = ld_cg(&p.meta[kMetaGateItems]) - n_pre;
      for (int j = lane; j < min(slot_capacity(p.E, p.S), kMaxSlots); j += 32) {
        const Slot sl = load_slot(&p.slots[j]);
        s_tab[j] = make_int4(sl.expert | (sl.kind << 16), sl.T, sl.q0, sl.item0);
      }
      __syncwarp();
      share = n_routed * 7 / 8 / (int)gridDim.x;
      dyn0 = share * (int)gridDim.x;
      cb = n_pre + blockIdx.x * share;
      ce = cb + share;
      n_items = n_pre + n_routed;
      routed_known = true;
    };
    int pre_next = 0, pre_end = 0;
    auto claim = [&]() -> int {
      if (!routed_known) {
        if (pre_next >= pre_end) {
          int b = 0;
          if (lane == 0 && n_pre > 0) b = (int)atomicAdd(&p.claim[2], (unsigned)kGateChunk);
          b = __shfl_sync(0xffffffffu, b, 0);
          if (n_pre > 0 && b < n_pre) {
            pre_next = b;
            pre_end = min(b + kGateChunk, n_pre);
          } else {
            learn_routing();
          }
        }
        if (!routed_known) return pre_next++;
      }
      if (cb >= ce) {
        int b = 0;
        if (lane == 0) b = dyn0 + (int)atomicAdd(&p.claim[0], (unsigned)kGateChunk);
        b = __shfl_sync(0xffffffffu, b, 0) + n_pre;
        if (b >= n_items) {
          cb = ce = n_items;
          return -1;
        }
        cb = b;
        ce = min(b + kGateChunk, n_items);
      }
      return cb++;
    };
    // An item's place: slot entry {expert | kind << 16, T, q0, first item} and its local index
    // within that slot's items.  Shared items carry the local shared expert's entry directly.
    struct Place {
      int4 sl;
      int local, key;
    };
    auto place = [&](int item) -> Place {
      Place pl;
      if (item < n_pre) {
        const int o = item / (sh_groups * Bt);  // o-th shared expert of this handle
        unsigned m = p.shared_mask;
        for (int i = 0; i < o; ++i) m &= m - 1;
        const int s_i = __ffs(m) - 1;
        pl.sl = make_int4(s_i | (1 << 16), p.B, p.B * p.k + s_i * p.B, 0);
        pl.local = item - o * sh_groups * Bt;
        pl.key = (1 << 20) + s_i * 1024 + pl.local / sh_groups;
      } else {
        const int r = item - n_pre;
        const int j = find_item_slot(s_tab, n_slots, r);
        pl.sl = s_tab[j];
        pl.local = r - pl.sl.w;
        const int I = (pl.sl.x >> 16) ? p.Ish : p.I;
        pl.key = j * 1024 + pl.local / (I / kTileRows);
      }
      return pl;
    };
    int key = -1, xb = rc.nxb - 1, tok_l = -1, mi = 0;
    int cur = claim();
    Place cpl = cur >= 0 ? place(cur) : Place{};
    for (; cur >= 0 && !*abort; ++mi) {
      const int nxt = claim();
      const Place npl = nxt >= 0 ? place(nxt) : Place{};
      const int cur_key = cpl.key, nxt_key = nxt >= 0 ? npl.key : -1;
      const int m = mi % kMetaRing;
      if (!mbar_wait(&mempty[m], ((mi / kMetaRing) & 1) ^ 1, abort, p.err)) break;
      const int4 sl = cpl.sl;
      const int kind = sl.x >> 16, ex = sl.x & 0xffff, T = sl.y, q0 = sl.z;
      const int I = kind ? p.Ish : p.I;
      const int local = cpl.local, tt = local / (I / kTileRows), rg = local % (I / kTileRows);
      const int nt = min(kTileTok, T - tt * kTileTok);
      if (lane == 0) {  // the copier's part first: it needs no token
        const __nv_bfloat16* base =
            kind == 0 ? static_cast<const __nv_bfloat16*>(p.gate_r) + (size_t)ex * p.I * H
                      : static_cast<const __nv_bfloat16*>(p.gate_s) + (size_t)ex * p.Ish * H;
        s_meta[m].rows = base + (size_t)rg * kTileRows * H;
        s_meta[m].q0 = q0 + tt * kTileTok;
        s_meta[m].nt = nt;
        s_meta[m].n0 = rg * kTileRows;
        s_meta[m].key = cur_key;
        s_meta[m].end = 0;
        mbar_arrive(&mrows[m]);
      }
      int xpar = 0;
      if (cur_key != key) {
        key = cur_key;
        // a shared expert's pair q0 + i is token i; a routed pair's token is in the pair table
        tok_l = lane >= nt ? -1
                : kind ? tt * kTileTok + lane
                       : __ldcg(&p.pair_token[q0 + tt * kTileTok + lane]);
        if constexpr (!kReg) {
          xb = (xb + 1) % rc.nxb;
          if (!mbar_wait(&xempty[xb], (xuse[xb] & 1) ^ 1, abort, p.err)) break;
          xpar = xuse[xb] & 1;
          xuse[xb]++;
          if (lane == 0) mbar_arrive_expect_tx(&xfull[xb], kTileTok * H * 2);
          __syncwarp();
          if (lane < kTileTok) {
            const void* src = tok_l >= 0 ? static_cast<const void*>(
                                               static_cast<const __nv_bfloat16*>(p.x) +
                                               (size_t)tok_l * H)
                                         : p.zero_row;
            bulk_g2s(xbuf + xb * rc.xs_bytes + lane * rc.xs_stride, src, H * 2, &xfull[xb]);
          }
        }
      } else if constexpr (!kReg) {
        xpar = (xuse[xb] - 1) & 1;
      }
      if (lane < kTileTok) s_meta[m].tok[lane] = tok_l;
      if (lane == 0) {
        s_meta[m].xb = xb;
        s_meta[m].xpar = xpar;
        s_meta[m].xlast = nxt_key != key;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&mfull[m]);
      cur = nxt;
      cpl = npl;
    }
    if (!routed_known) learn_routing();  // every CTA waits for the router before it exits
    {  // closing record
      const int m = mi % kMetaRing;
      mbar_wait(&mempty[m], ((mi / kMetaRing) & 1) ^ 1, abort, p.err);
      if (lane == 0) {
        s_meta[m].end = 1;
        mbar_arrive(&mrows[m]);
        mbar_arrive(&mfull[m]);
      }
    }
    // no token-tile copy may still be landing in shared memory when the CTA exits
    for (int b = 0; b < rc.nxb; ++b)
      if (xuse[b] > 0) mbar_drain(&xfull[b], (xuse[b] - 1) & 1);
    return;
  }

  if (warp == kCopier) {
    // ---------------- copier: the item's 16 rows, kc columns per stage, one bulk copy per row
    const uint32_t piece = rc.kc * 2;
    int it = 0;
    for (int mi = 0; !*abort; ++mi) {
      const int m = mi % kMetaRing;
      if (!mbar_wait(&mrows[m], (mi / kMetaRing) & 1, abort, p.err)) break;
      if (s_meta[m].end) break;
      const __nv_bfloat16* row = s_meta[m].rows + (size_t)(lane & 15) * H;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mempty[m]);
      for (int kc = 0; kc < rc.nk; ++kc, ++it) {
        const int st = it % rc.ns;
        if (!mbar_wait(&empty[st], ((it / rc.ns) & 1) ^ 1, abort, p.err)) break;
        if (lane == 0) mbar_arrive_expect_tx(&full[st], kTileRows * piece);
        __syncwarp();
        if (lane < kTileRows)
          bulk_g2s(ring + (size_t)st * rc.stage_bytes + lane * rc.rs_a, row + kc * rc.kc, piece,
                   &full[st]);
      }
    }
    for (int k = it - 1; k >= 0 && k >= it - rc.ns; --k) mbar_drain(&full[k % rc.ns], (k / rc.ns) & 1);
    return;
  }

  // ---------------- consumers
  constexpr int kXR = kReg ? NK : 1, kXB = kReg ? BPW : 1;
  uint4 xr[kXR][kXB];
  int it = 0, ib = 0, cur = -1;
  bool nan_seen = false;
  const int nblk = rc.kc / 32;
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  for (int mi = 0;; ++mi) {
    const int m = mi % kMetaRing;
    mbar_wait(&mfull[m], (mi / kMetaRing) & 1, abort, p.err);
    // the end (or an abort) is decided by all consumer warps together
    if (consumer_sync_or(kThreads, s_meta[m].end || *abort)) {
      trace_value(p.trace, 1, 5, (unsigned long long)mi);
      break;
    }
    if (mi == 0) trace_point(p.trace, 1, 2);
    trace_point(p.trace, 1, 6);
    const int q0 = s_meta[m].q0, nt = s_meta[m].nt, n0 = s_meta[m].n0, key = s_meta[m].key;
    const int xb = min(max(s_meta[m].xb, 0), max(rc.nxb - 1, 0));  // trusted only w/o abort
    const int xlast = s_meta[m].xlast;
    const unsigned char* xrow = xbuf + xb * rc.xs_bytes + g * rc.xs_stride;
    if constexpr (kReg) {
      if (key != cur) {  // this warp's token fragments for the new tile (one round trip)
        cur = key;
        const int tok = s_meta[m].tok[g];
#pragma unroll
        for (int kc = 0; kc < kXR; ++kc)
#pragma unroll
          for (int i = 0; i < kXB; ++i) {
            const int b = warp + kWarps * i;
            xr[kc][i] = (b < nblk && tok >= 0)
                            ? ld_nc(x + (size_t)tok * H + kc * rc.kc + b * 32 + t * 8)
                            : make_uint4(0, 0, 0, 0);
          }
      }
    } else {
      mbar_wait(&xfull[xb], s_meta[m].xpar, abort, p.err);
    }
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (kReg) {
#pragma unroll
      for (int kc = 0; kc < kXR; ++kc, ++it) {
        const int st = it % rc.ns;
        mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
        if (it == 0) trace_point(p.trace, 1, 3);
        const unsigned char* stage = ring + (size_t)st * rc.stage_bytes;
#pragma unroll
        for (int i = 0; i < kXB; ++i) {
          const int b = warp + kWarps * i;
          if (b < nblk) {
            const int col = (b * 32 + t * 8) * 2;
            const uint4 a0 = lds128(stage + g * rc.rs_a + col);
            const uint4 a1 = lds128(stage + (g + 8) * rc.rs_a + col);
            const uint4 xv = xr[kc][i];
            mma_16816(d, a0.x, a1.x, a0.y, a1.y, xv.x, xv.y);
            mma_16816(d, a0.z, a1.z, a0.w, a1.w, xv.z, xv.w);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
    } else {
      for (int kc = 0; kc < rc.nk; ++kc, ++it) {
        const int st = it % rc.ns;
        mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
        const unsigned char* stage = ring + (size_t)st * rc.stage_bytes;
        for (int b = warp; b < nblk; b += kWarps) {
          const int col = (b * 32 + t * 8) * 2;
          const uint4 a0 = lds128(stage + g * rc.rs_a + col);
          const uint4 a1 = lds128(stage + (g + 8) * rc.rs_a + col);
          const uint4 xv = lds128(xrow + kc * rc.kc * 2 + col);
          mma_16816(d, a0.x, a1.x, a0.y, a1.y, xv.x, xv.y);
          mma_16816(d, a0.z, a1.z, a0.w, a1.w, xv.z, xv.w);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
    }
    if (lane == 0) {
      mbar_arrive(&mempty[m]);
      if (!kReg && xlast) mbar_arrive(&xempty[xb]);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) red[ib][warp][c][lane] = d[c];
    const int aborted = consumer_sync_or(kThreads, *abort);
    if (threadIdx.x < 128 && !aborted) {
      // one output per thread: fragment element (c, lane), summed over the warps in order
      const int ln = threadIdx.x & 31, c = threadIdx.x >> 5;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[ib][w][c][ln];
      const int ti = 2 * (ln & 3) + (c & 1);
      if (ti < nt) {
        const float a = silu(v);
        nan_seen |= isnan(a);
        p.act[(size_t)(q0 + ti) * p.Imax + n0 + (ln >> 2) + (c >> 1) * 8] = a;
        if (uses_hist(p, q0 >= p.B * p.k)) hist_add(p, q0 + ti, a);
      }
    }
    if (mi == 0) trace_point(p.trace, 1, 4);
    ib ^= 1;
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
  trace_point(p.trace, 1, 7);
}

// fp32 variant: register loads, 8 warps split H, same items.
__global__ void __launch_bounds__(kThreads) gate_f32_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ int4 s_tab[kMaxSlots];
  __shared__ const float* s_x[kTileTok];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, Imax = p.Imax;
  const int n_slots = ld_cg(&p.meta[kMetaSlots]);
  const int n_items = ld_cg(&p.meta[kMetaGateItems]);
  load_slot_table(p, n_slots, s_tab);
  __syncthreads();
  const float* x = static_cast<const float*>(p.x);
  bool nan_seen = false;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int j = find_item_slot(s_tab, n_slots, item);
    const int4 sl = s_tab[j];
    const int kind = sl.x >> 16, ex = sl.x & 0xffff, T = sl.y, q0 = sl.z;
    const int I = kind ? p.Ish : p.I;
    const int local = item - sl.w, tt = local / (I / kTileRows), rg = local % (I / kTileRows);
    if (threadIdx.x < kTileTok) {
      const int ti = tt * kTileTok + threadIdx.x;
      s_x[threadIdx.x] = ti < T ? x + (size_t)__ldcg(&p.pair_token[q0 + ti]) * H : nullptr;
    }
    __syncthreads();
    const float* base = kind == 0 ? static_cast<const float*>(p.gate_r) + (size_t)ex * p.I * H
                                  : static_cast<const float*>(p.gate_s) + (size_t)ex * p.Ish * H;
    const int n0 = rg * kTileRows;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    tile_dot<1>(base + (size_t)(n0 + g) * H, base + (size_t)(n0 + g + 8) * H, s_x, warp, kWarps,
                H / 32, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
    __syncthreads();
    if (warp == 0) {
      reduce_fragments(red, d);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int ti = tt * kTileTok + 2 * t + (c & 1);
        if (ti < T) {
          const float a = silu(d[c]);
          nan_seen |= isnan(a);
          p.act[(size_t)(q0 + ti) * Imax + n0 + g + (c >> 1) * 8] = a;
          if (uses_hist(p, kind)) hist_add(p, q0 + ti, a);
        }
      }
    }
    __syncthreads();
  }
  if (nan_seen) set_error(p.err, kErrNanAct);
}

template <int NK, int BPW>
cudaError_t set_gate_smem(int budget) {
  return allow_max_smem(gate_tma_kernel<NK, BPW>, budget);
}

template <int NK, int BPW>
int gate_static_smem() {
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, gate_tma_kernel<NK, BPW>) == cudaSuccess
             ? (int)fa.sharedSizeBytes
             : 16384;
}

}  // namespace

// Register-fragment variants, by hidden size: {H, NK, BPW}.  H = NK stages of kc columns, and
// each of the 8 warps takes at most BPW 32-column blocks of a stage.
extern const int kRegVariants[4][3];
const int kRegVariants[4][3] = {{512, 1, 2}, {2048, 1, 8}, {2880, 3, 4}, {5120, 4, 5}};

int ring_variant(int H) {
  for (int v = 0; v < 4; ++v)
    if (kRegVariants[v][0] == H) return v + 1;
  return 0;
}

// Copy-ring shape.  Register variant (nk_fixed > 0): the whole budget goes to stages of kc =
// H/nk_fixed.  Generic variant (nk_fixed = 0): the widest row pieces (kc a multiple of 64
// dividing H) that still leave two stages next to two token tiles (or one).
Ring make_ring(int H, int nk_fixed, int smem_budget, int static_smem) {
  const int avail = smem_budget - static_smem - kBarBytes - kRedBytes;
  for (int nk = nk_fixed ? nk_fixed : 1; nk <= H / 64; ++nk) {
    if (H % nk || (H / nk) % 64) {
      if (nk_fixed) break;
      continue;
    }
    Ring r;
    r.nk = nk;
    r.kc = H / nk;
    r.rs_a = r.kc * 2 + 64;
    r.rs_d = r.kc * 2 + 16;
    r.stage_bytes = kTileRows * r.rs_a;
    r.xs_stride = H * 2 + 64;
    r.xs_bytes = kTileTok * r.xs_stride;
    for (int nxb = nk_fixed ? 0 : 2; nxb >= (nk_fixed ? 0 : 1); --nxb) {
      int ns = (avail - nxb * r.xs_bytes) / r.stage_bytes;
      if (ns > 16) ns = 16;
      if (ns >= 2) {
        r.nxb = nxb;
        r.ns = ns;
        r.smem_bytes = kBarBytes + kRedBytes + nxb * r.xs_bytes + ns * r.stage_bytes;
        return r;
      }
    }
    if (nk_fixed) break;
  }
  Ring none{};
  none.ns = 0;
  return none;
}

cudaError_t launch_gate(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                        bool pdl) {
  if (dtype != 0)
    return launch_pdl(gate_f32_kernel, dim3(ls.grid_gate), dim3(kThreads), 0, st, pdl, p);
  const Ring& r = ls.ring_gate;
  const dim3 grid(ls.nsm), block(kRingThreads);
  switch (ls.variant) {
    case 1: return launch_pdl(gate_tma_kernel<1, 2>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 2: return launch_pdl(gate_tma_kernel<1, 8>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 3: return launch_pdl(gate_tma_kernel<3, 4>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 4: return launch_pdl(gate_tma_kernel<4, 5>, grid, block, r.smem_bytes, st, pdl, p, r);
    default: return launch_pdl(gate_tma_kernel<0, 0>, grid, block, r.smem_bytes, st, pdl, p, r);
  }
}

cudaError_t configure_gate(int dtype, int H, int smem_budget, LaunchShape* ls) {
  if (dtype != 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gate_f32_kernel, kThreads, 0);
    ls->grid_gate = ls->nsm * (n > 0 ? n : 1);
    return e;
  }
  ls->variant = ring_variant(H);
  const int nk = ls->variant ? kRegVariants[ls->variant - 1][1] : 0;
  int stat = 0;
  switch (ls->variant) {
    case 1: stat = gate_static_smem<1, 2>(); break;
    case 2: stat = gate_static_smem<1, 8>(); break;
    case 3: stat = gate_static_smem<3, 4>(); break;
    case 4: stat = gate_static_smem<4, 5>(); break;
    default: stat = gate_static_smem<0, 0>(); break;
  }
  ls->ring_gate = make_ring(H, nk, smem_budget, stat + 1024);
  if (ls->ring_gate.ns < 2) return cudaErrorInvalidConfiguration;
  ls->grid_gate = ls->nsm;
  switch (ls->variant) {
    case 1: return set_gate_smem<1, 2>(smem_budget);
    case 2: return set_gate_smem<1, 8>(smem_budget);
    case 3: return set_gate_smem<3, 4>(smem_budget);
    case 4: return set_gate_smem<4, 5>(smem_budget);
    default: return set_gate_smem<0, 0>(smem_budget);
  }
}

}  // namespace moe
