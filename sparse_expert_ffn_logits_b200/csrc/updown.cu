// updown.cu - fused sparse up/down projection over the kept neurons, weighted into the output.
//
// Only the weights of active neurons are read ("Uncovering Intra-expert Activation Sparsity
// ...", technical summary, Methodology: fused up-down projection).  The packed layout keeps a
// neuron's W_up row and W_down column side by side ([I][2][H]), so the rows of the expert's
// kept-neuron union are gathered as contiguous pieces and a dropped neuron costs no bytes.
// Each row is read once per token tile of its expert; tokens of the tile whose own kept set
// lacks the neuron get coefficient 0.
//
// Work item = (slot, token tile of 8 pairs, 16 union rows), ordered slot, token tile, rows;
// each CTA takes a contiguous share of the items, then claims the rest one at a time from a
// counter.  Per item:
//   1. u[r][c] = W_up[n_r] . x_c           tensor cores, warps split H
//   2. hc[r][c] = mask * SiLU(g) * u        fp32, rounded to bf16 for the tensor cores
//   3. y[h][c] = sum_r W_down[h][n_r] hc    tensor cores, 64 h per warp step
//   4. out_acc[token][h] += w_c * y         fp32 vector reductions in L2
// bf16: one persistent CTA per SM; a producer warp gathers the 16 rows' up pieces, then their
// down pieces, through a ring of shared-memory stages (bulk asynchronous copies, mbarriers);
// eight consumer warps compute.  fp32: a plain CUDA-core variant with register loads.
#include "kernels.h"
#include "tile.cuh"
#include "tma.cuh"

namespace moe {
namespace {

// 8 consumer warps, the copier, the lead meta warp (token tiles) and kCoefWarps coefficient
// warps that fill alternate item records in parallel (each record costs two dependent L2 reads)
constexpr int kCoefWarps = 2;
constexpr int kRingThreads = kThreads + 64 + 32 * kCoefWarps;
constexpr int kCopier = kWarps, kMetaWarp = kWarps + 1, kCoefWarp0 = kWarps + 2;

// Items per slot = ceil(union rows / 16) * token tiles; exclusive prefix into s_item0[0..n],
// with s_item0[n_slots] = total.  Whole block.
__device__ int updown_items(const FwdParams& p, int n_slots, int* s_item0, int* scratch) {
  const int per = (n_slots + blockDim.x - 1) / blockDim.x;
  const int b0 = min(n_slots, (int)threadIdx.x * per), b1 = min(n_slots, b0 + per);
  int c = 0;
  for (int j = b0; j < b1; ++j) {
    const int rows = __ldcg(&p.ucnt[j]);
    const int T = __ldcg(&p.slots[j].T);
    const int v = ((rows + kTileRows - 1) / kTileRows) * ((T + kTileTok - 1) / kTileTok);
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
  return s_item0[n_slots];
}

struct UdPos {
  int j, tt, rg, rows;
};

__device__ __forceinline__ UdPos decode_ud_item(const FwdParams& p, const int* s_item0,
                                                int n_slots, int item) {
  UdPos u;
  u.j = find_slot(s_item0, n_slots, item);
  u.rows = __ldcg(&p.ucnt[u.j]);
  const int nrg = (u.rows + kTileRows - 1) / kTileRows;
  const int local = item - s_item0[u.j];
  u.tt = local / nrg;
  u.rg = local % nrg;
  return u;
}

__device__ __forceinline__ int union_row(const FwdParams& p, const UdPos& u, int r) {
  const int idx = u.rg * kTileRows + r;
  return __ldcg(&p.ulist[(size_t)u.j * p.Imax + (idx < u.rows ? idx : u.rg * kTileRows)]);
}

struct UdMeta {
  const __nv_bfloat16* ud;  // the expert's packed [I][2][H] block
  int rows[kTileRows];      // union neuron of each row (a repeated valid row past the end)
  float coef[kTileRows][kTileTok];  // SiLU(g) if the row is kept by the token's pair, else 0
  int tok[kTileTok];        // token of each tile column (-1 past the end)
  float w[kTileTok];        // routing weight of each tile column
  int key;                  // token tile id (slot * 1024 + tile)
  int xb, xpar, xlast;      // generic variant: token tile buffer, fill phase, last user
  int j, tt, rg;            // the item: slot, token tile, row group (for the coefficient warps)
  int end;                  // 1: no more items (the CTA's loops end here)
};

constexpr int kUdChunk = 1;  // items claimed at a time from the work counter

template <int NK, int BPW>
__global__ void __launch_bounds__(kRingThreads, 1) updown_tma_kernel(FwdParams p, Ring rc) {
  constexpr bool kReg = NK > 0;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int4 s_tab[kMaxSlots];  // {expert | kind << 16, T, q0, first up/down item}
  __shared__ int s_ucnt[kMaxSlots];
  __shared__ int scratch[33];
  __shared__ int s_total;
  __shared__ int s_abort;
  __shared__ UdMeta s_meta[kMetaRing];
  __shared__ __align__(16) uint32_t s_hcw[2][kTileTok][kTileRows / 2];
  __shared__ uint32_t s_tmem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + rc.ns;
  uint64_t* mfull = empty + rc.ns;
  uint64_t* mempty = mfull + kMetaRing;
  uint64_t* xfull = mempty + kMetaRing;
  uint64_t* xempty = xfull + 2;
  uint64_t* mhead = xempty + 2;  // the lead warp has written the record's item
  uint64_t* mrows = mhead + kMetaRing;  // the record's rows are written (all the copier needs)
  float(*red)[kWarps][4][32] = reinterpret_cast<float(*)[kWarps][4][32]>(smem + kBarBytes);
  unsigned char* xbuf = smem + kBarBytes + kRedBytes;
  unsigned char* ring = xbuf + rc.nxb * rc.xs_bytes;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  trace_point(p.trace, 3, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < rc.ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    for (int i = 0; i < kMetaRing; ++i) {
      mbar_init(&mfull[i], 2);  // lead meta warp + the coefficient warp of that record
      mbar_init(&mempty[i], kWarps + 1);
      mbar_init(&mhead[i], 1);
      mbar_init(&mrows[i], 2);  // lead meta warp + the coefficient warp of that record
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], kWarps);
    }
    s_abort = 0;
    mbar_init_fence();
  }
  for (int i = threadIdx.x; i < kMetaRing * (int)(sizeof(UdMeta) / 4); i += blockDim.x)
    reinterpret_cast<int*>(s_meta)[i] = 0;
  // Down-projection accumulators in tensor memory: consumer warp w keeps the 16 values of each
  // of its 64-column sub-chunks (spw per stage, nk stages) in lane quarter w % 4, columns
  // 256 (w / 4) + 16 (kc spw + local sub-chunk), while consecutive items of one (expert, token
  // tile) follow each other, and flushes them to the output accumulator once per such run.
  // Hidden sizes that would need more than 256 columns per warp group reduce every item.
  const int spw = (rc.kc / 64 + kWarps - 1) / kWarps;
  const bool tmem_acc = rc.nk * spw * 16 <= 256;
  if (tmem_acc && warp == 0) tmem_alloc(&s_tmem, 512);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = tmem_acc ? s_tmem : 0u;
  pdl_trigger();
  pdl_wait();
  trace_point(p.trace, 3, 1);
  const int n_slots = ld_cg(&p.meta[kMetaSlots]);
  {
    // items per slot = ceil(union rows / 16) * token tiles; exclusive prefix into s_tab[].w.
    // Every slot entry that can exist (E + S) is read together with the slot count (one round
    // trip); entries at n_slots and beyond count as empty.
    const int n_max = min(slot_capacity(p.E, p.S), kMaxSlots);
    const int per = (n_max + blockDim.x - 1) / blockDim.x;
    const int b0 = min(n_max, (int)threadIdx.x * per), b1 = min(n_max, b0 + per);
    int c = 0;
    for (int j = b0; j < b1; ++j) {
      const Slot sl = load_slot(&p.slots[j]);
      const int rows_any = __ldcg(&p.ucnt[j]);  // issued before n_slots is known
      const int rows = j < n_slots && sl.T < p.dense_min ? rows_any : 0;  // dense: not here
      s_ucnt[j] = rows;
      const int v = ((rows + kTileRows - 1) / kTileRows) * ((sl.T + kTileTok - 1) / kTileTok);
      s_tab[j] = make_int4(sl.expert | (sl.kind << 16), sl.T, sl.q0, v);
      c += v;
    }
    int total;
    int run = block_exclusive_scan(c, scratch, &total);
    for (int j = b0; j < b1; ++j) {
      const int v = s_tab[j].w;
      s_tab[j].w = run;
      run += v;
    }
    if (threadIdx.x == 0) s_total = total;
    __syncthreads();
  }
  const int n_items = s_total;
  const int H = p.H, Imax = p.Imax, Wmax = p.Imax / 32;
  volatile int* abort = &s_abort;

  if (warp == kMetaWarp) {
    // ---------------- lead meta warp: claims items (its own contiguous share of 3/4 of them
    // first, then one at a time from the work counter, so that fast CTAs take more of the tail),
    // owns the token tiles and the record fields ud, key, xb, xpar, xlast; publishes the item
    // (mhead) for the coefficient warp of the record.  Two records with end = 1 close the
    // stream: one for the copier and consumers, one more so that both coefficient warps see it.
    int xuse[2] = {0, 0};
    const int share = n_items * 3 / 4 / (int)gridDim.x;
    const int dyn0 = share * (int)gridDim.x;
    int cb = blockIdx.x * share, ce = cb + share;
    auto claim = [&]() -> int {
      if (cb >= ce) {
        int b = 0;
        if (lane == 0) b = dyn0 + (int)atomicAdd(&p.claim[1], (unsigned)kUdChunk);
        b = __shfl_sync(0xffffffffu, b, 0);
        if (b >= n_items) {
          cb = ce = n_items;
          return -1;
        }
        cb = b;
        ce = min(b + kUdChunk, n_items);
      }
      return cb++;
    };
    struct Pos {
      int j, tt, rg;
    };
    auto decode = [&](int item) -> Pos {
      Pos d;
      d.j = find_item_slot(s_tab, n_slots, item);
      const int nrg = (s_ucnt[d.j] + kTileRows - 1) / kTileRows;
      const int local = item - s_tab[d.j].w;
      d.tt = local / nrg;
      d.rg = local % nrg;
      return d;
    };
    int key = -1, xb = rc.nxb - 1, mi = 0;
    int cur = claim();
    Pos cp = cur >= 0 ? decode(cur) : Pos{0, 0, 0};
    for (; cur >= 0 && !*abort; ++mi) {
      const int nxt = claim();
      const Pos np = nxt >= 0 ? decode(nxt) : Pos{0, 0, 0};
      const int nxt_key = nxt >= 0 ? np.j * 1024 + np.tt : -1;
      const int m = mi % kMetaRing;
      if (!mbar_wait(&mempty[m], ((mi / kMetaRing) & 1) ^ 1, abort, p.err)) break;
      const int4 sl = s_tab[cp.j];
      const int kind = sl.x >> 16, ex = sl.x & 0xffff, T = sl.y, q0 = sl.z;
      const int nt = min(kTileTok, T - cp.tt * kTileTok);
      const int qt = q0 + cp.tt * kTileTok;
      int xpar = 0;
      if (cp.j * 1024 + cp.tt != key) {
        key = cp.j * 1024 + cp.tt;
        if constexpr (!kReg) {
          xb = (xb + 1) % rc.nxb;
          if (!mbar_wait(&xempty[xb], (xuse[xb] & 1) ^ 1, abort, p.err)) break;
          xpar = xuse[xb] & 1;
          xuse[xb]++;
          const int tok_l = lane < nt ? __ldcg(&p.pair_token[qt + lane]) : -1;
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
      if (lane == 0) {
        s_meta[m].ud = kind == 0 ? static_cast<const __nv_bfloat16*>(p.updown_r) +
                                       (size_t)ex * p.I * 2 * H
                                 : static_cast<const __nv_bfloat16*>(p.updown_s) +
                                       (size_t)ex * p.Ish * 2 * H;
        s_meta[m].key = key;
        s_meta[m].xb = xb;
        s_meta[m].xpar = xpar;
        s_meta[m].xlast = nxt_key != key;
        s_meta[m].j = cp.j;
        s_meta[m].tt = cp.tt;
        s_meta[m].rg = cp.rg;
        s_meta[m].end = 0;
        mbar_arrive(&mhead[m]);
        mbar_arrive(&mrows[m]);
        mbar_arrive(&mfull[m]);
      }
      __syncwarp();
      cur = nxt;
      cp = np;
    }
    for (int e = 0; e < 2; ++e, ++mi) {  // closing records
      const int m = mi % kMetaRing;
      mbar_wait(&mempty[m], ((mi / kMetaRing) & 1) ^ 1, abort, p.err);
      if (lane == 0) {
        s_meta[m].end = 1;
        mbar_arrive(&mhead[m]);
        mbar_arrive(&mrows[m]);
        mbar_arrive(&mfull[m]);
      }
      __syncwarp();
    }
    for (int b = 0; b < rc.nxb; ++b)
      if (xuse[b] > 0) mbar_drain(&xfull[b], (xuse[b] - 1) & 1);
    return;
  }

  if (warp >= kCoefWarp0) {
    // ---------------- coefficient warp c: rows, coef, tok and w of the records mi with
    // mi % kCoefWarps == c (so it always uses the same meta slots)
    const int cw = warp - kCoefWarp0;
    for (int mi = cw;; mi += kCoefWarps) {
      const int m = mi % kMetaRing;
      if (!mbar_wait(&mhead[m], (mi / kMetaRing) & 1, abort, p.err)) break;
      if (s_meta[m].end) {
        if (lane == 0) {
          mbar_arrive(&mrows[m]);
          mbar_arrive(&mfull[m]);
        }
        break;
      }
      const int j = s_meta[m].j, tt = s_meta[m].tt, rg = s_meta[m].rg;
      const int4 sl = s_tab[j];
      const int T = sl.y, q0 = sl.z, rows = s_ucnt[j];
      const int nt = min(kTileTok, T - tt * kTileTok);
      const int qt = q0 + tt * kTileTok;
      // row of this lane (lanes 0..15) and token of this lane (lanes 0..7); the rows go out
      // first (mrows: all the copier needs), the coefficients after one more round trip
      const int ridx = rg * kTileRows + (lane & 15);
      const int n_l = __ldcg(&p.ulist[(size_t)j * Imax + (ridx < rows ? ridx : rg * kTileRows)]);
      const int tok_l = lane < nt ? __ldcg(&p.pair_token[qt + lane]) : -1;
      const float w_l = lane < nt ? __ldcg(&p.pair_w[qt + lane]) : 0.f;
      if (lane < kTileRows) s_meta[m].rows[lane] = n_l;
      if (lane < kTileTok) {
        s_meta[m].tok[lane] = tok_l;
        s_meta[m].w[lane] = w_l;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&mrows[m]);
      // coefficients: lane l covers row l/2, columns 4*(l&1) .. +3
      const int r = lane >> 1, c0 = (lane & 1) * 4;
      const int n = __shfl_sync(0xffffffffu, n_l, r);
      const bool rvalid = rg * kTileRows + r < rows;
      uint32_t bits[4];
      float av[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int q = qt + c0 + c;
        const bool ok = rvalid && c0 + c < nt;
        bits[c] = ok ? __ldcg(&p.maskbits[(size_t)q * Wmax + (n >> 5)]) : 0u;
        av[c] = ok ? __ldcg(&p.act[(size_t)q * Imax + n]) : 0.f;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c)
        s_meta[m].coef[r][c0 + c] = ((bits[c] >> (n & 31)) & 1u) ? av[c] : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mfull[m]);
    }
    return;
  }

  if (warp == kCopier) {
    // ---------------- copier: up pieces, then down pieces, of the item's 16 rows
    const uint32_t piece = rc.kc * 2;
    int it = 0;
    for (int mi = 0; !*abort; ++mi) {
      const int m = mi % kMetaRing;
      if (!mbar_wait(&mrows[m], (mi / kMetaRing) & 1, abort, p.err)) break;
      if (s_meta[m].end) break;
      const __nv_bfloat16* row = s_meta[m].ud + (size_t)s_meta[m].rows[lane & 15] * 2 * H;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mempty[m]);
      bool stop = false;
      for (int half = 0; half < 2 && !stop; ++half) {
        const int rs = half ? rc.rs_d : rc.rs_a;
        for (int kc = 0; kc < rc.nk; ++kc, ++it) {
          const int st = it % rc.ns;
          if (!mbar_wait(&empty[st], ((it / rc.ns) & 1) ^ 1, abort, p.err)) {
            stop = true;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(&full[st], kTileRows * piece);
          __syncwarp();
          if (lane < kTileRows)
            bulk_g2s(ring + (size_t)st * rc.stage_bytes + lane * rs, row + half * H + kc * rc.kc,
                     piece, &full[st]);
        }
      }
    }
    for (int k = it - 1; k >= 0 && k >= it - rc.ns; --k) mbar_drain(&full[k % rc.ns], (k / rc.ns) & 1);
    return;
  }

  // ---------------- consumers
  constexpr int kXR = kReg ? NK : 1, kXB = kReg ? BPW : 1;
  uint4 xr[kXR][kXB];
  int it = 0, ib = 0, cur = -1, run_key = -1;
  const int nblk = rc.kc / 32, nsub = rc.kc / 64;
  const uint32_t tmem_warp = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + 256u * (warp >> 2);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  for (int mi = 0;; ++mi) {
    const int m = mi % kMetaRing;
    // rows, tokens and weights (mrows) are enough for the up projection; the coefficients
    // (mfull, one more L2 round trip) are awaited before the epilogue
    mbar_wait(&mrows[m], (mi / kMetaRing) & 1, abort, p.err);
    // the end (or an abort) is decided by all consumer warps together
    if (consumer_sync_or(kThreads, s_meta[m].end || *abort)) {
      trace_value(p.trace, 3, 5, (unsigned long long)mi);
      break;
    }
    if (mi == 0) trace_point(p.trace, 3, 2);
    trace_point(p.trace, 3, 6);
    const UdMeta& mt = s_meta[m];
    const int xb = min(max(mt.xb, 0), max(rc.nxb - 1, 0));  // a record is trusted only w/o abort
    const int xlast = mt.xlast;
    const int item_key = mt.key;  // the record is handed back to the meta warp before the down
                                  // projection: everything read from it is read here
    const int tok0 = mt.tok[2 * t], tok1 = mt.tok[2 * t + 1];
    const float w0 = mt.w[2 * t], w1 = mt.w[2 * t + 1];
    const unsigned char* xrow = xbuf + xb * rc.xs_bytes + g * rc.xs_stride;
    if constexpr (kReg) {
      if (mt.key != cur) {  // this warp's token fragments for the new tile (one round trip)
        cur = mt.key;
        const int tok = mt.tok[g];
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
      mbar_wait(&xfull[xb], mt.xpar, abort, p.err);
    }
    // 1. up projection
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (kReg) {
#pragma unroll
      for (int kc = 0; kc < kXR; ++kc, ++it) {
        const int st = it % rc.ns;
        mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
        if (it == 0) trace_point(p.trace, 3, 3);
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
    if (!kReg && lane == 0 && xlast) mbar_arrive(&xempty[xb]);
#pragma unroll
    for (int c = 0; c < 4; ++c) red[ib][warp][c][lane] = d[c];
    mbar_wait(&mfull[m], (mi / kMetaRing) & 1, abort, p.err);
    const int aborted = consumer_sync_or(kThreads, *abort);
    // 2. coefficients times u, rounded to bf16, token-major (one element per thread)
    if (threadIdx.x < 128) {
      const int ln = threadIdx.x & 31, c = threadIdx.x >> 5;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[ib][w][c][ln];
      const int r = (ln >> 2) + (c >> 1) * 8, tok = 2 * (ln & 3) + (c & 1);
      reinterpret_cast<__nv_bfloat16*>(&s_hcw[ib][tok][0])[r] =
          __float2bfloat16_rn(mt.coef[r][tok] * v);
    }
    consumer_sync(kThreads);
    if (lane == 0) mbar_arrive(&mempty[m]);
    // 3-4. down projection of each stage's 64-column sub-chunks, kept in tensor memory while
    // the run of items of this (expert, token tile) goes on, reduced into out_acc at its end
    const uint32_t b0 = s_hcw[ib][g][t], b1 = s_hcw[ib][g][4 + t];
    const bool first = item_key != run_key, last = xlast != 0 || !tmem_acc;
    run_key = last ? -1 : item_key;
    for (int kc = 0; kc < rc.nk; ++kc, ++it) {
      const int st = it % rc.ns;
      mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
      const unsigned char* stage = ring + (size_t)st * rc.stage_bytes;
      for (int sc = warp; sc < nsub; sc += kWarps) {
        const int off = (sc * 64 + 8 * g) * 2;
        const uint4 r0 = lds128(stage + (2 * t) * rc.rs_d + off);
        const uint4 r1 = lds128(stage + (2 * t + 1) * rc.rs_d + off);
        const uint4 r2 = lds128(stage + (2 * t + 8) * rc.rs_d + off);
        const uint4 r3 = lds128(stage + (2 * t + 9) * rc.rs_d + off);
        const uint32_t w0v[4] = {r0.x, r0.y, r0.z, r0.w}, w1v[4] = {r1.x, r1.y, r1.z, r1.w};
        const uint32_t w2v[4] = {r2.x, r2.y, r2.z, r2.w}, w3v[4] = {r3.x, r3.y, r3.z, r3.w};
        const int hb = kc * rc.kc + sc * 64 + 8 * g;
        // mma i gives h = hb + 2i, 2i + 1 for the thread's two tokens: eight consecutive h per
        // token, reduced as two 16-byte vectors (the L2 reductions are the costly part here)
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
          mma_16816(acc[i], __byte_perm(w0v[i], w1v[i], 0x5410),
                    __byte_perm(w0v[i], w1v[i], 0x7632), __byte_perm(w2v[i], w3v[i], 0x5410),
                    __byte_perm(w2v[i], w3v[i], 0x7632), b0, b1);
        }
        if (!(first && last)) {
          float v[16];
          const uint32_t col = tmem_warp + 16u * (uint32_t)(kc * spw + (sc - warp) / kWarps);
          if (!first) {  // earlier items of the run, summed in the same order every time
            tmem_ld16(col, v);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int c = 0; c < 4; ++c) acc[i][c] += v[4 * i + c];
          }
          if (!last) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int c = 0; c < 4; ++c) v[4 * i + c] = acc[i][c];
            tmem_st16(col, v);
          }
        }
        if (last && !aborted && tok0 >= 0) {
          float* o = p.out_acc + (size_t)tok0 * H + hb;
          red_add_v4(o, w0 * acc[0][0], w0 * acc[0][2], w0 * acc[1][0], w0 * acc[1][2]);
          red_add_v4(o + 4, w0 * acc[2][0], w0 * acc[2][2], w0 * acc[3][0], w0 * acc[3][2]);
        }
        if (last && !aborted && tok1 >= 0) {
          float* o = p.out_acc + (size_t)tok1 * H + hb;
          red_add_v4(o, w1 * acc[0][1], w1 * acc[0][3], w1 * acc[1][1], w1 * acc[1][3]);
          red_add_v4(o + 4, w1 * acc[2][1], w1 * acc[2][3], w1 * acc[3][1], w1 * acc[3][3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (!last) tmem_wait_st();  // the next item of the run loads these columns
    if (mi == 0) trace_point(p.trace, 3, 4);
    ib ^= 1;
  }
  trace_point(p.trace, 3, 7);
  // every consumer warp is done with tensor memory before warp 0 frees it
  tmem_fence_before();
  consumer_sync(kThreads);
  tmem_fence_after();
  if (tmem_acc && warp == 0) tmem_dealloc(tmem_base, 512);
}

// fp32 variant: register loads, same items and fragment layout.
__global__ void __launch_bounds__(kThreads) updown_f32_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ int s_item0[kMaxSlots + 1];
  __shared__ int scratch[33];
  __shared__ const float* s_x[kTileTok];
  __shared__ const float* s_up[kTileRows];
  __shared__ const float* s_dn[kTileRows];
  __shared__ int s_tok[kTileTok];
  __shared__ float s_w[kTileTok];
  __shared__ float s_coef[kTileRows][kTileTok];
  __shared__ float s_hcf[kTileRows][kTileTok];
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, Imax = p.Imax, Wmax = p.Imax / 32;
  const int n_slots = ld_cg(&p.meta[kMetaSlots]);
  const int n_items = updown_items(p, n_slots, s_item0, scratch);
  const float* x = static_cast<const float*>(p.x);
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const UdPos u = decode_ud_item(p, s_item0, n_slots, item);
    const Slot s = load_slot(&p.slots[u.j]);
    const float* ud = s.kind == 0 ? static_cast<const float*>(p.updown_r) + (size_t)s.expert * p.I * 2 * H
                                  : static_cast<const float*>(p.updown_s) + (size_t)s.expert * p.Ish * 2 * H;
    if (threadIdx.x < kTileRows) {
      const int n = union_row(p, u, threadIdx.x);
      s_up[threadIdx.x] = ud + (size_t)n * 2 * H;
      s_dn[threadIdx.x] = ud + (size_t)n * 2 * H + H;
    } else if (threadIdx.x >= 32 && threadIdx.x < 32 + kTileTok) {
      const int c = threadIdx.x - 32, ti = u.tt * kTileTok + c;
      const bool ok = ti < s.T;
      const int tok = ok ? __ldcg(&p.pair_token[s.q0 + ti]) : -1;
      s_tok[c] = tok;
      s_w[c] = ok ? __ldcg(&p.pair_w[s.q0 + ti]) : 0.f;
      s_x[c] = ok ? x + (size_t)tok * H : nullptr;
    }
    if (threadIdx.x >= 64 && threadIdx.x < 64 + kTileRows * kTileTok) {
      const int r = (threadIdx.x - 64) >> 3, c = (threadIdx.x - 64) & 7;
      const int ti = u.tt * kTileTok + c, n = union_row(p, u, r);
      float coef = 0.f;
      if (ti < s.T && u.rg * kTileRows + r < u.rows) {
        const int q = s.q0 + ti;
        if ((__ldcg(&p.maskbits[(size_t)q * Wmax + (n >> 5)]) >> (n & 31)) & 1u)
          coef = __ldcg(&p.act[(size_t)q * Imax + n]);
      }
      s_coef[r][c] = coef;
    }
    __syncthreads();
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    tile_dot<1>(s_up[g], s_up[g + 8], s_x, warp, kWarps, H / 32, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
    __syncthreads();
    if (warp == 0) {
      reduce_fragments(red, d);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = g + (c >> 1) * 8, tok = 2 * t + (c & 1);
        s_hcf[r][tok] = s_coef[r][tok] * d[c];
      }
    }
    __syncthreads();
    const int tok0 = s_tok[2 * t], tok1 = s_tok[2 * t + 1];
    const float w0 = s_w[2 * t], w1 = s_w[2 * t + 1];
    for (int ch = warp; ch < H / 64; ch += kWarps) {
      const int h0 = ch * 64;
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
      tile_down(s_dn, h0, 0u, 0u, s_hcf, acc);
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

template <int NK, int BPW>
cudaError_t set_ud_smem(int budget) {
  return allow_max_smem(updown_tma_kernel<NK, BPW>, budget);
}

template <int NK, int BPW>
int ud_static_smem() {
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, updown_tma_kernel<NK, BPW>) == cudaSuccess
             ? (int)fa.sharedSizeBytes
             : 16384;
}

cudaError_t launch_updown(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                          bool pdl) {
  if (dtype != 0)
    return launch_pdl(updown_f32_kernel, dim3(ls.grid_updown), dim3(kThreads), 0, st, pdl, p);
  const Ring& r = ls.ring_ud;
  const dim3 grid(ls.nsm), block(kRingThreads);
  switch (ls.variant) {
    case 1: return launch_pdl(updown_tma_kernel<1, 2>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 2: return launch_pdl(updown_tma_kernel<1, 8>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 3: return launch_pdl(updown_tma_kernel<3, 4>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 4: return launch_pdl(updown_tma_kernel<4, 5>, grid, block, r.smem_bytes, st, pdl, p, r);
    default: return launch_pdl(updown_tma_kernel<0, 0>, grid, block, r.smem_bytes, st, pdl, p, r);
  }
}

extern const int kRegVariants[4][3];
Ring make_ring(int H, int nk_fixed, int smem_budget, int static_smem);

cudaError_t configure_updown(int dtype, int H, int smem_budget, LaunchShape* ls) {
  if (dtype != 0) {
    int n = 0;
    cudaError_t e =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, updown_f32_kernel, kThreads, 0);
    ls->grid_updown = ls->nsm * (n > 0 ? n : 1);
    return e;
  }
  // ls->variant was chosen by configure_gate for the same H
  const int nk = ls->variant ? kRegVariants[ls->variant - 1][1] : 0;
  int stat = 0;
  switch (ls->variant) {
    case 1: stat = ud_static_smem<1, 2>(); break;
    case 2: stat = ud_static_smem<1, 8>(); break;
    case 3: stat = ud_static_smem<3, 4>(); break;
    case 4: stat = ud_static_smem<4, 5>(); break;
    default: stat = ud_static_smem<0, 0>(); break;
  }
  ls->ring_ud = make_ring(H, nk, smem_budget, stat + 1024);
  if (ls->ring_ud.ns < 2) return cudaErrorInvalidConfiguration;
  ls->grid_updown = ls->nsm;
  switch (ls->variant) {
    case 1: return set_ud_smem<1, 2>(smem_budget);
    case 2: return set_ud_smem<1, 8>(smem_budget);
    case 3: return set_ud_smem<3, 4>(smem_budget);
    case 4: return set_ud_smem<4, 5>(smem_budget);
    default: return set_ud_smem<0, 0>(smem_budget);
  }
}

}  // namespace moe
