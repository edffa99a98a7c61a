// dense.cu - the dense masked fallback for experts with many tokens, on tcgen05 tensor cores.
//
// "Uncovering Intra-expert Activation Sparsity ..." (technical summary, Methodology) switches
// between its sparse kernel and dense kernels by batch size: once an expert has enough tokens,
// nearly every neuron is kept by some token and the layer is a dense contraction again.  The
// function does not change: the gate runs densely, selection keeps the same neurons, the up
// projection's result is multiplied by the 0/1 mask (times SiLU(g)), and the down projection
// sums over all neurons.  Here a slot (one expert and its tokens) is dense when its token count
// reaches the handle's threshold; the sparse kernels skip such slots.
//
// One kernel, three epilogues (mode):
//   gate  D[n][t] = W_g[n] . x_t           -> act[pair][n] = SiLU(D)
//   up    D[n][t] = W_up[n] . x_t          -> hbuf[pair][n] = bf16(mask * act * D)
//   down  D[h][t] = sum_n W_down[h][n] hbuf[pair][n]   -> out_acc[token][h] += w * D
// D = A . B^T with A = weights (M = neurons or h, K-major rows of the packed layout; for down the
// packed layout stores W_down transposed, so A is read M-major) and B = the slot's token rows
// (K-major): x rows gathered per pair (xp), or hbuf rows.  Tile 128 (M) x up to 256 tokens (N) x
// 64 (K) per stage, bf16 in, fp32 accumulated in tensor memory.
//
// Persistent CTAs (one per SM), 6 warps: warps 0-3 drain the accumulator (each owns 32 TMEM
// lanes), warp 4 issues the 2-D TMA loads (128-byte swizzle) into a 4-stage ring, warp 5 issues
// tcgen05.mma from one thread.  Two accumulators alternate so one tile's epilogue overlaps the
// next tile's main loop.  Every mbarrier wait is bounded; on time-out the CTA stops issuing,
// waits (bounded) for its copies and MMAs in flight, frees tensor memory and returns.
#include <cuda.h>

#include "kernels.h"
#include "tma.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxBN = 256;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB
constexpr int kBBytes = kMaxBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kDenseThreads = 192;
constexpr int kProducerWarp = 4, kMmaWarp = 5;
constexpr int kTmemCols = 512;             // two accumulators of 256 fp32 columns
constexpr int kDenseSmem = kStages * kStageBytes + 1024;  // + alignment slack

// ---- tcgen05 / TMA primitives -----------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] . B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate)
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (warp's quarter + i)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), sm_100 version 1.
// Addresses and byte offsets are encoded in 16-byte units.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 D, bf16 A and B, A major (0 K, 1 M), B K-major,
// N = n (multiple of 16, <= 256), M = 128.
__host__ __device__ constexpr uint32_t instr_desc(int a_mn_major, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn_major << 15) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ bool slot_is_dense(int T, int dense_min) { return T >= dense_min; }

struct DenseMaps {
  CUtensorMap a_r, a_s;  // weights of the routed / shared experts
  CUtensorMap b;         // token rows: xp (gate, up) or hbuf (down)
};

// Tile t of the launch: slot j, M tile mt, N tile nt (all M tiles of one N tile are consecutive),
// and the range [kb0, kb1) of 64-wide K blocks it contracts (all of them, except for a down
// GEMM split over K).
struct TileRef {
  int j, kind, expert, T, q0, m0, n0, ntok, mext, kb0, kb1;
};

// Largest K split of the down GEMM.  Its epilogue adds w * D into the output accumulator, so
// partial sums over K ranges may be added separately.  A down GEMM with fewer tiles than CTAs
// (a large shared expert alone on this path: H / 128 tiles) is split until its tiles cover the
// grid.  The gate and up GEMMs are never split over K: their epilogues are not linear in D.
constexpr int kMaxKSplit = 4;

// A gate or up launch with fewer tiles than CTAs (a large shared expert alone on this path:
// I / 128 tiles) splits each slot's tokens into up to f N tiles, f = CTAs / tiles, at most
// kMaxNSplit, each at least 16 tokens wide.  The CTAs of one M tile's N tiles run at the same
// time, so the weights come from HBM once and from L2 for the others.  Every (neuron, token)
// dot product keeps its K order, so the activations do not depend on the split.
constexpr int kMaxNSplit = 8;

// Token columns of one N tile of a slot with T tokens split f ways: a multiple of 16, at most
// kMaxBN (f = 1: ceil(T / 256) tiles, 256 tokens wide but the last).
__device__ __forceinline__ int ntile_width(int T, int f) {
  return min(kMaxBN, ((T + f - 1) / f + 15) / 16 * 16);
}

template <int kMode>
__global__ void __launch_bounds__(kDenseThreads, 1)
    dense_gemm_kernel(const __grid_constant__ DenseMaps maps, FwdParams p) {
  extern __shared__ __align__(1024) unsigned char dsmem_raw[];
  __shared__ uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], done_bar;
  __shared__ int4 s_tab[kMaxSlots];   // {expert | kind << 16, T, q0, first tile}
  __shared__ int s_mt[kMaxSlots];     // M tiles of the slot
  __shared__ int scratch[33];
  __shared__ int s_total, s_abort;
  __shared__ uint32_t s_tmem;
  __shared__ int s_tok[2][kMaxBN];
  __shared__ float s_w[2][kMaxBN];
  unsigned char* dsmem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &s_abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(&done_bar, 1);
    s_abort = 0;
    mbar_init_fence();
  }
  if (warp == kMmaWarp) {  // the whole warp allocates tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_trigger();
  pdl_wait();
  // tile table over the dense slots (every slot entry that can exist is read speculatively)
  int nsplit = 1;  // N split of the gate and up GEMMs (kMaxNSplit)
  {
    const int n_slots = ld_cg(&p.meta[kMetaSlots]);
    const int n_max = min(slot_capacity(p.E, p.S), kMaxSlots);
    const int per = (n_max + blockDim.x - 1) / blockDim.x;
    const int b0 = min(n_max, (int)threadIdx.x * per), b1 = min(n_max, b0 + per);
    int c = 0;
    for (int j = b0; j < b1; ++j) {
      const Slot sl = load_slot(&p.slots[j]);
      const bool dense = j < n_slots && slot_is_dense(sl.T, p.dense_min);
      const int mext = kMode == 2 ? p.H : (sl.kind ? p.Ish : p.I);
      const int mt = (mext + kBM - 1) / kBM;
      const int v = dense ? mt * ((sl.T + kMaxBN - 1) / kMaxBN) : 0;
      s_tab[j] = make_int4(sl.expert | (sl.kind << 16), sl.T, sl.q0, v);
      s_mt[j] = mt;
      c += v;
    }
    int total;
    int run = block_exclusive_scan(c, scratch, &total);
    if (kMode != 2 && total > 0 && total < (int)gridDim.x) {
      nsplit = min(kMaxNSplit, (int)gridDim.x / total);
      if (nsplit > 1) {  // the same for every thread: recount the slots' tiles
        c = 0;
        for (int j = b0; j < b1; ++j) {
          const int T = s_tab[j].y, w = ntile_width(T, nsplit);
          const int v = s_tab[j].w ? s_mt[j] * ((T + w - 1) / w) : 0;
          s_tab[j].w = v;
          c += v;
        }
        run = block_exclusive_scan(c, scratch, &total);
      }
    }
    for (int j = b0; j < b1; ++j) {
      const int v = s_tab[j].w;
      s_tab[j].w = run;
      run += v;
    }
    if (threadIdx.x == 0) s_total = total;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n_tiles = s_total;
  const int n_max = min(slot_capacity(p.E, p.S), kMaxSlots);
  int ksplit = 1;
  if (kMode == 2 && n_tiles > 0 && n_tiles < (int)gridDim.x) {
    const int kb_min = (min(p.I, p.S > 0 ? p.Ish : p.I) + kBK - 1) / kBK;  // no part is empty
    ksplit = max(1, min(min(kMaxKSplit, kb_min), (int)gridDim.x / n_tiles));
  }
  const int n_work = n_tiles * ksplit;  // work item w: K part w / n_tiles of tile w % n_tiles
  const uint32_t tmem_base = s_tmem;
  auto tile_at = [&](int w) -> TileRef {
    TileRef r;
    const int t = w % n_tiles, part = w / n_tiles;
    r.j = find_item_slot(s_tab, n_max, t);
    const int4 sl = s_tab[r.j];
    r.kind = sl.x >> 16;
    r.expert = sl.x & 0xffff;
    r.T = sl.y;
    r.q0 = sl.z;
    const int local = t - sl.w, mt = s_mt[r.j], wn = ntile_width(r.T, nsplit);
    r.m0 = (local % mt) * kBM;
    r.n0 = (local / mt) * wn;
    r.ntok = min(wn, r.T - r.n0);
    r.mext = kMode == 2 ? p.H : (r.kind ? p.Ish : p.I);
    // contraction length: H for gate and up, the expert's I for down
    const int kb = kMode == 2 ? ((r.kind ? p.Ish : p.I) + kBK - 1) / kBK : p.H / kBK;
    r.kb0 = kb * part / ksplit;
    r.kb1 = kb * (part + 1) / ksplit;
    return r;
  };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < n_work && !*abort; t += gridDim.x) {
        const TileRef r = tile_at(t);
        const int nb = (r.ntok + 31) / 32;  // 32-token boxes of B
        const CUtensorMap* ma = r.kind ? &maps.a_s : &maps.a_r;
        const int kb_rows = kMode == 2 ? r.expert * (r.kind ? p.Ish : p.I) : 0;
        const int a_row0 = kMode == 2 ? 0 : r.expert * r.mext + r.m0;
        for (int k = r.kb0; k < r.kb1; ++k, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort, p.err)) break;
          unsigned char* sa = dsmem + s * kStageBytes;
          unsigned char* sb = sa + kABytes;
          mbar_arrive_expect_tx(&full[s], kABytes + nb * 32 * kBK * 2);
          if (kMode == 2) {
            // A = W_down read M-major: two boxes of 64 h x 64 neurons
            tma_load_2d(sa, ma, &full[s], r.m0, kb_rows + k * kBK);
            tma_load_2d(sa + kABytes / 2, ma, &full[s], r.m0 + 64, kb_rows + k * kBK);
          } else {
            tma_load_2d(sa, ma, &full[s], k * kBK, a_row0);
          }
          for (int b = 0; b < nb; ++b)
            tma_load_2d(sb + b * 32 * kBK * 2, &maps.b, &full[s], k * kBK, r.q0 + r.n0 + 32 * b);
        }
      }
      // no copy may still be landing when the CTA exits
      for (int k = it - 1; k >= 0 && k >= it - kStages; --k)
        mbar_drain(&full[k % kStages], (k / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      int it = 0, tl = 0;
      for (int t = blockIdx.x; t < n_work && !*abort; t += gridDim.x, ++tl) {
        const TileRef r = tile_at(t);
        const int nmma = (r.ntok + 15) & ~15;  // N of the instruction, a multiple of 16
        const uint32_t idesc = instr_desc(kMode == 2 ? 1 : 0, nmma);
        const int ab = tl & 1;
        if (!mbar_wait(&acc_empty[ab], ((tl >> 1) & 1) ^ 1, abort, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * kMaxBN;
        bool ok = true;
        for (int k = r.kb0; k < r.kb1; ++k, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], (it / kStages) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(dsmem + s * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major rows of 128 B (16 k per instruction = 32 B further along the row), or
            // M-major 64-h rows per k (two 8-k swizzle atoms = 2048 B per instruction)
            const uint64_t ad = kMode == 2 ? smem_desc(a_addr + kk * 2048, kABytes / 2, 1024)
                                           : smem_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc(b_addr + kk * 32, 16, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (k > r.kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
      umma_commit(&done_bar);  // every MMA of this CTA has completed when this arrives
      mbar_drain(&done_bar, 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warps 0-3, thread = one accumulator row (TMEM lane)
    int tl = 0;
    bool nan_seen = false;
    for (int t = blockIdx.x; t < n_work; t += gridDim.x, ++tl) {
      // the four warps leave together (the named barriers below must never miss a warp)
      if (consumer_sync_or(128, *abort)) break;
      const TileRef r = tile_at(t);
      const int ab = tl & 1;
      if (kMode == 2) {  // tokens and routing weights of the tile's columns
        for (int c = threadIdx.x; c < r.ntok; c += 128) {
          s_tok[ab][c] = __ldcg(&p.pair_token[r.q0 + r.n0 + c]);
          s_w[ab][c] = __ldcg(&p.pair_w[r.q0 + r.n0 + c]);
        }
        consumer_sync(128);
      }
      if (!mbar_wait(&acc_full[ab], (tl >> 1) & 1, abort, p.err)) continue;  // leaves above
      tc_fence_after();
      const int row = r.m0 + warp * 32 + lane;  // neuron (gate, up) or h (down)
      const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16) + ab * kMaxBN;
      for (int c0 = 0; c0 < r.ntok; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + c0, v);
        const int nc = min(32, r.ntok - c0);
        if (kMode == 0) {
          if (row < r.mext) {
            const bool hist = uses_hist(p, r.kind);
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c < nc) {
                const float a = silu(__uint_as_float(v[c]));
                nan_seen |= isnan(a);
                p.act[(size_t)(r.q0 + r.n0 + c0 + c) * p.Imax + row] = a;
                if (hist) hist_add(p, r.q0 + r.n0 + c0 + c, a);
              }
            }
          }
        } else if (kMode == 1) {
          // every load of the chunk first (they are independent), then the products and stores
          uint32_t bits[32];
          float a[32];
          const bool live = row < r.mext;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const size_t q = (size_t)(r.q0 + r.n0 + c0 + min(c, nc - 1));
            bits[c] = live ? __ldcg(&p.maskbits[q * (p.Imax / 32) + (row >> 5)]) : 0u;
            a[c] = live ? __ldcg(&p.act[q * p.Imax + row]) : 0.f;
          }
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c >= nc) continue;
            const size_t q = (size_t)(r.q0 + r.n0 + c0 + c);
            const float h = ((bits[c] >> (row & 31)) & 1u) ? a[c] * __uint_as_float(v[c]) : 0.f;
            p.hbuf[q * p.imax_pad + row] = __float2bfloat16_rn(h);
          }
        } else {
          if (row < p.H) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c >= nc) continue;
              const int cc = c0 + c;
              red_add_f32(p.out_acc + (size_t)s_tok[ab][cc] * p.H + row,
                          s_w[ab][cc] * __uint_as_float(v[c]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
    if (nan_seen) set_error(p.err, kErrNanAct);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kTmemCols)
                 : "memory");
}

// x rows of the pairs of dense slots, gathered into xp [pairs][H]: one warp per pair
__global__ void gather_kernel(FwdParams p) {
  pdl_trigger();
  pdl_wait();
  const int n_pairs = ld_cg(&p.meta[kMetaPairs]);
  const int lane = threadIdx.x & 31;
  const int w0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = (gridDim.x * blockDim.x) >> 5;
  for (int q = w0; q < n_pairs; q += nw) {
    const int j = __ldcg(&p.pair_slot[q]);
    if (j < 0 || !slot_is_dense(__ldcg(&p.slots[j].T), p.dense_min)) continue;
    const int tok = __ldcg(&p.pair_token[q]);
    const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.x) + (size_t)tok * p.H;
    for (int v = lane; v < p.H / 8; v += 32)
      *reinterpret_cast<uint4*>(p.xp + (size_t)q * p.H + v * 8) = ld_nc(src + v * 8);
  }
}

// ---- host: tensor maps ------------------------------------------------------------------------
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(f);
  }
  return fn;
}

// 2-D bf16 map: inner extent `inner` (contiguous), `rows` rows `row_bytes` apart, box
// box_inner x box_rows, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
              uint32_t box_inner, uint32_t box_rows) {
  EncodeTiled enc = encoder();
  if (!enc || !base) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t dense_smem_bytes() { return kDenseSmem; }

cudaError_t configure_dense(int budget) {
  cudaError_t e = allow_max_smem(dense_gemm_kernel<0>, budget);
  if (e == cudaSuccess) e = allow_max_smem(dense_gemm_kernel<1>, budget);
  if (e == cudaSuccess) e = allow_max_smem(dense_gemm_kernel<2>, budget);
  return e;
}

// Launches gather + the gate GEMM (stage 0), or the up and down GEMMs (stage 1), for the dense
// slots of this call.  Weights are the packed layouts: gate [n][I][H], updown [n][I][2][H].
cudaError_t launch_dense(const FwdParams& p, const LaunchShape& ls, int stage, cudaStream_t st,
                         bool pdl) {
  const uint64_t H = (uint64_t)p.H;
  // the routed weights are the handle's local block of experts [e_begin, e_end)
  const uint64_t rows_r = (uint64_t)(p.e_end - p.e_begin) * p.I, rows_s = (uint64_t)p.S * p.Ish;
  const __nv_bfloat16* gr = static_cast<const __nv_bfloat16*>(p.gate_r);
  const __nv_bfloat16* gs = static_cast<const __nv_bfloat16*>(p.gate_s);
  const __nv_bfloat16* ur = static_cast<const __nv_bfloat16*>(p.updown_r);
  const __nv_bfloat16* us = static_cast<const __nv_bfloat16*>(p.updown_s);
  DenseMaps m;
  memset(&m, 0, sizeof(m));
  const dim3 grid(ls.nsm), block(kDenseThreads);
  if (stage == 0) {
    cudaError_t e = launch_pdl(gather_kernel, dim3(ls.nsm), dim3(256), 0, st, pdl, p);
    if (e != cudaSuccess) return e;
    if (!make_map(&m.a_r, gr, H, rows_r, H * 2, kBK, kBM)) return cudaErrorInvalidValue;
    if (p.S > 0 && !make_map(&m.a_s, gs, H, rows_s, H * 2, kBK, kBM)) return cudaErrorInvalidValue;
    if (!make_map(&m.b, p.xp, H, (uint64_t)p.Bmax * (p.k + p.S), H * 2, kBK, 32))
      return cudaErrorInvalidValue;
    return launch_pdl(dense_gemm_kernel<0>, grid, block, kDenseSmem, st, pdl, m, p);
  }
  // up: the W_up halves of the packed rows
  if (!make_map(&m.a_r, ur, H, rows_r, H * 4, kBK, kBM)) return cudaErrorInvalidValue;
  if (p.S > 0 && !make_map(&m.a_s, us, H, rows_s, H * 4, kBK, kBM)) return cudaErrorInvalidValue;
  if (!make_map(&m.b, p.xp, H, (uint64_t)p.Bmax * (p.k + p.S), H * 2, kBK, 32))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(dense_gemm_kernel<1>, grid, block, kDenseSmem, st, pdl, m, p);
  if (e != cudaSuccess) return e;
  // down: the W_down halves (h contiguous per neuron), read M-major in boxes of 64 h x 64 n
  DenseMaps d;
  memset(&d, 0, sizeof(d));
  if (!make_map(&d.a_r, ur + H, H, rows_r, H * 4, 64, kBK)) return cudaErrorInvalidValue;
  if (p.S > 0 && !make_map(&d.a_s, us + H, H, rows_s, H * 4, 64, kBK)) return cudaErrorInvalidValue;
  if (!make_map(&d.b, p.hbuf, (uint64_t)p.imax_pad, (uint64_t)p.Bmax * (p.k + p.S),
                (uint64_t)p.imax_pad * 2, kBK, 32))
    return cudaErrorInvalidValue;
  return launch_pdl(dense_gemm_kernel<2>, grid, block, kDenseSmem, st, pdl, d, p);
}

}  // namespace moe
