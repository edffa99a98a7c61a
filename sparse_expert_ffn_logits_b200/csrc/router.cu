// router.cu - router logits, top-k + routing weights, and the grouping of (token, expert) pairs
// by expert, fused in one launch.
//
// The router of the paper's layer is the standard MoE router, kept unchanged ("Uncovering
// Intra-expert Activation Sparsity ...", technical summary, Methodology): logits W_r x, the k
// largest per token (ties: lower expert index), weights by softmax over the chosen logits,
// softmax over all logits, or a sigmoid of the chosen logit.
//
// Grid (ceil(E/16), ceil(B/8)): CTA (eg, tt) computes the logits of experts 16eg.. for tokens
// 8tt.. on the tensor cores.  The last CTA of a token tile (atomic ticket) picks the top-k of
// its 8 tokens, one warp per token; the last token tile to finish groups every pair by expert
// (a stable counting sort: tokens ascending within an expert) and writes the slot table that
// the later kernels walk.  No CTA waits on another: the tickets only elect who continues.
#include <math.h>

#include "kernels.h"
#include "tile.cuh"

namespace moe {
namespace {

constexpr size_t kRouterClusterPartBytes = 64 * 1024;  // partial logits of one cluster CTA

// Order key of (logit, expert): larger key = larger logit, then lower expert index; 0 = none.
__device__ __forceinline__ unsigned long long topk_key(float v, int e) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)e);
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  uint32_t u = (uint32_t)(k >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}

// Top-k of one token's logits (lg, shared memory) by one warp; writes topk_idx / topk_w.
// PER = logits per lane (E <= 32 * PER).  sv / si: this warp's k-entry scratch.  With roster
// routing the choice is by logit + bias (the bias row of the token's sequence), the weights come
// from the unbiased logits, and the sequence's counts of the chosen experts grow by one.
template <int PER>
__device__ void topk_token(const FwdParams& p, int tok, const float* lg, float* sv, int* si) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, k = p.k;
  const float* bias = p.router_bias ? p.router_bias + (size_t)tok * E : nullptr;
  unsigned long long key[PER];
  bool nan_seen = false;
  float mx = -INFINITY;  // largest unbiased logit (the softmax-over-all shift)
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    key[j] = 0ull;
    if (e < E) {
      float f = lg[e];
      if (isnan(f)) {
        nan_seen = true;
        f = -INFINITY;
      }
      mx = fmaxf(mx, f);
      if (bias) f = f + __ldg(bias + e);
      if (isnan(f)) f = -INFINITY;
      key[j] = topk_key(f, e);
    }
  }
  if (__any_sync(0xffffffffu, nan_seen) && lane == 0) set_error(p.err, kErrNanLogit);
  for (int r = 0; r < k; ++r) {
    unsigned long long best = key[0];
#pragma unroll
    for (int j = 1; j < PER; ++j) best = key[j] > best ? key[j] : best;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    const int e = (int)(0xFFFFFFFFu - (uint32_t)best);
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (lane + 32 * j == e) key[j] = 0ull;
    if (lane == 0) {
      si[r] = e;
      const float f = lg[e];
      sv[r] = isnan(f) ? -INFINITY : f;  // the unbiased logit of the chosen expert
    }
  }
  __syncwarp();
  // routing weights: lane r < k computes entry r.  The shift is the largest chosen logit
  // (softmax over the chosen) or the largest logit (softmax over all); without a bias both are
  // the first chosen logit.
  float z = 0.f;
  float m = sv[0];
  if (bias) {
    if (p.route == 1) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      m = mx;
    } else {
      for (int r = 1; r < k; ++r) m = fmaxf(m, sv[r]);
    }
  }
  if (p.route == 1) {
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane + 32 * j;
      if (e < E) {
        const float f = lg[e];
        z += expf((isnan(f) ? -INFINITY : f) - m);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  } else if (p.route == 0) {
    for (int r = 0; r < k; ++r) z += expf(sv[r] - m);
  }
  if (lane < k) {
    const float v = sv[lane];
    const float w = p.route == 2 ? 1.0f / (1.0f + expf(-v)) : expf(v - m) / z;
    p.topk_idx[(size_t)tok * k + lane] = si[lane];
    p.topk_w[(size_t)tok * k + lane] = w;
    if (p.roster_counts) p.roster_counts[(size_t)tok * E + si[lane]] += 1;
  }
}

// Exclusive prefix of a 64-bit value over the block; scratch holds 33 x 64 bits.
__device__ unsigned long long block_scan64(unsigned long long v, unsigned long long* scratch,
                                           unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const unsigned long long s = lane < nw ? scratch[lane] : 0ull;
    unsigned long long si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    if (lane < nw) scratch[lane] = si - s;
    if (lane == 31) scratch[32] = si;
  }
  __syncthreads();
  const unsigned long long res = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

// Groups all pairs by expert (tokens ascending within an expert) and writes the slot table,
// the pair arrays and meta (one CTA).  One 64-bit block scan over the experts gives, packed,
// each expert's first pair, its slot index and its first gate item.  Under expert parallelism
// only the routed experts [e_begin, e_end) and the shared experts of shared_mask are this
// handle's: the others get no slot, their pairs no pair index (pair_slot -1), and a slot names
// its routed expert by its index in the handle's local block of weights (e - e_begin).
__device__ void group_pairs(const FwdParams& p, uint32_t* dyn, unsigned long long* scratch) {
  const int B = p.B, E = p.E, k = p.k, S = p.S;
  const int W = (B + 31) / 32;
  int* cnt = reinterpret_cast<int*>(dyn);                          // [E]
  unsigned long long* pre = reinterpret_cast<unsigned long long*>(
      dyn + ((E + 1) & ~1));                                      // [E] packed prefixes
  uint32_t* tokmask = reinterpret_cast<uint32_t*>(pre + E);        // [E][W]
  int* sidx = reinterpret_cast<int*>(tokmask + E * W);             // [B*k]
  float* sw = reinterpret_cast<float*>(sidx + B * k);              // [B*k]
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) tokmask[i] = 0;
  for (int i = threadIdx.x; i < B * k; i += blockDim.x) {
    sidx[i] = ld_cg(&p.topk_idx[i]);
    sw[i] = ld_cg(&p.topk_w[i]);
  }
  __syncthreads();
  for (int pi = threadIdx.x; pi < B * k; pi += blockDim.x) {
    const int t = pi / k, e = sidx[pi];
    atomicAdd(&cnt[e], 1);
    atomicOr(&tokmask[e * W + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  // packed per local expert: pairs (bits 0..19) | touched (bits 20..31) | gate items (32..63)
  auto packed = [&](int e) -> unsigned long long {
    if (e < p.e_begin || e >= p.e_end) return 0ull;
    const unsigned long long c = (unsigned)cnt[e];
    // a dense slot (c >= dense_min) has no sparse gate items: the tensor-core path covers it
    const unsigned long long items =
        c && (int)c < p.dense_min
            ? (unsigned long long)(p.I / kTileRows) * ((c + kTileTok - 1) / kTileTok)
            : 0ull;
    return c | ((c ? 1ull : 0ull) << 20) | (items << 32);
  };
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
  unsigned long long mine = 0ull;
  for (int e = e0; e < e1; ++e) mine += packed(e);
  unsigned long long tot;
  unsigned long long run = block_scan64(mine, scratch, &tot);
  for (int e = e0; e < e1; ++e) {
    pre[e] = run;
    run += packed(e);
  }
  __syncthreads();
  const int n_local_pairs = (int)(tot & 0xFFFFF);
  const int n_touched = (int)((tot >> 20) & 0xFFF);
  const int routed_items = (int)(tot >> 32);
  const unsigned smask = p.shared_mask;
  const int n_shared_local = __popc(smask & ((1u << S) - 1u));
  // A sparse shared expert with at most kMaxSharedTiles token tiles has a slot per tile (each
  // with its own union); otherwise one slot for all B tokens.
  const int Bt = (B + kTileTok - 1) / kTileTok;
  const bool split = B < p.dense_min && Bt <= kMaxSharedTiles;
  const int sh_tiles = split ? Bt : 1;
  const int n_slots = n_touched + n_shared_local * sh_tiles;
  const int sh_items = B < p.dense_min ? (p.Ish / kTileRows) * (split ? 1 : Bt) : 0;  // per slot
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (cnt[e] > 0 && e >= p.e_begin && e < p.e_end) {
      const unsigned long long pr = pre[e];
      Slot s;
      s.kind = 0;
      s.expert = e - p.e_begin;
      s.T = cnt[e];
      s.q0 = (int)(pr & 0xFFFFF);
      s.I = p.I;
      s.item0 = (int)(pr >> 32);
      s.pad0 = s.pad1 = 0;
      p.slots[(int)((pr >> 20) & 0xFFF)] = s;
    }
  }
  // local shared expert s_i: first slot n_touched + sh_tiles (its rank among the local shared
  // experts); its tile tt is that slot + tt when split
  auto shared_slot = [&](int s_i) -> int {
    return ((smask >> s_i) & 1u) ? n_touched + sh_tiles * __popc(smask & ((1u << s_i) - 1u))
                                 : -1;
  };
  for (int i = threadIdx.x; i < S * sh_tiles; i += blockDim.x) {
    const int s_i = i / sh_tiles, tt = i % sh_tiles;
    const int j0 = shared_slot(s_i);
    if (j0 < 0) continue;
    const int j = j0 + tt;
    Slot s;
    s.kind = 1;
    s.expert = s_i;
    s.T = split ? min(kTileTok, B - tt * kTileTok) : B;
    s.q0 = B * k + s_i * B + tt * kTileTok;
    s.I = p.Ish;
    s.item0 = routed_items + (j - n_touched) * sh_items;
    s.pad0 = s.pad1 = 0;
    p.slots[j] = s;
  }
  // routed pairs: rank of token t among the tokens of its expert
  for (int pi = threadIdx.x; pi < B * k; pi += blockDim.x) {
    const int t = pi / k, e = sidx[pi];
    if (e < p.e_begin || e >= p.e_end) {
      p.pair_index[t * (k + S) + (pi % k)] = -1;
      continue;
    }
    int rank = __popc(tokmask[e * W + (t >> 5)] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(tokmask[e * W + w]);
    const unsigned long long pr = pre[e];
    const int q = (int)(pr & 0xFFFFF) + rank;
    p.pair_token[q] = t;
    p.pair_w[q] = sw[pi];
    p.pair_slot[q] = (int)((pr >> 20) & 0xFFF);
    p.pair_index[t * (k + S) + (pi % k)] = q;
  }
  // the routed pair indices past the local ones belong to no slot
  for (int q = n_local_pairs + threadIdx.x; q < B * k; q += blockDim.x) p.pair_slot[q] = -1;
  for (int i = threadIdx.x; i < B * S; i += blockDim.x) {
    const int s_i = i / B, t = i % B;
    const int q = B * k + s_i * B + t;
    const int j0 = shared_slot(s_i);
    const int j = j0 < 0 ? -1 : j0 + (split ? t / kTileTok : 0);
    p.pair_token[q] = t;
    p.pair_w[q] = 1.0f;
    p.pair_slot[q] = j;
    p.pair_index[t * (k + S) + k + s_i] = j < 0 ? -1 : q;
  }
  if (threadIdx.x == 0) {
    p.meta[kMetaSlots] = n_slots;
    p.meta[kMetaPairs] = B * (k + S);
    p.meta[kMetaGateItems] = routed_items + n_shared_local * sh_tiles * sh_items;
    p.meta[kMetaTouched] = n_touched;
  }
}

// Grid (egroups * hsplit, token tiles).  CTA (eg, hs, tt): partial logits of experts 16eg..
// over the hs-th slice of H for the 8 tokens of tile tt; the last CTA of the tile (ticket) sums
// the slices in a fixed order, picks the top-k, and the last tile groups the pairs.
template <typename T, int PER>
__global__ void __launch_bounds__(kThreads) router_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ const T* s_x[kTileTok];
  __shared__ int s_last;
  __shared__ unsigned long long scratch[33];
  __shared__ float s_lg[kTileTok][kMaxRouted];
  __shared__ float s_tv[kWarps][kMaxTopK];
  __shared__ int s_ti[kWarps][kMaxTopK];
  extern __shared__ uint32_t dyn[];
  pdl_trigger();
  trace_point(p.trace, 0, 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, E = p.E, B = p.B, hsplit = p.hsplit;
  const int eg = blockIdx.x / hsplit, hs = blockIdx.x % hsplit, tt = blockIdx.y;
  const int e0 = eg * kTileRows;
  const int nblk = H / 32;
  const int blo = hs * nblk / hsplit, bhi = (hs + 1) * nblk / hsplit;
  const T* x = static_cast<const T*>(p.x);
  const T* wr = static_cast<const T*>(p.router);
  if (threadIdx.x < kTileTok) {
    const int tok = tt * kTileTok + threadIdx.x;
    s_x[threadIdx.x] = tok < B ? x + (size_t)tok * H : nullptr;
  }
  __syncthreads();
  const T* rowA = wr + (size_t)min(e0 + g, E - 1) * H;
  const T* rowB = wr + (size_t)min(e0 + g + 8, E - 1) * H;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  tile_dot<4>(rowA, rowB, s_x, blo + warp, kWarps, bhi, d);
#pragma unroll
  for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
  __syncthreads();
  if (warp == 0) {
    reduce_fragments(red, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = e0 + g + (c >> 1) * 8;
      const int tok = tt * kTileTok + 2 * t + (c & 1);
      if (e < E && tok < B) p.logit_part[((size_t)hs * p.Bmax + tok) * E + e] = d[c];
    }
  }
  trace_point(p.trace, 0, 1);
  __threadfence();
  __syncthreads();
  trace_point(p.trace, 0, 2);
  if (threadIdx.x == 0) {
    const unsigned ticket = atomicAdd(&p.tile_ticket[tt], 1u);
    s_last = ticket == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // logits of the tile's tokens: the H slices summed in a fixed order
  bool nan_seen = false;
  for (int i = threadIdx.x; i < kTileTok * E; i += blockDim.x) {
    const int c = i / E, e = i % E, tok = tt * kTileTok + c;
    float v = 0.f;
    if (tok < B) {
      float pv[kMaxHsplit];  // all slices in flight at once, then summed in slice order
#pragma unroll
      for (int h = 0; h < kMaxHsplit; ++h)
        pv[h] = h < hsplit ? ld_cg(&p.logit_part[((size_t)h * p.Bmax + tok) * E + e]) : 0.f;
#pragma unroll
      for (int h = 0; h < kMaxHsplit; ++h) v += pv[h];
      p.logits[(size_t)tok * E + e] = v;
      nan_seen |= isnan(v);
    }
    s_lg[c][e] = v;
  }
  if (nan_seen) set_error(p.err, kErrNanLogit);
  __syncthreads();
  trace_point(p.trace, 0, 3);
  {
    const int tok = tt * kTileTok + warp;
    if (tok < B) topk_token<PER>(p, tok, s_lg[warp], s_tv[warp], s_ti[warp]);
  }
  trace_point(p.trace, 0, 4);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    p.tile_ticket[tt] = 0;
    const unsigned ticket = atomicAdd(p.global_ticket, 1u);
    s_last = ticket == gridDim.y - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  trace_point(p.trace, 0, 5);
  group_pairs(p, dyn, scratch);
  if (threadIdx.x == 0) *p.global_ticket = 0;
  trace_point(p.trace, 0, 6);
}

// ---- single-cluster variant for small batches ------------------------------------------------
// One thread-block cluster does the whole step: CTA r of the C CTAs computes the partial logits
// of every (expert, token) over the r-th slice of H into its own shared memory; after a cluster
// barrier each CTA sums, for its tokens (t = r, r + C, ...), the C partials in rank order through
// distributed shared memory, picks the top-k; after a second barrier CTA 0 groups the pairs.
// No global tickets, no fences between CTAs of different SMs' L1s, no second wave of loads.

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// f32 at the same shared-memory offset as `local`, in the shared memory of cluster CTA `rank`
// (no ordering constraint of its own: the cluster barrier before the reads orders them)
__device__ __forceinline__ float ld_dsmem(const float* local, uint32_t rank) {
  uint32_t ra;
  asm("mapa.shared::cluster.u32 %0, %1, %2;"
      : "=r"(ra)
      : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra));
  return v;
}
constexpr int kMaxClusterCtas = 16;

template <typename T, int PER>
__global__ void __launch_bounds__(kThreads) router_cluster_kernel(FwdParams p) {
  extern __shared__ uint32_t dyn[];  // partial logits [B][E], later group_pairs' scratch
  __shared__ const T* s_xt[kWarps][kTileTok];
  __shared__ unsigned long long scratch[33];
  __shared__ float s_lg[kWarps][kMaxRouted];
  __shared__ float s_tv[kWarps][kMaxTopK];
  __shared__ int s_ti[kWarps][kMaxTopK];
  pdl_trigger();  // the gate kernel may start its prologue now
  trace_point(p.trace, 0, 0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const uint32_t rank = cluster_rank(), C = cluster_size();
  const int H = p.H, E = p.E, B = p.B;
  const int nblk = H / 32;
  const int blo = (int)(rank * nblk / C), bhi = (int)((rank + 1) * nblk / C);
  const T* x = static_cast<const T*>(p.x);
  const T* wr = static_cast<const T*>(p.router);
  float* part = reinterpret_cast<float*>(dyn);
  const int etiles = (E + kTileRows - 1) / kTileRows, ttiles = (B + kTileTok - 1) / kTileTok;
  for (int tile = warp; tile < etiles * ttiles; tile += kWarps) {
    const int e0 = (tile % etiles) * kTileRows, t0 = (tile / etiles) * kTileTok;
    if (lane < kTileTok) s_xt[warp][lane] = t0 + lane < B ? x + (size_t)(t0 + lane) * H : nullptr;
    __syncwarp();
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    // every block of the CTA's slice of H in flight at once (up to 10 x 32 columns: one round
    // trip to HBM for H <= 5120 with 16 CTAs)
    tile_dot<10>(wr + (size_t)min(e0 + g, E - 1) * H, wr + (size_t)min(e0 + g + 8, E - 1) * H,
                s_xt[warp], blo, 1, bhi, d);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = e0 + g + (c >> 1) * 8, tok = t0 + 2 * t + (c & 1);
      if (e < E && tok < B) part[tok * E + e] = d[c];
    }
    __syncwarp();
  }
  trace_point(p.trace, 0, 1);
  cluster_sync_all();
  trace_point(p.trace, 0, 2);
  bool nan_seen = false;
  for (int i = warp;; i += kWarps) {
    const int tok = (int)rank + (int)C * i;
    if (tok >= B) break;
    for (int e = lane; e < E; e += 32) {
      float pv[kMaxClusterCtas];  // every rank's partial in flight, then summed in rank order
#pragma unroll
      for (uint32_t r = 0; r < kMaxClusterCtas; ++r)
        pv[r] = r < C ? ld_dsmem(&part[tok * E + e], r) : 0.f;
      float v = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxClusterCtas; ++r) v += pv[r];
      s_lg[warp][e] = v;
      p.logits[(size_t)tok * E + e] = v;
      nan_seen |= isnan(v);
    }
    __syncwarp();
    topk_token<PER>(p, tok, s_lg[warp], s_tv[warp], s_ti[warp]);
    __syncwarp();
  }
  if (nan_seen) set_error(p.err, kErrNanLogit);
  trace_point(p.trace, 0, 3);
  __threadfence();
  cluster_sync_all();  // every top-k is written; no CTA reads another's shared memory after this
  if (rank == 0) {
    trace_point(p.trace, 0, 5);
    group_pairs(p, dyn, scratch);
    trace_point(p.trace, 0, 6);
  }
}

}  // namespace

size_t router_smem_bytes(int E, int B) {
  const int W = (B + 31) / 32;
  // cnt [E] (padded to even) | packed prefixes [E] x 8 | tokmask [E][W] | topk idx, w [B*k]
  return sizeof(int) * (size_t)((E + 1) & ~1) + 8 * (size_t)E + 4 * (size_t)E * W +
         (size_t)B * kMaxTopK * 8;
}

// H slices of the router: enough CTAs to keep ~96 in flight, at least 2 blocks of 32 per slice.
int router_hsplit(int E, int B, int H) {
  const int ctas = ((E + kTileRows - 1) / kTileRows) * ((B + kTileTok - 1) / kTileTok);
  int hs = (96 + ctas - 1) / ctas;
  const int cap = H / 64;
  if (hs > cap) hs = cap;
  if (hs > kMaxHsplit) hs = kMaxHsplit;
  return hs < 1 ? 1 : hs;
}

template <typename T>
cudaError_t launch_router_t(const FwdParams& p, dim3 grid, size_t smem, cudaStream_t st) {
  if (p.E <= 32) return launch_pdl(router_kernel<T, 1>, grid, dim3(kThreads), smem, st, false, p);
  if (p.E <= 64) return launch_pdl(router_kernel<T, 2>, grid, dim3(kThreads), smem, st, false, p);
  if (p.E <= 128) return launch_pdl(router_kernel<T, 4>, grid, dim3(kThreads), smem, st, false, p);
  if (p.E <= 256) return launch_pdl(router_kernel<T, 8>, grid, dim3(kThreads), smem, st, false, p);
  return launch_pdl(router_kernel<T, 16>, grid, dim3(kThreads), smem, st, false, p);
}

// The single-cluster router holds the batch's partial logits in each CTA's shared memory, and
// one of its CTAs groups all B k pairs.  Measured on B200 (OLMoE shape, 256 tokens: 64 KB of
// partials, 2048 pairs) it took 43 us where the multi-CTA router takes 23 us, so it is used up to
// half of its shared-memory room.
constexpr size_t kRouterClusterUseBytes = kRouterClusterPartBytes / 2;
bool router_uses_cluster(int cluster, int E, int B) {
  return cluster > 0 && (size_t)E * B * 4 <= kRouterClusterUseBytes;
}

template <typename T, int PER>
cudaError_t launch_router_cluster_t(const FwdParams& p, size_t smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.router_cluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.router_cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_cluster_kernel<T, PER>, p);
}

template <typename T>
cudaError_t launch_router_cluster(const FwdParams& p, cudaStream_t st) {
  const size_t part = (size_t)p.E * p.B * 4, grp = router_smem_bytes(p.E, p.B);
  const size_t smem = part > grp ? part : grp;
  if (p.E <= 32) return launch_router_cluster_t<T, 1>(p, smem, st);
  if (p.E <= 64) return launch_router_cluster_t<T, 2>(p, smem, st);
  if (p.E <= 128) return launch_router_cluster_t<T, 4>(p, smem, st);
  if (p.E <= 256) return launch_router_cluster_t<T, 8>(p, smem, st);
  return launch_router_cluster_t<T, 16>(p, smem, st);
}

cudaError_t launch_router(const FwdParams& p, int dtype, cudaStream_t st) {
  if (router_uses_cluster(p.router_cluster, p.E, p.B))
    return dtype == 0 ? launch_router_cluster<__nv_bfloat16>(p, st)
                      : launch_router_cluster<float>(p, st);
  dim3 grid(((p.E + kTileRows - 1) / kTileRows) * p.hsplit, (p.B + kTileTok - 1) / kTileTok);
  const size_t smem = router_smem_bytes(p.E, p.B);
  if (dtype == 0) return launch_router_t<__nv_bfloat16>(p, grid, smem, st);
  return launch_router_t<float>(p, grid, smem, st);
}

template <typename T>
cudaError_t configure_router_t(int budget) {
  cudaError_t e = allow_max_smem(router_kernel<T, 1>, budget);
  if (e == cudaSuccess) e = allow_max_smem(router_kernel<T, 2>, budget);
  if (e == cudaSuccess) e = allow_max_smem(router_kernel<T, 4>, budget);
  if (e == cudaSuccess) e = allow_max_smem(router_kernel<T, 8>, budget);
  if (e == cudaSuccess) e = allow_max_smem(router_kernel<T, 16>, budget);
  return e;
}

template <typename T>
cudaError_t configure_router_cluster_t(int budget, bool wide) {
  cudaError_t e = cudaSuccess;
  auto one = [&](auto kernel) {
    if (e != cudaSuccess) return;
    e = allow_max_smem(kernel, budget);
    if (e == cudaSuccess && wide)
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  };
  one(router_cluster_kernel<T, 1>);
  one(router_cluster_kernel<T, 2>);
  one(router_cluster_kernel<T, 4>);
  one(router_cluster_kernel<T, 8>);
  one(router_cluster_kernel<T, 16>);
  return e;
}

// Shared-memory limits of every router kernel and, for the single-cluster router, the widest
// cluster the device accepts (16 CTAs where allowed, else 8; 0: only the multi-CTA router).
// Function attributes belong to the current device's context, so this runs for every handle
// and every context (the caller holds the set-up lock); the width found is kept per context.
cudaError_t configure_router(int budget, int* cluster_out) {
  cudaError_t e = configure_router_t<__nv_bfloat16>(budget);
  if (e != cudaSuccess) return e;
  e = configure_router_t<float>(budget);
  if (e != cudaSuccess) return e;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static unsigned long long known_ctx[kMaxDevices];
  static int known_width[kMaxDevices];
  const unsigned long long ctx = current_context_id();
  if (dev >= 0 && dev < kMaxDevices && ctx != 0 && known_ctx[dev] == ctx) {
    const int c = known_width[dev];
    if (c > 0 && (configure_router_cluster_t<__nv_bfloat16>(budget, c > 8) != cudaSuccess ||
                  configure_router_cluster_t<float>(budget, c > 8) != cudaSuccess))
      return cudaErrorInvalidConfiguration;
    *cluster_out = c;
    return cudaSuccess;
  }
  int c = 0;
  for (int want : {16, 8}) {
    if (configure_router_cluster_t<__nv_bfloat16>(budget, want > 8) != cudaSuccess ||
        configure_router_cluster_t<float>(budget, want > 8) != cudaSuccess)
      continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(want);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kRouterClusterPartBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = want;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, router_cluster_kernel<__nv_bfloat16, 16>, &cfg) ==
            cudaSuccess &&
        n > 0) {
      c = want;
      break;
    }
  }
  cudaGetLastError();  // a refused cluster width is not an error of this call
  if (dev >= 0 && dev < kMaxDevices && ctx != 0) {
    known_ctx[dev] = ctx;
    known_width[dev] = c;
  }
  *cluster_out = c;
  return cudaSuccess;
}

}  // namespace moe
