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

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

// Top-k of one token's logits by one warp; writes topk_idx / topk_w.
__device__ void topk_token(const FwdParams& p, int tok) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, k = p.k;
  constexpr int kPer = kMaxRouted / 32;
  float v[kPer];
  bool nan_seen = false;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = lane + 32 * j;
    float f = -INFINITY;
    if (e < E) {
      f = ld_cg(&p.logits[(size_t)tok * E + e]);
      if (isnan(f)) {
        nan_seen = true;
        f = -INFINITY;
      }
    }
    v[j] = f;
  }
  if (__any_sync(0xffffffffu, nan_seen) && lane == 0) set_error(p.err, kErrNanLogit);
  unsigned taken = 0;
  float sel_v[kMaxTopK];
  int sel_e[kMaxTopK];
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    sel_v[r] = -INFINITY;
    sel_e[r] = 0;
    if (r < k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((taken >> j) & 1u) && better(v[j], e, bv, be)) {
          bv = v[j];
          be = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (better(ov, oe, bv, be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      sel_v[r] = bv;
      sel_e[r] = be;
    }
  }
  float w[kMaxTopK];
  if (p.route == 2) {
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) w[r] = 1.0f / (1.0f + expf(-sel_v[r]));
  } else {
    const float m = sel_v[0];
    float z = 0.f;
    if (p.route == 1) {
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (lane + 32 * j < E) z += expf(v[j] - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    } else {
#pragma unroll
      for (int r = 0; r < kMaxTopK; ++r)
        if (r < k) z += expf(sel_v[r] - m);
    }
#pragma unroll
    for (int r = 0; r < kMaxTopK; ++r) w[r] = expf(sel_v[r] - m) / z;
  }
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < k && lane == r) {
      p.topk_idx[(size_t)tok * k + r] = sel_e[r];
      p.topk_w[(size_t)tok * k + r] = w[r];
    }
  }
}

// Exclusive scan of n ints in place (shared memory), by the whole block; returns the total.
__device__ int block_scan_array(int* a, int n, int* scratch) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, (int)threadIdx.x * per), end = min(n, beg + per);
  int s = 0;
  for (int i = beg; i < end; ++i) s += a[i];
  int total;
  int run = block_exclusive_scan(s, scratch, &total);
  for (int i = beg; i < end; ++i) {
    const int v = a[i];
    a[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

// Groups all pairs by expert and writes the slot table, pair arrays and meta (one CTA).
__device__ void group_pairs(const FwdParams& p, uint32_t* dyn, int* scratch) {
  const int B = p.B, E = p.E, k = p.k, S = p.S;
  const int W = (B + 31) / 32;
  int* cnt = reinterpret_cast<int*>(dyn);  // [E]
  int* qoff = cnt + E;                     // [E] exclusive prefix of cnt
  int* touched = qoff + E;                 // [E] -> slot index after the scan
  int* items = touched + E;                // [E + S] gate items per slot -> item0
  uint32_t* tokmask = reinterpret_cast<uint32_t*>(items + E + S);  // [E][W]
  for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
  for (int i = threadIdx.x; i < E * W; i += blockDim.x) tokmask[i] = 0;
  __syncthreads();
  for (int pi = threadIdx.x; pi < B * k; pi += blockDim.x) {
    const int t = pi / k;
    const int e = ld_cg(&p.topk_idx[pi]);
    atomicAdd(&cnt[e], 1);
    atomicOr(&tokmask[e * W + (t >> 5)], 1u << (t & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    qoff[e] = cnt[e];
    touched[e] = cnt[e] > 0 ? 1 : 0;
  }
  __syncthreads();
  block_scan_array(qoff, E, scratch);
  const int n_touched = block_scan_array(touched, E, scratch);
  const int n_slots = n_touched + S;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (cnt[e] > 0) {
      Slot s;
      s.kind = 0;
      s.expert = e;
      s.T = cnt[e];
      s.q0 = qoff[e];
      s.I = p.I;
      s.item0 = 0;
      s.pad0 = s.pad1 = 0;
      p.slots[touched[e]] = s;
      items[touched[e]] = (p.I / kTileRows) * ((cnt[e] + kTileTok - 1) / kTileTok);
    }
  }
  for (int s_i = threadIdx.x; s_i < S; s_i += blockDim.x) {
    Slot s;
    s.kind = 1;
    s.expert = s_i;
    s.T = B;
    s.q0 = B * k + s_i * B;
    s.I = p.Ish;
    s.item0 = 0;
    s.pad0 = s.pad1 = 0;
    p.slots[n_touched + s_i] = s;
    items[n_touched + s_i] = (p.Ish / kTileRows) * ((B + kTileTok - 1) / kTileTok);
  }
  // routed pairs: rank of token t among the tokens of its expert
  for (int pi = threadIdx.x; pi < B * k; pi += blockDim.x) {
    const int t = pi / k;
    const int e = ld_cg(&p.topk_idx[pi]);
    int rank = __popc(tokmask[e * W + (t >> 5)] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(tokmask[e * W + w]);
    const int q = qoff[e] + rank;
    p.pair_token[q] = t;
    p.pair_w[q] = ld_cg(&p.topk_w[pi]);
    p.pair_slot[q] = touched[e];
    p.pair_index[t * (k + S) + (pi % k)] = q;
  }
  for (int i = threadIdx.x; i < B * S; i += blockDim.x) {
    const int s_i = i / B, t = i % B;
    const int q = B * k + s_i * B + t;
    p.pair_token[q] = t;
    p.pair_w[q] = 1.0f;
    p.pair_slot[q] = n_touched + s_i;
    p.pair_index[t * (k + S) + k + s_i] = q;
  }
  __syncthreads();
  const int n_items = block_scan_array(items, n_slots, scratch);
  for (int j = threadIdx.x; j < n_slots; j += blockDim.x) p.slots[j].item0 = items[j];
  if (threadIdx.x == 0) {
    p.meta[kMetaSlots] = n_slots;
    p.meta[kMetaPairs] = B * (k + S);
    p.meta[kMetaGateItems] = n_items;
    p.meta[kMetaTouched] = n_touched;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) router_kernel(FwdParams p) {
  __shared__ float red[kWarps][32][4];
  __shared__ const T* s_x[kTileTok];
  __shared__ int s_last;
  __shared__ int scratch[33];
  extern __shared__ uint32_t dyn[];
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int H = p.H, E = p.E, B = p.B;
  const int e0 = blockIdx.x * kTileRows, tt = blockIdx.y;
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
  tile_dot<2>(rowA, rowB, s_x, warp, kWarps, H / 32, d);
#pragma unroll
  for (int c = 0; c < 4; ++c) red[warp][lane][c] = d[c];
  __syncthreads();
  if (warp == 0) {
    reduce_fragments(red, d);
    bool nan_seen = false;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = e0 + g + (c >> 1) * 8;
      const int tok = tt * kTileTok + 2 * t + (c & 1);
      if (e < E && tok < B) {
        p.logits[(size_t)tok * E + e] = d[c];
        nan_seen |= isnan(d[c]);
      }
    }
    if (nan_seen) set_error(p.err, kErrNanLogit);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned ticket = atomicAdd(&p.tile_ticket[tt], 1u);
    s_last = ticket == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  {
    const int tok = tt * kTileTok + warp;
    if (tok < B) topk_token(p, tok);
  }
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
  group_pairs(p, dyn, scratch);
  if (threadIdx.x == 0) *p.global_ticket = 0;
}

}  // namespace

size_t router_smem_bytes(int E, int B) {
  const int W = (B + 31) / 32;
  return sizeof(int) * (size_t)(3 * E + E + kMaxShared) + sizeof(uint32_t) * (size_t)E * W;
}

cudaError_t launch_router(const FwdParams& p, int dtype, cudaStream_t st) {
  dim3 grid((p.E + kTileRows - 1) / kTileRows, (p.B + kTileTok - 1) / kTileTok);
  const size_t smem = router_smem_bytes(p.E, p.B);
  if (dtype == 0)
    return launch_pdl(router_kernel<__nv_bfloat16>, grid, dim3(kThreads), smem, st, false, p);
  return launch_pdl(router_kernel<float>, grid, dim3(kThreads), smem, st, false, p);
}

cudaError_t configure_router(int max_E, int max_B) {
  const size_t smem = router_smem_bytes(max_E, max_B);
  cudaError_t e = cudaFuncSetAttribute(router_kernel<__nv_bfloat16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(router_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem);
}

}  // namespace moe
