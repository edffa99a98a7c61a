// misc.cu - output cast, weight packing, debug export and per-handle kernel configuration.
#include <cuda.h>

#include "kernels.h"
#include "tma.cuh"

namespace moe {

cudaError_t configure_select(int imax, int budget, int* occupancy);
cudaError_t configure_gate(int dtype, int H, int smem_budget, LaunchShape* ls);
cudaError_t configure_updown(int dtype, int H, int smem_budget, LaunchShape* ls);

namespace {

// out[t][h] = dtype(out_acc[t][h]); out_acc is cleared for the next call.
template <typename T>
__global__ void finalize_kernel(FwdParams p) {
  pdl_trigger();
  trace_point(p.trace, 4, 0);
  pdl_wait();
  trace_point(p.trace, 4, 1);
  if (blockIdx.x == 0 && threadIdx.x < 3) p.claim[threadIdx.x] = 0;  // work counters, next call
  // the fused layer kernel's readiness state, for the next call
  const int n_pairs = p.B * (p.k + p.S);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_pairs; i += gridDim.x * blockDim.x) {
    p.tile_done[i] = 0;
    p.s_task[i] = 0;
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < slot_capacity(p.E, p.S);
       i += gridDim.x * blockDim.x)
    p.u_ent[i] = make_int4(0, 0, 0, 0);
  if (blockIdx.x == 0 && threadIdx.x < 4) p.fq[threadIdx.x] = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.u_res = 0ull;
  const size_t n4 = (size_t)p.B * p.H / 4;
  float4* acc = reinterpret_cast<float4*>(p.out_acc);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = __ldcg(acc + i);
    acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (sizeof(T) == 2) {
      uint2 o;
      o.x = pack_bf16x2(v.x, v.y);
      o.y = pack_bf16x2(v.z, v.w);
      reinterpret_cast<uint2*>(p.out)[i] = o;
    } else {
      reinterpret_cast<float4*>(p.out)[i] = v;
    }
  }
}

// Roster routing bias ("Predatory MoE", technical summary, Methodology 2): one CTA per sequence
// t.  The roster is the m experts with the most selections so far (equal counts: lower index),
// found by each expert's rank among the counts.  bias[t][e] = 0 while fewer than m distinct
// experts have been used; then +delta for roster members and -delta for the others; for a
// pinned sequence 0 for members and -inf for the others.
__global__ void roster_bias_kernel(const int* __restrict__ counts, const int* __restrict__ pinned,
                                   int E, int m, float delta, float* __restrict__ bias) {
  __shared__ int c[kMaxRouted];
  __shared__ int s_distinct;
  const int t = blockIdx.x;
  if (threadIdx.x == 0) s_distinct = 0;
  __syncthreads();
  int mine = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    c[e] = counts[(size_t)t * E + e];
    mine += c[e] > 0;
  }
  if (mine) atomicAdd(&s_distinct, mine);
  __syncthreads();
  const bool pin = pinned[t] != 0;
  const bool explore = s_distinct < m;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int ce = c[e];
    int rank = 0;
    for (int f = 0; f < E; ++f) rank += c[f] > ce || (c[f] == ce && f < e);
    const bool member = rank < m;
    float b;
    if (pin) b = member ? 0.f : -INFINITY;
    else if (explore) b = 0.f;
    else b = member ? delta : -delta;
    bias[(size_t)t * E + e] = b;
  }
}

// out[i] = dtype(sum[i]): the layer output from the sum of the partial outputs of all handles
// (expert parallelism).
template <typename T>
__global__ void cast_output_kernel(const float* __restrict__ sum, T* __restrict__ out, size_t n4) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(sum)[i];
    if constexpr (sizeof(T) == 2) {
      uint2 o;
      o.x = pack_bf16x2(v.x, v.y);
      o.y = pack_bf16x2(v.z, v.w);
      reinterpret_cast<uint2*>(out)[i] = o;
    } else {
      reinterpret_cast<float4*>(out)[i] = v;
    }
  }
}

// packed[e][n][1][h] = w_down[e][h][n]: 32x32 tiles through shared memory.
template <typename T>
__global__ void pack_down_kernel(const T* __restrict__ wd, T* __restrict__ ud, int I, int H) {
  __shared__ T tile[32][33];
  const int e = blockIdx.z;
  const int n0 = blockIdx.x * 32, h0 = blockIdx.y * 32;
  const T* src = wd + (size_t)e * H * I;
  T* dst = ud + (size_t)e * I * 2 * H;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int h = h0 + r, n = n0 + threadIdx.x;
    if (h < H && n < I) tile[r][threadIdx.x] = src[(size_t)h * I + n];
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int n = n0 + r, h = h0 + threadIdx.x;
    if (h < H && n < I) dst[(size_t)n * 2 * H + H + h] = tile[threadIdx.x][r];
  }
}

// Reorders the last call's per-pair results into [token][pair] order for export: the kept
// neurons as an ascending index list (from the pair's mask row; -1 after the last) and their
// count, and the activations.  One CTA per (token, pair); warp 0 writes the list.
__global__ void debug_gather_kernel(FwdParams p, int* cnt, int* lists, float* act) {
  const int P = p.k + p.S;
  const int tj = blockIdx.x;  // token * P + pair
  const int t = tj / P, jj = tj % P;
  const int q = p.pair_index[t * P + jj];
  const int I = jj < p.k ? p.I : p.Ish;
  const int lane = threadIdx.x & 31;
  if (q < 0) {  // an expert another handle evaluates: no kept neuron, no activation here
    for (int n = threadIdx.x; n < p.Imax; n += blockDim.x) {
      if (lists) lists[(size_t)tj * p.Imax + n] = -1;
      if (act) act[(size_t)tj * p.Imax + n] = 0.f;
    }
    if (threadIdx.x == 0 && cnt) cnt[tj] = 0;
    return;
  }
  const uint32_t* mrow = p.maskbits + (size_t)q * (p.Imax / 32);
  if (threadIdx.x < 32) {
    const int W = I / 32, wpl = (W + 31) / 32;
    const int w0 = min(W, lane * wpl), w1 = min(W, w0 + wpl);
    int c = 0;
    for (int w = w0; w < w1; ++w) c += __popc(mrow[w]);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - c;
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (lists) {
      int* out = lists + (size_t)tj * p.Imax;
      for (int w = w0; w < w1; ++w) {
        uint32_t b = mrow[w];
        while (b) {
          out[pos++] = w * 32 + __ffs(b) - 1;
          b &= b - 1;
        }
      }
      for (int n = total + lane; n < p.Imax; n += 32) out[n] = -1;
    }
    if (lane == 0 && cnt) cnt[tj] = total;
  }
  if (act)
    for (int n = threadIdx.x; n < p.Imax; n += blockDim.x)
      act[(size_t)tj * p.Imax + n] = n < I ? p.act[(size_t)q * p.Imax + n] : 0.f;
}

}  // namespace

cudaError_t launch_finalize(const FwdParams& p, int dtype, const LaunchShape& ls, cudaStream_t st,
                            bool pdl) {
  const size_t n4 = (size_t)p.B * p.H / 4;
  size_t blocks = (n4 + 255) / 256;
  const size_t cap = (size_t)ls.nsm * 4;
  if (blocks > cap) blocks = cap;
  if (dtype == 0)
    return launch_pdl(finalize_kernel<__nv_bfloat16>, dim3((unsigned)blocks), dim3(256), 0, st,
                      pdl, p);
  return launch_pdl(finalize_kernel<float>, dim3((unsigned)blocks), dim3(256), 0, st, pdl, p);
}

cudaError_t launch_pack_down(const void* w_down, void* packed_updown, int n, int I, int H,
                             int elt, cudaStream_t st) {
  dim3 grid((I + 31) / 32, (H + 31) / 32, n), block(32, 8);
  if (elt == 2)
    pack_down_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w_down), static_cast<__nv_bfloat16*>(packed_updown), I,
        H);
  else
    pack_down_kernel<float><<<grid, block, 0, st>>>(static_cast<const float*>(w_down),
                                                    static_cast<float*>(packed_updown), I, H);
  return cudaGetLastError();
}

// Failure-detection hook: one warp waits, with the same bounded wait as the ring kernels, on an
// mbarrier that nothing ever completes.  The wait gives up after its time limit, sets the error
// word (timeout) and the kernel returns: the path that a stalled pipeline takes, exercised
// without a stalled pipeline.
__global__ void force_timeout_kernel(FwdParams p) {
  __shared__ uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    s_abort = 0;
    mbar_init_fence();
  }
  __syncwarp();
  volatile int* abort = &s_abort;
  if (threadIdx.x == 0) mbar_wait(&bar, 0, abort, p.err);  // phase 0 never completes
}

cudaError_t launch_cast_output(const float* sum, void* out, size_t n, int dtype, int nsm,
                               cudaStream_t st) {
  const size_t n4 = n / 4;
  size_t blocks = (n4 + 255) / 256;
  if (blocks > (size_t)nsm * 4) blocks = (size_t)nsm * 4;
  if (blocks == 0) return cudaSuccess;
  if (dtype == 0)
    cast_output_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
        sum, static_cast<__nv_bfloat16*>(out), n4);
  else
    cast_output_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(sum, static_cast<float*>(out), n4);
  return cudaGetLastError();
}

cudaError_t launch_roster_bias(const int* counts, const int* pinned, int B, int E, int m,
                               float delta, float* bias, cudaStream_t st) {
  roster_bias_kernel<<<B, 128, 0, st>>>(counts, pinned, E, m, delta, bias);
  return cudaGetLastError();
}

cudaError_t launch_force_timeout(const FwdParams& p, cudaStream_t st) {
  force_timeout_kernel<<<1, 32, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_debug_gather(const FwdParams& p, int n_tokens, int* cnt, int* lists,
                                float* act, cudaStream_t st) {
  const int P = p.k + p.S;
  debug_gather_kernel<<<n_tokens * P, 256, 0, st>>>(p, cnt, lists, act);
  return cudaGetLastError();
}

std::mutex& setup_mutex() {
  static std::mutex mu;
  return mu;
}

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

cudaError_t configure_kernels(int dtype, int imax, int n_slot_max, int max_B, int H, LaunchShape* ls) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&ls->nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  int budget = 0;
  e = cudaDeviceGetAttribute(&budget, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  e = configure_router(budget, &ls->router_cluster);
  if (e != cudaSuccess) return e;
  int occ_sel = 0;
  e = configure_select(imax, budget, &occ_sel);
  if (e != cudaSuccess) return e;
  ls->grid_select = ls->nsm * (occ_sel > 0 ? occ_sel : 1);
  e = configure_gate(dtype, H, budget, ls);
  if (e != cudaSuccess) return e;
  e = configure_updown(dtype, H, budget, ls);
  if (e != cudaSuccess) return e;
  if (dtype == 0) {
    e = configure_dense(budget);
    if (e != cudaSuccess) return e;
    e = configure_layer(H, imax, n_slot_max, budget, ls);
    if (e != cudaSuccess) return e;
  } else {
    ls->ring_layer.ns = 0;
  }
  return cudaGetLastError();
}

}  // namespace moe
