// route_noalloc.cu - routing only (router logits, top-k experts, routing weights) for one batch,
// with no handle and no device allocation.
//
// Who calls it.  moe_create allocates the whole layer workspace.  Some callers need only the
// expert choice of each token, and cannot allocate device memory where they ask for it:
//   - a scheduler that prefetches or places experts from the next batch's routing, running
//     while a caching allocator has reserved all free device memory (a cudaMalloc there would
//     fail, or force the allocator to release and fragment its pool);
//   - code that must not change the device's memory footprint, such as a memory-budgeted
//     service whose footprint was measured at start-up.
// For them this entry point runs the router kernel of the layer (logit tiles, top-k, grouping)
// on a fixed scratch area compiled into the library, instead of a handle's workspace.
//
// The scratch area is one static device array, which every device that loads the library
// holds until the process exits.  The first call in a device's CUDA context looks up the array's
// address there (cudaGetSymbolAddress, which may load the module) and sets the router kernels'
// limits; that first call should therefore come before any stream capture.  A later call checks
// that the context is still the one set up (a device reset ends a context; the call after it
// sets up again), clears the zero-at-start words and launches.  Calls that overlap in time on
// one device, from two streams or two threads, share the scratch area and race: the caller
// serialises them.
#include <climits>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = (size_t)2 << 20;  // 2 MiB: room for 256 tokens x 512 experts
constexpr int kNoAllocMaxTokens = 256;

// The scratch area (zero at module load; the zero-at-start words are cleared again by every call).
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

// per device: the context that was set up, the scratch area's address there and the width of
// the single-cluster router (ctx 0 = not set up yet)
struct DeviceSetup {
  unsigned long long ctx;
  void* scratch;
  int router_cluster;
};
DeviceSetup g_setup[moe::kMaxDevices];

// The scratch area's address and the router's cluster width for the current device, set up
// once per device context with that device current.  Returns false (with *err set) on failure.
bool setup_current_device(void** scratch, int* cluster, cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return false;
  if (dev < 0 || dev >= moe::kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return false;
  }
  std::lock_guard<std::mutex> lock(moe::setup_mutex());
  // the context identity is read after the first runtime call, so the context exists
  const unsigned long long ctx = moe::current_context_id();
  DeviceSetup& d = g_setup[dev];
  if (ctx == 0 || d.ctx != ctx) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_route_scratch);
    if (*err != cudaSuccess || !ptr) {
      if (*err == cudaSuccess) *err = cudaErrorInvalidSymbol;
      return false;
    }
    int budget = 0;
    *err = cudaDeviceGetAttribute(&budget, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (*err != cudaSuccess) return false;
    int c = 0;
    *err = moe::configure_router(budget, &c);
    if (*err != cudaSuccess) return false;
    d.scratch = ptr;
    d.router_cluster = c;
    d.ctx = ctx;  // 0 when the identity cannot be read: set up again on every call
  }
  *scratch = d.scratch;
  *cluster = d.router_cluster;
  return true;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_config* cfg, const void* x, int n_tokens,
                                        const void* router, int* topk_idx, float* topk_w,
                                        void* stream) {
  if (!cfg) return MOE_ERR_INVALID_ARG;
  if (cfg->dtype != MOE_BF16 && cfg->dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (cfg->route < MOE_ROUTE_SOFTMAX_TOPK || cfg->route > MOE_ROUTE_SIGMOID)
    return MOE_ERR_INVALID_ARG;
  if (cfg->hidden <= 0 || cfg->n_routed <= 0 || cfg->top_k <= 0 || cfg->top_k > cfg->n_routed)
    return MOE_ERR_INVALID_ARG;
  if (cfg->hidden % 64 || cfg->hidden > 8192 || cfg->n_routed > moe::kMaxRouted ||
      cfg->top_k > moe::kMaxTopK)
    return MOE_ERR_UNSUPPORTED;
  if (n_tokens < 0) return MOE_ERR_INVALID_ARG;
  if (n_tokens > kNoAllocMaxTokens) return MOE_ERR_UNSUPPORTED;  // beyond the scratch area
  if (n_tokens == 0) return MOE_OK;
  if (!x || !router || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(router)) & 15u)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(topk_idx) | reinterpret_cast<uintptr_t>(topk_w)) & 3u)
    return MOE_ERR_INVALID_ARG;

  const int B = n_tokens, E = cfg->n_routed, k = cfg->top_k, H = cfg->hidden;
  const int hsplit = moe::router_hsplit(E, B, H);
  const int tiles = (B + moe::kTileTok - 1) / moe::kTileTok;
  // scratch layout: everything the router kernel writes, then the words that start at zero
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t o_logits = take(sizeof(float) * B * E);
  const size_t o_part = take(sizeof(float) * hsplit * B * E);
  const size_t o_pidx = take(sizeof(int) * B * k);
  const size_t o_ptok = take(sizeof(int) * B * k);
  const size_t o_pw = take(sizeof(float) * B * k);
  const size_t o_pslot = take(sizeof(int) * B * k);
  const size_t o_slots = take(sizeof(moe::Slot) * E);
  const size_t o_meta = take(sizeof(int) * moe::kMetaWords);
  const size_t o_zero = off;  // tile tickets, the batch ticket and the error word start at zero
  const size_t o_tick = take(sizeof(unsigned) * tiles);
  const size_t o_gtick = take(sizeof(unsigned));
  const size_t o_err = take(sizeof(int));
  const size_t zero_bytes = off - o_zero;
  if (off > kScratchBytes) return MOE_ERR_UNSUPPORTED;

  cudaError_t ce = cudaSuccess;
  void* scratch = nullptr;
  int cluster = 0;
  if (!setup_current_device(&scratch, &cluster, &ce)) return MOE_ERR_CUDA;
  char* base = static_cast<char*>(scratch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(base + o_zero, 0, zero_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;

  moe::FwdParams p = {};
  p.H = H;
  p.E = E;
  p.k = k;
  p.S = 0;
  p.I = moe::kTileRows;  // the grouping phase counts gate items; no later kernel reads them
  p.Ish = moe::kTileRows;
  p.B = B;
  p.Imax = moe::kTileRows;
  p.Bmax = B;
  p.hsplit = hsplit;
  p.router_cluster = cluster;
  p.route = (int)cfg->route;
  p.dense_min = INT_MAX;  // only the grouping's item counts read it; no later kernel runs
  p.e_begin = 0;
  p.e_end = E;
  p.shared_mask = 0;
  p.x = x;
  p.router = router;
  p.logits = reinterpret_cast<float*>(base + o_logits);
  p.logit_part = reinterpret_cast<float*>(base + o_part);
  p.topk_idx = topk_idx;
  p.topk_w = topk_w;
  p.pair_index = reinterpret_cast<int*>(base + o_pidx);
  p.pair_token = reinterpret_cast<int*>(base + o_ptok);
  p.pair_w = reinterpret_cast<float*>(base + o_pw);
  p.pair_slot = reinterpret_cast<int*>(base + o_pslot);
  p.slots = reinterpret_cast<moe::Slot*>(base + o_slots);
  p.meta = reinterpret_cast<int*>(base + o_meta);
  p.tile_ticket = reinterpret_cast<unsigned*>(base + o_tick);
  p.global_ticket = reinterpret_cast<unsigned*>(base + o_gtick);
  p.err = reinterpret_cast<int*>(base + o_err);
  p.trace = nullptr;
  return moe::launch_router(p, cfg->dtype == MOE_BF16 ? 0 : 1, st) == cudaSuccess ? MOE_OK
                                                                                  : MOE_ERR_CUDA;
}
