// moe_api.cu - the C ABI declared in include/moe.h: argument checks, the workspace, packing,
// and the launch sequence of one layer call.
//
// One call runs five kernels on the caller's stream, each (after the first) launched with
// programmatic dependent launch so that it is resident before its predecessor drains:
//   router   logits, top-k, routing weights, pair grouping and slot table
//   gate     dense gate + SiLU of every evaluated pair
//   select   per-pair kept set, per-expert union of kept neurons
//   updown   sparse up/down over the kept rows, weighted into an fp32 accumulator
//   finalize accumulator -> out (dtype), accumulator cleared
// Nothing is allocated and nothing waits on the host, so a call can be captured in a graph.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include <climits>

#include "../../include/moe.h"
#include "kernels.h"
#include "tma.cuh"

using moe::FwdParams;
using moe::LaunchShape;

struct moe_handle {
  moe_config cfg;
  int device;
  int elt;
  int imax;
  LaunchShape ls;
  FwdParams base;  // workspace pointers and sizes
  void* ws;
  size_t ws_bytes;
  void* zero_begin;  // [zero_begin, zero_begin + zero_bytes) is all-zero between calls
  size_t zero_bytes;
  void* x_stage;    // device staging of moe_forward_host
  void* out_stage;
  bool dirty;       // a call failed mid-way: re-zero before the next one
  int last_tokens;
  int last_launches;  // kernels the last moe_forward launched
  cudaEvent_t stage_events[MOE_STAGE_EVENTS];
  bool timing;
  int dense_min;  // MOE_DENSE_AUTO, 0 (never dense) or a per-slot token threshold
  unsigned long long* trace_buf;  // device, kTraceKernels * kTraceCtas * kTracePoints stamps
  float* roster_bias;  // device [max_tokens][E]: the roster bias of the current call
  int e_begin, e_end;     // routed experts this handle evaluates (all by default)
  unsigned shared_mask;   // shared experts this handle evaluates (all by default)
  bool fused;             // the fused layer kernel where it applies (default off)
};

namespace {

// Automatic path choice (the default): the whole call takes the tensor-core path when the
// batch's average tokens per routed expert, n_tokens * k / E, reaches kDenseTpe, or
// kDenseTpeSparse when the routed experts keep 30 % of their neurons or fewer.  Measured on B200
// (layer time with every expert sparse against every expert dense, OLMoE, DeepSeek-V2-Lite and
// GPT-OSS shapes, sparsity 0 / 0.5 / 0.9): the dense path wins from 4-8 tokens per expert at
// sparsity <= 0.5 and from 8-16 at 0.9.  Mixing the two paths in one call was slower than either.
constexpr double kDenseTpe = 6.0, kDenseTpeSparse = 10.0;

// Shared experts see every token, so at large batches the sparse kernels read their weights once
// per 8-token tile.  Where a shared expert's packed weights exceed the L2 cache (so that those
// re-reads come from HBM), the shared experts alone take the tensor-core path from
// kSharedDenseTokens tokens on (kSharedDenseTokensDense when the routed experts keep 70 % of their
// neurons or more), the routed experts staying sparse.  Measured on B200 (Llama-4-Maverick shape,
// one 8192-neuron shared expert of 252 MB): the split wins from 32 tokens at sparsity 0.5 and
// 0.9 (2.30 ms against 3.42 ms all-sparse at 256 tokens, s = 0.9) and from 128 at sparsity 0;
// DeepSeek-V2-Lite's shared experts (17 MB each) stay in L2 and never gain.
constexpr int kSharedDenseTokens = 32, kSharedDenseTokensDense = 128;
constexpr double kL2Bytes = 126.0 * 1024 * 1024;

// The per-call threshold of automatic mode: 1 (every slot dense), n_tokens (only slots with every
// token: the shared experts) or INT_MAX (every slot sparse).
int auto_dense_min(const moe_config& c, int n_tokens, const moe_sparsity* sp) {
  const double tpe = (double)n_tokens * c.top_k / c.n_routed;
  const bool very_sparse = sp->mode == MOE_SEL_TOPK && sp->sparsity > 0.7;
  if (tpe >= (very_sparse ? kDenseTpeSparse : kDenseTpe)) return 1;
  const double sh_bytes = 3.0 * c.inter_shared * c.hidden * (c.dtype == MOE_BF16 ? 2 : 4);
  const bool mostly_kept = sp->mode == MOE_SEL_TOPK && sp->sparsity < 0.3;
  if (c.n_shared > 0 && sh_bytes > kL2Bytes &&
      n_tokens >= (mostly_kept ? kSharedDenseTokensDense : kSharedDenseTokens))
    return n_tokens;
  return INT_MAX;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Makes the handle's device current for one call and restores the caller's device after it,
// so that a handle works whichever device the calling thread has selected.
struct DeviceScope {
  int prev = -1;
  bool switched = false;
  bool ok = true;
  explicit DeviceScope(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev) {
      ok = cudaSetDevice(dev) == cudaSuccess;
      switched = ok;
    }
  }
  ~DeviceScope() {
    if (switched) cudaSetDevice(prev);
  }
};

moe_status check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_BF16 && c->dtype != MOE_F32) return MOE_ERR_INVALID_ARG;
  if (c->route < MOE_ROUTE_SOFTMAX_TOPK || c->route > MOE_ROUTE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->n_routed <= 0 || c->top_k <= 0 || c->inter <= 0 ||
      c->max_tokens <= 0 || c->n_shared < 0 || (c->n_shared > 0 && c->inter_shared <= 0))
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->n_routed) return MOE_ERR_INVALID_ARG;
  if (c->hidden % 64 || c->hidden < 64 || c->hidden > 8192) return MOE_ERR_UNSUPPORTED;
  if (c->inter % 32 || c->inter < 32 || c->inter > 16384) return MOE_ERR_UNSUPPORTED;
  if (c->n_shared > 0 && (c->inter_shared % 32 || c->inter_shared < 32 || c->inter_shared > 16384))
    return MOE_ERR_UNSUPPORTED;
  if (c->top_k > moe::kMaxTopK || c->n_routed > moe::kMaxRouted || c->n_shared > moe::kMaxShared ||
      c->max_tokens > moe::kMaxTokens)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_sparsity(const moe_sparsity* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->mode == MOE_SEL_TOPK) {
    if (!(s->sparsity >= 0.0 && s->sparsity <= 1.0)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
  }
  if (s->mode == MOE_SEL_THRESHOLD) return isnan(s->threshold) ? MOE_ERR_INVALID_ARG : MOE_OK;
  return MOE_ERR_INVALID_ARG;
}

// K = ceil((1 - s) I), evaluated as I - floor(s I + 1e-9) and clamped to [0, I].
int keep_count(int I, double s) {
  long k = (long)I - (long)floor(s * (double)I + 1e-9);
  if (k < 0) k = 0;
  if (k > I) k = I;
  return (int)k;
}

struct Carve {
  char* base;
  size_t off;
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~(size_t)255;
    T* p = reinterpret_cast<T*>(base + off);
    off += n * sizeof(T);
    return p;
  }
};

// Lays the workspace out (base == nullptr only measures it).
size_t carve(moe_handle* h, char* base) {
  const moe_config& c = h->cfg;
  const size_t Bm = (size_t)c.max_tokens, E = c.n_routed, k = c.top_k, S = c.n_shared;
  const size_t Pm = Bm * (k + S), Im = h->imax, Wm = Im / 32,
               slots = (size_t)moe::slot_capacity((int)E, (int)S);
  Carve cv{base, 0};
  FwdParams& p = h->base;
  p.logits = cv.take<float>(Bm * E);
  p.logit_part = cv.take<float>((size_t)moe::kMaxHsplit * Bm * E);
  p.topk_idx = cv.take<int>(Bm * k);
  p.topk_w = cv.take<float>(Bm * k);
  p.pair_index = cv.take<int>(Bm * (k + S));
  p.pair_token = cv.take<int>(Pm);
  p.pair_w = cv.take<float>(Pm);
  p.pair_slot = cv.take<int>(Pm);
  p.slots = cv.take<moe::Slot>(slots);
  p.meta = cv.take<int>(moe::kMetaWords);
  p.act = cv.take<float>(Pm * Im);
  p.maskbits = cv.take<uint32_t>(Pm * Wm);
  p.ulist = cv.take<int>(slots * Im);
  p.ucnt = cv.take<int>(slots);
  p.err = cv.take<int>(1);
  h->roster_bias = cv.take<float>(Bm * E);
  p.zero_row = cv.take<char>((size_t)c.hidden * h->elt);
  h->trace_buf = cv.take<unsigned long long>((size_t)moe::kTraceKernels * moe::kTraceCtas *
                                             moe::kTracePoints);
  p.trace = nullptr;
  h->x_stage = cv.take<char>(Bm * c.hidden * h->elt);
  h->out_stage = cv.take<char>(Bm * c.hidden * h->elt);
  // dense fallback buffers (bf16 layers only)
  p.imax_pad = (int)((Im + 127) / 128 * 128);
  const bool dense_ok = c.dtype == MOE_BF16;
  p.xp = dense_ok ? cv.take<__nv_bfloat16>(Pm * c.hidden) : nullptr;
  p.hbuf = dense_ok ? cv.take<__nv_bfloat16>(Pm * (size_t)p.imax_pad) : nullptr;
  // zero-at-rest region: tickets, union bitmasks, score histograms, output accumulator
  char* zb = cv.take<char>(0);
  p.tile_ticket = cv.take<unsigned>((Bm + moe::kTileTok - 1) / moe::kTileTok);
  p.global_ticket = cv.take<unsigned>(1);
  p.claim = cv.take<unsigned>(3);
  p.slot_ticket = cv.take<unsigned>(slots);
  p.ubits = cv.take<uint32_t>(slots * Wm);
  p.hist = cv.take<unsigned>(Pm * moe::kHistBins);
  p.tile_done = cv.take<unsigned>(Pm);
  p.s_task = cv.take<int>(Pm);
  p.fq = cv.take<unsigned>(4);
  p.u_res = cv.take<unsigned long long>(1);
  p.u_ent = cv.take<int4>(slots);
  p.out_acc = cv.take<float>(Bm * c.hidden);
  h->zero_begin = zb;
  h->zero_bytes = (size_t)((base + cv.off) - zb);
  return cv.off + 256;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status forward_impl(moe_handle* h, const void* x, int n_tokens, const void* router,
                        const moe_roster* roster, const moe_expert_weights* routed,
                        const moe_expert_weights* shared, const moe_sparsity* sp_routed,
                        const moe_sparsity* sp_shared, void* out, cudaStream_t st,
                        bool partial = false) {
  const moe_config& c = h->cfg;
  FwdParams p = h->base;
  p.H = c.hidden;
  p.E = c.n_routed;
  p.k = c.top_k;
  p.S = c.n_shared;
  p.I = c.inter;
  p.Ish = c.n_shared > 0 ? c.inter_shared : 0;
  p.B = n_tokens;
  p.Imax = h->imax;
  p.Bmax = c.max_tokens;
  p.hsplit = moe::router_hsplit(c.n_routed, n_tokens, c.hidden);
  p.router_cluster = h->ls.router_cluster;
  p.e_begin = h->e_begin;
  p.e_end = h->e_end;
  p.shared_mask = h->shared_mask;
  p.route = (int)c.route;
  p.sel_mode[0] = sp_routed->mode == MOE_SEL_THRESHOLD ? 1 : 0;
  p.sel_K[0] = keep_count(c.inter, sp_routed->sparsity);
  p.sel_t[0] = sp_routed->threshold;
  if (c.n_shared > 0) {
    p.sel_mode[1] = sp_shared->mode == MOE_SEL_THRESHOLD ? 1 : 0;
    p.sel_K[1] = keep_count(c.inter_shared, sp_shared->sparsity);
    p.sel_t[1] = sp_shared->threshold;
  } else {
    p.sel_mode[1] = 0;
    p.sel_K[1] = 0;
    p.sel_t[1] = 0.f;
  }
  p.x = x;
  p.router = router;
  p.gate_r = routed->gate;
  p.updown_r = routed->updown;
  p.gate_s = c.n_shared > 0 ? shared->gate : nullptr;
  p.updown_s = c.n_shared > 0 ? shared->updown : nullptr;
  p.out = out;
  if (h->dirty) {
    if (cudaMemsetAsync(h->zero_begin, 0, h->zero_bytes, st) != cudaSuccess) return MOE_ERR_CUDA;
    h->dirty = false;
  }
  const int dt = c.dtype == MOE_BF16 ? 0 : 1;
  // MOE_NO_PDL=1 in the environment launches the chain without programmatic overlap (a tuning
  // switch; results are identical either way)
  static const bool no_pdl = getenv("MOE_NO_PDL") != nullptr && getenv("MOE_NO_PDL")[0] == '1';
  const bool tm = h->timing, pdl = !tm && !no_pdl;
  p.trace = tm ? h->trace_buf : nullptr;
  // dense fallback: slots with at least dense_min tokens (bf16 only; no slot has more than
  // n_tokens tokens, so below that nothing is launched for it).  The router already needs it:
  // it gives dense slots no sparse gate items.
  p.dense_min = dt != 0 || h->dense_min == 0 ? INT_MAX
                : h->dense_min == MOE_DENSE_AUTO ? auto_dense_min(c, n_tokens, sp_routed)
                                                 : h->dense_min;
  const bool dense = p.dense_min <= n_tokens;
  cudaEvent_t* ev = h->stage_events;
  cudaError_t e = tm ? cudaEventRecord(ev[0], st) : cudaSuccess;
  p.router_bias = nullptr;
  p.roster_counts = nullptr;
  if (roster) {
    p.router_bias = h->roster_bias;
    p.roster_counts = roster->counts;
    if (e == cudaSuccess)
      e = moe::launch_roster_bias(roster->counts, roster->pinned, n_tokens, c.n_routed, roster->m,
                                  roster->delta, h->roster_bias, st);
  }
  // The fused layer kernel does gate, selection and up/down in one launch (bf16, register
  // token fragments, no slot on the tensor-core path).  Under stage timing its event pair is the
  // gate stage's, and the selection and up/down stages are empty.
  const bool fused = dt == 0 && !dense && h->fused && moe::layer_available(h->ls);
  if (e == cudaSuccess) e = moe::launch_router(p, dt, st);
  if (e == cudaSuccess && tm) e = cudaEventRecord(ev[1], st);
  if (fused) {
    if (e == cudaSuccess) e = moe::launch_layer(p, h->ls, st, pdl);
    for (int k = 2; k <= 4 && tm && e == cudaSuccess; ++k) e = cudaEventRecord(ev[k], st);
  } else {
    if (e == cudaSuccess) e = moe::launch_gate(p, dt, h->ls, st, pdl);
    if (e == cudaSuccess && dense) e = moe::launch_dense(p, h->ls, 0, st, pdl);
    if (e == cudaSuccess && tm) e = cudaEventRecord(ev[2], st);
    if (e == cudaSuccess) e = moe::launch_select(p, h->ls, st, pdl);
    if (e == cudaSuccess && tm) e = cudaEventRecord(ev[3], st);
    if (e == cudaSuccess && dense) e = moe::launch_dense(p, h->ls, 1, st, pdl);
    if (e == cudaSuccess) e = moe::launch_updown(p, dt, h->ls, st, pdl);
    if (e == cudaSuccess && tm) e = cudaEventRecord(ev[4], st);
  }
  // a partial output stays fp32: the sum over the handles is cast once (moe_cast_output)
  if (e == cudaSuccess) e = moe::launch_finalize(p, partial ? 1 : dt, h->ls, st, pdl);
  if (e == cudaSuccess && tm) e = cudaEventRecord(ev[5], st);
  if (e != cudaSuccess) {
    h->dirty = true;
    return MOE_ERR_CUDA;
  }
  h->last_tokens = n_tokens;
  // router, fused layer, finalize; or the chain of five (+ gather and three GEMMs on the
  // tensor-core path); + the roster bias kernel
  h->last_launches = (fused ? 3 : dense ? 9 : 5) + (roster ? 1 : 0);
  return MOE_OK;
}

moe_status check_forward(moe_handle* h, const void* x, int n_tokens, const void* router,
                         const moe_expert_weights* routed, const moe_expert_weights* shared,
                         const moe_sparsity* sp_routed, const moe_sparsity* sp_shared,
                         const void* out, bool host_io) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;  // a no-op: nothing is read
  if (!x || !router || !routed || !out || !sp_routed) return MOE_ERR_INVALID_ARG;
  if (!routed->gate || !routed->updown) return MOE_ERR_INVALID_ARG;
  if (!aligned16(router) || !aligned16(routed->gate) || !aligned16(routed->updown))
    return MOE_ERR_INVALID_ARG;
  if (!host_io && (!aligned16(x) || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  moe_status s = check_sparsity(sp_routed);
  if (s != MOE_OK) return s;
  if (h->cfg.n_shared > 0) {
    if (!shared || !shared->gate || !shared->updown || !sp_shared) return MOE_ERR_INVALID_ARG;
    if (!aligned16(shared->gate) || !aligned16(shared->updown)) return MOE_ERR_INVALID_ARG;
    s = check_sparsity(sp_shared);
    if (s != MOE_OK) return s;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_create(const moe_config* cfg, moe_handle** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  moe_handle* h = new (std::nothrow) moe_handle();
  if (!h) return MOE_ERR_OOM;
  h->cfg = *cfg;
  h->elt = cfg->dtype == MOE_BF16 ? 2 : 4;
  h->imax = cfg->inter;
  if (cfg->n_shared > 0 && cfg->inter_shared > h->imax) h->imax = cfg->inter_shared;
  if (cudaGetDevice(&h->device) != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  cudaError_t e;
  {
    std::lock_guard<std::mutex> lock(moe::setup_mutex());
    e = moe::configure_kernels(cfg->dtype == MOE_BF16 ? 0 : 1, h->imax,
                               moe::slot_capacity(cfg->n_routed, cfg->n_shared),
                               cfg->max_tokens, cfg->hidden, &h->ls);
  }
  if (e != cudaSuccess) {
    delete h;
    return MOE_ERR_CUDA;
  }
  h->ws_bytes = carve(h, nullptr);
  if (cudaMalloc(&h->ws, h->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_OOM;
  }
  h->dense_min = MOE_DENSE_AUTO;
  h->fused = false;
  h->e_begin = 0;
  h->e_end = cfg->n_routed;
  h->shared_mask = (1u << cfg->n_shared) - 1u;
  carve(h, static_cast<char*>(h->ws));
  if (cudaMemset(h->ws, 0, h->ws_bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

moe_status moe_packed_bytes(const moe_config* cfg, int shared, size_t* gate_bytes,
                            size_t* updown_bytes) {
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (shared && cfg->n_shared == 0) return MOE_ERR_INVALID_ARG;
  const size_t elt = cfg->dtype == MOE_BF16 ? 2 : 4;
  const size_t I = shared ? cfg->inter_shared : cfg->inter;
  if (gate_bytes) *gate_bytes = I * cfg->hidden * elt;
  if (updown_bytes) *updown_bytes = 2 * I * cfg->hidden * elt;
  return MOE_OK;
}

moe_status moe_pack_experts(moe_handle* h, int shared, const void* w_gate, const void* w_up,
                            const void* w_down, int n, void* packed_gate, void* packed_updown,
                            void* stream) {
  if (!h || !w_gate || !w_up || !w_down || !packed_gate || !packed_updown || n < 0)
    return MOE_ERR_INVALID_ARG;
  if (shared && h->cfg.n_shared == 0) return MOE_ERR_INVALID_ARG;
  if (n > (shared ? h->cfg.n_shared : h->cfg.n_routed)) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t H = h->cfg.hidden, I = shared ? h->cfg.inter_shared : h->cfg.inter, elt = h->elt;
  cudaError_t e = cudaSuccess;
  if (packed_gate != w_gate)
    e = cudaMemcpyAsync(packed_gate, w_gate, (size_t)n * I * H * elt, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = cudaMemcpy2DAsync(packed_updown, 2 * H * elt, w_up, H * elt, H * elt, (size_t)n * I,
                          cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess)
    e = moe::launch_pack_down(w_down, packed_updown, n, (int)I, (int)H, (int)elt, st);
  return cuda_status(e);
}

moe_status moe_forward(moe_handle* h, const void* x, int n_tokens, const void* router,
                       const moe_expert_weights* routed, const moe_expert_weights* shared,
                       const moe_sparsity* sp_routed, const moe_sparsity* sp_shared, void* out,
                       void* stream) {
  moe_status s = check_forward(h, x, n_tokens, router, routed, shared, sp_routed, sp_shared, out,
                               false);
  if (s != MOE_OK) return s;
  if (n_tokens == 0) return MOE_OK;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  return forward_impl(h, x, n_tokens, router, nullptr, routed, shared, sp_routed, sp_shared, out,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_roster(moe_handle* h, const void* x, int n_tokens, const void* router,
                              const moe_roster* roster, const moe_expert_weights* routed,
                              const moe_expert_weights* shared, const moe_sparsity* sp_routed,
                              const moe_sparsity* sp_shared, void* out, void* stream) {
  moe_status s = check_forward(h, x, n_tokens, router, routed, shared, sp_routed, sp_shared, out,
                               false);
  if (s != MOE_OK) return s;
  if (n_tokens == 0) return MOE_OK;
  if (!roster || !roster->counts || !roster->pinned) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(roster->counts) | reinterpret_cast<uintptr_t>(roster->pinned)) &
      3u)
    return MOE_ERR_INVALID_ARG;
  if (roster->m < h->cfg.top_k || roster->m > h->cfg.n_routed) return MOE_ERR_INVALID_ARG;
  if (!(roster->delta >= 0.f) || isinf(roster->delta)) return MOE_ERR_INVALID_ARG;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  return forward_impl(h, x, n_tokens, router, roster, routed, shared, sp_routed, sp_shared, out,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_forward_host(moe_handle* h, const void* x_host, int n_tokens, const void* router,
                            const moe_expert_weights* routed, const moe_expert_weights* shared,
                            const moe_sparsity* sp_routed, const moe_sparsity* sp_shared,
                            void* out_host, void* stream) {
  moe_status s = check_forward(h, x_host, n_tokens, router, routed, shared, sp_routed, sp_shared,
                               out_host, true);
  if (s != MOE_OK) return s;
  if (n_tokens == 0) return MOE_OK;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)n_tokens * h->cfg.hidden * h->elt;
  if (cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  s = forward_impl(h, h->x_stage, n_tokens, router, nullptr, routed, shared, sp_routed, sp_shared,
                   h->out_stage, st);
  if (s != MOE_OK) return s;
  if (cudaMemcpyAsync(out_host, h->out_stage, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_debug_lists(moe_handle* h, int n_tokens, int* idx, float* w, float* logits,
                           int* cnt, int* lists, float* act, void* stream) {
  if (!h || n_tokens <= 0 || n_tokens != h->last_tokens) return MOE_ERR_INVALID_ARG;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const moe_config& c = h->cfg;
  FwdParams p = h->base;
  p.H = c.hidden;
  p.E = c.n_routed;
  p.k = c.top_k;
  p.S = c.n_shared;
  p.I = c.inter;
  p.Ish = c.n_shared > 0 ? c.inter_shared : 0;
  p.B = n_tokens;
  p.Imax = h->imax;
  cudaError_t e = cudaSuccess;
  const size_t nk = (size_t)n_tokens * c.top_k;
  if (idx) e = cudaMemcpyAsync(idx, p.topk_idx, nk * sizeof(int), cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && w)
    e = cudaMemcpyAsync(w, p.topk_w, nk * sizeof(float), cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && logits)
    e = cudaMemcpyAsync(logits, p.logits, (size_t)n_tokens * c.n_routed * sizeof(float),
                        cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && (cnt || lists || act))
    e = moe::launch_debug_gather(p, n_tokens, cnt, lists, act, st);
  return cuda_status(e);
}

moe_status moe_profile_stages(moe_handle* h, void* const* events, int n_events) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!events) {
    h->timing = false;
    return MOE_OK;
  }
  if (n_events != MOE_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_STAGE_EVENTS; ++i) {
    if (!events[i]) return MOE_ERR_INVALID_ARG;
    h->stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  }
  h->timing = true;
  return MOE_OK;
}

moe_status moe_read_trace(moe_handle* h, unsigned long long* host, size_t n) {
  if (!h || !host) return MOE_ERR_INVALID_ARG;
  const size_t cap = (size_t)moe::kTraceKernels * moe::kTraceCtas * moe::kTracePoints;
  if (n > cap) n = cap;
  DeviceScope dev(h->device);
  if (!dev.ok || cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpy(host, h->trace_buf, n * sizeof(unsigned long long), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(cudaMemset(h->trace_buf, 0, n * sizeof(unsigned long long)));
}

moe_status moe_get_error(moe_handle* h, int* device_code) {
  if (!h || !device_code) return MOE_ERR_INVALID_ARG;
  *device_code = 0;
  DeviceScope dev(h->device);
  if (!dev.ok || cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, h->base.err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (v == 0) return MOE_OK;
  *device_code = v;
  if (cudaMemset(h->base.err, 0, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return v == moe::kErrTimeout ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE;
}

moe_status moe_debug_force_timeout(moe_handle* h, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  return cuda_status(moe::launch_force_timeout(h->base, static_cast<cudaStream_t>(stream)));
}

moe_status moe_set_expert_range(moe_handle* h, int e_begin, int e_end, unsigned shared_mask) {
  if (!h || e_begin < 0 || e_end > h->cfg.n_routed || e_begin > e_end) return MOE_ERR_INVALID_ARG;
  if (h->cfg.n_shared < 32 && (shared_mask >> h->cfg.n_shared) != 0u) return MOE_ERR_INVALID_ARG;
  h->e_begin = e_begin;
  h->e_end = e_end;
  h->shared_mask = shared_mask;
  return MOE_OK;
}

moe_status moe_forward_partial(moe_handle* h, const void* x, int n_tokens, const void* router,
                               const moe_expert_weights* routed, const moe_expert_weights* shared,
                               const moe_sparsity* sp_routed, const moe_sparsity* sp_shared,
                               float* partial, void* stream) {
  moe_status s = check_forward(h, x, n_tokens, router, routed, shared, sp_routed, sp_shared,
                               partial, false);
  if (s != MOE_OK) return s;
  if (n_tokens == 0) return MOE_OK;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  return forward_impl(h, x, n_tokens, router, nullptr, routed, shared, sp_routed, sp_shared,
                      partial, static_cast<cudaStream_t>(stream), true);
}

moe_status moe_cast_output(moe_handle* h, const float* sum, int n_tokens, void* out,
                           void* stream) {
  if (!h || n_tokens < 0 || n_tokens > h->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
  if (n_tokens == 0) return MOE_OK;
  if (!sum || !out || !aligned16(sum) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  DeviceScope dev(h->device);
  if (!dev.ok) return MOE_ERR_CUDA;
  return cuda_status(moe::launch_cast_output(sum, out, (size_t)n_tokens * h->cfg.hidden,
                                             h->cfg.dtype == MOE_BF16 ? 0 : 1, h->ls.nsm,
                                             static_cast<cudaStream_t>(stream)));
}

moe_status moe_last_launches(moe_handle* h, int* n) {
  if (!h || !n) return MOE_ERR_INVALID_ARG;
  *n = h->last_launches;
  return MOE_OK;
}

moe_status moe_set_dense_min_tokens(moe_handle* h, int min_tokens) {
  if (!h || min_tokens < MOE_DENSE_AUTO) return MOE_ERR_INVALID_ARG;
  h->dense_min = min_tokens;
  return MOE_OK;
}

moe_status moe_set_fused(moe_handle* h, int enable) {
  if (!h || (enable != 0 && enable != 1)) return MOE_ERR_INVALID_ARG;
  h->fused = enable != 0;
  return MOE_OK;
}

moe_status moe_destroy(moe_handle* h) {
  if (!h) return MOE_OK;
  moe_status s = MOE_OK;
  {
    DeviceScope dev(h->device);
    cudaError_t e = dev.ok ? cudaDeviceSynchronize() : cudaErrorInvalidDevice;
    cudaError_t f = cudaFree(h->ws);
    if (e != cudaSuccess || f != cudaSuccess) s = MOE_ERR_CUDA;
  }
  delete h;
  return s;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_OOM: return "out of device memory";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE: return "device-side error flag set";
    case MOE_ERR_TIMEOUT: return "timeout";
  }
  return "unknown status";
}

}  // extern "C"
