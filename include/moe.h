/*
 * moe.h - C ABI of the sparse-expert MoE FFN decode layer for NVIDIA B200 (sm_100a).
 *
 * The layer is the one of "Uncovering Intra-expert Activation Sparsity for Efficient
 * Mixture-of-Expert Model Execution" (technical summary, Methodology): the router picks the
 * top-k experts of each token; every routed and every always-on shared expert computes its
 * gate projection densely, which scores its neurons; inside each (token, expert) pair only the
 * neurons that survive the sparsity cut are kept, and the up and down projections read and
 * compute those neurons only; the expert outputs are combined with the routing weights.
 *
 * Conventions shared by every entry point
 *   - Plain C types only.  `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device pointers are CUDA global-memory addresses.
 *   - A handle belongs to the device that was current at moe_create.  Every call on it makes
 *     that device current for the call's duration and then restores the caller's device.
 *     Its buffers and `stream` must belong to that device.  Calls without a handle, such as
 *     moe_route_noalloc, run on the current device.
 *   - The caller owns every buffer it passes.  The handle owns its workspace (allocated once
 *     by moe_create, sized for cfg.max_tokens) and never allocates afterwards, so moe_forward
 *     makes no allocation and no host synchronisation and may be captured in a CUDA graph.
 *   - Element type: every x, router, weight and out buffer holds cfg.dtype (bf16 or binary32),
 *     row-major and contiguous, 16-byte aligned.
 *   - Errors are status codes; nothing is thrown across the ABI.  Arguments are validated
 *     before any launch.  Faults the kernels detect (NaN router logits or activations) set an
 *     error word on the device that moe_get_error reads.
 *   - A handle serves one stream at a time: calls that overlap on the GPU race on its
 *     workspace.
 */
#ifndef SPARSE_MOE_H_
#define SPARSE_MOE_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* a null pointer, a size out of range, a misaligned buffer */
  MOE_ERR_UNSUPPORTED = 2, /* a shape outside the supported limits (see moe_config) */
  MOE_ERR_OOM = 3,         /* the workspace allocation failed */
  MOE_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  MOE_ERR_DEVICE = 5,      /* the kernels set the device error word (moe_get_error) */
  MOE_ERR_TIMEOUT = 6      /* a bounded wait inside a kernel gave up (moe_get_error) */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_F32 = 1 } moe_dtype;

/* Routing weight of a chosen expert (the weight scales that expert's output):
 *   SOFTMAX_TOPK  softmax over the k chosen logits
 *   SOFTMAX_ALL   softmax over all E logits, evaluated at the chosen ones
 *   SIGMOID       1 / (1 + exp(-logit)) of the chosen logit
 * In every mode the k experts with the largest logits are chosen; equal logits keep the
 * lower expert index. */
typedef enum {
  MOE_ROUTE_SOFTMAX_TOPK = 0,
  MOE_ROUTE_SOFTMAX_ALL = 1,
  MOE_ROUTE_SIGMOID = 2
} moe_route;

/* Neuron selection inside each (token, expert) pair, on the score |SiLU(g_n)|:
 *   TOPK       keep K = I - floor(s*I + 1e-9) neurons (= ceil((1-s) I)), the largest scores;
 *              equal scores keep the lower neuron index
 *   THRESHOLD  keep the neurons whose score is strictly greater than `threshold` */
typedef enum { MOE_SEL_TOPK = 0, MOE_SEL_THRESHOLD = 1 } moe_sel;

/* Layer shape.  Limits: hidden in [64, 8192] and a multiple of 64; inter and inter_shared in
 * [32, 16384] and multiples of 32; 1 <= top_k <= min(16, n_routed); n_routed <= 512;
 * 0 <= n_shared <= 8; 1 <= max_tokens <= 1024. */
typedef struct {
  int hidden;       /* H */
  int n_routed;     /* E routed experts */
  int top_k;        /* k experts per token */
  int inter;        /* I, intermediate size of a routed expert */
  int n_shared;     /* S always-on shared experts (weight 1) */
  int inter_shared; /* Ish, intermediate size of a shared expert (ignored when S = 0) */
  int max_tokens;   /* largest n_tokens any call will pass */
  moe_dtype dtype;
  moe_route route;
} moe_config;

/* Selection rule for one group of experts (routed, or shared).  sparsity in [0, 1] is used in
 * TOPK mode; threshold (binary32, may be -inf or +inf) in THRESHOLD mode. */
typedef struct {
  moe_sel mode;
  double sparsity;
  float threshold;
} moe_sparsity;

/* Packed, neuron-major expert weights (device pointers, produced by moe_pack_experts):
 *   gate    [n][I][H]      row n = the gate weights of neuron n
 *   updown  [n][I][2][H]   for neuron n: its W_up row, then its W_down column, contiguous,
 *                          so a skipped neuron is 2*H*elt skipped bytes */
typedef struct {
  const void* gate;
  const void* updown;
} moe_expert_weights;

typedef struct moe_handle moe_handle;

/* Validates cfg, allocates the workspace for cfg->max_tokens on the current device and returns
 * a handle in *out.  INVALID_ARG / UNSUPPORTED for a bad config, OOM if the allocation fails. */
moe_status moe_create(const moe_config* cfg, moe_handle** out);

/* Bytes of one expert's packed gate block (I*H*elt) and up/down block (2*I*H*elt); shared = 1
 * gives the shared-expert sizes.  Either output may be NULL. */
moe_status moe_packed_bytes(const moe_config* cfg, int shared, size_t* gate_bytes,
                            size_t* updown_bytes);

/* Re-lays n experts' logical weights into the packed layout, asynchronously on `stream`.
 *   w_gate [n][I][H], w_up [n][I][H], w_down [n][H][I]   (device, cfg.dtype; I = Ish if shared)
 *   packed_gate [n][I][H], packed_updown [n][I][2][H]    (device, caller-allocated)
 * Input and output buffers must not overlap, except packed_gate == w_gate (then no copy). */
moe_status moe_pack_experts(moe_handle* h, int shared, const void* w_gate, const void* w_up,
                            const void* w_down, int n, void* packed_gate, void* packed_updown,
                            void* stream);

/* The layer for n_tokens tokens, asynchronously on `stream`.
 *   x       [n_tokens][H]      device
 *   router  [E][H]             device
 *   routed  packed weights of the E routed experts
 *   shared  packed weights of the S shared experts (NULL allowed when S = 0)
 *   sp_routed, sp_shared  selection rules (sp_shared may be NULL when S = 0)
 *   out     [n_tokens][H]      device, written
 * n_tokens = 0 returns MOE_OK, reads no other argument and launches nothing; n_tokens < 0 or
 * n_tokens > max_tokens is INVALID_ARG. */
moe_status moe_forward(moe_handle* h, const void* x, int n_tokens, const void* router,
                       const moe_expert_weights* routed, const moe_expert_weights* shared,
                       const moe_sparsity* sp_routed, const moe_sparsity* sp_shared, void* out,
                       void* stream);

/* Roster routing state of the batch's sequences ("Predatory MoE", technical summary,
 * Methodology 2, the roster rule), one row per token: token t of a call is the decode token of
 * the sequence whose state is row t.
 *   counts  [n_tokens][E] int32, device, read and updated: how often each expert of this layer
 *           was selected for the sequence so far (the call adds its own choice)
 *   pinned  [n_tokens] int32, device, read: nonzero = the sequence's roster is pinned
 *   m       roster budget, top_k <= m <= E
 *   delta   barrier bonus, finite and >= 0
 * The roster of a sequence is its m most-selected experts (equal counts: lower index).  While
 * fewer than m distinct experts have been selected the router is unchanged (exploration); then
 * the choice is the top-k of logit + delta for members and logit - delta for the others; a
 * pinned sequence chooses among its roster only.  The bias acts on the choice: the routing
 * weights are those of the unbiased logits of the chosen experts. */
typedef struct {
  int* counts;
  const int* pinned;
  int m;
  float delta;
} moe_roster;

/* moe_forward with roster routing (one more kernel before the router computes each sequence's
 * bias; the router adds the choice to the counts).  INVALID_ARG for a NULL roster or buffer, a
 * buffer that is not 4-byte aligned, m outside [top_k, E] or a negative or non-finite delta;
 * otherwise as moe_forward.  The calls of one decode step must not overlap on the GPU with
 * another call that updates the same counts. */
moe_status moe_forward_roster(moe_handle* h, const void* x, int n_tokens, const void* router,
                              const moe_roster* roster, const moe_expert_weights* routed,
                              const moe_expert_weights* shared, const moe_sparsity* sp_routed,
                              const moe_sparsity* sp_shared, void* out, void* stream);

/* moe_forward with x and out in HOST memory: copies x to the handle's device staging buffer,
 * runs the layer and copies the result back, all asynchronously on `stream` (page-locked host
 * buffers make the copies asynchronous; the caller synchronises the stream before reading
 * out).  Weights and router stay device pointers. */
moe_status moe_forward_host(moe_handle* h, const void* x_host, int n_tokens, const void* router,
                            const moe_expert_weights* routed, const moe_expert_weights* shared,
                            const moe_sparsity* sp_routed, const moe_sparsity* sp_shared,
                            void* out_host, void* stream);

/* Copies the intermediate results of the last moe_forward (for parity checks), asynchronously
 * on `stream`, into caller-allocated device buffers; any output may be NULL.  n_tokens must be
 * the n_tokens of that call.  P = k + S pairs per token: pair j < k is the token's j-th routed
 * expert (in idx order), pair k + s is shared expert s; Imax = max(I, Ish).
 *   idx    [n_tokens][k] int32  chosen experts, by (logit desc, index asc)
 *   w      [n_tokens][k] float  routing weights
 *   logits [n_tokens][E] float  router logits
 *   cnt    [n_tokens][P] int32  kept-neuron count of each pair
 *   lists  [n_tokens][P][Imax] int32  kept neurons in ascending order, then -1 padding
 *   act    [n_tokens][P][Imax] float  SiLU(g) of every neuron (before selection), 0 padding */
moe_status moe_debug_lists(moe_handle* h, int n_tokens, int* idx, float* w, float* logits,
                           int* cnt, int* lists, float* act, void* stream);

/* Stage timing.  events = MOE_STAGE_EVENTS cudaEvent_t handles (as void*), or NULL to turn
 * timing off.  While set, every moe_forward records events[0] before its first kernel and
 * events[i] after its i-th kernel (1 router+top-k+grouping, 2 gate, 3 select, 4 up/down,
 * 5 output cast), and launches the kernels without programmatic overlap so that the interval
 * between consecutive events is that kernel alone.  A call on the fused layer kernel
 * (moe_set_fused) records events 2, 3 and 4 after it: its duration is the gate stage's, the
 * selection and up/down stages are empty.  The handle keeps the event handles, not
 * copies; the caller owns and destroys them. */
#define MOE_STAGE_EVENTS 6
moe_status moe_profile_stages(moe_handle* h, void* const* events, int n_events);

/* Phase timestamps of the last calls made while stage timing was on (%globaltimer ns, 0 where a
 * point was not reached): host[(kernel * 1024 + cta) * 8 + point] for kernel 0..4 in launch
 * order and the first 1024 CTAs.  In the gate and up/down kernels point 5 holds a count (the
 * CTA's work items), not a time.  Synchronises the device, copies min(n, 5*1024*8) values into
 * host memory, then clears the device buffer. */
moe_status moe_read_trace(moe_handle* h, unsigned long long* host, size_t n);

/* Synchronises the device, reads and clears the device error word.  Returns MOE_ERR_DEVICE
 * (code in *device_code: 1 = NaN router logit, 2 = NaN activation) or MOE_ERR_TIMEOUT (code 3:
 * a bounded wait inside a kernel gave up after 0.2 s; the output of that call is then invalid)
 * if it was set, else MOE_OK with *device_code = 0. */
moe_status moe_get_error(moe_handle* h, int* device_code);

/* Failure-detection test hook (the paper has none): launches one warp that waits, with the
 * kernels' own bounded wait, on a barrier that nothing completes.  After the wait's 0.2 s limit
 * it records a timeout in the handle's error word and returns; the GPU context stays usable and
 * the next moe_get_error returns MOE_ERR_TIMEOUT.  Asynchronous on `stream`. */
moe_status moe_debug_force_timeout(moe_handle* h, void* stream);

/* Path choice.  Both paths compute the same function ("Uncovering Intra-expert Activation
 * Sparsity ...", technical summary, Methodology: sparse or dense kernels chosen by batch size):
 * the sparse kernels read only the kept neurons' rows; the dense masked path runs the gate, up and
 * down projections as tcgen05 GEMMs, keeps the same neurons and multiplies the up projection by
 * the 0/1 mask and SiLU(g).  bf16 layers only (fp32 layers always take the sparse kernels).
 *   MOE_DENSE_AUTO (-1, the default)  per call: every expert takes the dense path when the
 *                      batch's average tokens per routed expert n_tokens * top_k / n_routed is
 *                      >= 6 (>= 10 when the routed sparsity is above 0.7); otherwise, when a
 *                      shared expert's packed weights exceed the 126 MB L2 cache, the shared
 *                      experts alone take it from 32 tokens on (128 when the routed sparsity is
 *                      below 0.3); else every expert takes the sparse path.  Thresholds measured
 *                      on B200
 *   0                  never the dense path
 *   n > 0              per expert: an expert (routed or shared) with >= n tokens in the call
 *                      takes the dense path, the others the sparse kernels
 * INVALID_ARG for a NULL handle or a value below -1.  Takes effect from the next moe_forward. */
#define MOE_DENSE_AUTO (-1)
moe_status moe_set_dense_min_tokens(moe_handle* h, int min_tokens);

/* Fused layer kernel ("Uncovering Intra-expert Activation Sparsity ...", technical summary, Key
 * contributions: the layer stays one fused, graph-capturable unit).  enable = 1: a bf16 call
 * whose slots all take the sparse kernels, on a hidden size with register token fragments (512,
 * 2048, 2880, 5120), runs gate, selection and up/down as one persistent kernel between the router
 * and the output cast (3 launches instead of 5): a token tile's selections start as soon as its
 * gate rows are done and an expert's up/down as soon as its union is known.  enable = 0 (the
 * default): the chain of separate kernels, which measured faster on B200 at every batch size
 * tried (the selections cost the fused kernel's consumer warps as much time as the separate
 * selection kernel costs the chain, and the last slots' selections stay on its critical path).  The results are the same within rounding of
 * the fp32 output sums (the up/down runs accumulate in another grouping); routing and kept sets
 * are identical.  Under stage timing (moe_profile_stages) the fused kernel's duration is the
 * gate stage's, and the selection and up/down stages are empty.  INVALID_ARG for a
 * NULL handle or enable outside {0, 1}.  Takes effect from the next moe_forward. */
moe_status moe_set_fused(moe_handle* h, int enable);

/* Expert parallelism ("Uncovering Intra-expert Activation Sparsity ...", technical summary,
 * Methodology: the serving system keeps expert parallelism).  Each of G ranks holds a handle of
 * the same configuration restricted to the routed experts [e_begin, e_end) and to the shared
 * experts whose bit is set in shared_mask; together the ranks' ranges and masks cover every
 * expert once.  Every handle still routes every token over all E experts (the router weights
 * and the tokens are replicated), so the ranks agree on the routing.  A restricted handle reads
 * routed weights of its own experts only: `routed` of its calls points at the packed blocks of
 * experts e_begin .. e_end - 1 (expert e at local index e - e_begin); `shared` still points at
 * all S shared experts' blocks, of which it reads the masked ones.  Default: all experts.
 * INVALID_ARG for a NULL handle, a range outside [0, E] or a mask bit at or above S. */
moe_status moe_set_expert_range(moe_handle* h, int e_begin, int e_end, unsigned shared_mask);

/* moe_forward that writes this handle's part of the layer output in fp32 instead of the cast
 * output: partial [n_tokens][H] (device, fp32, 16-byte aligned) = the weighted sum over the
 * (token, expert) pairs of the handle's experts.  The sum of the ranks' partials (an
 * all-reduce) is the layer output before rounding; moe_cast_output rounds it. */
moe_status moe_forward_partial(moe_handle* h, const void* x, int n_tokens, const void* router,
                               const moe_expert_weights* routed, const moe_expert_weights* shared,
                               const moe_sparsity* sp_routed, const moe_sparsity* sp_shared,
                               float* partial, void* stream);

/* out [n_tokens][H] (cfg.dtype) = sum [n_tokens][H] (fp32) rounded to the layer dtype, on
 * `stream`.  Both device buffers 16-byte aligned. */
moe_status moe_cast_output(moe_handle* h, const float* sum, int n_tokens, void* out,
                           void* stream);

/* How many kernels the last successful moe_forward on this handle launched (5 on the sparse
 * path: router, gate, select, up/down, output cast; 9 when the tensor-core path ran as well;
 * one more with roster routing; 0 before the first call).  Host-side only: reads no device memory.  INVALID_ARG for NULL. */
moe_status moe_last_launches(moe_handle* h, int* n);

/* Frees the workspace and the handle (synchronises the device first).  NULL is a no-op. */
moe_status moe_destroy(moe_handle* h);

/* Routing only, with no handle and no device allocation.  The paper has no counterpart: its
 * router runs inside the layer.  This is for callers that need only each token's expert choice
 * and cannot allocate device memory at that point (for instance a scheduler that plans expert
 * placement while a caching allocator holds all free memory).  It computes exactly what
 * moe_forward's router step computes:
 *   cfg       hidden, n_routed, top_k, dtype and route are read (the other fields are ignored);
 *             the limits of moe_config apply
 *   x         [n_tokens][hidden]  device, dtype, 16-byte aligned, read
 *   router    [n_routed][hidden]  device, dtype, 16-byte aligned, read
 *   topk_idx  [n_tokens][top_k]   device int32, written: experts by logit descending, ties to
 *                                 the lower expert index
 *   topk_w    [n_tokens][top_k]   device fp32, written: the routing weights of cfg->route
 *   stream    cudaStream_t, or NULL for the default stream; the call is asynchronous
 * It runs on a 2 MiB scratch area that the library holds on every device that loads it, until
 * the process exits.  n_tokens <= 256; n_tokens > 256 is UNSUPPORTED, n_tokens < 0 INVALID_ARG,
 * n_tokens = 0 a no-op.  The first call in a device's CUDA context (the first call on the device,
 * and the first after a device reset) sets the scratch area up (it may load the module), so make
 * it before any stream capture.  Calls that overlap in time on one device share the scratch area
 * and race: serialise them.  A NaN logit ranks lowest; no device error word is reported. */
moe_status moe_route_noalloc(const moe_config* cfg, const void* x, int n_tokens,
                             const void* router, int* topk_idx, float* topk_w, void* stream);

/* Static description of a status code. */
const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MOE_H_ */
