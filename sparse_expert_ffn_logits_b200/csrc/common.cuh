// common.cuh - device helpers shared by the layer's kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kThreads = 256;      // threads of the gate / up-down / router CTAs
constexpr int kWarps = kThreads / 32;
constexpr int kTileTok = 8;        // tokens per tile (the n of an m16n8k16 mma)
constexpr int kTileRows = 16;      // rows per tile (the m of an m16n8k16 mma)
constexpr int kMaxTopK = 16;
constexpr int kMaxShared = 8;
constexpr int kMaxRouted = 512;
constexpr int kMaxTokens = 1024;
// A sparse shared expert evaluates every token; up to kMaxSharedTiles token tiles (64 tokens)
// each of its tiles is a slot of its own, with its own union of kept neurons (the up/down rows
// a tile reads are those its own tokens keep).  Slot table capacity: routed experts + shared
// experts' tiles.
constexpr int kMaxSharedTiles = 8;
constexpr int kMaxSlots = kMaxRouted + kMaxShared * kMaxSharedTiles;
__host__ __device__ constexpr int slot_capacity(int E, int S) { return E + S * kMaxSharedTiles; }
constexpr int kMaxHsplit = 16;     // router slices of H
constexpr int kMaxI = 16384;       // largest intermediate size

// Per-pair histogram of the selection scores, filled by the gate epilogues and read by the
// selection: bin = the top 12 bits of the score's fp32 pattern (its sign bit is 0), i.e. the
// exponent and the 3 leading mantissa bits.  The 20 bits below are five 4-bit radix digits.
constexpr int kHistBins = 2048;
constexpr int kHistShift = 20;

// device error word codes
constexpr int kErrNanLogit = 1;
constexpr int kErrNanAct = 2;

// One expert that this call evaluates: a routed expert with >= 1 token, or a shared expert.
struct Slot {
  int kind;    // 0 routed, 1 shared
  int expert;  // routed expert index, or shared expert index
  int T;       // tokens of this expert
  int q0;      // first pair index of its tokens (pairs of a slot are contiguous, tokens ascending)
  int I;       // intermediate size
  int item0;   // first gate work item of this slot
  int pad0, pad1;
};

// A slot written by an earlier kernel of the same call, read through L2 (never a stale L1 line).
__device__ __forceinline__ Slot load_slot(const Slot* s) {
  const int4 a = __ldcg(reinterpret_cast<const int4*>(s));
  const int4 b = __ldcg(reinterpret_cast<const int4*>(s) + 1);
  Slot r;
  r.kind = a.x; r.expert = a.y; r.T = a.z; r.q0 = a.w;
  r.I = b.x; r.item0 = b.y; r.pad0 = b.z; r.pad1 = b.w;
  return r;
}

// Index j of the last table entry with tab[j].w <= item (entries ascending in .w).
__device__ __forceinline__ int find_item_slot(const int4* tab, int n, int item) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid].w <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// meta words written by the router kernel
enum { kMetaSlots = 0, kMetaPairs = 1, kMetaGateItems = 2, kMetaTouched = 3, kMetaWords = 8 };

struct FwdParams {
  int H, E, k, S, I, Ish, B, Imax;
  int Bmax;         // max_tokens of the handle
  int hsplit;       // router slices of H
  int e_begin, e_end;     // routed experts this handle evaluates (expert parallelism)
  unsigned shared_mask;   // shared experts this handle evaluates (bit s = shared expert s)
  int router_cluster;  // CTAs of the single-cluster router on this device (0: multi-CTA only)
  int route;
  int sel_mode[2];  // [0] routed, [1] shared: 0 top-K, 1 threshold
  int sel_K[2];
  float sel_t[2];
  const void* x;
  const void* router;
  const void* gate_r;
  const void* updown_r;
  const void* gate_s;
  const void* updown_s;
  void* out;
  // workspace
  float* logits;       // [Bmax][E]
  float* logit_part;   // [kMaxHsplit][Bmax][E] partial router logits
  int* topk_idx;       // [Bmax][k]
  float* topk_w;       // [Bmax][k]
  int* pair_index;     // [Bmax][k+S]
  int* pair_token;     // [Pmax]
  float* pair_w;       // [Pmax]
  int* pair_slot;      // [Pmax]
  Slot* slots;         // [slot_capacity(E, S)]
  int* meta;           // [kMetaWords]
  unsigned* tile_ticket;   // [ceil(Bmax/8)]
  unsigned* global_ticket; // [1]
  unsigned* slot_ticket;   // [slot_capacity(E, S)]
  float* act;          // [Pmax][Imax]
  uint32_t* maskbits;  // [Pmax][Imax/32]
  uint32_t* ubits;     // [slot_capacity(E, S)][Imax/32]
  int* ulist;          // [slot_capacity(E, S)][Imax] ascending union rows of each slot
  int* ucnt;           // [slot_capacity(E, S)]
  float* out_acc;      // [Bmax][H]
  int* err;            // device error word
  const void* zero_row;  // H zero elements (source of the copies of absent tokens)
  unsigned long long* trace;  // per-CTA phase timestamps (nullptr: tracing off)
  unsigned* claim;            // [3] work-item counters: gate (routed), up/down, gate (shared)
  unsigned* hist;             // [Pmax][kHistBins] score histograms of top-K pairs (zero at rest)
  // roster routing (nullptr: off): the router picks the top-k of logits + router_bias and adds
  // its choice to roster_counts; the weights stay those of the unbiased logits
  const float* router_bias;   // [B][E]
  int* roster_counts;         // [B][E] per-sequence selection counts (the caller's)
  // dense masked fallback: a slot with T >= dense_min tokens is computed by the tcgen05 GEMMs
  int dense_min;              // INT_MAX: never
  int imax_pad;               // Imax rounded up to 128 (row length of hbuf)
  __nv_bfloat16* xp;          // [Pmax][H] x rows of the pairs of dense slots
  __nv_bfloat16* hbuf;        // [Pmax][imax_pad] mask * SiLU(g) * u of dense slots, bf16
  // fused layer kernel: readiness of the work that depends on other CTAs (zero at rest)
  unsigned* tile_done;        // [Pmax] gate items finished per token tile, at its first pair
  int* s_task;                // [Pmax] selection tasks in the order they became ready: pair + 1
  unsigned* fq;               // [4] selection tasks reserved, claimed; up/down items claimed
  unsigned long long* u_res;  // [1] up/down entries published << 32 | up/down items reserved
  int4* u_ent;                // [slot_capacity(E, S)] per entry: {slot + 1, first item, items, union rows}
};

// Phase timestamps for tracing: kernel k, CTA b, point i (i < kTracePoints).
constexpr int kTraceKernels = 5, kTraceCtas = 1024, kTracePoints = 8;
__device__ __forceinline__ void trace_point(const unsigned long long* tr_base, int kernel, int i) {
  if (tr_base && threadIdx.x == 0 && blockIdx.x + blockIdx.y * gridDim.x < kTraceCtas) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    const_cast<unsigned long long*>(tr_base)[((size_t)kernel * kTraceCtas + blockIdx.x +
                                              blockIdx.y * gridDim.x) * kTracePoints + i] = t;
  }
}

// A plain value (not a time) in a trace slot, e.g. how many items a CTA processed.
__device__ __forceinline__ void trace_value(const unsigned long long* tr_base, int kernel, int i,
                                            unsigned long long v) {
  if (tr_base && threadIdx.x == 0 && blockIdx.x + blockIdx.y * gridDim.x < kTraceCtas)
    const_cast<unsigned long long*>(tr_base)[((size_t)kernel * kTraceCtas + blockIdx.x +
                                              blockIdx.y * gridDim.x) * kTracePoints + i] = v;
}

// Slot table in shared memory as int4 {expert | kind << 16, T, q0, item0}.
__device__ __forceinline__ void load_slot_table(const FwdParams& p, int n_slots, int4* s_tab) {
  for (int j = threadIdx.x; j < n_slots; j += blockDim.x) {
    const Slot s = load_slot(&p.slots[j]);
    s_tab[j] = make_int4(s.expert | (s.kind << 16), s.T, s.q0, s.item0);
  }
}

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch: a kernel launched with the programmatic-serialization attribute
// may start while its predecessor runs; it must wait before it reads the predecessor's output.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// loads
__device__ __forceinline__ uint4 ld_stream(const void* p) {  // read-once weights: skip L1
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_nc(const void* p) {  // read-only, reused: through L1
  return __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ int ld_cg(const int* p) { return __ldcg(p); }
__device__ __forceinline__ unsigned ld_cg(const unsigned* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }

// bitwise OR into global memory, no value returned (an atomicOr whose result is unused may
// still wait for it)
__device__ __forceinline__ void red_or(uint32_t* p, uint32_t v) {
  asm volatile("red.global.or.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// fp32 vector reductions into global memory (sm_90+); v4 needs a 16-byte aligned address
__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_add_f32(float* p, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// ---------------------------------------------------------------------------------------------
// bf16 helpers
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------------------------
// scans and reductions
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Exclusive prefix sum of v over the block (blockDim.x a multiple of 32, <= 1024); scratch holds
// 33 ints.  Returns the exclusive prefix; *total gets the block sum.  Contains __syncthreads.
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? scratch[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += y;
    }
    if (lane < nw) scratch[lane] = si - s;
    if (lane == 31) scratch[32] = si;
  }
  __syncthreads();
  int res = scratch[warp] + incl - v;
  if (total) *total = scratch[32];
  __syncthreads();
  return res;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Selection key of an activation: the fp32 pattern of |a|, which orders like the score; a NaN
// activation scores 0.
__device__ __forceinline__ uint32_t score_key(float a) {
  return isnan(a) ? 0u : __float_as_uint(fabsf(a));
}

__device__ __forceinline__ void red_add_u32(unsigned* p, unsigned v) {
  asm volatile("red.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Whether the pairs of kind (0 routed, 1 shared) are cut by the top-K radix selection, which
// reads the score histogram (threshold mode, K = 0 and K = I need none).
__device__ __forceinline__ bool uses_hist(const FwdParams& p, int kind) {
  const int I = kind ? p.Ish : p.I;
  return p.hist && p.sel_mode[kind] == 0 && p.sel_K[kind] > 0 && p.sel_K[kind] < I;
}

// Counts activation a of pair q in the pair's score histogram.
__device__ __forceinline__ void hist_add(const FwdParams& p, int q, float a) {
  red_add_u32(&p.hist[(size_t)q * kHistBins + (score_key(a) >> kHistShift)], 1u);
}

__device__ __forceinline__ void set_error(int* err, int code) { atomicCAS(err, 0, code); }

template <typename T>
struct Elt;
template <>
struct Elt<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr int kPerVec = 8;  // elements per 16-byte vector
};
template <>
struct Elt<float> {
  static constexpr int kBytes = 4;
  static constexpr int kPerVec = 4;
};

// Slot lookup: index j with items[j] <= i < items[j+1] (items ascending, n entries + sentinel).
__device__ __forceinline__ int find_slot(const int* items, int n, int i) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (items[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace moe
