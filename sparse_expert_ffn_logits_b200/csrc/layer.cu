// layer.cu - the fused decode layer: gate, selection and sparse up/down of one call in one
// persistent kernel, so that the selection of a token tile starts as soon as the tile's gate rows
// are done and an expert's up/down starts as soon as its union of kept neurons is known, while
// the weight streams of the other experts go on ("Uncovering Intra-expert Activation Sparsity
// ...", technical summary, Methodology: dense gate, activation masking, fused sparse up-down; Key
// contributions: the layer stays one graph-capturable unit).
//
// One CTA per SM, the roles of the gate and up/down ring kernels:
//   meta warp     decides the CTA's next piece of work and publishes it as a record in a ring of
//                 kLayerRing shared-memory records;
//   copier warp   streams the record's weight rows into a ring of shared-memory stages (bulk
//                 asynchronous copies completed on mbarriers);
//   2 coefficient warps  fill the up/down records' rows and coefficients;
//   8 consumer warps     compute: tensor-core tiles (m16n8k16) for gate and up/down, the radix
//                 selection for a selection record.
// Work comes in three kinds, taken in this order of priority:
//   S  the selection of one pair (select_pair.cuh), ready once every gate item of its token tile
//      is done.  The meta warp of the CTA whose report completes a tile's count reserves the
//      tile's pairs in a task list; any CTA claims them.
//   G  a gate item (slot, token tile, 16 neurons), numbered as in the gate kernel: the shared
//      experts' items first (no routing needed), then the routed ones, a contiguous share per CTA
//      and the rest claimed from a counter.  After its consumers finish a run of items of one
//      token tile, the meta warp adds the run's length to the tile's counter.
//   U  an up/down item (slot, token tile, 16 union rows), ready once the slot's union is
//      compacted: the CTA that compacts it reserves the slot's items in one range of a growing
//      index space and publishes an entry; CTAs claim items from a counter.
// No wait depends on another CTA's progress except for work that another CTA already holds (a
// claimed gate item, a claimed selection), and every wait is bounded by %globaltimer, so the
// kernel cannot deadlock on work that nobody will do; a time-out sets the device error word.
#include "kernels.h"
#include "select_pair.cuh"
#include "tile.cuh"
#include "tma.cuh"

namespace moe {
namespace {

constexpr int kCoefWarps = 2;
constexpr int kLayerThreads = kThreads + 64 + 32 * kCoefWarps;
constexpr int kCopier = kWarps, kMetaWarp = kWarps + 1, kCoefWarp0 = kWarps + 2;
constexpr int kGateChunk = 2;  // gate items claimed at a time from the work counter
constexpr int kGateRun = 8;    // consecutive gate items of a CTA's static rounds
// Records in flight per CTA: the meta warp publishes up to kLayerRing - 1 records ahead of the
// consumers (record i reuses the slot of record i - kLayerRing once that one is finished).
constexpr int kLayerRing = 6;
static_assert((2 * 16 + 4 * kLayerRing) * 8 <= kBarBytes, "mbarriers of the fused kernel");

enum : int { kRecG = 0, kRecU = 1, kRecS = 2 };

struct LayerMeta {
  const __nv_bfloat16* base;  // G: first of the item's 16 gate rows; U: the expert's [I][2][H]
  int type;                   // kRecG, kRecU, kRecS
  int end;                    // 1: no more records (the CTA's loops end here)
  int key;                    // token tile id of G and U records (-1 for S)
  int xlast;                  // G, U: the CTA's next record of this kind is of another tile
                              // (G: 2 when no gate record follows in this CTA)
  int q0, nt, n0;             // G: first pair of the tile, its tokens, first neuron
  int q;                      // S: the pair
  int j, tt, rg;              // U: slot, token tile, row group
  int tok[kTileTok];          // G, U: token of each tile column (-1 past the end)
  float w[kTileTok];          // U: routing weight of each tile column
  int rows[kTileRows];        // U: union neuron of each row (a repeated valid row past the end)
  float coef[kTileRows][kTileTok];  // U: SiLU(g) where the token's pair keeps the row, else 0
};

// Named barrier 2 over the 256 consumer threads, for the selection (barrier 1 is taken by the
// consumer handshakes of the tile loops).
struct ConsumerBar {
  __device__ __forceinline__ void operator()() const {
    asm volatile("bar.sync 2, %0;" ::"n"(kThreads) : "memory");
  }
};

__device__ __forceinline__ unsigned ld_volatile(const unsigned* p) {
  return *reinterpret_cast<const volatile unsigned*>(p);
}
__device__ __forceinline__ int ld_volatile(const int* p) {
  return *reinterpret_cast<const volatile int*>(p);
}
__device__ __forceinline__ unsigned long long ld_volatile(const unsigned long long* p) {
  return *reinterpret_cast<const volatile unsigned long long*>(p);
}

__device__ __forceinline__ void nanosleep_ns(unsigned ns) {
  asm volatile("nanosleep.u32 %0;" ::"r"(ns));
}

// Dynamic shared memory of the fused kernel: barriers | cross-warp sums | slot table | entry
// cache | union sizes | ring stages.  A selection takes one ring stage: the copier brings the
// pair's activations into it, and the consumers turn them into keys in place.
struct LayerSmem {
  int tab_off, ent_off, ucnt_off, ring_off;
};
__host__ __device__ inline LayerSmem layer_smem(int n_slot_max) {
  LayerSmem l;
  l.tab_off = kBarBytes + kRedBytes;
  l.ent_off = l.tab_off + n_slot_max * 16;
  l.ucnt_off = l.ent_off + n_slot_max * 8;
  l.ring_off = (l.ucnt_off + n_slot_max * 4 + 127) / 128 * 128;
  return l;
}

// Publishes slot j's union (urows rows) as the next up/down entry: its items are reserved as one
// range of the item index space.  One thread; the union list was written by the CTA's consumer
// threads before the barrier that precedes this call.
__device__ void publish_entry(const FwdParams& p, const int4* s_tab, int j, int urows) {
  const int T = s_tab[j].y;
  const int n = ((urows + kTileRows - 1) / kTileRows) * ((T + kTileTok - 1) / kTileTok);
  __threadfence();
  const unsigned long long old = atomicAdd(p.u_res, (1ull << 32) | (unsigned long long)n);
  int4* ent = p.u_ent + (int)(old >> 32);
  ent->y = (int)(old & 0xffffffffull);
  ent->z = n;
  ent->w = urows;
  __threadfence();
  *reinterpret_cast<volatile int*>(&ent->x) = j + 1;
}

template <int NK, int BPW>
__global__ void __launch_bounds__(kLayerThreads, 1) layer_kernel(FwdParams p, Ring rc) {
  static_assert(NK > 0, "the fused kernel keeps the token fragments in registers");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ LayerMeta s_meta[kLayerRing];
  __shared__ __align__(16) uint32_t s_hcw[2][kTileTok][kTileRows / 2];
  __shared__ SelShared<kThreads> s_sel;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int n_slot_max = min(slot_capacity(p.E, p.S), kMaxSlots);
  const LayerSmem L = layer_smem(n_slot_max);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + rc.ns;
  uint64_t* mfull = empty + rc.ns;  // the record's coefficients are written (U)
  uint64_t* mrows = mfull + kLayerRing;  // the record is complete for the copier and the tiles
  uint64_t* mhead = mrows + kLayerRing;  // the meta warp has written the record
  uint64_t* edone = mhead + kLayerRing;  // consumers and copier are done with the record
  float(*red)[kWarps][4][32] = reinterpret_cast<float(*)[kWarps][4][32]>(smem + kBarBytes);
  int4* s_tab = reinterpret_cast<int4*>(smem + L.tab_off);  // {expert | kind << 16, T, q0, item0}
  int2* s_ent = reinterpret_cast<int2*>(smem + L.ent_off);  // up/down entries {slot, first item}
  int* s_ucnt = reinterpret_cast<int*>(smem + L.ucnt_off);  // union rows of each slot
  unsigned char* ring = smem + L.ring_off;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  trace_point(p.trace, 1, 0);
  if (threadIdx.x == 0) {
    for (int i = 0; i < rc.ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    for (int i = 0; i < kLayerRing; ++i) {
      mbar_init(&mfull[i], 2);  // meta warp + the coefficient warp of the record
      mbar_init(&mrows[i], 2);
      mbar_init(&mhead[i], 1);
      mbar_init(&edone[i], 2);  // consumer thread 0 + copier
    }
    s_abort = 0;
    mbar_init_fence();
  }
  for (int i = threadIdx.x; i < kLayerRing * (int)(sizeof(LayerMeta) / 4); i += blockDim.x)
    reinterpret_cast<int*>(s_meta)[i] = 0;
  // Down-projection accumulators in tensor memory, as in the up/down kernel: consumer warp w keeps
  // the 16 values of each of its 64-column sub-chunks (spw per stage, nk stages) in lane quarter
  // w % 4, columns 256 (w / 4) + 16 (kc spw + local sub-chunk), while consecutive up/down items of
  // one (expert, token tile) follow each other, and flushes them once per such run.
  const int spw = (rc.kc / 64 + kWarps - 1) / kWarps;
  const bool tmem_acc = rc.nk * spw * 16 <= 256;
  if (tmem_acc && warp == 0) tmem_alloc(&s_tmem, 512);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tmem_base = tmem_acc ? s_tmem : 0u;
  pdl_trigger();
  const int H = p.H, Imax = p.Imax, Wmax = p.Imax / 32;
  volatile int* abort = &s_abort;

  if (warp == kMetaWarp) {
    // ------------------------------------------------------------------ meta warp
    // Gate items: first the shared experts' items, which need no routing (shared expert s
    // evaluates every token: token t is pair B k + s B + t), a few at a time from a counter while
    // the router may still run; then, after the wait for the router, the routed items.  About
    // 7/8 of those go out in static rounds: in round r, CTA c takes the kGateRun items of run
    // c + r G, so that all CTAs move through the slots together and the slots' tiles complete
    // one after another (their selections and up/down items become ready while the gate goes
    // on); the rest is claimed from a second counter, so that fast CTAs take more of the tail.
    const int Bt = (p.B + kTileTok - 1) / kTileTok;
    const int sh_groups = p.Ish / kTileRows;
    const int n_pre = p.S > 0 ? __popc(p.shared_mask) * sh_groups * Bt : 0;
    int n_slots = 0, n_items = n_pre, dyn0 = 0, n_sp_pairs = 0;
    bool routed_known = false;
    int cb = 0, ce = 0, pre_next = 0, pre_end = 0, round = 0;
    auto learn_routing = [&]() {
      pdl_wait();
      if (p.trace && lane == 0 && blockIdx.x < kTraceCtas)
        const_cast<unsigned long long*>(p.trace)[((size_t)1 * kTraceCtas + blockIdx.x) *
                                                     kTracePoints + 1] = globaltimer();
      n_slots = ld_cg(&p.meta[kMetaSlots]);
      const int n_routed = ld_cg(&p.meta[kMetaGateItems]) - n_pre;
      int tsum = 0;
      for (int j = lane; j < n_slot_max; j += 32) {
        const Slot sl = load_slot(&p.slots[j]);
        s_tab[j] = make_int4(sl.expert | (sl.kind << 16), sl.T, sl.q0, sl.item0);
        if (j < n_slots) tsum += sl.T;
      }
      n_sp_pairs = __reduce_add_sync(0xffffffffu, tsum);  // one selection task per pair
      __syncwarp();
      const int per_round = (int)gridDim.x * kGateRun;
      dyn0 = n_routed * 7 / 8 / per_round * per_round;  // routed items of the static rounds
      cb = ce = 0;
      n_items = n_pre + n_routed;
      routed_known = true;
    };
    auto claim_g = [&]() -> int {
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
        const int run = blockIdx.x + round * (int)gridDim.x;
        if ((run + 1) * kGateRun <= dyn0) {  // the next static round
          ++round;
          cb = n_pre + run * kGateRun;
          ce = cb + kGateRun;
          return cb++;
        }
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

    int mi = 0, si = 0;
    // Frees the ring slot of record mi: waits until record mi - kLayerRing is finished
    // (consumers and copier).  False once the CTA aborts.
    auto slot_free = [&]() -> bool {
      for (; si <= mi - kLayerRing; ++si)
        if (!mbar_wait(&edone[si % kLayerRing], (si / kLayerRing) & 1, abort, p.err))
          return false;
      return true;
    };
    auto post = [&](int m) {  // the meta warp's arrivals for a written record
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&mhead[m]);
        mbar_arrive(&mrows[m]);
        mbar_arrive(&mfull[m]);
      }
      __syncwarp();
    };

    // selection tasks
    int pend_s = -1;  // claimed task whose pair is not written yet (-1 none, -2 all claimed)
    // sa, sc: the tasks reserved and claimed so far, as lane 0 read them
    auto take_s = [&](unsigned sa, unsigned sc) -> int {
      if (!routed_known || pend_s == -2) return -1;
      int q = -1, ps = pend_s;
      if (lane == 0) {
        if (ps == -1 && sc < sa) {
          const unsigned c = atomicAdd(&p.fq[1], 1u);
          ps = (int)c < n_sp_pairs ? (int)c : -2;
        }
        if (ps >= 0) {
          const int v = ld_volatile(&p.s_task[ps]);
          if (v > 0) {
            __threadfence();
            q = v - 1;
            ps = -1;
          }
        }
      }
      pend_s = __shfl_sync(0xffffffffu, ps, 0);
      return __shfl_sync(0xffffffffu, q, 0);
    };

    // up/down items
    int ub = 0, ue = 0;   // claimed items not yet published
    int ne = 0;           // entries cached in s_ent
    int cached_end = 0;   // first item past the cached entries
    int ecur = 0;         // entry of item ub (a CTA's items ascend)
    bool u_done = false;  // every entry is in and no claimed item is left
    auto cache_entries = [&]() -> int {  // returns the entries published so far
      const int n_pub = (int)(ld_volatile(p.u_res) >> 32);
      while (ne < n_pub) {
        const int e = ne + lane;
        const int f = e < n_pub ? ld_volatile(&p.u_ent[e].x) : 0;
        const unsigned ready = __ballot_sync(0xffffffffu, f > 0);
        const int nrdy = ready == 0xffffffffu ? 32 : __ffs(~ready) - 1;
        if (nrdy == 0) break;
        int end_e = 0;
        if (lane < nrdy) {
          __threadfence();
          const int base = __ldcg(&p.u_ent[e].y), n = __ldcg(&p.u_ent[e].z);
          const int urows = __ldcg(&p.u_ent[e].w);
          s_ent[e] = make_int2(f - 1, base);
          s_ucnt[f - 1] = urows;
          end_e = base + n;
        }
        cached_end = __shfl_sync(0xffffffffu, end_e, nrdy - 1);
        ne += nrdy;
        __syncwarp();
      }
      return n_pub;
    };
    // Up/down items are handed out as in the up/down kernel, on the items published when the
    // first CTA runs out of gate items: that CTA takes a snapshot of the reserved count (a CAS
    // on fq[3], so that every CTA sees the same one), and 3/4 of those items go out as one
    // contiguous share per CTA (runs of one token tile: the sums stay in tensor memory, the
    // token fragments in registers).  The rest, and every item published later, is claimed one
    // at a time from fq[2].
    int u_next = -1;      // lane 0: a dynamic item claimed ahead (-1: none)
    bool u_static = false;  // the item last taken is from this CTA's contiguous share
    int dyn_base = -1;    // first dynamic item (-1: no snapshot taken yet by this CTA)
    auto claim_u_ahead = [&]() {
      if (lane == 0 && u_next < 0 && dyn_base >= 0 && ub >= ue)
        u_next = (int)atomicAdd(&p.fq[2], 1u);
    };
    auto take_u = [&](int* item) -> bool {
      if (u_done || !routed_known) return false;
      if (dyn_base < 0) {
        int snap = 0;
        if (lane == 0) {
          const unsigned tot = (unsigned)(ld_volatile(p.u_res) & 0xffffffffull);
          const unsigned old = atomicCAS(&p.fq[3], 0u, tot + 1u);
          snap = (int)(old == 0u ? tot : old - 1u);
        }
        snap = __shfl_sync(0xffffffffu, snap, 0);
        const int share = snap * 3 / 4 / (int)gridDim.x;
        ub = blockIdx.x * share;
        ue = ub + share;
        dyn_base = share * (int)gridDim.x;
      }
      u_static = ub < ue;
      if (ub >= ue) {  // one dynamic item
        int b = u_next;
        if (lane == 0 && b < 0) b = (int)atomicAdd(&p.fq[2], 1u);
        ub = dyn_base + __shfl_sync(0xffffffffu, b, 0);
        ue = ub + 1;
        u_next = -1;
      }
      if (ub >= cached_end) {
        const int n_pub = cache_entries();
        if (ub >= cached_end) {
          if (n_pub == n_slots && ne == n_pub) u_done = true;  // the item will never exist
          return false;
        }
      }
      while (ecur + 1 < ne && s_ent[ecur + 1].y <= ub) ++ecur;
      *item = ub++;
      return true;
    };

    // Trace of the meta warp (tracing on): row 2 = selections (0 end of own gate items,
    // 1 first published, 2 count, 3 last published), row 3 = up/down items (0 first claim,
    // 1 first published, 2 count, 3 end; 4 ns waiting for a free record, 5 ns idle).
    auto tr = [&](int row, int point, unsigned long long v) {
      if (p.trace && lane == 0 && blockIdx.x < kTraceCtas)
        const_cast<unsigned long long*>(p.trace)[((size_t)row * kTraceCtas + blockIdx.x) *
                                                     kTracePoints + point] = v;
    };
    unsigned long long t_wait = 0, t_idle = 0;
    int n_s = 0, n_u = 0;
    // A gate item's slot entry, local index and token tile (shared items carry the local shared
    // expert's entry directly)
    struct GPlace {
      int4 sl;
      int local, key;
    };
    auto place_g = [&](int item) -> GPlace {
      GPlace g;
      if (item < n_pre) {
        const int o = item / (sh_groups * Bt);  // o-th shared expert of this handle
        unsigned msk = p.shared_mask;
        for (int i = 0; i < o; ++i) msk &= msk - 1;
        const int s_i = __ffs(msk) - 1;
        g.sl = make_int4(s_i | (1 << 16), p.B, p.B * p.k + s_i * p.B, 0);
        g.local = item - o * sh_groups * Bt;
        g.key = (1 << 20) + s_i * 1024 + g.local / sh_groups;
      } else {
        const int r = item - n_pre;
        const int j = find_item_slot(s_tab, n_slots, r);
        g.sl = s_tab[j];
        g.local = r - g.sl.w;
        g.key = j * 1024 + g.local / (p.I / kTileRows);
      }
      return g;
    };
    // the current gate item and the next one, claimed ahead: a record whose successor is of
    // another token tile (or none) ends its run, which its consumers then report
    int gcur = claim_g();
    GPlace gpl = gcur >= 0 ? place_g(gcur) : GPlace{};
    int gnxt = gcur >= 0 ? claim_g() : -1;
    GPlace npl = gnxt >= 0 ? place_g(gnxt) : GPlace{};
    int tok_key = -2, tok_l = -1;  // token of lane l in the last gate tile the warp looked up
    unsigned long long idle_t0 = 0;
    bool g_end_seen = false;
    unsigned sa_next = 0, sc_next = 0;
    while (!*abort) {
      // the task counters as lane 0 read them in the previous iteration (the loads of the next
      // iteration's values are issued here, so their round trip overlaps this one)
      const unsigned sa = sa_next, sc = sc_next;
      if (lane == 0 && routed_known) {
        sa_next = ld_volatile(&p.fq[0]);
        sc_next = ld_volatile(&p.fq[1]);
      }
      {
        const unsigned long long t0 = p.trace ? globaltimer() : 0ull;
        if (!slot_free()) break;
        if (p.trace) t_wait += globaltimer() - t0;
      }
      const int m = mi % kLayerRing;
      const int qs = take_s(sa, sc);
      if (qs >= 0) {
        if (lane == 0) {
          s_meta[m].type = kRecS;
          s_meta[m].end = 0;
          s_meta[m].key = -1;
          s_meta[m].q = qs;
        }
        post(m);
        if (n_s == 0) tr(2, 1, globaltimer());
        tr(2, 3, globaltimer());
        ++n_s;
        ++mi;
        idle_t0 = 0;
        continue;
      }
      if (gcur >= 0) {
        const int4 sl = gpl.sl;
        const int local = gpl.local, key = gpl.key;
        const int kind = sl.x >> 16, ex = sl.x & 0xffff, T = sl.y, q0 = sl.z;
        const int I = kind ? p.Ish : p.I;
        const int tt = local / (I / kTileRows), rg = local % (I / kTileRows);
        const int nt = min(kTileTok, T - tt * kTileTok);
        if (lane == 0) {  // the copier's part first: it needs no token
          const __nv_bfloat16* gb =
              kind == 0 ? static_cast<const __nv_bfloat16*>(p.gate_r) + (size_t)ex * p.I * H
                        : static_cast<const __nv_bfloat16*>(p.gate_s) + (size_t)ex * p.Ish * H;
          s_meta[m].base = gb + (size_t)rg * kTileRows * H;
          s_meta[m].type = kRecG;
          s_meta[m].end = 0;
          s_meta[m].key = key;
          // 2: the run ends and no gate record follows in this CTA (its report is settled at
          // once: nothing later would look at it)
          s_meta[m].xlast = gnxt < 0 ? 2 : npl.key != key ? 1 : 0;
          s_meta[m].q0 = q0 + tt * kTileTok;
          s_meta[m].nt = nt;
          s_meta[m].n0 = rg * kTileRows;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&mhead[m]);
          mbar_arrive(&mrows[m]);
        }
        if (key != tok_key) {
          // a new tile: a shared expert's pair q0 + i is token i; a routed pair's token is in
          // the pair table (one round trip)
          tok_key = key;
          tok_l = lane >= nt ? -1
                  : kind ? tt * kTileTok + lane
                         : __ldcg(&p.pair_token[q0 + tt * kTileTok + lane]);
        }
        if (lane < kTileTok) s_meta[m].tok[lane] = tok_l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&mfull[m]);
        __syncwarp();
        ++mi;
        gcur = gnxt;
        gpl = npl;
        gnxt = gcur >= 0 ? claim_g() : -1;
        if (gnxt >= 0) npl = place_g(gnxt);
        idle_t0 = 0;
        continue;
      }
      if (!g_end_seen) {
        g_end_seen = true;
        tr(2, 0, globaltimer());
      }
      int item;
      if (take_u(&item)) {
        const int j = s_ent[ecur].x, local = item - s_ent[ecur].y;
        const int nrg = (s_ucnt[j] + kTileRows - 1) / kTileRows;
        const int tt = local / nrg, rg = local % nrg;
        // within the contiguous share the next item is known: the run of this token tile goes
        // on if it is the next row group of the same tile; a claimed item ends its run
        const int e_end = ecur + 1 < ne ? s_ent[ecur + 1].y : cached_end;
        const bool more = u_static && ub < ue && ub < e_end && (local + 1) / nrg == tt;
        if (lane == 0) {
          const int4 sl = s_tab[j];
          const int kind = sl.x >> 16, ex = sl.x & 0xffff;
          s_meta[m].base = kind == 0 ? static_cast<const __nv_bfloat16*>(p.updown_r) +
                                           (size_t)ex * p.I * 2 * H
                                     : static_cast<const __nv_bfloat16*>(p.updown_s) +
                                           (size_t)ex * p.Ish * 2 * H;
          s_meta[m].type = kRecU;
          s_meta[m].end = 0;
          s_meta[m].key = j * 1024 + tt;
          s_meta[m].xlast = more ? 0 : 1;
          s_meta[m].j = j;
          s_meta[m].tt = tt;
          s_meta[m].rg = rg;
        }
        post(m);
        claim_u_ahead();
        if (n_u == 0) tr(3, 1, globaltimer());
        ++n_u;
        ++mi;
        idle_t0 = 0;
        continue;
      }
      if (routed_known && u_done) break;
      // nothing to publish yet
      const unsigned long long now = globaltimer();
      if (idle_t0 == 0) idle_t0 = now;
      if (now - idle_t0 > kWaitLimitNs) {
        if (lane == 0) {
          *abort = 1;
          set_error(p.err, kErrTimeout);
        }
        __syncwarp();
        break;
      }
      nanosleep_ns(64);
      if (p.trace) t_idle += globaltimer() - now;
    }
    tr(2, 2, (unsigned long long)n_s);
    tr(3, 2, (unsigned long long)n_u);
    tr(3, 3, globaltimer());
    tr(3, 4, t_wait);
    tr(3, 5, t_idle);
    if (!routed_known) learn_routing();  // every CTA waits for the router before it exits
    // closing records: one for the copier and consumers, one more so that both coefficient
    // warps see it
    for (int e = 0; e < 2; ++e, ++mi) {
      const int m = mi % kLayerRing;
      if (!*abort) slot_free();
      if (lane == 0) {
        s_meta[m].end = 1;
        mbar_arrive(&mhead[m]);
        mbar_arrive(&mrows[m]);
        mbar_arrive(&mfull[m]);
      }
      __syncwarp();
    }
    return;
  }


  if (warp >= kCoefWarp0) {
    // ------------------------------------------------------------------ coefficient warp c
    // Up/down records mi with mi % kCoefWarps == c: rows, tokens and weights (mrows), then the
    // coefficients after one more round trip (mfull).  Other records only get its arrivals, which
    // keeps it in step with the ring of records.
    const int cw = warp - kCoefWarp0;
    bool waited = false;
    for (int mi = cw;; mi += kCoefWarps) {
      const int m = mi % kLayerRing;
      if (!mbar_wait(&mhead[m], (mi / kLayerRing) & 1, abort, p.err)) break;
      const int end = s_meta[m].end, type = s_meta[m].type;
      if (end || type != kRecU) {
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&mrows[m]);
          mbar_arrive(&mfull[m]);
        }
        if (end) break;
        continue;
      }
      if (!waited) {  // the pair tables and the selections come from the router and other CTAs
        pdl_wait();
        waited = true;
      }
      const int j = s_meta[m].j, tt = s_meta[m].tt, rg = s_meta[m].rg;
      const int4 sl = s_tab[j];
      const int T = sl.y, q0 = sl.z, rows = s_ucnt[j];
      const int nt = min(kTileTok, T - tt * kTileTok);
      const int qt = q0 + tt * kTileTok;
      // row of this lane (lanes 0..15) and token of this lane (lanes 0..7)
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
    // ------------------------------------------------------------------ copier
    // G: the item's 16 gate rows, kc columns per stage; U: the up pieces of the item's 16 union
    // rows, then their down pieces; S: nothing.  One bulk copy per row piece.
    const uint32_t piece = rc.kc * 2;
    int it = 0;
    for (int mi = 0; !*abort; ++mi) {
      const int m = mi % kLayerRing;
      if (!mbar_wait(&mrows[m], (mi / kLayerRing) & 1, abort, p.err)) break;
      if (s_meta[m].end) break;
      const int type = s_meta[m].type;
      const __nv_bfloat16* row =
          type == kRecG ? s_meta[m].base + (size_t)(lane & 15) * H
                        : s_meta[m].base + (size_t)s_meta[m].rows[lane & 15] * 2 * H;
      const int q = s_meta[m].q;
      __syncwarp();
      if (lane == 0) mbar_arrive(&edone[m]);  // the record is read
      if (type == kRecS) {
        // the pair's activations (written by other CTAs' gate epilogues, published to this
        // CTA through the task list) into one stage, for the selection
        const int st = it % rc.ns;
        if (!mbar_wait(&empty[st], ((it / rc.ns) & 1) ^ 1, abort, p.err)) break;
        const uint32_t bytes = (uint32_t)((q >= p.B * p.k ? p.Ish : p.I) * 4);
        if (lane == 0) {
          asm volatile("fence.proxy.async;" ::: "memory");
          mbar_arrive_expect_tx(&full[st], bytes);
          bulk_g2s(ring + (size_t)st * rc.stage_bytes, p.act + (size_t)q * Imax, bytes, &full[st]);
        }
        __syncwarp();
        ++it;
        continue;
      }
      bool stop = false;
      for (int half = 0; half < (type == kRecU ? 2 : 1) && !stop; ++half) {
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
    for (int k = it - 1; k >= 0 && k >= it - rc.ns; --k)
      mbar_drain(&full[k % rc.ns], (k / rc.ns) & 1);
    return;
  }

  // -------------------------------------------------------------------- consumers
  uint4 xr[NK][BPW];
  int it = 0, ib = 0, cur = -1;
  int run_key = -1;  // token tile of the open run of up/down sums in tensor memory
  int g_run = 0;     // thread 0: gate records of the current run of one token tile
  // thread 0: the last run report, whose result is looked at one gate record later
  int rep_q0 = -1, rep_cnt = 0, rep_nt = 0;
  unsigned rep_old = 0, rep_target = 0;
  bool nan_seen = false, waited = false;
  const int nblk = rc.kc / 32, nsub = rc.kc / 64;
  const uint32_t tmem_warp = tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + 256u * (warp >> 2);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(p.x);
  int mi = 0;
  for (;; ++mi) {
    const int m = mi % kLayerRing;
    const uint32_t ph = (mi / kLayerRing) & 1;
    mbar_wait(&mrows[m], ph, abort, p.err);
    // the end (or an abort) is decided by all consumer warps together
    if (consumer_sync_or(kThreads, s_meta[m].end || *abort)) break;
    if (mi == 0) trace_point(p.trace, 1, 2);
    const LayerMeta& mt = s_meta[m];
    const int type = mt.type;
    if (type != kRecG && threadIdx.x == 0 && rep_q0 >= 0) {  // a pending run report
      if (rep_old + (unsigned)rep_cnt == rep_target && !*abort) {
        __threadfence();
        const unsigned k0 = atomicAdd(&p.fq[0], (unsigned)rep_nt);
        for (int i = 0; i < rep_nt; ++i)
          *reinterpret_cast<volatile int*>(&p.s_task[k0 + i]) = rep_q0 + i + 1;
      }
      rep_q0 = -1;
    }
    if (type == kRecS) {
      // ---- selection of pair mt.q; the CTA that completes the slot's union publishes it
      if (!waited) {
        pdl_wait();
        waited = true;
      }
      const int st = it % rc.ns;
      mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
      uint32_t* key = reinterpret_cast<uint32_t*>(ring + (size_t)st * rc.stage_bytes);
      int j;
      const int urows = select_pair<kThreads, true>(p, mt.q, (int)threadIdx.x, key, s_sel,
                                                    ConsumerBar{}, nan_seen, &j);
      // the stage was written through the generic proxy: ordered before the next bulk copy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      ++it;
      if (urows >= 0 && threadIdx.x == 0) publish_entry(p, s_tab, j, urows);
      if (threadIdx.x == 0) {  // both arrivals on mfull precede the record's release
        mbar_wait(&mfull[m], ph, abort, p.err);
        mbar_arrive(&edone[m]);
      }
      if (mi == 0) trace_point(p.trace, 1, 4);
      continue;
    }
    // ---- gate item or up/down item: first the 16 rows against the token tile
    const int key = mt.key;
    const int q0 = mt.q0, nt = mt.nt, n0 = mt.n0, xlast = mt.xlast;
    if (type == kRecG && key != cur) mbar_wait(&mfull[m], ph, abort, p.err);  // gate tokens
    const int tok0 = mt.tok[2 * t], tok1 = mt.tok[2 * t + 1];
    if (key != cur) {  // this warp's token fragments for the new tile (one round trip)
      cur = key;
      const int tok = mt.tok[g];
#pragma unroll
      for (int kc = 0; kc < NK; ++kc)
#pragma unroll
        for (int i = 0; i < BPW; ++i) {
          const int b = warp + kWarps * i;
          xr[kc][i] = (b < nblk && tok >= 0)
                          ? ld_nc(x + (size_t)tok * H + kc * rc.kc + b * 32 + t * 8)
                          : make_uint4(0, 0, 0, 0);
        }
    }
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kc = 0; kc < NK; ++kc, ++it) {
      const int st = it % rc.ns;
      mbar_wait(&full[st], (it / rc.ns) & 1, abort, p.err);
      if (it == 0) trace_point(p.trace, 1, 3);
      const unsigned char* stage = ring + (size_t)st * rc.stage_bytes;
#pragma unroll
      for (int i = 0; i < BPW; ++i) {
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
#pragma unroll
    for (int c = 0; c < 4; ++c) red[ib][warp][c][lane] = d[c];
    if (type == kRecG) {
      // ---- gate epilogue: one activation per thread of warps 0-3, summed over the warps in
      // order; act = SiLU(g) and its count in the pair's score histogram.  Warps 0-3 then meet
      // (named barrier 3) so that every store precedes the record's release.
      const int aborted = consumer_sync_or(kThreads, *abort);
      if (threadIdx.x < 128) {
        if (!aborted) {
          const int ln = threadIdx.x & 31, c = threadIdx.x >> 5;
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) v += red[ib][w][c][ln];
          const int ti = 2 * (ln & 3) + (c & 1);
          if (ti < nt) {
            const float a = silu(v);
            nan_seen |= isnan(a);
            p.act[(size_t)(q0 + ti) * Imax + n0 + (ln >> 2) + (c >> 1) * 8] = a;
            if (uses_hist(p, q0 >= p.B * p.k)) hist_add(p, q0 + ti, a);
          }
        }
        if (xlast) asm volatile("bar.sync 3, 128;" ::: "memory");  // the run's last stores
        if (threadIdx.x == 0) {
          // A pending report (of an earlier run) is checked first: its round trip overlapped
          // the records since.  The report that completes a tile's count makes the tile's pairs
          // selection tasks.
          if (rep_q0 >= 0) {
            if (rep_old + (unsigned)rep_cnt == rep_target && !aborted) {
              __threadfence();
              const unsigned k0 = atomicAdd(&p.fq[0], (unsigned)rep_nt);
              for (int i = 0; i < rep_nt; ++i)
                *reinterpret_cast<volatile int*>(&p.s_task[k0 + i]) = rep_q0 + i + 1;
            }
            rep_q0 = -1;
          }
          // The run of gate records of this token tile ends here: its count goes to the tile's
          // counter, after a fence that makes these records' activations and histogram counts
          // visible.
          ++g_run;
          if (xlast) {
            const int I = q0 >= p.B * p.k ? p.Ish : p.I;
            __threadfence();
            rep_old = atomicAdd(&p.tile_done[q0], (unsigned)g_run);
            rep_cnt = g_run;
            rep_target = (unsigned)(I / kTileRows);
            rep_q0 = q0;
            rep_nt = nt;
            g_run = 0;
            if (xlast == 2) {
              if (rep_old + (unsigned)rep_cnt == rep_target && !aborted) {
                __threadfence();
                const unsigned k0 = atomicAdd(&p.fq[0], (unsigned)rep_nt);
                for (int i = 0; i < rep_nt; ++i)
                  *reinterpret_cast<volatile int*>(&p.s_task[k0 + i]) = rep_q0 + i + 1;
              }
              rep_q0 = -1;
            }
          }
          // both arrivals on mfull precede the record's release
          mbar_wait(&mfull[m], ph, abort, p.err);
          mbar_arrive(&edone[m]);
        }
      }
      if (mi == 0) trace_point(p.trace, 1, 4);
      ib ^= 1;
      continue;
    }
    // ---- up/down item
    if (!waited) {
      pdl_wait();
      waited = true;
    }
    const float w0 = mt.w[2 * t], w1 = mt.w[2 * t + 1];
    mbar_wait(&mfull[m], ph, abort, p.err);
    const int aborted = consumer_sync_or(kThreads, *abort);
    // 2. coefficients times u, rounded to bf16, token-major (one element per thread)
    if (threadIdx.x < 128) {
      const int ln = threadIdx.x & 31, c = threadIdx.x >> 5;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[ib][w][c][ln];
      const int r = (ln >> 2) + (c >> 1) * 8, tk = 2 * (ln & 3) + (c & 1);
      reinterpret_cast<__nv_bfloat16*>(&s_hcw[ib][tk][0])[r] =
          __float2bfloat16_rn(mt.coef[r][tk] * v);
    }
    consumer_sync(kThreads);
    if (threadIdx.x == 0) mbar_arrive(&edone[m]);  // nothing more is read from the record
    // 3-4. down projection of each stage's 64-column sub-chunks, kept in tensor memory while
    // the run of records of this (expert, token tile) goes on, reduced into out_acc in its last
    // record (interleaved with that record's tiles)
    const uint32_t b0 = s_hcw[ib][g][t], b1 = s_hcw[ib][g][4 + t];
    const bool first = key != run_key, last = xlast != 0 || !tmem_acc;
    run_key = last ? -1 : key;
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
        // token, reduced as two 16-byte vectors
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
          if (!first) {  // earlier records of the run, summed in the same order every time
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
    if (!last) tmem_wait_st();  // the next record of the run loads these columns
    if (mi == 0) trace_point(p.trace, 1, 4);
    ib ^= 1;
  }
  trace_value(p.trace, 1, 5, (unsigned long long)mi);
  if (nan_seen) set_error(p.err, kErrNanAct);
  trace_point(p.trace, 1, 7);
  // every consumer warp is done with tensor memory before warp 0 frees it
  tmem_fence_before();
  consumer_sync(kThreads);
  tmem_fence_after();
  if (tmem_acc && warp == 0) tmem_dealloc(tmem_base, 512);
}

template <int NK, int BPW>
int layer_static_smem() {
  cudaFuncAttributes fa;
  return cudaFuncGetAttributes(&fa, layer_kernel<NK, BPW>) == cudaSuccess
             ? (int)fa.sharedSizeBytes
             : 16384;
}

}  // namespace

extern const int kRegVariants[4][3];
Ring make_ring(int H, int nk_fixed, int smem_budget, int static_smem);

// Ring of the fused kernel: the stages take what the barriers, sums, selection keys and tables
// leave of the budget.
cudaError_t configure_layer(int H, int imax, int n_slot_max, int smem_budget, LaunchShape* ls) {
  ls->ring_layer.ns = 0;
  if (ls->variant == 0) return cudaSuccess;  // token tiles in shared memory: not fused
  const int nk = kRegVariants[ls->variant - 1][1];
  int stat = 0;
  cudaError_t e = cudaSuccess;
  switch (ls->variant) {
    case 1: stat = layer_static_smem<1, 2>(); e = allow_max_smem(layer_kernel<1, 2>, smem_budget); break;
    case 2: stat = layer_static_smem<1, 8>(); e = allow_max_smem(layer_kernel<1, 8>, smem_budget); break;
    case 3: stat = layer_static_smem<3, 4>(); e = allow_max_smem(layer_kernel<3, 4>, smem_budget); break;
    default: stat = layer_static_smem<4, 5>(); e = allow_max_smem(layer_kernel<4, 5>, smem_budget); break;
  }
  if (e != cudaSuccess) return e;
  const LayerSmem L = layer_smem(n_slot_max < kMaxSlots ? n_slot_max : kMaxSlots);
  Ring r = make_ring(H, nk, smem_budget, stat + 1024 + (L.ring_off - kBarBytes - kRedBytes));
  // too little room, or a selection's keys do not fit one stage: the launch chain stays in use
  if (r.ns < 2 || sel_key_bytes(imax) > (size_t)r.stage_bytes) return cudaSuccess;
  r.smem_bytes = L.ring_off + r.ns * r.stage_bytes;
  ls->ring_layer = r;
  return cudaSuccess;
}

bool layer_available(const LaunchShape& ls) { return ls.variant != 0 && ls.ring_layer.ns >= 2; }

cudaError_t launch_layer(const FwdParams& p, const LaunchShape& ls, cudaStream_t st, bool pdl) {
  const Ring& r = ls.ring_layer;
  const dim3 grid(ls.nsm), block(kLayerThreads);
  switch (ls.variant) {
    case 1: return launch_pdl(layer_kernel<1, 2>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 2: return launch_pdl(layer_kernel<1, 8>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 3: return launch_pdl(layer_kernel<3, 4>, grid, block, r.smem_bytes, st, pdl, p, r);
    case 4: return launch_pdl(layer_kernel<4, 5>, grid, block, r.smem_bytes, st, pdl, p, r);
    default: return cudaErrorInvalidConfiguration;
  }
}

}  // namespace moe
