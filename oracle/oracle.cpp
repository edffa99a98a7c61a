/*
 * oracle.cpp - plain fp64 CPU reference of the intra-expert activation-sparse MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code with the CUDA library: it reads the logical
 * (unpacked) weight tensors, computes everything in double precision with straightforward
 * loops and library sorts, and takes no blocking, fusion or reordering beyond the definition.
 *
 * What it computes follows "Uncovering Intra-expert Activation Sparsity for Efficient
 * Mixture-of-Expert Model Execution" (technical summary, Methodology):
 *   - the router is kept as in a standard MoE: top-k experts per token;
 *   - every selected (and every always-on shared) expert computes its gate projection densely,
 *     which yields the activation scores;
 *   - within each (token, expert) pair the lowest-scoring neuron activations are zeroed, either
 *     by keeping a target fraction or by a single-pass threshold mask;
 *   - the up and down projections are evaluated for the surviving neurons only.
 * Readings where the page is silent (each listed in the design notes):
 *   score of neuron n      sigma_n = |SiLU(g_n)|, SiLU(g) = g / (1 + exp(-g))
 *   keep count (top-K)     K = I - floor(s*I + 1e-9), clamped to [0, I]
 *   ties                   equal scores: lower neuron index kept; equal logits: lower expert
 *   threshold mode         keep sigma_n > t (strict)
 *   routing weights        softmax over the k chosen logits (default), softmax over all E,
 *                          or sigmoid of the chosen logit; the weight scales the expert output
 *   shared experts         weight 1, each with its own per-pair selection
 *   layer output           out_t = sum_{e in topk(t)} w_{t,e} y_{t,e} + sum_sh y_{t,sh}
 *                          y = sum_{n in A} SiLU(g_n) (W_up[n] . x) W_down[:, n]
 *
 * Optional roster routing ("Predatory MoE", technical summary, Methodology 2, the roster rule):
 * each sequence counts how often each expert of the layer was selected; its roster is the m
 * most-used experts (equal counts: lower expert index); while fewer than m distinct experts
 * have been used there is no bias (exploration), afterwards roster members get +delta and the
 * others -delta (barrier); a pinned sequence selects among its roster only (-inf for the
 * others).  Readings: the bias enters the top-k choice only, the routing weights stay those of
 * the unbiased logits; one decode token per sequence; the caller decides when to pin.
 *
 * Inputs are passed exactly as stored for the device: bf16 bit patterns (elt = 2) or binary32
 * (elt = 4), widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <thread>
#include <vector>

extern "C" {

typedef struct {
  int hidden;        /* H */
  int n_routed;      /* E */
  int top_k;         /* k */
  int inter;         /* I */
  int n_shared;      /* S */
  int inter_shared;  /* Ish */
  int route;         /* 0 softmax over top-k, 1 softmax over all E, 2 sigmoid */
  int elt;           /* 2: bf16 bit patterns, 4: binary32 */
  const void* router;             /* [E][H] */
  const void* const* gate;        /* E entries, each [I][H]; an entry may be NULL if unused */
  const void* const* up;          /* E entries, each [I][H] */
  const void* const* down;        /* E entries, each [H][I] */
  const void* const* sh_gate;     /* S entries, each [Ish][H] */
  const void* const* sh_up;       /* S entries, each [Ish][H] */
  const void* const* sh_down;     /* S entries, each [H][Ish] */
} oracle_layer;

typedef struct {
  int mode;          /* 0: keep the top K = I - floor(s*I + 1e-9); 1: keep sigma > threshold */
  double sparsity;   /* s in [0, 1] */
  double threshold;  /* t (mode 1) */
} oracle_sel;

enum { ORACLE_OK = 0, ORACLE_BAD_ARG = -1, ORACLE_MISSING_WEIGHT = -2 };

}  // extern "C"

namespace {

double load(const void* p, int elt, size_t i) {
  if (elt == 2) {
    uint32_t bits = (uint32_t)static_cast<const uint16_t*>(p)[i] << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
  }
  return (double)static_cast<const float*>(p)[i];
}

double silu(double g) { return g / (1.0 + exp(-g)); }

int keep_count(int I, double s) {
  long k = (long)I - (long)floor(s * (double)I + 1e-9);
  if (k < 0) k = 0;
  if (k > I) k = I;
  return (int)k;
}

/* Dense gate of one pair: g[n] = W_g[n] . x, a[n] = SiLU(g[n]). */
void gate_pair(const void* x, const void* wg, int elt, int H, int I, double* g, double* a) {
  std::vector<double> xd(H);
  for (int h = 0; h < H; ++h) xd[h] = load(x, elt, (size_t)h);
  for (int n = 0; n < I; ++n) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h) acc += load(wg, elt, (size_t)n * H + h) * xd[h];
    g[n] = acc;
    a[n] = silu(acc);
  }
}

/* Selection of the kept neurons from the scores. */
void select_keep(const double* score, int I, const oracle_sel& sel, unsigned char* keep) {
  if (sel.mode == 1) {
    for (int n = 0; n < I; ++n) keep[n] = score[n] > sel.threshold ? 1 : 0;
    return;
  }
  int K = keep_count(I, sel.sparsity);
  std::vector<int> order(I);
  for (int n = 0; n < I; ++n) order[n] = n;
  std::sort(order.begin(), order.end(), [&](int p, int q) {
    if (score[p] != score[q]) return score[p] > score[q];
    return p < q;
  });
  memset(keep, 0, (size_t)I);
  for (int r = 0; r < K; ++r) keep[order[r]] = 1;
}

/* y[h] = sum over kept n of a[n] * (W_up[n] . x) * W_down[h][n]. */
void expert_out(const void* x, const void* wu, const void* wd, int elt, int H, int I,
                const unsigned char* keep, const double* a, double* y) {
  std::vector<double> xd(H);
  for (int h = 0; h < H; ++h) xd[h] = load(x, elt, (size_t)h);
  for (int h = 0; h < H; ++h) y[h] = 0.0;
  for (int n = 0; n < I; ++n) {
    if (!keep[n]) continue;
    double u = 0.0;
    for (int h = 0; h < H; ++h) u += load(wu, elt, (size_t)n * H + h) * xd[h];
    double coef = a[n] * u;
    for (int h = 0; h < H; ++h) y[h] += coef * load(wd, elt, (size_t)h * I + n);
  }
}

/* Routing weights of the chosen experts idx[0..k) from the token's logits. */
void route_weights(const oracle_layer& L, const double* logits, const int* idx, double* w) {
  const int E = L.n_routed, k = L.top_k;
  if (L.route == 2) {
    for (int i = 0; i < k; ++i) w[i] = 1.0 / (1.0 + exp(-logits[idx[i]]));
    return;
  }
  double m = -INFINITY;
  if (L.route == 1) {
    for (int e = 0; e < E; ++e) m = std::max(m, logits[e]);
  } else {
    for (int i = 0; i < k; ++i) m = std::max(m, logits[idx[i]]);
  }
  double z = 0.0;
  if (L.route == 1) {
    for (int e = 0; e < E; ++e) z += exp(logits[e] - m);
  } else {
    for (int i = 0; i < k; ++i) z += exp(logits[idx[i]] - m);
  }
  for (int i = 0; i < k; ++i) w[i] = exp(logits[idx[i]] - m) / z;
}

/* Router logits of one token. */
void router_logits(const oracle_layer& L, const void* x_t, double* logits) {
  const int H = L.hidden, E = L.n_routed;
  std::vector<double> xd(H);
  for (int h = 0; h < H; ++h) xd[h] = load(x_t, L.elt, (size_t)h);
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h) acc += load(L.router, L.elt, (size_t)e * H + h) * xd[h];
    logits[e] = acc;
  }
}

/* The top-k experts by (logit descending, expert index ascending). */
void topk_experts(const double* logits, int E, int k, int* idx) {
  std::vector<int> order(E);
  for (int e = 0; e < E; ++e) order[e] = e;
  std::sort(order.begin(), order.end(), [&](int p, int q) {
    if (logits[p] != logits[q]) return logits[p] > logits[q];
    return p < q;
  });
  for (int i = 0; i < k; ++i) idx[i] = order[i];
}

bool layer_ok(const oracle_layer* L) {
  if (!L || L->hidden <= 0 || L->n_routed <= 0 || L->top_k <= 0 || L->top_k > L->n_routed ||
      L->inter <= 0 || L->n_shared < 0 || (L->n_shared > 0 && L->inter_shared <= 0) ||
      (L->elt != 2 && L->elt != 4) || L->route < 0 || L->route > 2 || !L->router)
    return false;
  if (!L->gate || !L->up || !L->down) return false;
  if (L->n_shared > 0 && (!L->sh_gate || !L->sh_up || !L->sh_down)) return false;
  return true;
}

bool sel_ok(const oracle_sel& s) {
  if (s.mode == 0) return s.sparsity >= 0.0 && s.sparsity <= 1.0;
  return s.mode == 1 && !isnan(s.threshold);
}

template <class F>
void parallel_for(int n, int nthreads, F&& fn) {
  int hw = (int)std::thread::hardware_concurrency();
  int nt = nthreads > 0 ? nthreads : (hw > 0 ? hw : 1);
  nt = std::min(nt, std::max(n, 1));
  std::atomic<int> next(0);
  auto worker = [&]() {
    for (int i = next.fetch_add(1); i < n; i = next.fetch_add(1)) fn(i);
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& t : pool) t.join();
}

}  // namespace

extern "C" {

/* K = ceil((1 - s) I), evaluated as I - floor(s I + 1e-9) and clamped to [0, I]. */
int oracle_keep_count(int I, double s) { return keep_count(I, s); }

int oracle_threads(void) {
  int hw = (int)std::thread::hardware_concurrency();
  return hw > 0 ? hw : 1;
}

/* Roster bias of B sequences: counts [B][E] selections so far, pinned [B] (0 / 1), budget m
 * (1 <= m <= E), delta >= 0  ->  bias [B][E]. */
int oracle_roster_bias(const int* counts, const int* pinned, int B, int E, int m, double delta,
                       double* bias) {
  if (!counts || !pinned || !bias || B < 0 || E <= 0 || m < 1 || m > E || !(delta >= 0.0))
    return ORACLE_BAD_ARG;
  std::vector<int> order(E);
  for (int t = 0; t < B; ++t) {
    const int* c = counts + (size_t)t * E;
    for (int e = 0; e < E; ++e) order[e] = e;
    std::sort(order.begin(), order.end(), [&](int p, int q) {
      if (c[p] != c[q]) return c[p] > c[q];
      return p < q;
    });
    std::vector<unsigned char> member(E, 0);
    for (int r = 0; r < m; ++r) member[order[r]] = 1;
    int distinct = 0;
    for (int e = 0; e < E; ++e) distinct += c[e] > 0;
    double* b = bias + (size_t)t * E;
    for (int e = 0; e < E; ++e) {
      if (pinned[t]) b[e] = member[e] ? 0.0 : -INFINITY;
      else if (distinct < m) b[e] = 0.0;
      else b[e] = member[e] ? delta : -delta;
    }
  }
  return ORACLE_OK;
}

/* counts[t][idx[t][j]] += 1 for the k experts each sequence's token selected. */
int oracle_roster_update(int* counts, const int* idx, int B, int E, int k) {
  if (!counts || !idx || B < 0 || E <= 0 || k <= 0) return ORACLE_BAD_ARG;
  for (int t = 0; t < B; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= E) return ORACLE_BAD_ARG;
      counts[(size_t)t * E + e] += 1;
    }
  return ORACLE_OK;
}

/* Router with an additive selection bias [B][E] (nullable): the top-k of logits + bias by
 * (value descending, expert index ascending); the weights of the chosen experts from the
 * unbiased logits.  logits [B][E] (nullable) are the unbiased ones. */
int oracle_route_biased(const oracle_layer* L, const void* x, int B, const double* bias,
                        double* logits, int* idx, double* w) {
  if (!L || !L->router || B < 0 || !x || !idx || !w || L->top_k <= 0 || L->top_k > L->n_routed)
    return ORACLE_BAD_ARG;
  const int E = L->n_routed, k = L->top_k;
  std::vector<double> lg(E), sel(E);
  for (int t = 0; t < B; ++t) {
    const void* xt = static_cast<const char*>(x) + (size_t)t * L->hidden * L->elt;
    router_logits(*L, xt, lg.data());
    for (int e = 0; e < E; ++e) sel[e] = lg[e] + (bias ? bias[(size_t)t * E + e] : 0.0);
    topk_experts(sel.data(), E, k, idx + (size_t)t * k);
    route_weights(*L, lg.data(), idx + (size_t)t * k, w + (size_t)t * k);
    if (logits) memcpy(logits + (size_t)t * E, lg.data(), sizeof(double) * E);
  }
  return ORACLE_OK;
}

/* Router for B tokens.  logits [B][E] (nullable), idx [B][k], w [B][k]. */
int oracle_route(const oracle_layer* L, const void* x, int B, double* logits, int* idx, double* w) {
  if (!L || !L->router || B < 0 || !x || !idx || !w || L->top_k <= 0 || L->top_k > L->n_routed)
    return ORACLE_BAD_ARG;
  const int E = L->n_routed, k = L->top_k;
  std::vector<double> lg(E);
  for (int t = 0; t < B; ++t) {
    const void* xt = static_cast<const char*>(x) + (size_t)t * L->hidden * L->elt;
    router_logits(*L, xt, lg.data());
    topk_experts(lg.data(), E, k, idx + (size_t)t * k);
    route_weights(*L, lg.data(), idx + (size_t)t * k, w + (size_t)t * k);
    if (logits) memcpy(logits + (size_t)t * E, lg.data(), sizeof(double) * E);
  }
  return ORACLE_OK;
}

/* The top-k experts of given logits [E] by (logit descending, index ascending). */
int oracle_topk(const double* logits, int E, int k, int* idx) {
  if (!logits || !idx || E <= 0 || k <= 0 || k > E) return ORACLE_BAD_ARG;
  topk_experts(logits, E, k, idx);
  return ORACLE_OK;
}

/* Routing weights for a given choice of experts idx[0..k) and the token's logits [E]. */
int oracle_route_weights(const oracle_layer* L, const double* logits, const int* idx, double* w) {
  if (!L || !logits || !idx || !w) return ORACLE_BAD_ARG;
  route_weights(*L, logits, idx, w);
  return ORACLE_OK;
}

/* Dense gate of one (token, expert) pair: g [I] and a = SiLU(g) [I]. */
int oracle_gate(const void* x_t, const void* wg, int elt, int H, int I, double* g, double* a) {
  if (!x_t || !wg || !g || !a || H <= 0 || I <= 0 || (elt != 2 && elt != 4)) return ORACLE_BAD_ARG;
  gate_pair(x_t, wg, elt, H, I, g, a);
  return ORACLE_OK;
}

/* Dense gate of one expert for T tokens: a [T][I] = SiLU(W_g x_t), the same loop as
 * oracle_gate, with the (token, block of 64 neurons) jobs spread over the host threads. */
int oracle_gate_tokens(const void* x, int T, const void* wg, int elt, int H, int I, double* a,
                       int nthreads) {
  if (!x || !wg || !a || T < 0 || H <= 0 || I <= 0 || (elt != 2 && elt != 4))
    return ORACLE_BAD_ARG;
  const int nb = (I + 63) / 64;
  parallel_for(T * nb, nthreads, [&](int job) {
    const int t = job / nb, n0 = (job % nb) * 64, n1 = std::min(I, n0 + 64);
    const void* xt = static_cast<const char*>(x) + (size_t)t * H * elt;
    const void* rows = static_cast<const char*>(wg) + (size_t)n0 * H * elt;
    std::vector<double> g(n1 - n0);
    gate_pair(xt, rows, elt, H, n1 - n0, g.data(), a + (size_t)t * I + n0);
  });
  return ORACLE_OK;
}

/* Kept-neuron mask keep [I] (0/1) from scores [I]. */
int oracle_select(const double* score, int I, oracle_sel sel, unsigned char* keep) {
  if (!score || !keep || I <= 0 || !sel_ok(sel)) return ORACLE_BAD_ARG;
  select_keep(score, I, sel, keep);
  return ORACLE_OK;
}

/* Expert output y [H] of one pair for a given mask keep [I] and activations a [I]. */
int oracle_expert(const void* x_t, const void* wu, const void* wd, int elt, int H, int I,
                  const unsigned char* keep, const double* a, double* y) {
  if (!x_t || !wu || !wd || !keep || !a || !y || H <= 0 || I <= 0 || (elt != 2 && elt != 4))
    return ORACLE_BAD_ARG;
  expert_out(x_t, wu, wd, elt, H, I, keep, a, y);
  return ORACLE_OK;
}

/*
 * The whole layer for B tokens.
 *   idx_in   [B][k]   nullable: use this routing instead of the top-k of the logits
 *   keep_in  [B][k+S][Imax], keep_flag [B][k+S]  nullable: for pairs whose flag is set, use
 *            this mask instead of the selection (Imax = max(I, Ish))
 *   out      [B][H]   the layer output
 *   idx_out  [B][k], w_out [B][k]           nullable
 *   keep_out [B][k+S][Imax], a_out [B][k+S][Imax], logits_out [B][E]   nullable
 * Pair j < k of token t is its j-th routed expert; pair k+s is shared expert s.
 */
int oracle_forward(const oracle_layer* L, const void* x, int B, oracle_sel routed,
                   oracle_sel shared, const int* idx_in, const unsigned char* keep_in,
                   const unsigned char* keep_flag, double* out, int* idx_out, double* w_out,
                   unsigned char* keep_out, double* a_out, double* logits_out, int nthreads) {
  if (!layer_ok(L) || B < 0 || (B > 0 && (!x || !out)) || !sel_ok(routed) ||
      (L->n_shared > 0 && !sel_ok(shared)))
    return ORACLE_BAD_ARG;
  if (B == 0) return ORACLE_OK;
  const int H = L->hidden, E = L->n_routed, k = L->top_k, S = L->n_shared;
  const int I = L->inter, Ish = L->inter_shared;
  const int Imax = std::max(I, S > 0 ? Ish : 0);
  const int P = k + S;
  const size_t xstride = (size_t)H * L->elt;

  std::vector<double> logits((size_t)B * E);
  std::vector<int> idx((size_t)B * k);
  std::vector<double> w((size_t)B * k);
  for (int t = 0; t < B; ++t) {
    const void* xt = static_cast<const char*>(x) + t * xstride;
    router_logits(*L, xt, &logits[(size_t)t * E]);
    if (idx_in) {
      for (int i = 0; i < k; ++i) {
        int e = idx_in[(size_t)t * k + i];
        if (e < 0 || e >= E) return ORACLE_BAD_ARG;
        idx[(size_t)t * k + i] = e;
      }
    } else {
      topk_experts(&logits[(size_t)t * E], E, k, &idx[(size_t)t * k]);
    }
    route_weights(*L, &logits[(size_t)t * E], &idx[(size_t)t * k], &w[(size_t)t * k]);
  }
  for (int t = 0; t < B; ++t)
    for (int i = 0; i < k; ++i)
      if (!L->gate[idx[(size_t)t * k + i]] || !L->up[idx[(size_t)t * k + i]] ||
          !L->down[idx[(size_t)t * k + i]])
        return ORACLE_MISSING_WEIGHT;
  for (int s = 0; s < S; ++s)
    if (!L->sh_gate[s] || !L->sh_up[s] || !L->sh_down[s]) return ORACLE_MISSING_WEIGHT;

  /* every (token, pair) independently */
  std::vector<double> y((size_t)B * P * H);
  std::vector<unsigned char> keep_all((size_t)B * P * Imax, 0);
  std::vector<double> a_all((size_t)B * P * Imax, 0.0);
  parallel_for(B * P, nthreads, [&](int job) {
    const int t = job / P, j = job % P;
    const void* xt = static_cast<const char*>(x) + t * xstride;
    const void *wg, *wu, *wd;
    int In;
    oracle_sel sel;
    if (j < k) {
      int e = idx[(size_t)t * k + j];
      wg = L->gate[e];
      wu = L->up[e];
      wd = L->down[e];
      In = I;
      sel = routed;
    } else {
      wg = L->sh_gate[j - k];
      wu = L->sh_up[j - k];
      wd = L->sh_down[j - k];
      In = Ish;
      sel = shared;
    }
    std::vector<double> g(In), a(In), score(In);
    gate_pair(xt, wg, L->elt, H, In, g.data(), a.data());
    unsigned char* keep = &keep_all[(size_t)job * Imax];
    if (keep_in && keep_flag && keep_flag[job]) {
      memcpy(keep, keep_in + (size_t)job * Imax, (size_t)In);
    } else {
      for (int n = 0; n < In; ++n) score[n] = fabs(a[n]);
      select_keep(score.data(), In, sel, keep);
    }
    memcpy(&a_all[(size_t)job * Imax], a.data(), sizeof(double) * In);
    expert_out(xt, wu, wd, L->elt, H, In, keep, a.data(), &y[(size_t)job * H]);
  });

  /* combine in a fixed order: routed pairs by rank, then the shared experts */
  for (int t = 0; t < B; ++t) {
    double* o = out + (size_t)t * H;
    for (int h = 0; h < H; ++h) o[h] = 0.0;
    for (int j = 0; j < P; ++j) {
      const double wj = j < k ? w[(size_t)t * k + j] : 1.0;
      const double* yj = &y[((size_t)t * P + j) * H];
      for (int h = 0; h < H; ++h) o[h] += wj * yj[h];
    }
  }
  if (idx_out) memcpy(idx_out, idx.data(), sizeof(int) * idx.size());
  if (w_out) memcpy(w_out, w.data(), sizeof(double) * w.size());
  if (keep_out) memcpy(keep_out, keep_all.data(), keep_all.size());
  if (a_out) memcpy(a_out, a_all.data(), sizeof(double) * a_all.size());
  if (logits_out) memcpy(logits_out, logits.data(), sizeof(double) * logits.size());
  return ORACLE_OK;
}

/*
 * Threshold calibration (the threshold approach of the paper's results reaches a target
 * sparsity with one fixed cut).  Collects the scores sigma = |SiLU(g)| of every routed pair
 * (shared = 0) or every shared-expert pair (shared = 1) of the B calibration tokens, sorts
 * them ascending as S[0..N), and returns t = S[m-1] with m = floor(s N), or -inf when m = 0,
 * so that the scores above t are the top N - m.  The count N is written to *n_scores.
 */
int oracle_calibrate(const oracle_layer* L, const void* x, int B, int shared, double s,
                     double* t_out, long long* n_scores, int nthreads) {
  if (!layer_ok(L) || B <= 0 || !x || !t_out || s < 0.0 || s > 1.0) return ORACLE_BAD_ARG;
  if (shared && L->n_shared == 0) return ORACLE_BAD_ARG;
  const int H = L->hidden, E = L->n_routed, k = L->top_k, S = L->n_shared;
  const int In = shared ? L->inter_shared : L->inter;
  const int P = shared ? S : k;
  const size_t xstride = (size_t)H * L->elt;
  std::vector<int> idx((size_t)B * k);
  if (!shared) {
    std::vector<double> lg(E);
    for (int t = 0; t < B; ++t) {
      router_logits(*L, static_cast<const char*>(x) + t * xstride, lg.data());
      topk_experts(lg.data(), E, k, &idx[(size_t)t * k]);
      for (int i = 0; i < k; ++i)
        if (!L->gate[idx[(size_t)t * k + i]]) return ORACLE_MISSING_WEIGHT;
    }
  } else {
    for (int j = 0; j < S; ++j)
      if (!L->sh_gate[j]) return ORACLE_MISSING_WEIGHT;
  }
  std::vector<double> scores((size_t)B * P * In);
  parallel_for(B * P, nthreads, [&](int job) {
    const int t = job / P, j = job % P;
    const void* wg = shared ? L->sh_gate[j] : L->gate[idx[(size_t)t * k + j]];
    std::vector<double> g(In), a(In);
    gate_pair(static_cast<const char*>(x) + t * xstride, wg, L->elt, H, In, g.data(), a.data());
    for (int n = 0; n < In; ++n) scores[(size_t)job * In + n] = fabs(a[n]);
  });
  std::sort(scores.begin(), scores.end());
  const long long N = (long long)scores.size();
  const long long m = (long long)floor(s * (double)N);
  *t_out = m > 0 ? scores[(size_t)(m - 1)] : -INFINITY;
  if (n_scores) *n_scores = N;
  return ORACLE_OK;
}

}  // extern "C"
