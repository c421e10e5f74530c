// ep.cu -- expert-parallel forward of the layer over G ranks, one GPU each (include/moe.h,
// "expert parallelism").
//
// Experts sit on devices and tokens travel to them by an all-to-all and come back by a
// second one ("GShard (Expert Parallelism)", "In plain words"; with 256 experts on 8
// GPUs, 32 per GPU, and "a second all-to-all" returning the results: the "WideEP"
// claim).  Rank g holds a contiguous block of the batch's tokens and the experts
// [g*E/G, (g+1)*E/G); the router is replicated (W_g is small).
//
// Capacity keeps its one-device meaning: C = ceil(cf * k * S_total / E) over the whole
// batch, and slots are handed out rank-major over the batch in token order -- all first
// choices, then all second choices.  Tokens are ordered rank by rank, so the slot of a
// choice (t, r) of rank g at expert e is
//     base[g][r][e] + (its position among rank g's own rank-r choices of e),
//     base[g][r][e] = sum_{r' < r} sum_h cnt[h][r'][e] + sum_{h < g} cnt[h][r][e],
// where cnt[h][r][e] is rank h's rank-r demand of e.  Every rank computes the same table
// from the exchanged counts (moe_ep_plan), so the routing -- expert ids, slots, drops --
// equals the single-GPU layer's on the concatenated batch, bit for bit.
//
// One forward on rank g:
//   moe_ep_route     router on the rank's tokens + per-rank scan -> stats (counts, loss partials)
//   [caller]         all-gather the stats of every rank
//   moe_ep_dispatch  plan from the gathered counts; kept rows packed into the send buffer,
//                    ordered by destination rank, then expert, then choice rank, then token
//   [caller]         all-to-all of the send buffer (send / recv row counts per peer given)
//   moe_ep_experts   received rows -> the local experts' slot buffers, the two grouped GEMMs,
//                    the outputs written back over the received rows (same order)
//   [caller]         all-to-all back (the same counts, reversed)
//   moe_ep_combine   y[t] = sum_{r kept} g_r * (returned row of (t, r)), r ascending, fp32
// The losses use the gathered stats: f_j and P_j over the whole batch.
//
// Over peer memory (moe_ep_set_peers, moe_ep_dispatch_to_peers, moe_ep_combine_from_peers):
// the pack writes each kept row straight into its owner's receive buffer, at the row the
// all-to-all would have put it, and the combine reads each expert output from there, so
// neither exchange is a separate step.  The caller maps the buffers and orders the ranks
// (every rank's dispatch before any rank's experts, every rank's experts before any
// combine, every combine before the next dispatch).
//
// Two phases (moe_ep_set_phases): each expert's slots are split at
//     split_e = 256 * floor((n_e + 256) / 512)   (about half, a whole number of GEMM tiles),
// slots below it travel in phase 0 and the rest in phase 1.  The send and receive buffers
// hold the phase-0 rows first, each phase ordered as above, and each phase has its own
// row counts per peer, so a caller can exchange phase 1 while the experts compute phase 0
// (moe_ep_experts_phase) and return phase 0 while they compute phase 1.  The rows, their
// slots and every output are those of the one-phase forward: a GEMM tile never straddles
// the split.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"
#include "internal.h"

using namespace moe;

struct moe_ep_layer {
  int G, g;
  int64_t S_max, S_total_max, M, H;
  int32_t E, k, El;      // El = E / G experts on this rank: [g*El, (g+1)*El)
  double cf;
  moe_dtype act;
  const float* Wg;
  const float* bias;
  const void* W1;
  const void* W2;
  int64_t Cbuf;          // rows per local expert
  int device, num_sms;
  void* ws;
  Routing R;             // tables of the rank's own tokens; R.off holds the per-rank prefix
  int32_t* spos;         // [S_max, k] row of each kept choice in the send buffer, else -1
  void* xbuf;
  void* hbuf;
  void* ybuf;
  // base [k][E] | soff0 [k][E] | soff1 [k][E] | a0 [k][E] | seg_start [2][nseg] |
  // seg_dst [2][nseg] | nexp [2][El] | rowb [2][El]   (per phase: segments, rows, first row)
  int32_t* plan_dev;
  int32_t* rowmap;       // [El * Cbuf] expert row of each received row
  int nseg;              // received segments per phase: G * El * k
  int phases;            // 1 or 2
  int64_t recv_off[2], recv_cnt[2];   // each phase's rows in the receive buffer
  EpPeer* peers_dev;     // [G] every rank's receive buffer and this rank's row offset in it
  std::vector<void*> peer_ptrs;       // [G] set by moe_ep_set_peers (empty: not set)
  std::vector<EpPeer> peers_host;
  bool to_peers;         // the last dispatch wrote into the peers' buffers
  std::vector<int32_t> plan_host;
  GemmPlan plan1, plan2;
  void* wsplit;
  CUtensorMap wmap, xmap, xmap64;
  const void* xmap_ptr;
  int64_t xmap_S;
  uint64_t wait_limit_ns;
  // state of the current forward
  int64_t S;             // tokens routed by the last moe_ep_route
  bool routed, planned, computed;
  int64_t C;             // capacity of the planned batch
  int64_t S_total;       // tokens of the planned batch over all ranks
  int64_t send_total, recv_total;
  double l_aux, z;
};

namespace {

size_t act_bytes(moe_dtype a) { return a == MOE_BF16 ? 2 : 4; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  if (e == cudaErrorMemoryAllocation) return MOE_ERR_OOM;
  return MOE_ERR_CUDA;
}

#define EP_TRY(call)                             \
  do {                                           \
    cudaError_t _e = (call);                     \
    if (_e != cudaSuccess) return from_cuda(_e); \
  } while (0)

struct Carver {
  char* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~(size_t)255;
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    return p;
  }
};

size_t plan_ints(const moe_ep_layer* h) {
  return (size_t)4 * h->k * h->E + 4 * (size_t)h->nseg + 4 * (size_t)h->El;
}

size_t carve(moe_ep_layer* h, char* base) {
  Carver c{base};
  const int64_t S = h->S_max, E = h->E, k = h->k;
  const int64_t nchunk = (S + kChunk - 1) / kChunk;
  const size_t as = act_bytes(h->act);
  Routing& R = h->R;
  R.logits = c.take<float>(S * E);
  R.eidx = c.take<int32_t>(S * k);
  R.gate = c.take<float>(S * k);
  R.lrank = c.take<int32_t>(S * k);
  R.slot = c.take<int32_t>(S * k);
  R.hist = c.take<int32_t>(k * nchunk * E);
  R.off = c.take<int32_t>(k * nchunk * E);
  R.cnt = c.take<int32_t>(E);
  R.nexp = nullptr;                            // the local experts' counts live in the plan
  R.first = c.take<int32_t>(E);
  R.psum = c.take<float>(nchunk * E);
  R.lse2 = c.take<float>(nchunk);
  R.losses = c.take<float>(2);
  R.err = c.take<unsigned>(1);
  h->spos = c.take<int32_t>(S * k);
  h->xbuf = c.take<char>((size_t)h->El * h->Cbuf * h->M * as);
  h->hbuf = c.take<char>((size_t)h->El * h->Cbuf * h->H * as);
  h->ybuf = c.take<char>((size_t)h->El * h->Cbuf * h->M * as);
  h->plan_dev = c.take<int32_t>(plan_ints(h));
  h->rowmap = c.take<int32_t>((size_t)h->El * h->Cbuf);
  h->peers_dev = c.take<EpPeer>((size_t)h->G);
  h->wsplit = h->act == MOE_BF16 ? c.take<char>((size_t)3 * router_tc_pad(h->E) * h->M * 2) : nullptr;
  return c.off + 256;
}

// The exchange plan of rank g from every rank's counts.
struct Plan {
  int64_t C = 0, S_total = 0;
  std::vector<int64_t> base, kept;           // [G][k][E]
  std::vector<int64_t> n, split;             // [E] kept rows of each expert, first phase-1 slot
  std::vector<int64_t> a0;                   // [G][k][E] leading rows of each run in phase 0
  std::vector<int64_t> send_rows, recv_rows; // [phases][G]
};

int64_t phase_split(int64_t n, int phases) { return phases == 2 ? 256 * ((n + 256) / 512) : n; }

moe_status make_plan(int G, int g, int E, int k, double cf, const int64_t* cnt, const int64_t* S, Plan& p,
                     int phases = 1) {
  if (phases != 1 && phases != 2) return MOE_ERR_INVALID_ARG;
  if (G < 1 || g < 0 || g >= G || E < 1 || k < 1 || k > E || (E % G) || !cnt || !S ||
      !(cf > 0.0) || !isfinite(cf))
    return MOE_ERR_INVALID_ARG;
  const int El = E / G;
  p.S_total = 0;
  for (int q = 0; q < G; ++q) {
    if (S[q] < 0) return MOE_ERR_INVALID_ARG;
    p.S_total += S[q];
  }
  for (int64_t i = 0; i < (int64_t)G * k * E; ++i)
    if (cnt[i] < 0) return MOE_ERR_INVALID_ARG;
  for (int q = 0; q < G; ++q)                  // every rank's choices are k per token
    for (int r = 0; r < k; ++r) {
      int64_t s = 0;
      for (int e = 0; e < E; ++e) s += cnt[((int64_t)q * k + r) * E + e];
      if (s != S[q]) return MOE_ERR_INVALID_ARG;
    }
  if (p.S_total * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;
  p.C = capacity_of(cf, k, p.S_total, E);
  const size_t n = (size_t)G * k * E;
  p.base.assign(n, 0);
  p.kept.assign(n, 0);
  for (int e = 0; e < E; ++e) {
    int64_t run = 0;
    for (int r = 0; r < k; ++r)
      for (int q = 0; q < G; ++q) {
        const size_t i = ((size_t)q * k + r) * E + e;
        p.base[i] = run;
        const int64_t room = p.C - run;
        p.kept[i] = room <= 0 ? 0 : (room < cnt[i] ? room : cnt[i]);
        run += cnt[i];
      }
  }
  p.n.assign(E, 0);
  p.split.assign(E, 0);
  for (int e = 0; e < E; ++e) {
    for (int q = 0; q < G; ++q)
      for (int r = 0; r < k; ++r) p.n[e] += p.kept[((size_t)q * k + r) * E + e];
    p.split[e] = phase_split(p.n[e], phases);
  }
  p.a0.assign(n, 0);
  for (int q = 0; q < G; ++q)
    for (int r = 0; r < k; ++r)
      for (int e = 0; e < E; ++e) {
        const size_t i = ((size_t)q * k + r) * E + e;
        const int64_t a = p.split[e] - p.base[i];      // the run's slots below the split
        p.a0[i] = a <= 0 ? 0 : (a < p.kept[i] ? a : p.kept[i]);
      }
  p.send_rows.assign((size_t)phases * G, 0);
  p.recv_rows.assign((size_t)phases * G, 0);
  for (int ph = 0; ph < phases; ++ph)
    for (int q = 0; q < G; ++q)
      for (int r = 0; r < k; ++r)
        for (int e = 0; e < E; ++e) {
          const size_t i = ((size_t)q * k + r) * E + e;
          const int64_t v = ph == 0 ? p.a0[i] : p.kept[i] - p.a0[i];
          if (q == g) p.send_rows[(size_t)ph * G + e / El] += v;   // to the rank that holds expert e
          if (e / El == g) p.recv_rows[(size_t)ph * G + q] += v;   // from rank q, for one of our experts
        }
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_ep_stats_len(int32_t E, int32_t k) { return (E < 1 || k < 1) ? 0 : ep_stats_len(E, k); }

moe_status moe_ep_plan(int32_t G, int32_t g, int32_t E, int32_t k, double capacity_factor,
                       const int64_t* counts_host, const int64_t* S_host, int64_t* C_out,
                       int64_t* send_rows_host, int64_t* recv_rows_host, int64_t* base_host,
                       int64_t* kept_host) {
  Plan p;
  const moe_status s = make_plan(G, g, E, k, capacity_factor, counts_host, S_host, p);
  if (s != MOE_OK) return s;
  if (C_out) *C_out = p.C;
  if (send_rows_host) memcpy(send_rows_host, p.send_rows.data(), G * sizeof(int64_t));
  if (recv_rows_host) memcpy(recv_rows_host, p.recv_rows.data(), G * sizeof(int64_t));
  if (base_host) memcpy(base_host, p.base.data(), p.base.size() * sizeof(int64_t));
  if (kept_host) memcpy(kept_host, p.kept.data(), p.kept.size() * sizeof(int64_t));
  return MOE_OK;
}

moe_status moe_ep_phase_plan(int32_t G, int32_t g, int32_t E, int32_t k, double capacity_factor,
                             const int64_t* counts_host, const int64_t* S_host, int32_t phases,
                             int64_t* send_rows_host, int64_t* recv_rows_host, int64_t* split_host) {
  Plan p;
  const moe_status s = make_plan(G, g, E, k, capacity_factor, counts_host, S_host, p, phases);
  if (s != MOE_OK) return s;
  const size_t n = (size_t)phases * G;
  if (send_rows_host) memcpy(send_rows_host, p.send_rows.data(), n * sizeof(int64_t));
  if (recv_rows_host) memcpy(recv_rows_host, p.recv_rows.data(), n * sizeof(int64_t));
  if (split_host) memcpy(split_host, p.split.data(), (size_t)E * sizeof(int64_t));
  return MOE_OK;
}

moe_status moe_ep_create(moe_ep_handle* out, int32_t G, int32_t g, int64_t S_max, int64_t S_total_max,
                         int64_t M, int64_t H, int32_t E, int32_t k, double capacity_factor, moe_dtype act,
                         const float* Wg, const float* bias, const void* W1_local, const void* W2_local) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (G < 1 || g < 0 || g >= G || E < 1 || (E % G) || S_max < 1 || S_total_max < S_max || M < 64 ||
      H < 64 || (M % 64) || (H % 64) || k < 1 || k > E)
    return MOE_ERR_INVALID_ARG;
  if (!(capacity_factor > 0.0) || !isfinite(capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (act != MOE_F32 && act != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (!Wg || !W1_local || !W2_local || !aligned(Wg, 4) || !aligned(W1_local, 16) ||
      !aligned(W2_local, 16) || (bias && !aligned(bias, 4)))
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (S_total_max > (int64_t)1 << 30 || M > (1 << 16) || H > (1 << 16)) return MOE_ERR_UNSUPPORTED;
  const int64_t C = capacity_of(capacity_factor, k, S_total_max, E);
  const int64_t rows = C < S_total_max ? C : S_total_max;
  const int64_t Cbuf = (rows + 255) / 256 * 256;
  if ((int64_t)(E / G) * Cbuf > INT32_MAX || S_total_max * k > INT32_MAX) return MOE_ERR_UNSUPPORTED;

  moe_ep_layer* h = new (std::nothrow) moe_ep_layer();
  if (!h) return MOE_ERR_OOM;
  h->G = G;
  h->g = g;
  h->S_max = S_max;
  h->S_total_max = S_total_max;
  h->M = M;
  h->H = H;
  h->E = E;
  h->k = k;
  h->El = E / G;
  h->cf = capacity_factor;
  h->act = act;
  h->Wg = Wg;
  h->bias = bias;
  h->W1 = W1_local;
  h->W2 = W2_local;
  h->Cbuf = Cbuf;
  h->nseg = G * h->El * k;
  h->phases = 1;
  h->wait_limit_ns = 2000000000ull;
  cudaError_t ce = cudaGetDevice(&h->device);
  if (ce == cudaSuccess) ce = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  if (ce != cudaSuccess) {
    delete h;
    return from_cuda(ce);
  }
  const size_t bytes = carve(h, nullptr);
  ce = cudaMalloc(&h->ws, bytes);
  if (ce != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return from_cuda(ce);
  }
  carve(h, static_cast<char*>(h->ws));
  ce = cudaMemset(h->R.err, 0, sizeof(unsigned));
  if (ce == cudaSuccess) ce = cudaMemset(h->plan_dev, 0, plan_ints(h) * 4);
  if (ce != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return from_cuda(ce);
  }
  if (act == MOE_BF16) {
    const bool ok1 = make_gemm_plan(h->plan1, h->xbuf, W1_local, h->hbuf, h->El, Cbuf, (int)M, (int)H, true);
    const bool ok2 = make_gemm_plan(h->plan2, h->hbuf, W2_local, h->ybuf, h->El, Cbuf, (int)H, (int)M, false);
    ce = split_gate_weights(Wg, (int)M, E, h->wsplit, 0);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(0);
    const bool ok3 = ce == cudaSuccess && make_router_wmap(&h->wmap, h->wsplit, (int)M, E);
    if (!ok1 || !ok2 || !ok3) {
      cudaFree(h->ws);
      delete h;
      return MOE_ERR_CUDA;
    }
  }
  h->plan_host.assign(plan_ints(h), 0);
  *out = h;
  return MOE_OK;
}

moe_status moe_ep_set_phases(moe_ep_handle h, int32_t phases) {
  if (!h || (phases != 1 && phases != 2)) return MOE_ERR_INVALID_ARG;
  if (phases == 2 && h->act != MOE_BF16) return MOE_ERR_UNSUPPORTED;   // the FFMA GEMMs take no row base
  h->phases = phases;
  h->planned = h->computed = false;
  return MOE_OK;
}

moe_status moe_ep_destroy(moe_ep_handle h) {
  if (!h) return MOE_OK;
  cudaError_t ce = cudaDeviceSynchronize();
  cudaError_t fe = cudaFree(h->ws);
  delete h;
  if (ce != cudaSuccess) return from_cuda(ce);
  return from_cuda(fe);
}

moe_status moe_ep_buffer_rows(moe_ep_handle h, int64_t* send_rows_max, int64_t* recv_rows_max) {
  if (!h || !send_rows_max || !recv_rows_max) return MOE_ERR_INVALID_ARG;
  *send_rows_max = h->S_max * h->k;
  const int64_t C = capacity_of(h->cf, h->k, h->S_total_max, h->E);
  *recv_rows_max = (int64_t)h->El * (C < h->S_total_max ? C : h->S_total_max);
  return MOE_OK;
}

moe_status moe_ep_route(moe_ep_handle h, int64_t S, const void* x, double* stats_dev, void* stream) {
  if (!h || S < 0 || S > h->S_max || !stats_dev || !aligned(stats_dev, 8)) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!x || !aligned(x, 16))) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->S = S;
  h->routed = true;
  h->planned = h->computed = false;
  if (S == 0) {                                // no tokens: zero demand, zero partials
    EP_TRY(cudaMemsetAsync(stats_dev, 0, (size_t)ep_stats_len(h->E, h->k) * sizeof(double), st));
    return MOE_OK;
  }
  const int iS = (int)S, iM = (int)h->M;
  if (h->act == MOE_BF16) {
    const bool persistent = router_persistent(h->E, iS);
    if (h->xmap_ptr != x || h->xmap_S != S) {
      if (!make_router_xmap(&h->xmap, x, iS, iM, h->E)) return MOE_ERR_CUDA;
      if (persistent && !make_router_xmap64(&h->xmap64, x, iS, iM)) return MOE_ERR_CUDA;
      h->xmap_ptr = x;
      h->xmap_S = S;
    }
    EP_TRY(launch_router_tc(h->xmap, persistent ? &h->xmap64 : nullptr, x, h->wmap, h->bias, iS, iM, h->E,
                            h->k, h->R, h->wait_limit_ns, st));
  } else {
    EP_TRY(launch_router(x, false, h->Wg, h->bias, iS, iM, h->E, h->k, h->R, st));
  }
  EP_TRY(launch_ep_scan(iS, h->E, h->k, h->R, stats_dev, st));
  return MOE_OK;
}

}  // extern "C"

namespace {

// moe_ep_dispatch (sendbuf) and moe_ep_dispatch_to_peers (to_peers: the owners' receive
// buffers set by moe_ep_set_peers).
moe_status dispatch_impl(moe_ep_layer* h, const double* stats_all_host, const void* x, void* sendbuf,
                         bool to_peers, int64_t* send_rows_host, int64_t* recv_rows_host, void* stream) {
  if (!h || !stats_all_host || !send_rows_host || !recv_rows_host) return MOE_ERR_INVALID_ARG;
  if (!h->routed) return MOE_ERR_STATE;
  if (to_peers && (h->peer_ptrs.empty() || h->phases != 1)) return MOE_ERR_STATE;
  const int G = h->G, E = h->E, k = h->k, El = h->El, L = ep_stats_len(E, k);
  // the gathered counts must be exact non-negative integers, and this rank's must be its own
  std::vector<int64_t> cnt((size_t)G * k * E), Sv(G);
  for (int q = 0; q < G; ++q) {
    const double* st_q = stats_all_host + (size_t)q * L;
    for (int i = 0; i < k * E; ++i) {
      const double v = st_q[i];
      if (!(v >= 0.0) || v != floor(v) || v > 2147483647.0) return MOE_ERR_INVALID_ARG;
      cnt[(size_t)q * k * E + i] = (int64_t)v;
    }
    const double s = st_q[k * E + E + 1];
    if (!(s >= 0.0) || s != floor(s) || s > 1073741824.0) return MOE_ERR_INVALID_ARG;
    Sv[q] = (int64_t)s;
  }
  if (Sv[h->g] != h->S) return MOE_ERR_INVALID_ARG;
  Plan p;
  moe_status s = make_plan(G, h->g, E, k, h->cf, cnt.data(), Sv.data(), p, h->phases);
  if (s != MOE_OK) return s;
  if (p.S_total > h->S_total_max) return MOE_ERR_INVALID_ARG;
  if (h->S > 0 && (!x || !aligned(x, 16) || (!to_peers && (!sendbuf || !aligned(sendbuf, 16)))))
    return MOE_ERR_INVALID_ARG;

  // device tables: base, send offsets (per phase) and phase-0 lengths of this rank's runs;
  // per phase, the received segments and the local experts' rows
  const size_t kE = (size_t)k * E;
  int32_t* base = h->plan_host.data();
  int32_t* soff0 = base + kE;
  int32_t* soff1 = soff0 + kE;
  int32_t* a0 = soff1 + kE;
  int32_t* seg_start = a0 + kE;                // [2][nseg]
  int32_t* seg_dst = seg_start + 2 * (size_t)h->nseg;
  int32_t* nexp = seg_dst + 2 * (size_t)h->nseg;   // [2][El]
  int32_t* rowb = nexp + 2 * (size_t)El;
  int64_t pos = 0;
  for (int ph = 0; ph < h->phases; ++ph)       // phase 0 rows first; destination ranks ascend with e
    for (int e = 0; e < E; ++e)
      for (int r = 0; r < k; ++r) {
        const size_t i = ((size_t)h->g * k + r) * E + e;
        if (ph == 0) {
          base[r * E + e] = (int32_t)p.base[i];
          a0[r * E + e] = (int32_t)p.a0[i];
          soff0[r * E + e] = (int32_t)pos;
          soff1[r * E + e] = 0;
          pos += p.a0[i];
        } else {
          soff1[r * E + e] = (int32_t)pos;
          pos += p.kept[i] - p.a0[i];
        }
      }
  int64_t rpos_all = 0;
  for (int ph = 0; ph < h->phases; ++ph) {     // arrival order in a phase: source rank, expert, choice rank
    int64_t rpos = 0;
    for (int q = 0; q < G; ++q)
      for (int el = 0; el < El; ++el)
        for (int r = 0; r < k; ++r) {
          const int e = h->g * El + el;
          const size_t i = ((size_t)q * k + r) * E + e;
          const size_t sq = (size_t)ph * h->nseg + ((size_t)q * El + el) * k + r;
          const int64_t lead = ph == 0 ? 0 : p.a0[i];
          seg_start[sq] = (int32_t)rpos;
          seg_dst[sq] = (int32_t)((int64_t)el * h->Cbuf + p.base[i] + lead);
          rpos += ph == 0 ? p.a0[i] : p.kept[i] - p.a0[i];
        }
    h->recv_off[ph] = rpos_all;
    h->recv_cnt[ph] = rpos;
    rpos_all += rpos;
    for (int el = 0; el < El; ++el) {
      const int e = h->g * El + el;
      nexp[(size_t)ph * El + el] = (int32_t)(ph == 0 ? p.split[e] : p.n[e] - p.split[e]);
      rowb[(size_t)ph * El + el] = (int32_t)(ph == 0 ? 0 : p.split[e]);
    }
  }
  const int64_t rpos = rpos_all;
  // from pageable memory: the call returns once the table is staged, so the host copy
  // may be rewritten by the next dispatch
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  EP_TRY(cudaMemcpyAsync(h->plan_dev, h->plan_host.data(), h->plan_host.size() * sizeof(int32_t),
                         cudaMemcpyHostToDevice, st));
  if (to_peers) {
    // rank d receives, source after source, rows[q][d] from each rank q; this rank's rows for
    // d start there after the earlier sources', and in this rank's send order after its
    // rows for the earlier destinations
    std::vector<int64_t> rows((size_t)G * G, 0);
    for (int q = 0; q < G; ++q)
      for (int r = 0; r < k; ++r)
        for (int e = 0; e < E; ++e) rows[(size_t)q * G + e / El] += p.kept[((size_t)q * k + r) * E + e];
    h->peers_host.assign(G, EpPeer{nullptr, 0});
    int64_t send_start = 0;
    for (int d = 0; d < G; ++d) {
      int64_t arrive = 0;
      for (int q = 0; q < h->g; ++q) arrive += rows[(size_t)q * G + d];
      h->peers_host[d] = EpPeer{h->peer_ptrs[d], arrive - send_start};
      send_start += rows[(size_t)h->g * G + d];
    }
    EP_TRY(cudaMemcpyAsync(h->peers_dev, h->peers_host.data(), (size_t)G * sizeof(EpPeer),
                           cudaMemcpyHostToDevice, st));
  }
  for (size_t i = 0; i < (size_t)h->phases * G; ++i) {
    send_rows_host[i] = p.send_rows[i];
    recv_rows_host[i] = p.recv_rows[i];
  }
  h->C = p.C;
  h->S_total = p.S_total;
  h->send_total = pos;
  h->recv_total = rpos;
  // losses over the whole batch: f_j from the first choices, P_j from the probability sums
  double term = 0.0, zs = 0.0;
  for (int j = 0; j < E; ++j) {
    double P = 0.0, f = 0.0;
    for (int q = 0; q < G; ++q) {
      P += stats_all_host[(size_t)q * L + k * E + j];
      f += (double)cnt[(size_t)q * k * E + j];
    }
    term += f * P;
  }
  for (int q = 0; q < G; ++q) zs += stats_all_host[(size_t)q * L + k * E + E];
  const double Sd = (double)p.S_total;
  h->l_aux = p.S_total ? (double)E * term / (Sd * Sd) : 0.0;
  h->z = p.S_total ? zs / Sd : 0.0;
  h->planned = true;
  h->computed = false;
  h->to_peers = to_peers;
  if (h->S == 0) return MOE_OK;
  EP_TRY(launch_ep_dispatch(x, h->act == MOE_BF16, (int)h->S, (int)h->M, E, k, (int)p.C, h->R,
                            h->plan_dev, h->plan_dev + kE, h->spos, sendbuf, st,
                            to_peers ? h->peers_dev : nullptr, El));
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_ep_dispatch(moe_ep_handle h, const double* stats_all_host, const void* x, void* sendbuf,
                           int64_t* send_rows_host, int64_t* recv_rows_host, void* stream) {
  return dispatch_impl(h, stats_all_host, x, sendbuf, false, send_rows_host, recv_rows_host, stream);
}

moe_status moe_ep_set_peers(moe_ep_handle h, const void* const* recv_bufs_host) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!recv_bufs_host) {                       // back to the caller's exchanges
    h->peer_ptrs.clear();
    return MOE_OK;
  }
  for (int d = 0; d < h->G; ++d)
    if (!recv_bufs_host[d] || !aligned(recv_bufs_host[d], 16)) return MOE_ERR_INVALID_ARG;
  h->peer_ptrs.resize(h->G);
  for (int d = 0; d < h->G; ++d) h->peer_ptrs[d] = const_cast<void*>(recv_bufs_host[d]);
  h->planned = h->computed = false;
  return MOE_OK;
}

moe_status moe_ep_dispatch_to_peers(moe_ep_handle h, const double* stats_all_host, const void* x,
                                    int64_t* send_rows_host, int64_t* recv_rows_host, void* stream) {
  return dispatch_impl(h, stats_all_host, x, nullptr, true, send_rows_host, recv_rows_host, stream);
}

moe_status moe_ep_combine_from_peers(moe_ep_handle h, void* y, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->planned || !h->to_peers || h->peer_ptrs.empty()) return MOE_ERR_STATE;
  if (h->S == 0) return MOE_OK;
  if (!y || !aligned(y, 16)) return MOE_ERR_INVALID_ARG;
  Routing R2 = h->R;
  R2.slot = h->spos;
  EP_TRY(launch_combine(nullptr, h->act == MOE_BF16, (int)h->S, (int)h->M, h->k, 0, R2, y,
                        static_cast<cudaStream_t>(stream), false, 0, h->peers_dev, h->El));
  return MOE_OK;
}

namespace {

// One phase: its received rows into the experts' slots, the two GEMMs over its slot
// ranges, the outputs back over its received rows.
moe_status experts_phase(moe_ep_layer* h, void* recvbuf, int ph, cudaStream_t st) {
  const bool bf16 = h->act == MOE_BF16;
  const int k = h->k, E = h->E, El = h->El;
  const size_t kE = (size_t)k * E;
  const int32_t* seg_start = h->plan_dev + 4 * kE + (size_t)ph * h->nseg;
  const int32_t* seg_dst = h->plan_dev + 4 * kE + 2 * (size_t)h->nseg + (size_t)ph * h->nseg;
  const int32_t* nexp = h->plan_dev + 4 * kE + 4 * (size_t)h->nseg + (size_t)ph * El;
  const int32_t* rowb = h->plan_dev + 4 * kE + 4 * (size_t)h->nseg + 2 * (size_t)El + (size_t)ph * El;
  const size_t as = act_bytes(h->act);
  char* rb = static_cast<char*>(recvbuf) + (size_t)h->recv_off[ph] * h->M * as;
  int32_t* rowmap = h->rowmap + h->recv_off[ph];
  const int nrows = (int)h->recv_cnt[ph];
  EP_TRY(launch_ep_unpack(rb, bf16, nrows, (int)h->M, seg_start, seg_dst, h->nseg, rowmap, h->xbuf, h->R.err,
                          (int64_t)El * h->Cbuf, st));
  if (bf16) {
    // CTA-pair (256-row) tiles when the batch's experts run at capacity, the rule of
    // the one-device layer on the same batch
    const bool pair = (double)h->S_total * h->k / E >= (double)h->C;
    GemmPlan p1 = h->plan1, p2 = h->plan2;
    p1.row_base = p2.row_base = rowb;
    EP_TRY(launch_ffn_bf16(p1, nexp, h->R.err, h->wait_limit_ns, h->num_sms, pair, st));
    EP_TRY(launch_ffn_bf16(p2, nexp, h->R.err, h->wait_limit_ns, h->num_sms, pair, st));
  } else {                                     // one phase only (moe_ep_set_phases)
    EP_TRY(launch_ffn_f32((const float*)h->xbuf, (const float*)h->W1, (float*)h->hbuf, nexp, El, h->Cbuf,
                          (int)h->M, (int)h->H, true, st));
    EP_TRY(launch_ffn_f32((const float*)h->hbuf, (const float*)h->W2, (float*)h->ybuf, nexp, El, h->Cbuf,
                          (int)h->H, (int)h->M, false, st));
  }
  EP_TRY(launch_ep_repack(h->ybuf, bf16, nrows, (int)h->M, rowmap, rb, st));
  return MOE_OK;
}

}  // namespace

moe_status moe_ep_experts(moe_ep_handle h, void* recvbuf, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->planned) return MOE_ERR_STATE;
  if (h->recv_total > 0 && (!recvbuf || !aligned(recvbuf, 16))) return MOE_ERR_INVALID_ARG;
  for (int ph = 0; ph < h->phases; ++ph) {
    const moe_status s = experts_phase(h, recvbuf, ph, static_cast<cudaStream_t>(stream));
    if (s != MOE_OK) return s;
  }
  h->computed = true;
  return MOE_OK;
}

moe_status moe_ep_experts_phase(moe_ep_handle h, void* recvbuf, int32_t phase, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->planned) return MOE_ERR_STATE;
  if (phase < 0 || phase >= h->phases) return MOE_ERR_INVALID_ARG;
  if (h->recv_cnt[phase] > 0 && (!recvbuf || !aligned(recvbuf, 16))) return MOE_ERR_INVALID_ARG;
  const moe_status s = experts_phase(h, recvbuf, phase, static_cast<cudaStream_t>(stream));
  if (s == MOE_OK && phase == h->phases - 1) h->computed = true;
  return s;
}

moe_status moe_ep_combine(moe_ep_handle h, const void* sendbuf, void* y, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->planned || h->to_peers) return MOE_ERR_STATE;   // rows went to the peers: combine_from_peers
  if (h->S == 0) return MOE_OK;
  if (!y || !aligned(y, 16) || (h->send_total > 0 && (!sendbuf || !aligned(sendbuf, 16))))
    return MOE_ERR_INVALID_ARG;
  // the returned rows sit where the dispatch packed them: combine by row index (with a
  // zero expert stride, row = e * 0 + spos)
  Routing R2 = h->R;
  R2.slot = h->spos;
  EP_TRY(launch_combine(sendbuf, h->act == MOE_BF16, (int)h->S, (int)h->M, h->k, 0, R2, y,
                        static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_ep_aux_loss(moe_ep_handle h, float* l_aux, float* z_loss) {
  if (!h || !l_aux || !z_loss) return MOE_ERR_INVALID_ARG;
  if (!h->planned) return MOE_ERR_STATE;
  *l_aux = (float)h->l_aux;
  *z_loss = (float)h->z;
  return MOE_OK;
}

moe_status moe_ep_get_routing(moe_ep_handle h, int32_t* eidx, float* gate, int32_t* slot, int32_t* spos,
                              float* logits, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!h->routed) return MOE_ERR_STATE;
  if ((slot || spos) && !h->planned) return MOE_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)h->S * h->k;
  if (n) {
    if (eidx) EP_TRY(cudaMemcpyAsync(eidx, h->R.eidx, n * 4, cudaMemcpyDeviceToDevice, st));
    if (gate) EP_TRY(cudaMemcpyAsync(gate, h->R.gate, n * 4, cudaMemcpyDeviceToDevice, st));
    if (slot) EP_TRY(cudaMemcpyAsync(slot, h->R.slot, n * 4, cudaMemcpyDeviceToDevice, st));
    if (spos) EP_TRY(cudaMemcpyAsync(spos, h->spos, n * 4, cudaMemcpyDeviceToDevice, st));
    if (logits)
      EP_TRY(cudaMemcpyAsync(logits, h->R.logits, (size_t)h->S * h->E * 4, cudaMemcpyDeviceToDevice, st));
  }
  return MOE_OK;
}

moe_status moe_ep_check(moe_ep_handle h, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned e = 0;
  cudaError_t ce = cudaMemcpyAsync(&e, h->R.err, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  if (ce != cudaSuccess) return from_cuda(ce);
  if (e) {
    cudaMemsetAsync(h->R.err, 0, sizeof(unsigned), st);
    cudaStreamSynchronize(st);
    return (e & DEVERR_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_ERR_CUDA;
  }
  return MOE_OK;
}

}  // extern "C"
