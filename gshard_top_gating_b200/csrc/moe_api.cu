// moe_api.cu -- the C ABI (include/moe.h): handle, workspace, launch sequence.
//
// One forward enqueues six kernels on the caller's stream and never waits on
// the host:
//   router  (gate GEMM, softmax, top-k, gates, loss partials, chunk tables)
//   scan    (rank-major capacity offsets per expert, kept counts, losses)
//   dispatch(slots, x rows -> per-expert buffers)
//   ffn1    (grouped relu(xbuf W1))      ffn2 (grouped hbuf W2)
//   combine (gate-weighted sum back to token order)
// The data-dependent per-expert counts stay on the device: the grouped GEMMs
// read them there.
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moe.h"
#include "common.cuh"
#include "internal.h"

using namespace moe;

struct moe_layer {
  int64_t S_max, M, H;
  int32_t E, k;
  double cf;
  moe_dtype act;
  const float* Wg;
  const float* bias;
  const void* W1;
  const void* W2;
  int64_t Cbuf;          // rows per expert in xbuf / hbuf / ybuf
  int device, num_sms;
  size_t ws_bytes;
  void* ws;              // the one device allocation
  Routing R;
  void* xbuf;
  void* hbuf;
  void* ybuf;
  void* xstage[2];       // moe_forward_host staging, two slots so calls overlap
  void* ystage[2];
  // moe_forward_host pipeline: copy-in, compute and copy-out streams (created on first use)
  bool host_ready;
  cudaStream_t hs_in, hs_comp, hs_out;
  cudaEvent_t ev_xready[2], ev_fwd[2], ev_yfree[2], ev_entry;
  int host_slot;
  bool last_was_host;    // the handle's last device work was a moe_forward_host
  GemmPlan plan1, plan2;
  void* wsplit;          // bf16 tokens: W_g split into three bf16 parts [3][EP][M]
  CUtensorMap wmap, xmap, xmap64;
  const void* xmap_ptr;  // x pointer / S the cached xmap describes
  int64_t xmap_S;
  int64_t last_S;
  bool have_forward;
  bool fwd_data;         // the expert buffers hold the last forward's (not a route-only call's)
  bool profiling;
  uint32_t route_flags;  // MOE_ROUTE_* flags of later forwards
  int32_t* slot_tok;     // top-1, fused combine: token of each expert-buffer row [E*Cbuf]
  float* slot_gate;      // its gate [E*Cbuf]
  bool last_fused;       // the last forward stored the expert outputs straight into y
  bool last_rerouted;    // the last routing call gave dropped choices a second chance
  // backward (moe_enable_backward)
  void* bws;             // the backward's one device allocation
  void* dybuf;           // [E, Cbuf, M] act: dY, then dX_e
  void* dpre;            // [E, Cbuf, H] act: dP
  float* dl;             // [S_max, E]
  float* dgate;          // [S_max, k]
  float* part;           // dW_g / dbias split-K partials
  size_t part_floats;
  GemmPlan plan_dp, plan_dx;        // dP = (dY W2^T)*[h>0],  dX = dP W1^T
  GemmPlan plan_dw2, plan_dw1;      // dW2 = h^T dY,  dW1 = X^T dP (output pointers cached)
  const void* dw2_ptr;
  const void* dw1_ptr;
  uint32_t bwd_flags;               // MOE_BWD_* flags
  uint32_t* hbits;                  // [H/32, E*Cbuf] bits of h > 0, written by FFN1 once enabled
  bool bits_valid;                  // the last forward wrote hbits
  // A forward was captured into a CUDA graph without the bits epilogue: a replay of
  // that graph rewrites h but not hbits, and the host cannot see replays, so from
  // then on the backward reads its ReLU mask from h.
  bool graph_without_bits;
  // bf16: tensor-core gate gradients
  int EPb;                          // E rounded up to 64
  void* dlb;                        // [S_max, 2*EPb] bf16 split of dl
  float* bpart;                     // [4*num_sms, E] bias partials
  int32_t* cnt_rows;                // [1 + max splits]
  GemmPlan plan_gdx, plan_dwg;      // dx = dl W_g^T;  dW_g partials = x^T [dl_hi | dl_lo]
  const void* gdx_ptr;
  const void* dwg_ptr;
  int64_t gdx_S, dwg_S;
  cudaEvent_t ev[MOE_NUM_STAGES + 1];
  cudaEvent_t evb[MOE_NUM_BWD_STAGES + 1];
  bool have_events;
  bool have_backward_times;
  uint64_t wait_limit_ns;
};

namespace {

// Top-1 routing on an inference handle (no backward workspace): the second expert GEMM
// stores its gate-scaled rows straight into y, and no combine kernel runs.
bool fuses_combine(const moe_layer* h) { return h->slot_tok != nullptr && !h->bws; }

// Forward expert GEMMs below capacity: CTA pairs for each expert's 256-row blocks and
// one-CTA tiles for a last block of at most 128 rows (else 128-row tiles throughout).
constexpr bool kMixedTiles = false;

// Token rows x model width from which the combine (which moves about 3 bytes per element)
// outlasts the loss block, so summing the losses beside it costs nothing; below that the
// scan keeps them (measured: beside the skewed workload's 12 us combine, 16 us).
constexpr double kLossBesideCombine = 33554432.0;

size_t act_bytes(moe_dtype a) { return a == MOE_BF16 ? 2 : 4; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  if (e == cudaErrorMemoryAllocation) return MOE_ERR_OOM;
  return MOE_ERR_CUDA;
}


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

// Lays out the workspace; with base == nullptr only measures it.
size_t carve(moe_layer* h, char* base) {
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
  R.nexp = c.take<int32_t>(E);
  R.first = c.take<int32_t>(E);
  R.psum = c.take<float>(nchunk * E);
  R.lse2 = c.take<float>(nchunk);
  R.losses = c.take<float>(2);
  R.err = c.take<unsigned>(1);
  R.dest = c.take<int32_t>(S * k);
  R.alt = c.take<int32_t>(S * k);
  R.lrank2 = c.take<int32_t>(S * k);
  R.hist2 = c.take<int32_t>(k * nchunk * E);
  R.off2 = c.take<int32_t>(k * nchunk * E);
  h->xbuf = c.take<char>((size_t)E * h->Cbuf * h->M * as);
  h->hbuf = c.take<char>((size_t)E * h->Cbuf * h->H * as);
  h->ybuf = c.take<char>((size_t)E * h->Cbuf * h->M * as);
  for (int b = 0; b < 2; ++b) {
    h->xstage[b] = c.take<char>((size_t)S * h->M * as);
    h->ystage[b] = c.take<char>((size_t)S * h->M * as);
  }
  h->wsplit = h->act == MOE_BF16 ? c.take<char>((size_t)3 * router_tc_pad(h->E) * h->M * 2) : nullptr;
  const bool top1 = h->act == MOE_BF16 && k == 1;
  h->slot_tok = top1 ? c.take<int32_t>((size_t)E * h->Cbuf) : nullptr;
  h->slot_gate = top1 ? c.take<float>((size_t)E * h->Cbuf) : nullptr;
  return c.off + 256;
}

moe_status read_device_error(moe_handle h, cudaStream_t st) {
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

#define MOE_TRY(call)                            \
  do {                                           \
    cudaError_t _e = (call);                     \
    if (_e != cudaSuccess) return from_cuda(_e); \
  } while (0)

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_OOM: return "out of device memory";
    case MOE_ERR_STATE: return "call out of order";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* moe_backward_stage_name(int32_t s) {
  static const char* names[MOE_NUM_BWD_STAGES] = {"gate_bwd", "pad_zero", "dW2", "dP",
                                                  "dW1",      "dX_e",     "dx",  "dWg"};
  return (s >= 0 && s < MOE_NUM_BWD_STAGES) ? names[s] : "?";
}

const char* moe_stage_name(int32_t s) {
  static const char* names[MOE_NUM_STAGES] = {"router", "scan", "dispatch", "ffn1", "ffn2", "combine"};
  return (s >= 0 && s < MOE_NUM_STAGES) ? names[s] : "?";
}

moe_status moe_create(moe_handle* out, int64_t S_max, int64_t M, int64_t H, int32_t E, int32_t k,
                      double capacity_factor, moe_dtype act, const float* Wg, const float* bias,
                      const void* W1, const void* W2) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (S_max < 1 || M < 64 || H < 64 || (M % 64) || (H % 64) || E < 1 || k < 1 || k > E)
    return MOE_ERR_INVALID_ARG;
  if (!(capacity_factor > 0.0) || !isfinite(capacity_factor)) return MOE_ERR_INVALID_ARG;
  if (act != MOE_F32 && act != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (!Wg || !W1 || !W2 || !aligned(Wg, 4) || !aligned(W1, 16) || !aligned(W2, 16) ||
      (bias && !aligned(bias, 4)))
    return MOE_ERR_INVALID_ARG;
  if (E > kMaxExperts || k > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (S_max > (int64_t)1 << 30 || M > (1 << 16) || H > (1 << 16)) return MOE_ERR_UNSUPPORTED;

  moe_layer* h = new (std::nothrow) moe_layer();
  if (!h) return MOE_ERR_OOM;
  h->S_max = S_max;
  h->M = M;
  h->H = H;
  h->E = E;
  h->k = k;
  h->cf = capacity_factor;
  h->act = act;
  h->Wg = Wg;
  h->bias = bias;
  h->W1 = W1;
  h->W2 = W2;
  const int64_t C = capacity_of(capacity_factor, k, S_max, E);
  // rows per expert: at most min(C, S_max) are kept; rounded up to 256 so every GEMM
  // tile (128 rows, or 256 for a CTA pair) and its whole-tile stores stay inside the
  // expert's own rows
  const int64_t rows = C < S_max ? C : S_max;
  h->Cbuf = (rows + 255) / 256 * 256;
  // expert-buffer rows and token choices are 32-bit indices (TMA coordinates, tables)
  if ((int64_t)E * h->Cbuf > INT32_MAX || S_max * k > INT32_MAX) {
    delete h;
    return MOE_ERR_UNSUPPORTED;
  }
  h->wait_limit_ns = 2000000000ull;   // 2 s per wait: far above any legitimate wait
  cudaError_t ce = cudaGetDevice(&h->device);
  if (ce == cudaSuccess)
    ce = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
  if (ce != cudaSuccess) {
    delete h;
    return from_cuda(ce);
  }
  h->ws_bytes = carve(h, nullptr);
  ce = cudaMalloc(&h->ws, h->ws_bytes);
  if (ce != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return from_cuda(ce);
  }
  carve(h, static_cast<char*>(h->ws));
  ce = cudaMemset(h->R.err, 0, sizeof(unsigned));
  if (ce == cudaSuccess) ce = cudaMemset(h->R.losses, 0, 2 * sizeof(float));
  if (ce != cudaSuccess) {
    cudaFree(h->ws);
    delete h;
    return from_cuda(ce);
  }
  if (act == MOE_BF16) {
    const bool ok1 = make_gemm_plan(h->plan1, h->xbuf, W1, h->hbuf, E, h->Cbuf, (int)M, (int)H, true);
    const bool ok2 = make_gemm_plan(h->plan2, h->hbuf, W2, h->ybuf, E, h->Cbuf, (int)H, (int)M, false);
    ce = split_gate_weights(Wg, (int)M, E, h->wsplit, 0);
    if (ce == cudaSuccess) ce = cudaStreamSynchronize(0);
    const bool ok3 = ce == cudaSuccess && make_router_wmap(&h->wmap, h->wsplit, (int)M, E);
    if (!ok1 || !ok2 || !ok3) {
      cudaFree(h->ws);
      delete h;
      return MOE_ERR_CUDA;
    }
  }
  *out = h;
  return MOE_OK;
}

moe_status moe_destroy(moe_handle h) {
  if (!h) return MOE_OK;
  cudaError_t ce = cudaDeviceSynchronize();
  if (h->have_events) {
    for (auto& e : h->ev) cudaEventDestroy(e);
    for (auto& e : h->evb) cudaEventDestroy(e);
  }
  if (h->host_ready) {
    for (cudaStream_t s_ : {h->hs_in, h->hs_comp, h->hs_out}) cudaStreamDestroy(s_);
    for (int b = 0; b < 2; ++b) {
      cudaEventDestroy(h->ev_xready[b]);
      cudaEventDestroy(h->ev_fwd[b]);
      cudaEventDestroy(h->ev_yfree[b]);
    }
    cudaEventDestroy(h->ev_entry);
  }
  cudaError_t fe = cudaFree(h->ws);
  delete h;
  if (ce != cudaSuccess) return from_cuda(ce);
  return from_cuda(fe);
}

moe_status moe_get_capacity(moe_handle h, int64_t S, int64_t* C_out) {
  if (!h || !C_out || S < 0) return MOE_ERR_INVALID_ARG;
  *C_out = capacity_of(h->cf, h->k, S, h->E);
  return MOE_OK;
}

int32_t moe_kernels_per_forward(moe_handle h, int64_t S) {
  if (!h || S <= 0) return 0;
  const bool reroute = (h->route_flags & MOE_ROUTE_REROUTE) != 0;
  int n = reroute ? 8 : (fuses_combine(h) ? 5 : 6);
  if (h->act == MOE_BF16 && kMixedTiles && h->Cbuf % 256 == 0) {
    const int64_t C = capacity_of(h->cf, h->k, S, h->E);
    const bool saturated = (double)S * h->k / h->E >= (double)C;
    if (!saturated) n += (h->plan1.pair ? 1 : 0) + (h->plan2.pair ? 1 : 0);   // pair + rest launches
  }
  return n;
}

moe_status moe_set_routing_flags(moe_handle h, uint32_t flags) {
  if (!h || (flags & ~(uint32_t)MOE_ROUTE_REROUTE)) return MOE_ERR_INVALID_ARG;
  h->route_flags = flags;
  return MOE_OK;
}

}  // extern "C"

namespace {

// NVTX ranges on the host timeline: one around a forward or backward, one per stage
// around its launches (header-only NVTX: without a tool attached, each push or pop
// is a call that returns at once).
struct NvtxStages {
  const char* (*name)(int32_t);
  int n, open = -1;
  NvtxStages(const char* top, const char* (*name_)(int32_t), int n_) : name(name_), n(n_) {
    nvtxRangePushA(top);
  }
  void stage(int i) {
    if (open >= 0) nvtxRangePop();
    open = -1;
    if (i < n) {
      nvtxRangePushA(name(i));
      open = i;
    }
  }
  ~NvtxStages() {
    if (open >= 0) nvtxRangePop();
    nvtxRangePop();
  }
};

moe_status forward_impl(moe_handle h, int64_t S, const void* x, void* y, cudaStream_t st) {
  if (!h || S < 0 || S > h->S_max) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!x || !y || !aligned(x, 16) || !aligned(y, 16))) return MOE_ERR_INVALID_ARG;
  h->last_S = S;
  h->have_forward = true;
  h->fwd_data = true;
  h->bits_valid = false;
  h->last_fused = false;
  if (h->act == MOE_BF16 && !h->plan1.bits) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    // an error (a capture elsewhere in global mode) counts as capturing
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
      h->graph_without_bits = true;
  }
  if (S == 0) {
    MOE_TRY(cudaMemsetAsync(h->R.losses, 0, 2 * sizeof(float), st));
    return MOE_OK;
  }
  const bool bf16 = h->act == MOE_BF16;
  const int C = (int)capacity_of(h->cf, h->k, S, h->E);
  const int iS = (int)S, iM = (int)h->M, iH = (int)h->H;
  const Routing& R = h->R;
  const bool prof = h->profiling && h->have_events;
  NvtxStages nv("moe_forward", moe_stage_name, MOE_NUM_STAGES);
  auto mark = [&](int i) -> cudaError_t {
    nv.stage(i);
    return prof ? cudaEventRecord(h->ev[i], st) : cudaSuccess;
  };

  MOE_TRY(mark(0));
  if (bf16) {
    const bool persistent = router_persistent(h->E, iS);
    if (h->xmap_ptr != x || h->xmap_S != S) {
      if (!make_router_xmap(&h->xmap, x, iS, iM, h->E)) return MOE_ERR_CUDA;
      if (persistent && !make_router_xmap64(&h->xmap64, x, iS, iM)) return MOE_ERR_CUDA;
      h->xmap_ptr = x;
      h->xmap_S = S;
    }
    MOE_TRY(launch_router_tc(h->xmap, persistent ? &h->xmap64 : nullptr, x, h->wmap, h->bias, iS, iM, h->E,
                             h->k, R, h->wait_limit_ns, st));
  } else {
    MOE_TRY(launch_router(x, bf16, h->Wg, h->bias, iS, iM, h->E, h->k, R, st));
  }
  MOE_TRY(mark(1));
  const bool reroute = (h->route_flags & MOE_ROUTE_REROUTE) != 0;
  // top-1 inference: the combine is fused into the second expert GEMM, whose epilogue
  // stores each row straight into y (the backward needs the expert outputs, so a
  // handle in training mode keeps the separate combine)
  const bool fused = fuses_combine(h) && !reroute;
  // the losses are summed beside a long combine, off the dispatch's critical path;
  // beside a short one (or without one) they stay in the scan
  const bool loss_in_combine = !fused && (double)S * h->M >= kLossBesideCombine;
  MOE_TRY(launch_scan(iS, h->E, h->k, C, h->Cbuf, R, st, !loss_in_combine));
  h->last_rerouted = reroute;
  if (reroute) {       // second chance for dropped choices: offers, their scan
    MOE_TRY(launch_reroute_offers(iS, h->E, h->k, (int)(C < h->Cbuf ? C : h->Cbuf), R, st));
    MOE_TRY(launch_reroute_scan(iS, h->E, h->k, C, h->Cbuf, R, st));
  }
  MOE_TRY(mark(2));
  h->last_fused = fused;
  if (fused)
    MOE_TRY(launch_dispatch_fused(x, iS, iM, h->E, C, h->Cbuf, R, h->xbuf, h->slot_tok, h->slot_gate, y, st));
  else if (reroute)
    MOE_TRY(launch_dispatch_rerouted(x, bf16, iS, iM, h->E, h->k, C, h->Cbuf, R, h->xbuf, st));
  else
    MOE_TRY(launch_dispatch(x, bf16, iS, iM, h->E, h->k, C, h->Cbuf, R, h->xbuf, st));
  MOE_TRY(mark(3));
  if (bf16) {
    // CTA-pair GEMMs (256-row tiles) when the experts run at capacity, so the
    // rows per expert are close to C and the 256-row padding stays small;
    // otherwise 128-row tiles waste less on partly filled last tiles.
    const bool saturated = (double)S * h->k / h->E >= (double)C;
    // below capacity: pairs for each expert's 256-row blocks, one-CTA tiles for the rest
    MOE_TRY(launch_ffn_bf16(h->plan1, R.nexp, R.err, h->wait_limit_ns, h->num_sms, saturated, st,
                            kMixedTiles));
    h->bits_valid = h->plan1.bits != nullptr;
    MOE_TRY(mark(4));
    GemmPlan p2 = h->plan2;
    if (fused) p2.sy = ScatterY{h->slot_tok, h->slot_gate, y, h->M};
    MOE_TRY(launch_ffn_bf16(p2, R.nexp, R.err, h->wait_limit_ns, h->num_sms, saturated, st, kMixedTiles));
  } else {
    MOE_TRY(launch_ffn_f32((const float*)h->xbuf, (const float*)h->W1, (float*)h->hbuf, R.nexp,
                           h->E, h->Cbuf, iM, iH, true, st));
    MOE_TRY(mark(4));
    MOE_TRY(launch_ffn_f32((const float*)h->hbuf, (const float*)h->W2, (float*)h->ybuf, R.nexp,
                           h->E, h->Cbuf, iH, iM, false, st));
  }
  MOE_TRY(mark(5));
  if (!fused) {
    Routing Rc = R;
    if (reroute) Rc.eidx = R.dest;     // combine from the expert that served each choice
    MOE_TRY(launch_combine(h->ybuf, bf16, iS, iM, h->k, h->Cbuf, Rc, y, st, loss_in_combine, h->E));
  }
  MOE_TRY(mark(6));
  return MOE_OK;
}

cudaError_t host_pipeline_init(moe_handle h) {
  if (h->host_ready) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  for (cudaStream_t* s_ : {&h->hs_in, &h->hs_comp, &h->hs_out})
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(s_, cudaStreamNonBlocking);
  for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
    e = cudaEventCreateWithFlags(&h->ev_xready[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fwd[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_yfree[b], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_entry, cudaEventDisableTiming);
  if (e == cudaSuccess) h->host_ready = true;    // (a failure leaks the few objects made)
  return e;
}

}  // namespace

extern "C" {

moe_status moe_forward(moe_handle h, int64_t S, const void* x, void* y, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  return forward_impl(h, S, x, y, static_cast<cudaStream_t>(stream));
}

// Three stages on the handle's own streams, so that consecutive calls overlap: the
// copy of call i+1's x runs during call i's compute, and call i's y travels back
// during call i+1's compute.  Staging slot b = call parity; events hand a slot
// from one stage to the next and back.  Ordering with the caller:
//  - `stream` waits for this call's copy back of y, so work later on `stream`
//    (or a synchronisation of it) sees the result;
//  - a call whose predecessor on this handle was not a host call first waits for
//    the work enqueued on `stream` so far (the handle's workspace may still be
//    read there); between host calls that wait is skipped, which is what lets
//    the copies overlap.
moe_status moe_forward_host(moe_handle h, int64_t S, const void* x_host, void* y_host, void* stream) {
  if (!h || S < 0 || S > h->S_max) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!x_host || !y_host)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (S == 0) {
    h->last_was_host = false;
    return forward_impl(h, 0, nullptr, nullptr, st);
  }
  MOE_TRY(host_pipeline_init(h));
  const size_t bytes = (size_t)S * h->M * act_bytes(h->act);
  const int b = h->host_slot;
  if (!h->last_was_host) {
    MOE_TRY(cudaEventRecord(h->ev_entry, st));
    MOE_TRY(cudaStreamWaitEvent(h->hs_in, h->ev_entry, 0));
    MOE_TRY(cudaStreamWaitEvent(h->hs_comp, h->ev_entry, 0));
  }
  // copy in: slot b's x was last read by the compute of call i-2
  MOE_TRY(cudaStreamWaitEvent(h->hs_in, h->ev_fwd[b], 0));
  MOE_TRY(cudaMemcpyAsync(h->xstage[b], x_host, bytes, cudaMemcpyHostToDevice, h->hs_in));
  MOE_TRY(cudaEventRecord(h->ev_xready[b], h->hs_in));
  // compute: needs this x, and slot b's y copied out by call i-2
  MOE_TRY(cudaStreamWaitEvent(h->hs_comp, h->ev_xready[b], 0));
  MOE_TRY(cudaStreamWaitEvent(h->hs_comp, h->ev_yfree[b], 0));
  moe_status s = forward_impl(h, S, h->xstage[b], h->ystage[b], h->hs_comp);
  if (s != MOE_OK) return s;
  MOE_TRY(cudaEventRecord(h->ev_fwd[b], h->hs_comp));
  // copy out, then make the caller's stream wait for it
  MOE_TRY(cudaStreamWaitEvent(h->hs_out, h->ev_fwd[b], 0));
  MOE_TRY(cudaMemcpyAsync(y_host, h->ystage[b], bytes, cudaMemcpyDeviceToHost, h->hs_out));
  MOE_TRY(cudaEventRecord(h->ev_yfree[b], h->hs_out));
  MOE_TRY(cudaStreamWaitEvent(st, h->ev_yfree[b], 0));
  h->host_slot = b ^ 1;
  h->last_was_host = true;
  return MOE_OK;
}

moe_status moe_aux_loss(moe_handle h, float* l_aux, float* z_loss, void* stream) {
  if (!h || !l_aux || !z_loss) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->have_forward) return MOE_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float v[2] = {0.f, 0.f};
  MOE_TRY(cudaMemcpyAsync(v, h->R.losses, sizeof(v), cudaMemcpyDeviceToHost, st));
  moe_status s = read_device_error(h, st);   // synchronises
  if (s != MOE_OK) return s;
  *l_aux = v[0];
  *z_loss = v[1];
  return MOE_OK;
}

moe_status moe_check(moe_handle h, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  return read_device_error(h, static_cast<cudaStream_t>(stream));
}

moe_status moe_get_logits(moe_handle h, float* logits, void* stream) {
  if (!h || !logits) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->have_forward) return MOE_ERR_STATE;
  if (h->last_S == 0) return MOE_OK;
  MOE_TRY(cudaMemcpyAsync(logits, h->R.logits, (size_t)h->last_S * h->E * sizeof(float),
                          cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_get_routing(moe_handle h, int32_t* eidx, float* gate, int32_t* slot, int32_t* cnt,
                           void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->have_forward) return MOE_ERR_STATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = (size_t)h->last_S * h->k;
  if (n) {
    if (eidx) MOE_TRY(cudaMemcpyAsync(eidx, h->R.eidx, n * 4, cudaMemcpyDeviceToDevice, st));
    if (gate) MOE_TRY(cudaMemcpyAsync(gate, h->R.gate, n * 4, cudaMemcpyDeviceToDevice, st));
    if (slot) MOE_TRY(cudaMemcpyAsync(slot, h->R.slot, n * 4, cudaMemcpyDeviceToDevice, st));
  }
  if (cnt) {
    if (h->last_S == 0)
      MOE_TRY(cudaMemsetAsync(cnt, 0, (size_t)h->E * 4, st));
    else
      MOE_TRY(cudaMemcpyAsync(cnt, h->R.cnt, (size_t)h->E * 4, cudaMemcpyDeviceToDevice, st));
  }
  return MOE_OK;
}

moe_status moe_get_serving_experts(moe_handle h, int32_t* dest, void* stream) {
  if (!h || !dest) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->have_forward) return MOE_ERR_STATE;
  const size_t n = (size_t)h->last_S * h->k;
  if (n)
    MOE_TRY(cudaMemcpyAsync(dest, h->last_rerouted ? h->R.dest : h->R.eidx, n * 4, cudaMemcpyDeviceToDevice,
                            static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_route_from_logits(moe_handle h, int64_t S, const float* logits, void* stream) {
  if (!h || S < 0 || S > h->S_max) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (S > 0 && (!logits || !aligned(logits, 4))) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  h->last_S = S;
  h->have_forward = true;
  h->fwd_data = false;
  h->bits_valid = false;
  if (S == 0) {
    MOE_TRY(cudaMemsetAsync(h->R.losses, 0, 2 * sizeof(float), st));
    return MOE_OK;
  }
  const int C = (int)capacity_of(h->cf, h->k, S, h->E);
  MOE_TRY(launch_route_logits(logits, (int)S, h->E, h->k, h->R, st));
  MOE_TRY(launch_scan((int)S, h->E, h->k, C, h->Cbuf, h->R, st));
  h->last_rerouted = (h->route_flags & MOE_ROUTE_REROUTE) != 0;
  if (h->last_rerouted) {
    MOE_TRY(launch_reroute_offers((int)S, h->E, h->k, (int)(C < h->Cbuf ? C : h->Cbuf), h->R, st));
    MOE_TRY(launch_reroute_scan((int)S, h->E, h->k, C, h->Cbuf, h->R, st));
    MOE_TRY(launch_dispatch_rerouted(nullptr, h->act == MOE_BF16, (int)S, (int)h->M, h->E, h->k, C,
                                     h->Cbuf, h->R, h->xbuf, st));
    return MOE_OK;
  }
  // slot pass of the dispatch kernel without moving any row
  MOE_TRY(launch_dispatch(nullptr, h->act == MOE_BF16, (int)S, (int)h->M, h->E, h->k, C, h->Cbuf,
                          h->R, h->xbuf, st));
  return MOE_OK;
}

moe_status moe_get_expert_rows(moe_handle h, int32_t which, int32_t e, int64_t nrows, void* dst,
                               void* stream) {
  if (!h || which < MOE_BUF_X || which > MOE_BUF_Y || e < 0 || e >= h->E || nrows < 0 ||
      nrows > h->Cbuf || (nrows > 0 && !dst))
    return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->have_forward || !h->fwd_data) return MOE_ERR_STATE;
  if (which == MOE_BUF_Y && h->last_fused) return MOE_ERR_STATE;   // stored straight into y
  if (nrows == 0) return MOE_OK;
  const size_t as = act_bytes(h->act);
  const int64_t width = which == MOE_BUF_H ? h->H : h->M;
  const void* base = which == MOE_BUF_X ? h->xbuf : which == MOE_BUF_H ? h->hbuf : h->ybuf;
  const size_t row_bytes = (size_t)width * as;
  const char* src = static_cast<const char*>(base) + (size_t)e * h->Cbuf * row_bytes;
  MOE_TRY(cudaMemcpyAsync(dst, src, (size_t)nrows * row_bytes, cudaMemcpyDeviceToDevice,
                          static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_set_profiling(moe_handle h, int32_t enable) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (enable && !h->have_events) {
    for (auto& e : h->ev) MOE_TRY(cudaEventCreate(&e));
    for (auto& e : h->evb) MOE_TRY(cudaEventCreate(&e));
    h->have_events = true;
  }
  h->profiling = enable != 0;
  return MOE_OK;
}

moe_status moe_get_stage_times(moe_handle h, float* ms, int32_t n) {
  if (!h || !ms || n < MOE_NUM_STAGES) return MOE_ERR_INVALID_ARG;
  if (!h->profiling || !h->have_events || !h->have_forward || h->last_S == 0) return MOE_ERR_STATE;
  MOE_TRY(cudaEventSynchronize(h->ev[MOE_NUM_STAGES]));
  for (int i = 0; i < MOE_NUM_STAGES; ++i) MOE_TRY(cudaEventElapsedTime(&ms[i], h->ev[i], h->ev[i + 1]));
  return MOE_OK;
}

moe_status moe_enable_backward(moe_handle h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (h->bws) return MOE_OK;
  const size_t as = act_bytes(h->act);
  const int64_t rowsE = (int64_t)h->E * h->Cbuf;
  const bool bf16 = h->act == MOE_BF16;
  h->EPb = (h->E + 63) / 64 * 64;
  const int ns_max = dwg_tc_split_bound((int)h->S_max, (int)h->M, h->EPb, h->num_sms);
  h->part_floats = bf16 ? (size_t)ns_max * h->M * 2 * h->EPb
                        : dwg_partial_floats((int)h->S_max, (int)h->M, h->E, h->num_sms);
  Carver c{nullptr};
  for (int pass = 0; pass < 2; ++pass) {
    c.off = 0;
    h->dybuf = c.take<char>((size_t)rowsE * h->M * as);
    h->dpre = c.take<char>((size_t)rowsE * h->H * as);
    h->dl = bf16 ? nullptr : c.take<float>((size_t)h->S_max * h->E);
    h->dgate = c.take<float>((size_t)h->S_max * h->k);
    h->part = c.take<float>(h->part_floats);
    h->dlb = bf16 ? c.take<char>((size_t)h->S_max * 2 * h->EPb * 2) : nullptr;
    h->bpart = bf16 ? c.take<float>((size_t)4 * h->num_sms * h->E) : nullptr;
    h->cnt_rows = bf16 ? c.take<int32_t>((size_t)1 + ns_max) : nullptr;
    h->hbits = bf16 ? c.take<uint32_t>((size_t)rowsE * (h->H / 32)) : nullptr;
    if (pass == 0) {
      const size_t bytes = c.off + 256;
      cudaError_t ce = cudaMalloc(&h->bws, bytes);
      if (ce != cudaSuccess) {
        cudaGetLastError();
        h->bws = nullptr;
        return from_cuda(ce);
      }
      c.base = static_cast<char*>(h->bws);
    }
  }
  if (h->act == MOE_BF16) {
    const int M = (int)h->M, H = (int)h->H;
    const bool ok = make_dgrad_plan(h->plan_dp, h->dybuf, h->W2, h->dpre, h->hbuf, h->E, h->Cbuf, M, H) &&
                    make_dgrad_plan(h->plan_dx, h->dpre, h->W1, h->dybuf, nullptr, h->E, h->Cbuf, H, M);
    if (!ok) {
      cudaFree(h->bws);
      h->bws = nullptr;
      return MOE_ERR_CUDA;
    }
    // from now on FFN1 also writes the bits of h > 0, which dP reads instead of h
    h->plan1.bits = h->hbits;
    h->plan_dp.bits = h->hbits;
    h->bits_valid = false;
  }
  h->dw1_ptr = h->dw2_ptr = nullptr;
  h->gdx_ptr = h->dwg_ptr = nullptr;
  h->gdx_S = h->dwg_S = -1;
  return MOE_OK;
}

moe_status moe_set_backward_flags(moe_handle h, uint32_t flags) {
  if (!h || (flags & ~(uint32_t)MOE_BWD_SKIP_EMPTY_EXPERTS)) return MOE_ERR_INVALID_ARG;
  h->bwd_flags = flags;
  return MOE_OK;
}

int32_t moe_kernels_per_backward(moe_handle h, int64_t S) {
  if (!h || S <= 0) return 0;
  return h->act == MOE_BF16 ? 10 : 8;
}

moe_status moe_backward(moe_handle h, int64_t S, const void* x, const void* dy, float a_aux, float a_z,
                        void* dx, float* dWg, float* dbias, void* dW1, void* dW2, void* stream) {
  if (!h || S < 0 || S > h->S_max) return MOE_ERR_INVALID_ARG;
  h->last_was_host = false;
  if (!h->bws || !h->have_forward || !h->fwd_data || S != h->last_S) return MOE_ERR_STATE;
  if (h->last_fused) return MOE_ERR_STATE;            // that forward kept no expert outputs
  if (!dWg || !dW1 || !dW2 || !aligned(dWg, 16) || !aligned(dW1, 16) || !aligned(dW2, 16) ||
      (dbias && !aligned(dbias, 4)))
    return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!x || !dy || !dx || !aligned(x, 16) || !aligned(dy, 16) || !aligned(dx, 16)))
    return MOE_ERR_INVALID_ARG;
  if (!isfinite(a_aux) || !isfinite(a_z)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t as = act_bytes(h->act);
  const int E = h->E, M = (int)h->M, H = (int)h->H;
  if (S == 0) {   // no tokens: every gradient is zero
    MOE_TRY(cudaMemsetAsync(dWg, 0, (size_t)M * E * 4, st));
    if (dbias) MOE_TRY(cudaMemsetAsync(dbias, 0, (size_t)E * 4, st));
    if (!(h->bwd_flags & MOE_BWD_SKIP_EMPTY_EXPERTS)) {   // every expert is empty
      MOE_TRY(cudaMemsetAsync(dW1, 0, (size_t)E * M * H * as, st));
      MOE_TRY(cudaMemsetAsync(dW2, 0, (size_t)E * H * M * as, st));
    }
    return MOE_OK;
  }
  const bool bf16 = h->act == MOE_BF16;
  BwdArgs a{};
  a.S = (int)S;
  a.M = M;
  a.H = H;
  a.E = E;
  a.k = h->k;
  a.Cbuf = h->Cbuf;
  a.bf16 = bf16;
  a.a_aux = a_aux;
  a.a_z = a_z;
  a.x = x;
  a.dy = dy;
  a.Wg = h->Wg;
  a.ybuf = h->ybuf;
  a.dybuf = h->dybuf;
  a.dl = h->dl;
  a.dgate = h->dgate;
  a.part = h->part;
  a.part_floats = h->part_floats;
  a.dx = dx;
  a.dWg = dWg;
  a.dbias = dbias;
  // a rerouted forward keeps a choice's rows at the expert serving it; its gate, and so
  // the gate gradient, belongs to the expert it chose
  a.dest = h->last_rerouted ? h->R.dest : nullptr;
  if (bf16) {
    a.dlb = h->dlb;
    a.EPb = h->EPb;
    a.bpart = h->bpart;
    a.cnt_rows = h->cnt_rows;
    dwg_tc_split((int)S, M, h->EPb, h->num_sms, a.nsplit, a.kchunk);
    if ((size_t)a.nsplit * M * 2 * h->EPb > h->part_floats) return MOE_ERR_STATE;
    if (h->gdx_ptr != dx || h->gdx_S != S) {
      if (!make_gate_dx_plan(h->plan_gdx, h->dlb, S, h->EPb, h->wsplit, router_tc_pad(E), dx, M))
        return MOE_ERR_CUDA;
      h->gdx_ptr = dx;
      h->gdx_S = S;
    }
    if (h->dwg_ptr != x || h->dwg_S != S) {
      if (!make_wgrad_plan(h->plan_dwg, x, h->dlb, h->part, a.nsplit, a.kchunk, M, 2 * h->EPb, true, S))
        return MOE_ERR_CUDA;
      h->dwg_ptr = x;
      h->dwg_S = S;
    }
  }
  const Routing& R = h->R;
  Routing Rrows = R;                   // row gathers address the serving expert's buffer
  if (h->last_rerouted) Rrows.eidx = R.dest;
  const bool prof = h->profiling && h->have_events;
  NvtxStages nv("moe_backward", moe_backward_stage_name, MOE_NUM_BWD_STAGES);
  auto mark = [&](int i) -> cudaError_t {
    nv.stage(i);
    return prof ? cudaEventRecord(h->evb[i], st) : cudaSuccess;
  };
  h->have_backward_times = false;
  MOE_TRY(mark(0));
  MOE_TRY(launch_gate_backward(a, R, st));
  MOE_TRY(mark(1));
  if (bf16) {
    if (h->dw2_ptr != dW2) {
      if (!make_wgrad_plan(h->plan_dw2, h->hbuf, h->dybuf, dW2, E, h->Cbuf, H, M)) return MOE_ERR_CUDA;
      h->dw2_ptr = dW2;
    }
    if (h->dw1_ptr != dW1) {
      if (!make_wgrad_plan(h->plan_dw1, h->xbuf, h->dpre, dW1, E, h->Cbuf, M, H)) return MOE_ERR_CUDA;
      h->dw1_ptr = dW1;
    }
    const bool skip = (h->bwd_flags & MOE_BWD_SKIP_EMPTY_EXPERTS) != 0;
    h->plan_dw2.skip_zero = skip;
    h->plan_dw1.skip_zero = skip;
    // else the mask is read from h itself
    h->plan_dp.use_bits = h->bits_valid && !h->graph_without_bits;
    // the weight-gradient GEMMs reduce over whole 64-slot blocks: clear the rows
    // between the kept count and the next multiple of 64
    void* bufs[3] = {h->xbuf, h->hbuf, h->dybuf};
    const int widths[3] = {M, H, M};
    MOE_TRY(launch_pad_zero(bufs, widths, 3, true, E, h->Cbuf, R, st));
    MOE_TRY(mark(2));
    const uint64_t lim = h->wait_limit_ns;
    // CTA pairs (256-row / 256-column tiles) under the forward's rule: experts at capacity
    const int C = (int)capacity_of(h->cf, h->k, S, E);
    const bool pair = (double)S * h->k / E >= (double)C;
    MOE_TRY(launch_ffn_bf16(h->plan_dw2, R.nexp, R.err, lim, h->num_sms, pair, st));
    MOE_TRY(mark(3));
    MOE_TRY(launch_ffn_bf16(h->plan_dp, R.nexp, R.err, lim, h->num_sms, pair, st));
    MOE_TRY(mark(4));
    MOE_TRY(launch_ffn_bf16(h->plan_dw1, R.nexp, R.err, lim, h->num_sms, pair, st));
    MOE_TRY(mark(5));
    MOE_TRY(launch_ffn_bf16(h->plan_dx, R.nexp, R.err, lim, h->num_sms, pair, st));
  } else {
    MOE_TRY(mark(2));
    MOE_TRY(launch_ffn_bwd_f32((const float*)h->xbuf, (const float*)h->hbuf, (float*)h->dybuf,
                               (float*)h->dpre, (const float*)h->W1, (const float*)h->W2, (float*)dW1,
                               (float*)dW2, R.nexp, E, h->Cbuf, M, H,
                               (h->bwd_flags & MOE_BWD_SKIP_EMPTY_EXPERTS) != 0, st));
    for (int i = 3; i <= 5; ++i) MOE_TRY(mark(i));   // the fp32 GEMMs are timed as one stage
  }
  MOE_TRY(mark(6));
  if (bf16) {
    const uint64_t lim = h->wait_limit_ns;
    MOE_TRY(launch_ffn_bf16(h->plan_gdx, h->cnt_rows, R.err, lim, h->num_sms, false, st));
    MOE_TRY(launch_dx_gather(a, Rrows, st));
    MOE_TRY(mark(7));
    MOE_TRY(launch_ffn_bf16(h->plan_dwg, h->cnt_rows + 1, R.err, lim, h->num_sms, false, st));
    MOE_TRY(launch_dwg_tc_reduce(a, gate_backward_grid((int)S, h->num_sms), h->num_sms, st));
  } else {
    MOE_TRY(launch_dx(a, Rrows, st));
    MOE_TRY(mark(7));
    MOE_TRY(launch_dwg(a, h->num_sms, st));
  }
  MOE_TRY(mark(8));
  h->have_backward_times = prof;
  return MOE_OK;
}

moe_status moe_get_backward_stage_times(moe_handle h, float* ms, int32_t n) {
  if (!h || !ms || n < MOE_NUM_BWD_STAGES) return MOE_ERR_INVALID_ARG;
  if (!h->have_backward_times) return MOE_ERR_STATE;
  MOE_TRY(cudaEventSynchronize(h->evb[MOE_NUM_BWD_STAGES]));
  for (int i = 0; i < MOE_NUM_BWD_STAGES; ++i)
    MOE_TRY(cudaEventElapsedTime(&ms[i], h->evb[i], h->evb[i + 1]));
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(int32_t limit_us, void* stream) {
  if (limit_us < 0 || limit_us > 10000000) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* buf = nullptr;
  MOE_TRY(cudaMalloc(&buf, 2 * sizeof(unsigned)));
  unsigned host[2] = {0, 0};
  cudaError_t ce = cudaMemsetAsync(buf, 0, 2 * sizeof(unsigned), st);
  if (ce == cudaSuccess) ce = launch_wait_selftest(buf, buf + 1, (uint64_t)limit_us * 1000ull, st);
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(host, buf, sizeof(host), cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(st);
  cudaFree(buf);
  if (ce != cudaSuccess) return from_cuda(ce);
  if (host[0] == 2u && (host[1] & DEVERR_TIMEOUT)) return MOE_ERR_TIMEOUT;
  return MOE_OK;
}

}  // extern "C"
