// internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <utility>

namespace moe {

constexpr int kMaxExperts = 256;
constexpr int kMaxK = 8;
constexpr int kChunk = 64;          // tokens per router CTA (= scan chunk)

// Expert capacity C = ceil(capacity_factor * k * S / E), evaluated in double left to
// right ("GShard: Scaling Giant Models with Conditional Computation and Automatic
// Sharding", paper-note summary: tokens beyond an expert's capacity, set by the
// capacity factor, are dropped); clamped to 2^31 - 1.
inline int64_t capacity_of(double cf, int k, int64_t S, int E) {
  const double c = ceil(cf * (double)k * (double)S / (double)E);
  if (!(c < 2147483647.0)) return 2147483647;
  return (int64_t)c;
}

// Launch with programmatic stream serialization: the kernel may begin while the
// previous kernel on the stream finishes, and orders itself with pdl_wait().
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Device tables of one forward (all owned by the handle's workspace).
struct Routing {
  float* logits;     // [S, E]   fp32 logits as routed (bias included)
  int32_t* eidx;     // [S, k]   expert of each choice, best first
  float* gate;       // [S, k]   normalised gate weight
  int32_t* lrank;    // [S, k]   rank of (t, r) among same-expert rank-r choices in t's chunk
  int32_t* slot;     // [S, k]   slot in the expert's buffer, -1 if dropped
  int32_t* hist;     // [k, nchunk, E] rank-r choices of each expert per chunk
  int32_t* off;      // [k, nchunk, E] exclusive rank-major prefix of hist per expert
  int32_t* cnt;      // [E] demand per expert (before capacity)
  int32_t* nexp;     // [E] kept rows per expert = min(cnt, C)
  int32_t* first;    // [E] tokens whose first choice is the expert (f_j * S)
  float* psum;       // [nchunk, E] per-chunk sum of softmax probabilities
  float* lse2;       // [nchunk]    per-chunk sum of lse^2
  float* losses;     // [2]  l_aux, z
  unsigned* err;     // device error word
  // rerouting of dropped choices (a second chance at the token's next-ranked expert)
  int32_t* dest;     // [S, k]   expert serving each choice (eidx unless rerouted)
  int32_t* alt;      // [S, k]   expert a dropped choice is offered, -1 if none
  int32_t* lrank2;   // [S, k]   rank of the offer among same-expert rank-r offers in t's chunk
  int32_t* hist2;    // [k, nchunk, E] rank-r offers to each expert per chunk
  int32_t* off2;     // [k, nchunk, E] first free slot of each chunk's offers (kept rows + prefix)
};

// router.cu
cudaError_t launch_router(const void* x, bool x_bf16, const float* Wg, const float* bias, int S,
                          int M, int E, int k, const Routing& R, cudaStream_t st);
cudaError_t launch_route_logits(const float* logits, int S, int E, int k, const Routing& R,
                                cudaStream_t st);
// router_tc.cu  (bf16 tokens: gate GEMM on tcgen05 with a bf16x3 split of W_g)
int router_tc_pad(int E);
cudaError_t split_gate_weights(const float* Wg, int M, int E, void* out3, cudaStream_t st);
bool make_router_wmap(CUtensorMap* tm, const void* wsplit, int M, int E);
bool make_router_xmap(CUtensorMap* tm, const void* x, int S, int M, int E);
// x map with 64-row boxes (the persistent router's last, one-chunk tiles)
bool make_router_xmap64(CUtensorMap* tm, const void* x, int S, int M);
// whether S tokens with E experts take the persistent router (E <= 64 and at least four
// 64-token chunks per SM), which needs the 64-row x map as well
bool router_persistent(int E, int S);
// x: the token rows themselves (unused by the current kernels; the maps describe them)
cudaError_t launch_router_tc(const CUtensorMap& tmX, const CUtensorMap* tmX64, const void* x,
                             const CUtensorMap& tmW, const float* bias, int S, int M, int E, int k,
                             const Routing& R, uint64_t limit_ns, cudaStream_t st);
// scan.cu
// with_losses: one more block computes the auxiliary losses (else the combine does)
cudaError_t launch_scan(int S, int E, int k, int C, int64_t Cbuf, const Routing& R, cudaStream_t st,
                        bool with_losses = true);
// scan.cu, expert parallelism: per-rank scan of one rank's tokens.  off[r][c][e] gets the
// exclusive prefix of hist[r][.][e] over chunks; stats (doubles, ep_stats_len(E, k)):
// [r*E + e] rank-r demand of expert e, [k*E + j] sum over tokens of p_tj,
// [k*E + E] sum of lse^2, [k*E + E + 1] the rank's token count S.
inline int ep_stats_len(int E, int k) { return k * E + E + 2; }
cudaError_t launch_ep_scan(int S, int E, int k, const Routing& R, double* stats, cudaStream_t st);
// Expert parallelism over peer memory: rank d's receive buffer as this GPU addresses it,
// and the row at which this rank's rows for d start there minus the row at which they
// start in this rank's send order (row in d's buffer = send row + delta).
struct EpPeer {
  void* base;
  int64_t delta;
};
// dispatch_combine.cu, expert parallelism (one rank's side of the two exchanges):
//   ep_dispatch: slot[t][r] = base[r][e] + off[r][c][e] + lrank (global rank-major slot),
//     kept iff < C; a kept row goes to sendbuf[soff[r][e] + off + lrank] (runs ordered by
//     destination rank, expert, rank r), spos[t][r] = that row or -1
//   ep_unpack: received row j of segment q (starts seg_start[q], sorted) goes to expert row
//     seg_dst[q] + (j - seg_start[q]); rowmap[j] records it
//   ep_repack: recvbuf[j] = ybuf[rowmap[j]] (the expert outputs go back in arrival order)
// peers (device [G], or null): each kept row goes straight to its owner's receive buffer
// (rank e / El) instead of into sendbuf
cudaError_t launch_ep_dispatch(const void* x, bool bf16, int S, int M, int E, int k, int C,
                               const Routing& R, const int32_t* base, const int32_t* soff,
                               int32_t* spos, void* sendbuf, cudaStream_t st,
                               const EpPeer* peers = nullptr, int El = 1);
cudaError_t launch_ep_unpack(const void* recvbuf, bool bf16, int nrows, int M, const int32_t* seg_start,
                             const int32_t* seg_dst, int nseg, int32_t* rowmap, void* xbuf,
                             unsigned* err, int64_t xrows, cudaStream_t st);
cudaError_t launch_ep_repack(const void* ybuf, bool bf16, int nrows, int M, const int32_t* rowmap,
                             void* recvbuf, cudaStream_t st);
// reroute.cu: primary slots, and for each dropped choice the alternative it is offered
// (the token's next-ranked expert it has not chosen or been offered), with the offers'
// chunk histograms and local ranks.  Needs the router's logits and the scan's offsets.
// C: the capacity, at most the rows per expert of the buffers.
cudaError_t launch_reroute_offers(int S, int E, int k, int C, const Routing& R, cudaStream_t st);
// scan.cu: offsets of the offers per expert, starting after the rows the first pass
// kept; nexp becomes the final kept rows per expert.
cudaError_t launch_reroute_scan(int S, int E, int k, int C, int64_t Cbuf, const Routing& R,
                                cudaStream_t st);
// dispatch_combine.cu: final slot and serving expert of every choice, then the row
// copies (x == nullptr: tables only).
cudaError_t launch_dispatch_rerouted(const void* x, bool bf16, int S, int M, int E, int k, int C,
                                     int64_t Cbuf, const Routing& R, void* xbuf, cudaStream_t st);
// dispatch_combine.cu
cudaError_t launch_dispatch(const void* x, bool bf16, int S, int M, int E, int k, int C,
                            int64_t Cbuf, const Routing& R, void* xbuf, cudaStream_t st);
// The dispatch of the fused top-1 combine: as launch_dispatch, and every kept slot's token
// and gate into tok / gsc [E*Cbuf]; a token whose choice was dropped gets y = 0.
cudaError_t launch_dispatch_fused(const void* x, int S, int M, int E, int C, int64_t Cbuf,
                                  const Routing& R, void* xbuf, int32_t* tok, float* gsc, void* y,
                                  cudaStream_t st);
// with_losses: one more block computes the auxiliary losses (E experts) beside the combine
// peers (device [G], or null): the row of choice (t, r) is read from its owner's receive
// buffer, peers[e / El].base + (slot + peers[e / El].delta) rows, instead of ybuf
cudaError_t launch_combine(const void* ybuf, bool bf16, int S, int M, int k, int64_t Cbuf,
                           const Routing& R, void* y, cudaStream_t st, bool with_losses = false,
                           int E = 0, const EpPeer* peers = nullptr, int El = 1);
// ffn_simt.cu  (fp32 activations)
cudaError_t launch_ffn_f32(const float* A, const float* B, float* D, const int32_t* nexp, int E,
                           int64_t Cbuf, int K, int N, bool relu, cudaStream_t st);
// ffn_tc.cu  (bf16 activations, tcgen05)
enum { kGemmFwd = 0, kGemmDgrad = 1, kGemmWgrad = 2 };
// Gate-scaled stores straight into the layer output (forward FFN2 under top-1 routing):
// row r of the expert buffers (expert r / Cbuf, slot r % Cbuf) is taken by token tok[r]
// with gate gsc[r]; its result g * row goes to y[tok[r]] (ldy elements per row).  Rows at
// or past the expert's kept count are not stored.
struct ScatterY {
  const int32_t* tok;   // [E*Cbuf]
  const float* gsc;     // [E*Cbuf]
  void* y;              // [S, ldy] bf16, or null: the plain store into D
  int64_t ldy;
};

struct GemmPlan {
  // kGemmFwd   D[e,:n_e] = act(A[e,:n_e] . B[e])     A [E*Cbuf, K], B [E*K, N]
  // kGemmDgrad D[e,:n_e] = (A[e,:n_e] . Bt[e]^T) (* [mask > 0])   Bt [E*N, K]
  // kGemmWgrad D[e] = A[e,:n_e]^T . B[e,:n_e]        A [E*Cbuf, K=P], B [E*Cbuf, N=Q], D [E*P, Q]
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmD;   // box {64, 32}, 128B swizzle (epilogue stores)
  CUtensorMap tmB2;  // kGemmDgrad CTA pairs: B box {64, 128} (each CTA's half of the N rows)
  void* D;
  const void* mask;  // kGemmDgrad: [E*Cbuf, N] bf16 values whose sign masks the result, or null
  uint32_t* bits;    // [N/32, E*Cbuf] mask bits, word-major: kGemmFwd with ReLU writes them (h > 0);
                     // kGemmDgrad reads them instead of `mask` when use_bits is set
  bool use_bits;
  int kind;
  int E, K, N, BN;
  int64_t Cbuf;
  bool relu;
  bool pair;         // the CTA-pair (cta_group::2, 256 x 256 tile) kernel can run (N % 256 == 0)
  bool f32out;       // kGemmWgrad: D is fp32
  bool skip_zero;    // kGemmWgrad: experts with no kept row leave D[e] untouched (else zeros)
  int64_t row_limit; // rows of D (0 = E*Cbuf): stores of 32-row groups starting past it are skipped
  ScatterY sy;       // kGemmFwd: with sy.y set, the epilogue stores gate-scaled rows into y instead of D
  const int32_t* row_base;  // kGemmFwd / kGemmDgrad: [E] device, expert e's rows start at row_base[e]
                            // (its n_e rows are [row_base[e], row_base[e] + n_e)); null = 0
};
bool make_gemm_plan(GemmPlan& p, const void* A, const void* B, void* D, int E, int64_t Cbuf, int K,
                    int N, bool relu);
bool make_dgrad_plan(GemmPlan& p, const void* A, const void* Bt, void* D, const void* mask, int E,
                     int64_t Cbuf, int K, int N);
// rows_ab: rows of the A / B tensor maps (0 = E*Cbuf); rows past it read as zeros
bool make_wgrad_plan(GemmPlan& p, const void* A, const void* B, void* D, int E, int64_t Cbuf, int P,
                     int Q, bool f32out = false, int64_t rows_ab = 0);
// dx = dl_hi . W_g,hi^T as a one-expert forward GEMM: A = dlb [S, 2*EPb] (hi half),
// B = the router's W_g split [3*EPr, M], D = dx [S, M]
bool make_gate_dx_plan(GemmPlan& p, const void* dlb, int64_t S, int EPb, const void* wsplit,
                       int EPr, void* dx, int M);
// want_pair: CTA-pair (256-row) tiles everywhere (experts at capacity).  mixed (forward
// GEMMs, when want_pair is off): pairs for each expert's 256-row blocks and one-CTA tiles
// for a last block of at most 128 rows -- two launches.  Otherwise 128-row tiles.
cudaError_t launch_ffn_bf16(const GemmPlan& p, const int32_t* nexp, unsigned* err,
                            uint64_t wait_limit_ns, int num_sms, bool want_pair, cudaStream_t st,
                            bool mixed = false);
// backward.cu
struct BwdArgs {
  int S, M, H, E, k;
  int64_t Cbuf;
  bool bf16;
  float a_aux, a_z;
  const void* x;       // [S, M] act
  const void* dy;      // [S, M] act
  const float* Wg;     // [M, E]
  const void* ybuf;    // [E*Cbuf, M] act (forward's expert outputs)
  void* dybuf;         // [E*Cbuf, M] act (dY, later dX_e)
  float* dl;           // [S, E]
  float* dgate;        // [S, k]
  float* part;         // split-K partials of dWg and dbias
  size_t part_floats;
  void* dx;            // [S, M] act
  float* dWg;          // [M, E]
  float* dbias;        // [E] or null
  // bf16 activations (tensor-core gate gradients)
  void* dlb;           // [S, 2*EPb] bf16: dl hi in columns [0, EPb), lo in [EPb, 2*EPb)
  int EPb;             // E rounded up to 64
  float* bpart;        // [gate_bwd CTAs, E] bias partials
  int32_t* cnt_rows;   // [1 + nsplit]: S, then the rows of each dW_g split
  int nsplit, kchunk;  // dW_g split-K: nsplit splits of kchunk tokens
  // rerouted forward: the expert serving each choice [S, k] (its rows' buffer), while
  // the gate gradient goes to the chosen expert (Routing::eidx); null otherwise
  const int32_t* dest;
};
cudaError_t launch_gate_backward(const BwdArgs& a, const Routing& R, cudaStream_t st);
cudaError_t launch_pad_zero(void* const* bufs, const int* widths, int nbuf, bool bf16, int E,
                            int64_t Cbuf, const Routing& R, cudaStream_t st);
cudaError_t launch_dx(const BwdArgs& a, const Routing& R, cudaStream_t st);
int gate_backward_grid(int S, int num_sms);
cudaError_t launch_dx_gather(const BwdArgs& a, const Routing& R, cudaStream_t st);
cudaError_t launch_dwg_tc_reduce(const BwdArgs& a, int nbpart, int num_sms, cudaStream_t st);
cudaError_t launch_dwg(const BwdArgs& a, int num_sms, cudaStream_t st);
size_t dwg_partial_floats(int S, int M, int E, int num_sms);
// bf16 dW_g: split-K over tokens, about one tile per SM; splits of kchunk (a multiple
// of 64) tokens.  nsplit(S) <= dwg_tc_split_bound(S_max) for every S <= S_max.
void dwg_tc_split(int S, int M, int EPb, int num_sms, int& nsplit, int& kchunk);
int dwg_tc_split_bound(int S, int M, int EPb, int num_sms);
// fp32 activations: the expert FFN's backward GEMMs on CUDA cores
cudaError_t launch_ffn_bwd_f32(const float* xbuf, const float* hbuf, float* dybuf, float* dpre,
                               const float* W1, const float* W2, float* dW1, float* dW2,
                               const int32_t* nexp, int E, int64_t Cbuf, int M, int H,
                               bool skip_empty, cudaStream_t st);
// selftest.cu
cudaError_t launch_wait_selftest(unsigned* flag, unsigned* err, uint64_t limit_ns, cudaStream_t st);

}  // namespace moe
