// reroute.cu -- a second chance for the choices the capacity pass dropped.
//
// "GShard: Scaling Giant Neural Networks with Conditional Computation", "Expert
// Capacity": tokens over an expert's capacity are either dropped or routed to
// alternative experts.  The page gives no rule for the alternative; the one taken
// here (off unless the handle's MOE_ROUTE_REROUTE flag is set):
//   - the token's j-th dropped choice (in choice-rank order) is offered its
//     (k + j)-th ranked expert: the best logit among the experts the token neither
//     chose nor was offered before, ties to the lower index;
//   - offers are taken in the capacity pass's order (rank r, then token) into the
//     room the pass left (C minus its kept rows), each accepted offer taking the
//     next free slot; an offer that finds no room stays dropped;
//   - a rerouted choice keeps its gate weight.
// The accepted offers are a rank-major capacity pass of their own, so the same
// machinery applies: per-chunk local ranks and histograms here, a per-expert
// prefix in reroute_scan_kernel (starting after the kept rows), the final slot in
// the dispatch.
//
// One CTA per 64-token chunk.  A warp takes one token at a time: the lanes of the
// first k read the choice's primary slot (off + lrank < C) and write it; if any
// choice was dropped the warp reads the token's logit row (lanes over experts) and
// picks the offers by warp argmax, skipping the chosen and already offered experts.
// Then one warp per rank r gives each offer its local rank among same-expert offers
// of the chunk (a match over 32 tokens at a time, a running count per expert).
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int RE>
__global__ void __launch_bounds__(kThreads) reroute_offers_kernel(int S, int E, int k, int C, int nchunk,
                                                                  Routing R) {
  __shared__ int32_t sel[kChunk][kMaxK];              // offer of each (token, rank), -1 if none
  __shared__ int32_t cnt[kMaxK][kMaxExperts];         // running offers per (rank, expert)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, tok0 = chunk * kChunk;
  const int ntok = min(kChunk, S - tok0);
  pdl_trigger();
  for (int i = threadIdx.x; i < kMaxK * kMaxExperts; i += kThreads) (&cnt[0][0])[i] = 0;
  pdl_wait();                                   // logits, choices, local ranks and offsets complete
  for (int tl = warp; tl < kChunk; tl += kWarps) {
    const bool live = tl < ntok;                // warp-uniform
    const int64_t t = tok0 + tl;
    int e = -1, s = -1;
    if (live && lane < k) {
      e = R.eidx[t * k + lane];
      if (e >= 0 && e < E) {
        const int pos = R.off[((int64_t)lane * nchunk + chunk) * E + e] + R.lrank[t * k + lane];
        s = pos < C ? pos : -1;
      } else {
        atomicOr(R.err, DEVERR_BOUNDS);
        e = -1;
      }
      R.slot[t * k + lane] = s;
    }
    const unsigned dropped = __ballot_sync(0xffffffffu, live && lane < k && e >= 0 && s < 0);
    int mine = -1;                              // this lane's offer (lane = choice rank)
    if (dropped) {
      float v[RE];
#pragma unroll
      for (int i = 0; i < RE; ++i) {
        const int j = lane + 32 * i;
        v[i] = j < E ? R.logits[t * E + j] : -INFINITY;
      }
      unsigned taken = 0;                       // bit i: expert lane + 32 i chosen or offered
      for (int r = 0; r < k; ++r) {
        const int er = __shfl_sync(0xffffffffu, e, r);
        if (er >= 0 && (er & 31) == lane) taken |= 1u << (er >> 5);
      }
      for (int r = 0; r < k; ++r) {
        if (!((dropped >> r) & 1u)) continue;   // warp-uniform
        float bv = -INFINITY;
        int bj = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < RE; ++i) {
          const int j = lane + 32 * i;
          if (j < E && !((taken >> i) & 1u) && (v[i] > bv || bj == 0x7fffffff)) {
            bv = v[i];
            bj = j;
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
          if (oj != 0x7fffffff && (bj == 0x7fffffff || ov > bv || (ov == bv && oj < bj))) {
            bv = ov;
            bj = oj;
          }
        }
        const int a = bj < E ? bj : -1;         // none left when k + j >= E
        if (a >= 0 && (a & 31) == lane) taken |= 1u << (a >> 5);
        if (lane == r) mine = a;
      }
    }
    if (lane < k) {
      sel[tl][lane] = live ? mine : -1;
      if (live) R.alt[t * k + lane] = mine;
    }
  }
  __syncthreads();
  for (int r = warp; r < k; r += kWarps) {
    for (int h = 0; h < kChunk / 32; ++h) {
      const int tl = h * 32 + lane;
      const int a = tl < ntok ? sel[tl][r] : -1;
      const unsigned m = __match_any_sync(0xffffffffu, a >= 0 ? a : kMaxExperts + lane);
      if (tl < ntok)
        R.lrank2[(int64_t)(tok0 + tl) * k + r] = a >= 0 ? cnt[r][a] + __popc(m & ((1u << lane) - 1u)) : -1;
      __syncwarp();
      if (a >= 0 && lane == __ffs(m) - 1) cnt[r][a] += __popc(m);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < k * E; i += kThreads) {
    const int r = i / E, ex = i - r * E;
    R.hist2[((int64_t)r * nchunk + chunk) * E + ex] = cnt[r][ex];
  }
}

}  // namespace

cudaError_t launch_reroute_offers(int S, int E, int k, int C, const Routing& R, cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int RE = (E + 31) / 32;
  if (RE <= 1) return launch_pdl(reroute_offers_kernel<1>, dim3(nchunk), dim3(kThreads), 0, st, S, E, k, C, nchunk, R);
  if (RE <= 2) return launch_pdl(reroute_offers_kernel<2>, dim3(nchunk), dim3(kThreads), 0, st, S, E, k, C, nchunk, R);
  if (RE <= 4) return launch_pdl(reroute_offers_kernel<4>, dim3(nchunk), dim3(kThreads), 0, st, S, E, k, C, nchunk, R);
  return launch_pdl(reroute_offers_kernel<8>, dim3(nchunk), dim3(kThreads), 0, st, S, E, k, C, nchunk, R);
}

}  // namespace moe
