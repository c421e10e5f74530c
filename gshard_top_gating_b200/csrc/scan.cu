// scan.cu -- capacity scan (rank-major slot offsets per expert) and loss finalize.
//
// Capacity: each expert takes at most C = ceil(capacity_factor * k * S / E)
// assignments and the rest are dropped ("GShard: Scaling Giant Models with
// Conditional Computation and Automatic Sharding", paper-note summary; "GShard:
// Scaling Giant Neural Networks with Conditional Computation", "Expert Capacity").
// Order: all first choices in token order, then all second choices, ...  The
// router leaves hist[r][chunk][e] (rank-r choices of expert e in a chunk of 64
// tokens); for each expert the exclusive prefix over (r, chunk) in that
// lexicographic order is the position of the chunk's first such choice.
//
// Losses ("GShard: Scaling Giant Models ...", paper-note summary: load-balance
// loss N * sum_j f_j P_j plus a z-loss): l_aux = E * sum_j f_j P_j with
// f_j = (first choices of j) / S and P_j = (sum_t p_tj) / S; z = sum_t lse_t^2 / S.
// Partials are summed in a fixed order in double, so results are deterministic.
#include "common.cuh"
#include "internal.h"
#include "losses.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (kThreads / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kThreads / 32) warp_sums[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  total = warp_sums[kThreads / 32 - 1];
  const int before = warp ? warp_sums[warp - 1] : 0;
  return before + x - v;
}

__global__ void __launch_bounds__(kThreads) scan_kernel(int S, int E, int k, int C, int Cbuf,
                                                        int nchunk, Routing R) {
  static_assert(kThreads == kLossThreads, "the loss block runs with the scan's block size");
  __shared__ int warp_sums[kThreads / 32];
  const int tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();                                  // router tables complete
  if (blockIdx.x < (unsigned)E) {
    const int e = blockIdx.x;
    const int L = k * nchunk;                 // entries (r, chunk), r-major
    const int seg = (L + kThreads - 1) / kThreads;
    const int a = min(L, tid * seg), b = min(L, a + seg);
    int local = 0;
    for (int q = a; q < b; ++q) local += R.hist[(int64_t)q * E + e];
    int total;
    int run = block_exclusive_scan(local, warp_sums, total);
    for (int q = a; q < b; ++q) {
      R.off[(int64_t)q * E + e] = run;
      run += R.hist[(int64_t)q * E + e];
    }
    if (tid == 0) {
      R.cnt[e] = total;
      R.nexp[e] = min(total, min(C, Cbuf));   // Cbuf bounds the buffers even on bad input
    }
    return;
  }
  // block E (launched when no combine kernel follows): the auxiliary losses
  aux_loss_block(S, E, nchunk, R);
}

// Expert parallelism: the scan of one rank's own tokens.  Block e (< E): for every
// rank r, the exclusive prefix of hist[r][.][e] over the rank's chunks (the position of
// each chunk's first rank-r choice of e among the rank's own rank-r choices of e) and
// the total.  Block E: the loss partials of the rank's tokens, summed in double in a
// fixed order (chunk groups as in scan_kernel), and the token count.
__global__ void __launch_bounds__(kThreads) ep_scan_kernel(int S, int E, int k, int nchunk, Routing R,
                                                           double* __restrict__ stats) {
  __shared__ int warp_sums[kThreads / 32];
  __shared__ double dsum[kThreads / 32];
  const int tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();                                  // router tables complete
  if (blockIdx.x < (unsigned)E) {
    const int e = blockIdx.x;
    const int seg = (nchunk + kThreads - 1) / kThreads;
    const int a = min(nchunk, tid * seg), b = min(nchunk, a + seg);
    for (int r = 0; r < k; ++r) {
      const int64_t q0 = (int64_t)r * nchunk;
      int local = 0;
      for (int c = a; c < b; ++c) local += R.hist[(q0 + c) * E + e];
      int total;
      int run = block_exclusive_scan(local, warp_sums, total);
      for (int c = a; c < b; ++c) {
        R.off[(q0 + c) * E + e] = run;
        run += R.hist[(q0 + c) * E + e];
      }
      if (tid == 0) stats[(int64_t)r * E + e] = (double)total;
      __syncthreads();                         // warp_sums is reused by the next rank
    }
    return;
  }
  __shared__ double part_P[kThreads];
  const int G = E >= kThreads ? 1 : kThreads / E;
  if (tid < E * G) {
    const int j = tid % E, g = tid / E;
    double P = 0.0;
    for (int c = g; c < nchunk; c += G) P += (double)R.psum[(int64_t)c * E + j];
    part_P[tid] = P;
  }
  __syncthreads();
  for (int j = tid; j < E; j += kThreads) {
    double P = 0.0;
    for (int g = 0; g < G; ++g) P += part_P[g * E + j];
    stats[(int64_t)k * E + j] = P;
  }
  double zl = 0.0;
  for (int c = tid; c < nchunk; c += kThreads) zl += (double)R.lse2[c];
  const double zs = block_sum_f64(zl, dsum);
  if (tid == 0) {
    stats[(int64_t)k * E + E] = zs;
    stats[(int64_t)k * E + E + 1] = (double)S;
  }
}

// Rerouting: one block per expert.  The offers to e form a rank-major sequence over
// (r, chunk) like the choices; their slots start after the rows the first pass kept
// (nexp), and an offer is accepted while its slot is below C.
__global__ void __launch_bounds__(kThreads) reroute_scan_kernel(int S, int E, int k, int C, int Cbuf,
                                                                int nchunk, Routing R) {
  __shared__ int warp_sums[kThreads / 32];
  const int tid = threadIdx.x, e = blockIdx.x;
  pdl_trigger();
  pdl_wait();                                  // offers and first-pass counts complete
  const int kept = R.nexp[e];
  const int L = k * nchunk;
  const int seg = (L + kThreads - 1) / kThreads;
  const int a = min(L, tid * seg), b = min(L, a + seg);
  int local = 0;
  for (int q = a; q < b; ++q) local += R.hist2[(int64_t)q * E + e];
  int total;
  int run = kept + block_exclusive_scan(local, warp_sums, total);
  for (int q = a; q < b; ++q) {
    R.off2[(int64_t)q * E + e] = run;
    run += R.hist2[(int64_t)q * E + e];
  }
  if (tid == 0) R.nexp[e] = min(kept + total, min(C, Cbuf));
}

}  // namespace

cudaError_t launch_reroute_scan(int S, int E, int k, int C, int64_t Cbuf, const Routing& R,
                                cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int cb = Cbuf < 0x7fffffff ? (int)Cbuf : 0x7fffffff;
  return launch_pdl(reroute_scan_kernel, dim3(E), dim3(kThreads), 0, st, S, E, k, C, cb, nchunk, R);
}

cudaError_t launch_ep_scan(int S, int E, int k, const Routing& R, double* stats, cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  return launch_pdl(ep_scan_kernel, dim3(E + 1), dim3(kThreads), 0, st, S, E, k, nchunk, R, stats);
}

cudaError_t launch_scan(int S, int E, int k, int C, int64_t Cbuf, const Routing& R, cudaStream_t st,
                        bool with_losses) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int cb = Cbuf < 0x7fffffff ? (int)Cbuf : 0x7fffffff;
  return launch_pdl(scan_kernel, dim3(E + (with_losses ? 1 : 0)), dim3(kThreads), 0, st, S, E, k, C, cb,
                    nchunk, R);
}

}  // namespace moe
