// losses.cuh -- the auxiliary losses of one forward, from the router's per-chunk partials.
//
// "GShard: Scaling Giant Models with Conditional Computation and Automatic Sharding",
// paper-note summary: a load-balance loss N * sum_j f_j P_j plus a z-loss.  Here
// l_aux = E * sum_j f_j P_j with f_j = (first choices of j) / S and P_j = (sum_t p_tj) / S,
// and z = sum_t lse_t^2 / S.  Partials are summed in a fixed order in double, so the
// result is deterministic.  One block of 256 threads computes it; the layer runs it as
// an extra block of the combine kernel (off the dispatch's critical path) or, where no
// combine kernel runs, of the capacity scan.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kLossThreads = 256;

__device__ __forceinline__ double block_sum_f64(double v, double* sm) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sm[warp] = v;
  __syncthreads();
  double s = 0.0;
#pragma unroll
  for (int w = 0; w < kLossThreads / 32; ++w) s += sm[w];
  __syncthreads();
  return s;
}

// G threads share each expert column j, thread (j, g) summing chunks g, g+G, ...; the
// G partials are then added in order.  Also leaves f_j * S in R.first for the backward.
__device__ __forceinline__ void aux_loss_block(int S, int E, int nchunk, const Routing& R) {
  __shared__ double part_P[kLossThreads];
  __shared__ long long part_f[kLossThreads];
  __shared__ double dsum[kLossThreads / 32];
  const int tid = threadIdx.x;
  const int G = E >= kLossThreads ? 1 : kLossThreads / E;
  if (tid < E * G) {
    const int j = tid % E, g = tid / E;
    double P = 0.0;
    long long f = 0;
    for (int c = g; c < nchunk; c += G) {
      P += (double)R.psum[(int64_t)c * E + j];
      f += R.hist[(int64_t)c * E + j];          // rank-0 plane of hist: first choices
    }
    part_P[tid] = P;
    part_f[tid] = f;
  }
  __syncthreads();
  double term = 0.0;
  for (int j = tid; j < E; j += kLossThreads) {
    double P = 0.0;
    long long f = 0;
    for (int g = 0; g < G; ++g) {
      P += part_P[g * E + j];
      f += part_f[g * E + j];
    }
    term += (double)f * P;
    R.first[j] = (int32_t)f;                   // kept for the backward's d l_aux / d logits
  }
  const double fp = block_sum_f64(term, dsum);
  double zl = 0.0;
  for (int c = tid; c < nchunk; c += kLossThreads) zl += (double)R.lse2[c];
  const double zs = block_sum_f64(zl, dsum);
  if (tid == 0) {
    const double Sd = (double)S;
    R.losses[0] = (float)((double)E * fp / (Sd * Sd));
    R.losses[1] = (float)(zs / Sd);
  }
}

}  // namespace moe
