// route_token.cuh -- per-token softmax, top-k and normalised gates, one warp per token.
//
// G(x) = Softmax(x . W_g) ("GShard: Scaling Giant Neural Networks with Conditional
// Computation", "Mixture-of-Experts Implementation"); the k largest logits are
// chosen, ties to the lower expert index, and their weights are the
// "softmax-normalised top-2 weights" of "GShard: Scaling Giant Models with
// Conditional Computation and Automatic Sharding" (paper-note summary):
// g_r = p[e_r] / sum_r' p[e_r'] = exp(l_r - l_0) / sum_r' exp(l_r' - l_0).
//
// Layout: lane l of the warp holds the logits of experts l, l+32, ..., l+32*(RE-1)
// (bias already added, -inf beyond E).  Used by both router kernels.
#pragma once

#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

// Routes NT tokens at once (their work interleaves, hiding shuffle and exp
// latency).  For each token n: writes logits (if asked), eidx / gate rows, the
// chosen experts into sel_row[n][0..k) (shared memory), and accumulates this
// lane's probabilities into psum and lse^2 into lse2 (identical on every lane).
template <int RE, int NT>
__device__ __forceinline__ void route_tokens(const float (&v)[NT][RE], const int64_t (&tok)[NT], int E,
                                             int k, bool write_logits, const Routing& R,
                                             float (&psum)[RE], float& lse2,
                                             int32_t* const (&sel_row)[NT]) {
  const int lane = threadIdx.x & 31;
  if (write_logits) {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < RE; ++i)
        if (lane + 32 * i < E) R.logits[tok[n] * E + lane + 32 * i] = v[n][i];
  }
  float mx[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    mx[n] = v[n][0];
#pragma unroll
    for (int i = 1; i < RE; ++i) mx[n] = fmaxf(mx[n], v[n][i]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int n = 0; n < NT; ++n) mx[n] = fmaxf(mx[n], __shfl_xor_sync(0xffffffffu, mx[n], o));
  float ex[NT][RE], s[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    s[n] = 0.f;
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      ex[n][i] = (lane + 32 * i < E) ? expf(v[n][i] - mx[n]) : 0.f;
      s[n] += ex[n][i];
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1)
#pragma unroll
    for (int n = 0; n < NT; ++n) s[n] += __shfl_xor_sync(0xffffffffu, s[n], o);
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float inv = 1.f / s[n];
#pragma unroll
    for (int i = 0; i < RE; ++i) psum[i] += ex[n][i] * inv;
    const float lse = mx[n] + logf(s[n]);
    lse2 += lse * lse;
  }

  // top-k on the logits by warp argmax, ties -> lower expert index
  unsigned taken[NT];
  int er[NT][kMaxK];
  float lr[NT][kMaxK];
#pragma unroll
  for (int n = 0; n < NT; ++n) taken[n] = 0;
#pragma unroll
  for (int r = 0; r < kMaxK; ++r) {
    if (r < k) {
      float bv[NT];
      int bj[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        bv[n] = -INFINITY;
        bj[n] = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < RE; ++i) {
          const int j = lane + 32 * i;
          if (j < E && !((taken[n] >> i) & 1u) && (v[n][i] > bv[n] || bj[n] == 0x7fffffff)) {
            bv[n] = v[n][i];
            bj[n] = j;
          }
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv[n], o);
          const int oj = __shfl_xor_sync(0xffffffffu, bj[n], o);
          if (ov > bv[n] || (ov == bv[n] && oj < bj[n])) {
            bv[n] = ov;
            bj[n] = oj;
          }
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (bj[n] >= E) {                  // only for non-finite logits
          if (lane == 0) atomicOr(R.err, DEVERR_BOUNDS);
          bj[n] = 0;
        }
        if ((bj[n] & 31) == lane) taken[n] |= 1u << (bj[n] >> 5);
        er[n][r] = bj[n];
        lr[n][r] = bv[n];
      }
    } else {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        er[n][r] = 0;
        lr[n][r] = 0.f;
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    float gs = 0.f, gr[kMaxK];
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
      gr[r] = (r < k) ? expf(lr[n][r] - lr[n][0]) : 0.f;
      gs += gr[r];
    }
    const float ginv = 1.f / gs;
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
      if (r < k && lane == r) {
        R.eidx[tok[n] * k + r] = er[n][r];
        R.gate[tok[n] * k + r] = gr[r] * ginv;
        sel_row[n][r] = er[n][r];
      }
    }
  }
}

// Routes one token (see route_tokens).
template <int RE>
__device__ __forceinline__ void route_token(const float (&v)[RE], int64_t tok, int E, int k,
                                            bool write_logits, const Routing& R, float (&psum)[RE],
                                            float& lse2, int32_t* sel_row) {
  const float(&vv)[1][RE] = *reinterpret_cast<const float(*)[1][RE]>(&v);
  const int64_t tt[1] = {tok};
  int32_t* const rows[1] = {sel_row};
  route_tokens<RE, 1>(vv, tt, E, k, write_logits, R, psum, lse2, rows);
}

}  // namespace moe
