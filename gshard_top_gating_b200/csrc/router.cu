// router.cu -- gate GEMM + softmax + top-k + normalised gates + loss partials.
//
// Gating as "GShard: Scaling Giant Neural Networks with Conditional Computation",
// section "Mixture-of-Experts Implementation", defines it: G(x) = Softmax(x . W_g),
// then the top-k experts per token (k = 2 typical); the selected weights are
// "softmax-normalised top-2 weights" ("GShard: Scaling Giant Models with
// Conditional Computation and Automatic Sharding", paper-note summary).
//
// One CTA = 64 tokens x all E experts (E padded to EP = 32*RE).  Warp w owns
// tokens 8w..8w+7; lane l owns experts l, l+32, ..., so the GEMM accumulators
// are already in the layout the per-token epilogue needs (no smem round trip).
// Top-k runs on the fp32 logits by warp argmax with ties to the lower index.
// The epilogue also writes, per CTA ("chunk"), the rank-r histogram of chosen
// experts and each choice's rank among same-expert choices in the chunk, which
// the capacity scan turns into slots.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "route_token.cuh"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kKC = 32;   // K-chunk of the SIMT GEMM

struct __align__(16) EpiSmem {
  float red[8][kMaxExperts];      // per-warp probability sums
  float lse2[8];
  int32_t sel[kChunk][kMaxK];     // chosen experts of the chunk
  int32_t hist[kMaxK][kMaxExperts];
};

template <int RE>
struct __align__(16) GemmSmem {
  float xs[kChunk][kKC + 1];
  float ws[kKC][32 * RE];
};

// Route the 8 tokens of this warp whose logits are in acc[t][i] (expert lane+32i).
template <int RE>
__device__ __forceinline__ void route_warp(float (&acc)[8][RE], int tok0, int S, int E, int k,
                                           const float* __restrict__ bias, bool write_logits,
                                           const Routing& R, EpiSmem& es) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float psum[RE];
#pragma unroll
  for (int i = 0; i < RE; ++i) psum[i] = 0.f;
  float lse2 = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int tl = warp * 8 + t;
    const int tok = tok0 + tl;
    if (tok >= S) break;                       // warp-uniform
    float v[RE];
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      const int j = lane + 32 * i;
      v[i] = (j < E) ? acc[t][i] + (bias ? __ldg(bias + j) : 0.f) : -INFINITY;
    }
    route_token<RE>(v, tok, E, k, write_logits, R, psum, lse2, es.sel[tl]);
  }
#pragma unroll
  for (int i = 0; i < RE; ++i) es.red[warp][lane + 32 * i] = psum[i];
  if (lane == 0) es.lse2[warp] = lse2;
}

// Per-chunk loss partials, local ranks and rank-r histogram (after route_warp).
template <int RE>
__device__ __forceinline__ void chunk_tables(int tok0, int chunk, int nchunk, int S, int E, int k,
                                             const Routing& R, EpiSmem& es) {
  const int tid = threadIdx.x;
  __syncthreads();
  for (int j = tid; j < E; j += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += es.red[w][j];
    R.psum[(int64_t)chunk * E + j] = s;
  }
  if (tid == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += es.lse2[w];
    R.lse2[chunk] = s;
  }
  const int ntok = min(kChunk, S - tok0);
  for (int idx = tid; idx < ntok * k; idx += kThreads) {
    const int t = idx / k, r = idx - t * k;
    const int e = es.sel[t][r];
    int c = 0;
    for (int u = 0; u < t; ++u) c += (es.sel[u][r] == e);
    R.lrank[(int64_t)(tok0 + t) * k + r] = c;
    atomicAdd(&es.hist[r][e], 1);
  }
  __syncthreads();
  for (int idx = tid; idx < k * E; idx += kThreads) {
    const int r = idx / E, e = idx - r * E;
    R.hist[((int64_t)r * nchunk + chunk) * E + e] = es.hist[r][e];
  }
}

__device__ __forceinline__ void zero_hist(EpiSmem& es) {
  for (int idx = threadIdx.x; idx < kMaxK * kMaxExperts; idx += kThreads)
    (&es.hist[0][0])[idx] = 0;
}

template <typename TX, int RE>
__global__ void __launch_bounds__(kThreads) router_kernel(const TX* __restrict__ x,
                                                          const float* __restrict__ Wg,
                                                          const float* __restrict__ bias, int S,
                                                          int M, int E, int k, int nchunk,
                                                          Routing R) {
  constexpr int EP = 32 * RE;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EpiSmem& es = *reinterpret_cast<EpiSmem*>(smem_raw);
  GemmSmem<RE>& gs = *reinterpret_cast<GemmSmem<RE>*>(smem_raw + sizeof(EpiSmem));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x, tok0 = chunk * kChunk;
  zero_hist(es);

  float acc[8][RE];
#pragma unroll
  for (int t = 0; t < 8; ++t)
#pragma unroll
    for (int i = 0; i < RE; ++i) acc[t][i] = 0.f;

  const int lrow = tid >> 2, lcol = (tid & 3) * 8;   // x tile loader: 8 elements per thread
  const int xtok = tok0 + lrow;
#pragma unroll 1
  for (int k0 = 0; k0 < M; k0 += kKC) {
    __syncthreads();
    float xv[8];
    if (xtok < S) {
      const TX* src = x + (int64_t)xtok * M + k0 + lcol;
      if constexpr (sizeof(TX) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(src);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          xv[2 * q] = bf16lo(w4[q]);
          xv[2 * q + 1] = bf16hi(w4[q]);
        }
      } else {
        const float4 a = *reinterpret_cast<const float4*>(src);
        const float4 b = *reinterpret_cast<const float4*>(src + 4);
        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
        xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) xv[q] = 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) gs.xs[lrow][lcol + q] = xv[q];
    for (int idx = tid; idx < kKC * EP; idx += kThreads) {
      const int kk = idx / EP, j = idx - kk * EP;
      gs.ws[kk][j] = (j < E) ? __ldg(Wg + (int64_t)(k0 + kk) * E + j) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKC; ++kk) {
      float b[RE];
#pragma unroll
      for (int i = 0; i < RE; ++i) b[i] = gs.ws[kk][lane + 32 * i];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float a = gs.xs[warp * 8 + t][kk];
#pragma unroll
        for (int i = 0; i < RE; ++i) acc[t][i] = fmaf(a, b[i], acc[t][i]);
      }
    }
  }
  route_warp<RE>(acc, tok0, S, E, k, bias, true, R, es);
  chunk_tables<RE>(tok0, chunk, nchunk, S, E, k, R, es);
}

template <int RE>
__global__ void __launch_bounds__(kThreads) route_logits_kernel(const float* __restrict__ logits,
                                                                int S, int E, int k, int nchunk,
                                                                Routing R) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EpiSmem& es = *reinterpret_cast<EpiSmem*>(smem_raw);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int chunk = blockIdx.x, tok0 = chunk * kChunk;
  zero_hist(es);
  float acc[8][RE];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int tok = tok0 + warp * 8 + t;
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      const int j = lane + 32 * i;
      acc[t][i] = (tok < S && j < E) ? __ldg(logits + (int64_t)tok * E + j) : 0.f;
    }
  }
  __syncthreads();
  route_warp<RE>(acc, tok0, S, E, k, nullptr, true, R, es);
  chunk_tables<RE>(tok0, chunk, nchunk, S, E, k, R, es);
}

template <typename TX, int RE>
cudaError_t launch_router_t(const TX* x, const float* Wg, const float* bias, int S, int M, int E,
                            int k, const Routing& R, cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const size_t smem = sizeof(EpiSmem) + sizeof(GemmSmem<RE>);
  auto kern = router_kernel<TX, RE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<nchunk, kThreads, smem, st>>>(x, Wg, bias, S, M, E, k, nchunk, R);
  return cudaGetLastError();
}

template <int RE>
cudaError_t launch_route_logits_t(const float* logits, int S, int E, int k, const Routing& R,
                                  cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const size_t smem = sizeof(EpiSmem);
  auto kern = route_logits_kernel<RE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<nchunk, kThreads, smem, st>>>(logits, S, E, k, nchunk, R);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const void* x, bool x_bf16, const float* Wg, const float* bias, int S,
                          int M, int E, int k, const Routing& R, cudaStream_t st) {
  const int re = (E + 31) / 32;
#define MOE_ROUTER_CASE(N)                                                                       \
  case N:                                                                                        \
    return x_bf16 ? launch_router_t<__nv_bfloat16, N>((const __nv_bfloat16*)x, Wg, bias, S, M, E, \
                                                      k, R, st)                                   \
                  : launch_router_t<float, N>((const float*)x, Wg, bias, S, M, E, k, R, st);
  switch (re) {
    MOE_ROUTER_CASE(1)
    MOE_ROUTER_CASE(2)
    MOE_ROUTER_CASE(3)
    MOE_ROUTER_CASE(4)
    MOE_ROUTER_CASE(5)
    MOE_ROUTER_CASE(6)
    MOE_ROUTER_CASE(7)
    MOE_ROUTER_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef MOE_ROUTER_CASE
}

cudaError_t launch_route_logits(const float* logits, int S, int E, int k, const Routing& R,
                                cudaStream_t st) {
  switch ((E + 31) / 32) {
    case 1: return launch_route_logits_t<1>(logits, S, E, k, R, st);
    case 2: return launch_route_logits_t<2>(logits, S, E, k, R, st);
    case 3: return launch_route_logits_t<3>(logits, S, E, k, R, st);
    case 4: return launch_route_logits_t<4>(logits, S, E, k, R, st);
    case 5: return launch_route_logits_t<5>(logits, S, E, k, R, st);
    case 6: return launch_route_logits_t<6>(logits, S, E, k, R, st);
    case 7: return launch_route_logits_t<7>(logits, S, E, k, R, st);
    case 8: return launch_route_logits_t<8>(logits, S, E, k, R, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
