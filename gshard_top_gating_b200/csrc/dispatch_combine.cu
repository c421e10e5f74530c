// dispatch_combine.cu -- token -> expert-buffer dispatch and gate-weighted combine.
//
// On several devices the tokens travel to their experts by an all-to-all and
// come back by a second one ("GShard (Expert Parallelism)", "In plain words").
// On one GPU both become permutations in HBM:
//   dispatch: xbuf[e_r, slot_r] = x[t] for every kept choice (t, r)
//   combine : y[t] = sum_{r kept} g_r * ybuf[e_r, slot_r]   (r ascending, fp32)
// A dropped choice contributes nothing and the kept gates are not renormalised
// ("GShard: Scaling Giant Models ...", paper-note summary: over-capacity tokens
// are dropped).  Both kernels are token-centric (one warp per token), read and
// write whole rows in 16-byte vectors, and need no atomics, so the result does
// not depend on scheduling.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// One warp per token.  The first slice of the token's row is loaded before the
// slot lookups (which depend on two chained table reads), so the row's memory
// latency overlaps them.
template <typename T, int KM>
__global__ void __launch_bounds__(kThreads, 4) dispatch_kernel(const T* __restrict__ x, int S, int M,
                                                               int E, int k, int C, int64_t Cbuf,
                                                               int nchunk, Routing R,
                                                               T* __restrict__ xbuf) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = (int)((int64_t)M * sizeof(T) / 16);
  pdl_trigger();
  bool waited = false;
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
    const uint4* src = x ? reinterpret_cast<const uint4*>(x + (int64_t)t * M) : nullptr;
    uint4 first[kUnroll];
    if (src) {                                 // x is an input: no need to wait for it
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (lane + 32 * u < nv) first[u] = ld_nc_v4(src + lane + 32 * u);
    }
    if (!waited) {
      pdl_wait();                              // routing tables and offsets complete
      waited = true;
    }
    int e = 0, s = -1;
    if (lane < k) {
      e = R.eidx[(int64_t)t * k + lane];
      const int c = t / kChunk;
      int pos = 0x7fffffff;
      if (e >= 0 && e < E) {
        pos = R.off[((int64_t)lane * nchunk + c) * E + e] + R.lrank[(int64_t)t * k + lane];
      } else {
        atomicOr(R.err, DEVERR_BOUNDS);
      }
      s = (pos < C && pos < Cbuf) ? pos : -1;
      R.slot[(int64_t)t * k + lane] = s;
    }
    if (src == nullptr) continue;              // slot-only pass (routing without data)
    uint4* dst[KM];
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      const int er = __shfl_sync(0xffffffffu, e, r);
      const int sr = __shfl_sync(0xffffffffu, s, r);
      dst[r] = (r < k && sr >= 0) ? reinterpret_cast<uint4*>(xbuf + ((int64_t)er * Cbuf + sr) * M)
                                  : nullptr;
    }
    for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
      uint4 val[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        if (v0 == lane) val[u] = first[u];
        else if (v0 + 32 * u < nv) val[u] = ld_nc_v4(src + v0 + 32 * u);
      }
#pragma unroll
      for (int r = 0; r < KM; ++r) {
        if (dst[r] == nullptr) continue;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u)
          if (v0 + 32 * u < nv) dst[r][v0 + 32 * u] = val[u];
      }
    }
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load_fma(float (&a)[8], const uint4& u, float g) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      a[2 * q] = fmaf(g, bf16lo(w[q]), a[2 * q]);
      a[2 * q + 1] = fmaf(g, bf16hi(w[q]), a[2 * q + 1]);
    }
  }
  __device__ static uint4 pack(const float (&a)[8]) {
    return make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                      pack_bf16x2(a[6], a[7]));
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load_fma(float (&a)[8], const uint4& u, float g) {
    a[0] = fmaf(g, __uint_as_float(u.x), a[0]);
    a[1] = fmaf(g, __uint_as_float(u.y), a[1]);
    a[2] = fmaf(g, __uint_as_float(u.z), a[2]);
    a[3] = fmaf(g, __uint_as_float(u.w), a[3]);
  }
  __device__ static uint4 pack(const float (&a)[8]) {
    return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                      __float_as_uint(a[3]));
  }
};

template <typename T, int KM>
__global__ void __launch_bounds__(kThreads, KM >= 8 ? 3 : 4) combine_kernel(const T* __restrict__ ybuf, int S, int M,
                                                              int k, int64_t Cbuf, Routing R,
                                                              T* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = (int)((int64_t)M * sizeof(T) / 16);
  constexpr int U = KM >= 4 ? 1 : 2;          // 16-byte vectors per lane per step
  pdl_trigger();
  pdl_wait();                                  // expert outputs complete
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
    int e = 0, s = -1;
    float g = 0.f;
    if (lane < k) {
      e = R.eidx[(int64_t)t * k + lane];
      s = R.slot[(int64_t)t * k + lane];
      g = R.gate[(int64_t)t * k + lane];
    }
    const uint4* srcs[KM];
    float gr[KM];
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      const int er = __shfl_sync(0xffffffffu, e, r);
      const int sr = __shfl_sync(0xffffffffu, s, r);
      gr[r] = __shfl_sync(0xffffffffu, g, r);
      srcs[r] = (r < k && sr >= 0)
                    ? reinterpret_cast<const uint4*>(ybuf + ((int64_t)er * Cbuf + sr) * M)
                    : nullptr;
    }
    uint4* dst = reinterpret_cast<uint4*>(y + (int64_t)t * M);
    for (int v0 = lane; v0 < nv; v0 += 32 * U) {
      float acc[U][8];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[u][q] = 0.f;
      // all k rows' loads first, then the fixed-order fp32 sum
      uint4 val[KM][U];
#pragma unroll
      for (int r = 0; r < KM; ++r)
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (srcs[r] != nullptr && v0 + 32 * u < nv) val[r][u] = ld_nc_v4(srcs[r] + v0 + 32 * u);
#pragma unroll
      for (int r = 0; r < KM; ++r)
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (srcs[r] != nullptr && v0 + 32 * u < nv) Vec<T>::load_fma(acc[u], val[r][u], gr[r]);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (v0 + 32 * u < nv) dst[v0 + 32 * u] = Vec<T>::pack(acc[u]);
    }
  }
}

int grid_for(int S) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int want = (S + (kThreads / 32) - 1) / (kThreads / 32);   // one warp per token
  return want < sms * 4 ? want : sms * 4;                          // 4 CTAs per SM resident
}

template <typename T, int KM>
void dispatch_t(const void* x, int S, int M, int E, int k, int C, int64_t Cbuf, int nchunk,
                const Routing& R, void* xbuf, int grid, cudaStream_t st) {
  launch_pdl(dispatch_kernel<T, KM>, dim3(grid), dim3(kThreads), 0, st, (const T*)x, S, M, E, k, C,
             Cbuf, nchunk, R, (T*)xbuf);
}

template <typename T, int KM>
void combine_t(const void* ybuf, int S, int M, int k, int64_t Cbuf, const Routing& R, void* y,
               int grid, cudaStream_t st) {
  launch_pdl(combine_kernel<T, KM>, dim3(grid), dim3(kThreads), 0, st, (const T*)ybuf, S, M, k, Cbuf,
             R, (T*)y);
}

template <typename T>
void dispatch_k(int k, const void* x, int S, int M, int E, int C, int64_t Cbuf, int nchunk,
                const Routing& R, void* xbuf, int grid, cudaStream_t st) {
  if (k <= 1) dispatch_t<T, 1>(x, S, M, E, k, C, Cbuf, nchunk, R, xbuf, grid, st);
  else if (k <= 2) dispatch_t<T, 2>(x, S, M, E, k, C, Cbuf, nchunk, R, xbuf, grid, st);
  else if (k <= 4) dispatch_t<T, 4>(x, S, M, E, k, C, Cbuf, nchunk, R, xbuf, grid, st);
  else dispatch_t<T, 8>(x, S, M, E, k, C, Cbuf, nchunk, R, xbuf, grid, st);
}

template <typename T>
void combine_k(int k, const void* ybuf, int S, int M, int64_t Cbuf, const Routing& R, void* y,
               int grid, cudaStream_t st) {
  if (k <= 1) combine_t<T, 1>(ybuf, S, M, k, Cbuf, R, y, grid, st);
  else if (k <= 2) combine_t<T, 2>(ybuf, S, M, k, Cbuf, R, y, grid, st);
  else if (k <= 4) combine_t<T, 4>(ybuf, S, M, k, Cbuf, R, y, grid, st);
  else combine_t<T, 8>(ybuf, S, M, k, Cbuf, R, y, grid, st);
}

}  // namespace

cudaError_t launch_dispatch(const void* x, bool bf16, int S, int M, int E, int k, int C,
                            int64_t Cbuf, const Routing& R, void* xbuf, cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int grid = grid_for(S);
  if (bf16)
    dispatch_k<__nv_bfloat16>(k, x, S, M, E, C, Cbuf, nchunk, R, xbuf, grid, st);
  else
    dispatch_k<float>(k, x, S, M, E, C, Cbuf, nchunk, R, xbuf, grid, st);
  return cudaGetLastError();
}

cudaError_t launch_combine(const void* ybuf, bool bf16, int S, int M, int k, int64_t Cbuf,
                           const Routing& R, void* y, cudaStream_t st) {
  const int grid = grid_for(S);
  if (bf16)
    combine_k<__nv_bfloat16>(k, ybuf, S, M, Cbuf, R, y, grid, st);
  else
    combine_k<float>(k, ybuf, S, M, Cbuf, R, y, grid, st);
  return cudaGetLastError();
}

}  // namespace moe
