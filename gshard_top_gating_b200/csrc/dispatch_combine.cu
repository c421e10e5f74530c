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
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "losses.cuh"

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

// Rerouting: the final slot and serving expert of every choice -- the first pass's
// slot, or for a dropped choice its offer's slot (off2 + lrank2) when that is below C
// -- then the row copies, as dispatch_kernel.  x == nullptr: tables only.
template <typename T, int KM>
__global__ void __launch_bounds__(kThreads, 4) dispatch_rerouted_kernel(const T* __restrict__ x, int S,
                                                                        int M, int E, int k, int C,
                                                                        int64_t Cbuf, int nchunk, Routing R,
                                                                        T* __restrict__ xbuf) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = (int)((int64_t)M * sizeof(T) / 16);
  pdl_trigger();
  pdl_wait();                                  // first-pass slots, offers and their offsets complete
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
    int d = 0, s = -1;
    if (lane < k) {
      const int64_t i = (int64_t)t * k + lane;
      d = R.eidx[i];
      s = R.slot[i];
      if (s < 0) {
        const int a = R.alt[i];
        if (a >= 0 && a < E) {
          const int q = R.off2[((int64_t)lane * nchunk + t / kChunk) * E + a] + R.lrank2[i];
          if (q < C && q < Cbuf) {
            s = q;
            d = a;
          }
        }
      }
      R.slot[i] = s;
      R.dest[i] = d;
    }
    if (x == nullptr) continue;
    uint4* dst[KM];
    bool any = false;
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      const int dr = __shfl_sync(0xffffffffu, d, r);
      const int sr = __shfl_sync(0xffffffffu, s, r);
      dst[r] = (r < k && sr >= 0) ? reinterpret_cast<uint4*>(xbuf + ((int64_t)dr * Cbuf + sr) * M) : nullptr;
      any |= dst[r] != nullptr;
    }
    if (!any) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)t * M);
    for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
      uint4 val[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (v0 + 32 * u < nv) val[u] = ld_nc_v4(src + v0 + 32 * u);
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

// Top-1 routing with the combine fused into the second expert GEMM: the dispatch also
// records, for every kept slot, the token that took it and its gate (the GEMM's
// epilogue stores g * row straight into y[token]), and writes y = 0 for a token whose
// choice was dropped (no expert row reaches it).
__global__ void __launch_bounds__(kThreads, 4) dispatch_fused_kernel(const __nv_bfloat16* __restrict__ x,
                                                                     int S, int M, int E, int C,
                                                                     int64_t Cbuf, int nchunk, Routing R,
                                                                     __nv_bfloat16* __restrict__ xbuf,
                                                                     int32_t* __restrict__ tok,
                                                                     float* __restrict__ gsc,
                                                                     __nv_bfloat16* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = M * 2 / 16;
  pdl_trigger();
  pdl_wait();                                  // routing tables and offsets complete
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
    int e = 0, s = -1;
    if (lane == 0) {
      e = R.eidx[t];
      int pos = 0x7fffffff;
      if (e >= 0 && e < E) {
        pos = R.off[(int64_t)(t / kChunk) * E + e] + R.lrank[t];
      } else {
        atomicOr(R.err, DEVERR_BOUNDS);
      }
      s = (pos < C && pos < Cbuf) ? pos : -1;
      R.slot[t] = s;
      if (s >= 0) {
        tok[(int64_t)e * Cbuf + s] = t;
        gsc[(int64_t)e * Cbuf + s] = R.gate[t];
      }
    }
    e = __shfl_sync(0xffffffffu, e, 0);
    s = __shfl_sync(0xffffffffu, s, 0);
    uint4* dst = s >= 0 ? reinterpret_cast<uint4*>(xbuf + ((int64_t)e * Cbuf + s) * M)
                        : reinterpret_cast<uint4*>(y + (int64_t)t * M);
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)t * M);
    for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
      uint4 val[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (v0 + 32 * u < nv) val[u] = s >= 0 ? ld_nc_v4(src + v0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (v0 + 32 * u < nv) dst[v0 + 32 * u] = val[u];
    }
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
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

// loss_blocks = 1: the grid's first block computes the auxiliary losses instead of
// combining tokens (the router's partials are long complete by then); being first,
// it is resident from the start and runs beside the token blocks.
template <typename T, int KM>
__global__ void __launch_bounds__(kThreads, KM >= 8 ? 3 : 4) combine_kernel(const T* __restrict__ ybuf, int S, int M,
                                                              int k, int64_t Cbuf, Routing R,
                                                              T* __restrict__ y, int loss_blocks, int E,
                                                              int nchunk, const EpPeer* __restrict__ peers,
                                                              int El) {
  static_assert(kThreads == kLossThreads, "the loss block runs with the combine's block size");
  const int lane = threadIdx.x & 31;
  const int warps = ((gridDim.x - loss_blocks) * kThreads) >> 5;
  const int blk = blockIdx.x - loss_blocks;    // this block's index among the token blocks
  const int nv = (int)((int64_t)M * sizeof(T) / 16);
  constexpr int U = KM >= 4 ? 1 : 2;          // 16-byte vectors per lane per step
  pdl_trigger();
  pdl_wait();                                  // expert outputs complete
  if (blk < 0) {
    aux_loss_block(S, E, nchunk, R);
    return;
  }
  for (int t = (blk * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
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
      const T* row = nullptr;
      if (r < k && sr >= 0) {
        if (peers) {                           // the owner's receive buffer (expert parallelism)
          const EpPeer p = peers[er / El];
          row = static_cast<const T*>(p.base) + ((int64_t)sr + p.delta) * M;
        } else {
          row = ybuf + ((int64_t)er * Cbuf + sr) * M;
        }
      }
      srcs[r] = reinterpret_cast<const uint4*>(row);
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

// Expert parallelism, sending side: the global rank-major slot of each of the rank's
// choices is base[r][e] (all earlier ranks' and earlier choice ranks' demand of e, from
// the exchanged counts) plus the rank-local position off[r][c][e] + lrank.  Kept rows go
// to the send buffer.  A run (this rank's kept choices of rank r at expert e) is a prefix
// of its choices; its first a0[r][e] rows travel in phase 0 from soff0[r][e], the rest in
// phase 1 from soff1[r][e] (soff = [soff0 | soff1 | a0], each [k][E]; with one phase,
// a0 covers the whole run).
template <typename T, int KM>
__global__ void __launch_bounds__(kThreads, 4) ep_dispatch_kernel(const T* __restrict__ x, int S, int M,
                                                                  int E, int k, int C, int nchunk,
                                                                  Routing R, const int32_t* __restrict__ base,
                                                                  const int32_t* __restrict__ soff,
                                                                  int32_t* __restrict__ spos,
                                                                  T* __restrict__ sendbuf,
                                                                  const EpPeer* __restrict__ peers, int El) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = (int)((int64_t)M * sizeof(T) / 16);
  pdl_trigger();
  pdl_wait();                                  // local offsets and the exchanged plan complete
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < S; t += warps) {
    int sp = -1, ev = 0;
    if (lane < k) {
      const int e = R.eidx[(int64_t)t * k + lane];
      ev = e;
      int s = -1;
      if (e >= 0 && e < E) {
        const int local = R.off[((int64_t)lane * nchunk + t / kChunk) * E + e] + R.lrank[(int64_t)t * k + lane];
        const int i = lane * E + e;
        const int g = base[i] + local;
        if (g < C) {
          s = g;
          const int a = soff[2 * k * E + i];
          sp = local < a ? soff[i] + local : soff[k * E + i] + (local - a);
        }
      } else {
        atomicOr(R.err, DEVERR_BOUNDS);
      }
      R.slot[(int64_t)t * k + lane] = s;
      spos[(int64_t)t * k + lane] = sp;
    }
    const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)t * M);
    uint4* dst[KM];
    bool any = false;
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      const int pr = __shfl_sync(0xffffffffu, sp, r);
      const int er = __shfl_sync(0xffffffffu, ev, r);
      T* row = nullptr;
      if (r < k && pr >= 0) {
        if (peers) {                           // straight into the owner's receive buffer
          const EpPeer p = peers[er / El];
          row = static_cast<T*>(p.base) + ((int64_t)pr + p.delta) * M;
        } else {
          row = sendbuf + (int64_t)pr * M;
        }
      }
      dst[r] = reinterpret_cast<uint4*>(row);
      any |= dst[r] != nullptr;
    }
    if (!any) continue;                        // every choice dropped: the row is not sent
    for (int v0 = lane; v0 < nv; v0 += 32 * kUnroll) {
      uint4 val[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (v0 + 32 * u < nv) val[u] = ld_nc_v4(src + v0 + 32 * u);
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

// Expert parallelism, receiving side: one warp per received row.  The row's segment is
// the last q with seg_start[q] <= j (empty segments share their start with the next
// one, so the last such q is the non-empty segment holding j).
__global__ void __launch_bounds__(kThreads) ep_unpack_kernel(const uint4* __restrict__ recv, int nrows,
                                                             int nv, const int32_t* __restrict__ seg_start,
                                                             const int32_t* __restrict__ seg_dst, int nseg,
                                                             int32_t* __restrict__ rowmap,
                                                             uint4* __restrict__ xbuf, unsigned* err,
                                                             int64_t xrows) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  pdl_trigger();
  pdl_wait();
  for (int j = (blockIdx.x * kThreads + threadIdx.x) >> 5; j < nrows; j += warps) {
    int lo = 0, hi = nseg;                     // first q with seg_start[q] > j
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (seg_start[mid] <= j) lo = mid + 1;
      else hi = mid;
    }
    const int q = lo - 1;
    const int64_t row = q >= 0 ? (int64_t)seg_dst[q] + (j - seg_start[q]) : -1;
    if (row < 0 || row >= xrows) {             // a plan inconsistent with the rows received
      if (lane == 0) {
        atomicOr(err, DEVERR_BOUNDS);
        rowmap[j] = -1;
      }
      continue;
    }
    if (lane == 0) rowmap[j] = (int32_t)row;
    const uint4* s = recv + (int64_t)j * nv;
    uint4* d = xbuf + row * nv;
    for (int v = lane; v < nv; v += 32) d[v] = ld_nc_v4(s + v);
  }
}

__global__ void __launch_bounds__(kThreads) ep_repack_kernel(const uint4* __restrict__ ybuf, int nrows, int nv,
                                                             const int32_t* __restrict__ rowmap,
                                                             uint4* __restrict__ recv) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  pdl_trigger();
  pdl_wait();                                  // expert outputs complete
  for (int j = (blockIdx.x * kThreads + threadIdx.x) >> 5; j < nrows; j += warps) {
    const int row = rowmap[j];
    if (row < 0) continue;
    const uint4* s = ybuf + (int64_t)row * nv;
    uint4* d = recv + (int64_t)j * nv;
    for (int v = lane; v < nv; v += 32) d[v] = ld_nc_v4(s + v);
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
               int grid, cudaStream_t st, int loss_blocks, int E, const EpPeer* peers, int El) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  launch_pdl(combine_kernel<T, KM>, dim3(grid + loss_blocks), dim3(kThreads), 0, st, (const T*)ybuf, S, M,
             k, Cbuf, R, (T*)y, loss_blocks, E, nchunk, peers, El);
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
               int grid, cudaStream_t st, int loss_blocks, int E, const EpPeer* peers, int El) {
  if (k <= 1) combine_t<T, 1>(ybuf, S, M, k, Cbuf, R, y, grid, st, loss_blocks, E, peers, El);
  else if (k <= 2) combine_t<T, 2>(ybuf, S, M, k, Cbuf, R, y, grid, st, loss_blocks, E, peers, El);
  else if (k <= 4) combine_t<T, 4>(ybuf, S, M, k, Cbuf, R, y, grid, st, loss_blocks, E, peers, El);
  else combine_t<T, 8>(ybuf, S, M, k, Cbuf, R, y, grid, st, loss_blocks, E, peers, El);
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

cudaError_t launch_dispatch_fused(const void* x, int S, int M, int E, int C, int64_t Cbuf,
                                  const Routing& R, void* xbuf, int32_t* tok, float* gsc, void* y,
                                  cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  return launch_pdl(dispatch_fused_kernel, dim3(grid_for(S)), dim3(kThreads), 0, st,
                    (const __nv_bfloat16*)x, S, M, E, C, Cbuf, nchunk, R, (__nv_bfloat16*)xbuf, tok, gsc,
                    (__nv_bfloat16*)y);
}

cudaError_t launch_dispatch_rerouted(const void* x, bool bf16, int S, int M, int E, int k, int C,
                                     int64_t Cbuf, const Routing& R, void* xbuf, cudaStream_t st) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int grid = grid_for(S);
  auto go = [&](auto tag, auto km) {
    using T = decltype(tag);
    constexpr int KM = decltype(km)::value;
    return launch_pdl(dispatch_rerouted_kernel<T, KM>, dim3(grid), dim3(kThreads), 0, st, (const T*)x, S,
                      M, E, k, C, Cbuf, nchunk, R, (T*)xbuf);
  };
  using I1 = std::integral_constant<int, 1>;
  using I2 = std::integral_constant<int, 2>;
  using I4 = std::integral_constant<int, 4>;
  using I8 = std::integral_constant<int, 8>;
  if (bf16) {
    const __nv_bfloat16 b{};
    return k <= 1 ? go(b, I1{}) : k <= 2 ? go(b, I2{}) : k <= 4 ? go(b, I4{}) : go(b, I8{});
  }
  return k <= 1 ? go(0.f, I1{}) : k <= 2 ? go(0.f, I2{}) : k <= 4 ? go(0.f, I4{}) : go(0.f, I8{});
}

cudaError_t launch_ep_dispatch(const void* x, bool bf16, int S, int M, int E, int k, int C,
                               const Routing& R, const int32_t* base, const int32_t* soff,
                               int32_t* spos, void* sendbuf, cudaStream_t st, const EpPeer* peers,
                               int El) {
  const int nchunk = (S + kChunk - 1) / kChunk;
  const int grid = grid_for(S);
  auto go = [&](auto tag, auto km) {
    using T = decltype(tag);
    constexpr int KM = decltype(km)::value;
    return launch_pdl(ep_dispatch_kernel<T, KM>, dim3(grid), dim3(kThreads), 0, st, (const T*)x, S, M, E,
                      k, C, nchunk, R, base, soff, spos, (T*)sendbuf, peers, El);
  };
  using I1 = std::integral_constant<int, 1>;
  using I2 = std::integral_constant<int, 2>;
  using I4 = std::integral_constant<int, 4>;
  using I8 = std::integral_constant<int, 8>;
  if (bf16) {
    const __nv_bfloat16 b{};
    return k <= 1 ? go(b, I1{}) : k <= 2 ? go(b, I2{}) : k <= 4 ? go(b, I4{}) : go(b, I8{});
  }
  return k <= 1 ? go(0.f, I1{}) : k <= 2 ? go(0.f, I2{}) : k <= 4 ? go(0.f, I4{}) : go(0.f, I8{});
}

cudaError_t launch_ep_unpack(const void* recvbuf, bool bf16, int nrows, int M, const int32_t* seg_start,
                             const int32_t* seg_dst, int nseg, int32_t* rowmap, void* xbuf,
                             unsigned* err, int64_t xrows, cudaStream_t st) {
  if (nrows <= 0) return cudaSuccess;
  const int nv = (int)((int64_t)M * (bf16 ? 2 : 4) / 16);
  return launch_pdl(ep_unpack_kernel, dim3(grid_for(nrows)), dim3(kThreads), 0, st,
                    (const uint4*)recvbuf, nrows, nv, seg_start, seg_dst, nseg, rowmap, (uint4*)xbuf, err,
                    xrows);
}

cudaError_t launch_ep_repack(const void* ybuf, bool bf16, int nrows, int M, const int32_t* rowmap,
                             void* recvbuf, cudaStream_t st) {
  if (nrows <= 0) return cudaSuccess;
  const int nv = (int)((int64_t)M * (bf16 ? 2 : 4) / 16);
  return launch_pdl(ep_repack_kernel, dim3(grid_for(nrows)), dim3(kThreads), 0, st, (const uint4*)ybuf,
                    nrows, nv, rowmap, (uint4*)recvbuf);
}

cudaError_t launch_combine(const void* ybuf, bool bf16, int S, int M, int k, int64_t Cbuf,
                           const Routing& R, void* y, cudaStream_t st, bool with_losses, int E,
                           const EpPeer* peers, int El) {
  // with the loss block, one token block fewer: grid_for fills the SMs' resident slots
  // exactly, and a block past them would run alone after the others
  const int lb = with_losses ? 1 : 0;
  const int grid = grid_for(S) > 1 ? grid_for(S) - lb : grid_for(S);
  if (bf16)
    combine_k<__nv_bfloat16>(k, ybuf, S, M, Cbuf, R, y, grid, st, lb, E, peers, El);
  else
    combine_k<float>(k, ybuf, S, M, Cbuf, R, y, grid, st, lb, E, peers, El);
  return cudaGetLastError();
}

}  // namespace moe
