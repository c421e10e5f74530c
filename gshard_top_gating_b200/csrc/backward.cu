// backward.cu -- the layer's backward pass outside the tensor-core expert GEMMs.
//
// Gradients of L = <dy, y> + a_aux * l_aux + a_z * z ("GShard: Scaling Giant
// Neural Networks with Conditional Computation", "Training Methodology": the
// auxiliary loss joins the task loss with a small weight; only experts that
// received tokens get a gradient).  The routing -- choices, slots, drops -- and
// the first-choice fractions f_j are piecewise constant and carry no gradient.
//
//   gate_bwd   one warp per token: dY_e[slot_r] = g_r dy[t] and
//              dgate_r = <dy[t], y_e[slot_r]> for kept r (the combine's
//              backward), then the logit gradient
//                dl[t] = a_aux E/S p_t (f - <p_t, f>) + a_z 2/S lse_t p_t
//                        + sum_r onehot(e_r) g_r (dgate_r - sum_r' g_r' dgate_r')
//              (softmax recomputed from the saved logits; the gates g_r are a
//              softmax over the chosen logits, "softmax-normalised top-2 weights")
//   pad_zero   rows n_e .. ceil64(n_e) - 1 of the per-expert buffers the
//              weight-gradient GEMMs reduce over are cleared
//   dx         dx[t] = sum_{r kept} dX_e[slot_r] + dl[t] W_g^T
//   dwg        dW_g = x^T dl and dbias = sum_t dl: split-K partials in a fixed
//              order, then a fixed-order sum (no atomics: bitwise reproducible)
// bf16 activations: dl also leaves gate_bwd as a two-term bf16 split
// (hi = bf16(dl), lo = bf16(dl - hi)), the operand of two tensor-core GEMMs in
// ffn_tc.cu: dl_hi W_g,hi^T straight into dx (which dx_gather then adds the
// expert rows to), and x^T [dl_hi | dl_lo] as fp32 split-K partials that
// dwg_tc_reduce sums with the bias partials gate_bwd leaves per CTA.
// fp32 activations: dx, dW_g and the four expert GEMMs of the backward run on
// the tiled FFMA kernel below (tensor cores would lose fp32 accuracy).
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

template <typename T>
struct V16;
template <>
struct V16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      f[2 * q] = bf16lo(w[q]);
      f[2 * q + 1] = bf16hi(w[q]);
    }
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct V16<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- combine + gate backward
template <typename T, int KM, int RE, bool TC>
__global__ void __launch_bounds__(kThreads) gate_bwd_kernel(BwdArgs a, Routing R) {
  __shared__ float bred[TC ? kThreads / 32 : 1][TC ? 32 * RE : 1];
  float bacc[RE];
#pragma unroll
  for (int i = 0; i < RE; ++i) bacc[i] = 0.f;
  if (TC && blockIdx.x == 0 && threadIdx.x == 0) {
    a.cnt_rows[0] = a.S;                       // rows of the one-expert gate GEMMs
    for (int z = 0; z < a.nsplit; ++z) a.cnt_rows[1 + z] = max(0, min(a.kchunk, a.S - z * a.kchunk));
  }
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = (int)((int64_t)a.M * sizeof(T) / 16);
  const int E = a.E, k = a.k;
  const float invS = 1.f / (float)a.S;
  const T* dy = static_cast<const T*>(a.dy);
  const T* ybuf = static_cast<const T*>(a.ybuf);
  T* dybuf = static_cast<T*>(a.dybuf);
  // f_j for this lane's experts (the same for every token)
  float fj[RE];
#pragma unroll
  for (int i = 0; i < RE; ++i) {
    const int j = lane + 32 * i;
    fj[i] = j < E ? (float)R.first[j] * invS : 0.f;
  }
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < a.S; t += warps) {
    int e = 0, d = 0, s = -1;
    float g = 0.f;
    if (lane < k) {
      e = R.eidx[(int64_t)t * k + lane];
      d = a.dest ? a.dest[(int64_t)t * k + lane] : e;    // the buffer of its rows
      s = R.slot[(int64_t)t * k + lane];
      g = R.gate[(int64_t)t * k + lane];
    }
    const uint4* src[KM];
    uint4* dst[KM];
    float gr[KM], dot[KM];
    int er[KM];
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      er[r] = __shfl_sync(0xffffffffu, e, r);
      const int dr = __shfl_sync(0xffffffffu, d, r);
      const int sr = __shfl_sync(0xffffffffu, s, r);
      gr[r] = __shfl_sync(0xffffffffu, g, r);
      dot[r] = 0.f;
      const bool kept = r < k && sr >= 0;
      const int64_t row = ((int64_t)dr * a.Cbuf + sr) * a.M;
      src[r] = kept ? reinterpret_cast<const uint4*>(ybuf + row) : nullptr;
      dst[r] = kept ? reinterpret_cast<uint4*>(dybuf + row) : nullptr;
    }
    const uint4* dyr = reinterpret_cast<const uint4*>(dy + (int64_t)t * a.M);
    for (int v = lane; v < nv; v += 32) {
      float d[8];
      V16<T>::unpack(ld_nc_v4(dyr + v), d);
#pragma unroll
      for (int r = 0; r < KM; ++r) {
        if (src[r] == nullptr) continue;
        float yv[8], o[8];
        V16<T>::unpack(ld_nc_v4(src[r] + v), yv);
#pragma unroll
        for (int q = 0; q < V16<T>::N; ++q) {
          dot[r] = fmaf(d[q], yv[q], dot[r]);
          o[q] = gr[r] * d[q];
        }
        dst[r][v] = V16<T>::pack(o);
      }
    }
    float inner = 0.f;
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      dot[r] = warp_sum(dot[r]);
      if (r < k) inner = fmaf(gr[r], dot[r], inner);
    }
    if (lane < k) {
      float mine = 0.f;
#pragma unroll
      for (int r = 0; r < KM; ++r)
        if (r == lane) mine = dot[r];
      a.dgate[(int64_t)t * k + lane] = mine;
    }
    // softmax of the saved logits, then the logit gradient
    const float* lrow = R.logits + (int64_t)t * E;
    float v[RE], mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      const int j = lane + 32 * i;
      v[i] = j < E ? lrow[j] : -INFINITY;
      mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float ssum = 0.f;
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      v[i] = (lane + 32 * i < E) ? expf(v[i] - mx) : 0.f;
      ssum += v[i];
    }
    ssum = warp_sum(ssum);
    const float inv = 1.f / ssum;
    const float lse = mx + logf(ssum);
    float pf = 0.f;
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      v[i] *= inv;                            // p_tj
      pf = fmaf(v[i], fj[i], pf);
    }
    pf = warp_sum(pf);
    const float ca = a.a_aux * (float)E * invS, cz = a.a_z * 2.f * invS * lse;
    float dd[RE];
#pragma unroll
    for (int i = 0; i < RE; ++i) {
      const int j = lane + 32 * i;
      float d = ca * v[i] * (fj[i] - pf) + cz * v[i];
#pragma unroll
      for (int r = 0; r < KM; ++r)
        if (r < k && er[r] == j) d += gr[r] * (dot[r] - inner);
      dd[i] = j < E ? d : 0.f;
    }
    if (TC) {
      __nv_bfloat16* hrow = static_cast<__nv_bfloat16*>(a.dlb) + (int64_t)t * 2 * a.EPb;
      const int nI = a.EPb / 32;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i >= nI) break;
        float d = 0.f;
#pragma unroll
        for (int q = 0; q < RE; ++q)
          if (q == i) d = dd[q];
        const __nv_bfloat16 hi = __float2bfloat16_rn(d);
        const __nv_bfloat16 lo = __float2bfloat16_rn(d - __bfloat162float(hi));
        hrow[lane + 32 * i] = hi;
        hrow[a.EPb + lane + 32 * i] = lo;
      }
#pragma unroll
      for (int i = 0; i < RE; ++i) bacc[i] += dd[i];
    } else {
      float* drow = a.dl + (int64_t)t * E;
#pragma unroll
      for (int i = 0; i < RE; ++i)
        if (lane + 32 * i < E) drow[lane + 32 * i] = dd[i];
    }
  }
  if (TC) {
    // bias partial of this CTA: its warps' sums added in warp order
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int i = 0; i < RE; ++i) bred[warp][lane + 32 * i] = bacc[i];
    __syncthreads();
    for (int j = threadIdx.x; j < E; j += kThreads) {
      float sum = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) sum += bred[w][j];
      a.bpart[(int64_t)blockIdx.x * E + j] = sum;
    }
  }
}

template <typename T, int KM>
void gate_bwd_re(const BwdArgs& a, const Routing& R, int grid, cudaStream_t st) {
  constexpr bool TC = sizeof(T) == 2;
  const int re = (a.E + 31) / 32;
  if (re <= 1) gate_bwd_kernel<T, KM, 1, TC><<<grid, kThreads, 0, st>>>(a, R);
  else if (re <= 2) gate_bwd_kernel<T, KM, 2, TC><<<grid, kThreads, 0, st>>>(a, R);
  else if (re <= 4) gate_bwd_kernel<T, KM, 4, TC><<<grid, kThreads, 0, st>>>(a, R);
  else gate_bwd_kernel<T, KM, 8, TC><<<grid, kThreads, 0, st>>>(a, R);
}

// dx[t] += sum over kept choices of dX_e[slot] (r ascending, fp32), in place on
// the bf16 dx that holds dl W_g^T; one warp per token, 16-byte vectors.
template <int KM>
__global__ void __launch_bounds__(kThreads) dx_gather_kernel(BwdArgs a, Routing R) {
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * kThreads) >> 5;
  const int nv = a.M / 8;
  const int k = a.k;
  const __nv_bfloat16* dxe = static_cast<const __nv_bfloat16*>(a.dybuf);
  for (int t = (blockIdx.x * kThreads + threadIdx.x) >> 5; t < a.S; t += warps) {
    int e = 0, s = -1;
    if (lane < k) {
      e = R.eidx[(int64_t)t * k + lane];
      s = R.slot[(int64_t)t * k + lane];
    }
    const uint4* src[KM];
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      const int er = __shfl_sync(0xffffffffu, e, r);
      const int sr = __shfl_sync(0xffffffffu, s, r);
      src[r] = (r < k && sr >= 0) ? reinterpret_cast<const uint4*>(dxe + ((int64_t)er * a.Cbuf + sr) * a.M)
                                  : nullptr;
    }
    uint4* row = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dx) + (int64_t)t * a.M);
    for (int v = lane; v < nv; v += 32) {
      uint4 val[KM];
#pragma unroll
      for (int r = 0; r < KM; ++r)
        if (src[r] != nullptr) val[r] = ld_nc_v4(src[r] + v);
      float acc[8];
      V16<__nv_bfloat16>::unpack(row[v], acc);
#pragma unroll
      for (int r = 0; r < KM; ++r) {
        if (src[r] == nullptr) continue;
        float f[8];
        V16<__nv_bfloat16>::unpack(val[r], f);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += f[q];
      }
      row[v] = V16<__nv_bfloat16>::pack(acc);
    }
  }
}

// dW_g[m, e] = sum over splits z of (P[z][m][e] + P[z][m][EPb + e]) (hi and lo
// halves of dl), dbias[e] = sum over gate_bwd's CTAs of their partials, both in order.
__global__ void __launch_bounds__(kThreads) dwg_tc_reduce_kernel(const float* __restrict__ part,
                                                                int nsplit, int M, int E, int EPb,
                                                                const float* __restrict__ bpart,
                                                                int nbpart, float* dWg, float* dbias) {
  const int64_t n = (int64_t)M * E;
  const int64_t zstride = (int64_t)M * 2 * EPb;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n + E;
       i += (int64_t)gridDim.x * kThreads) {
    if (i < n) {
      const int64_t m = i / E, e = i - m * E;
      const float* p = part + m * 2 * EPb + e;
      float s = 0.f;
#pragma unroll 8
      for (int z = 0; z < nsplit; ++z) s += __ldg(p + z * zstride) + __ldg(p + z * zstride + EPb);
      dWg[i] = s;
    } else if (dbias) {
      const int64_t e = i - n;
      float s = 0.f;
      for (int b = 0; b < nbpart; ++b) s += bpart[(int64_t)b * E + e];
      dbias[e] = s;
    }
  }
}

template <typename T>
void gate_bwd_k(const BwdArgs& a, const Routing& R, int grid, cudaStream_t st) {
  if (a.k <= 1) gate_bwd_re<T, 1>(a, R, grid, st);
  else if (a.k <= 2) gate_bwd_re<T, 2>(a, R, grid, st);
  else if (a.k <= 4) gate_bwd_re<T, 4>(a, R, grid, st);
  else gate_bwd_re<T, 8>(a, R, grid, st);
}

// ---------------------------------------------------------------- padding rows
struct PadBufs {
  char* p[4];
  int64_t row_bytes[4];
  int n;
};

__global__ void __launch_bounds__(kThreads) pad_zero_kernel(PadBufs b, int64_t Cbuf, Routing R) {
  const int e = blockIdx.y;
  const int n = min((int64_t)R.nexp[e], Cbuf);
  const int64_t end = min(Cbuf, (int64_t)((n + 63) / 64) * 64);
  for (int q = 0; q < b.n; ++q) {
    const int64_t vecs_per_row = b.row_bytes[q] / 16;
    const int64_t total = (end - n) * vecs_per_row;
    uint4* base = reinterpret_cast<uint4*>(b.p[q] + ((int64_t)e * Cbuf + n) * b.row_bytes[q]);
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * kThreads)
      base[i] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// ---------------------------------------------------------------- tiled FFMA GEMM
//
//   C(i, j) = sum_{kk in [k0, k1)} A(i, kk) B(kk, j),   i < rows, j < cols
//
// with A(i, kk) = A[z*a_z + i*a_i + kk*a_k] and B(kk, j) = B[z*b_z + kk*b_k + j*b_j]
// for the batch index z = blockIdx.z (an expert, or a split of K).  rows / K may
// come per expert from the kept counts.  64 x 64 tiles, 16-deep k-steps, 4 x 4
// outputs per thread.  Epilogues: plain store, ReLU-mask store, the dx sum, the
// split-K partial.
constexpr int TM = 64, TN = 64, TK = 16;
enum { kSgStore = 0, kSgMask = 1, kSgDx = 2, kSgPartial = 3 };

struct SimtGemm {
  const void* A;
  const void* B;
  int64_t a_z, a_i, a_k, b_z, b_k, b_j;
  int rows, cols, K;
  bool rows_from_n, k_from_n;   // rows / K = the expert's kept count
  bool skip_empty;              // k_from_n: an expert with no kept row leaves D untouched
  int ones_row;                 // A(i, kk) = 1 for i == ones_row (bias gradient), else -1
  int kchunk;                   // split-K: z covers [z*kchunk, (z+1)*kchunk)
  void* D;
  int64_t d_z, d_i;             // D[z*d_z + i*d_i + j]
  const float* mask;            // kSgMask: same indexing as D
  // kSgDx: dX_e rows gathered by the routing
  const void* dxe;
  int64_t Cbuf;
  int k;
  const int32_t* nexp;
};

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i) {
  return static_cast<float>(p[i]);
}
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <typename TA, typename TB, typename TD, int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtGemm g, Routing R) {
  const int z = blockIdx.z;
  int rows = g.rows, k0 = 0, k1 = g.K;
  if (g.rows_from_n) rows = min(g.nexp[z], (int)g.Cbuf);
  if (g.k_from_n) k1 = min(g.nexp[z], (int)g.Cbuf);
  if (g.kchunk > 0) {
    k0 = z * g.kchunk;
    k1 = min(g.K, k0 + g.kchunk);
  }
  const int i0 = blockIdx.y * TM, j0 = blockIdx.x * TN;
  if (i0 >= rows) return;
  if (g.skip_empty && g.k_from_n && k1 <= 0) return;
  const TA* A = static_cast<const TA*>(g.A) + (g.kchunk > 0 ? 0 : z * g.a_z);
  const TB* B = static_cast<const TB*>(g.B) + (g.kchunk > 0 ? 0 : z * g.b_z);
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const bool a_icont = g.a_i == 1, b_jcont = g.b_j == 1;
  float acc[4][4] = {};
  for (int kb = k0; kb < k1; kb += TK) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = tid + 256 * u;
      const int ii = a_icont ? (idx & 63) : (idx >> 4);
      const int kk = a_icont ? (idx >> 6) : (idx & 15);
      const int i = i0 + ii, kq = kb + kk;
      float v = 0.f;
      if (i < rows && kq < k1) v = (i == g.ones_row) ? 1.f : ldf(A, i * g.a_i + kq * g.a_k);
      As[kk][ii] = v;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int idx = tid + 256 * u;
      const int jj = b_jcont ? (idx & 63) : (idx >> 4);
      const int kk = b_jcont ? (idx >> 6) : (idx & 15);
      const int j = j0 + jj, kq = kb + kk;
      Bs[kk][jj] = (j < g.cols && kq < k1) ? ldf(B, kq * g.b_k + (int64_t)j * g.b_j) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) av[q] = As[kk][ty * 4 + q];
#pragma unroll
      for (int q = 0; q < 4; ++q) bv[q] = Bs[kk][tx * 4 + q];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[q][w] = fmaf(av[q], bv[w], acc[q][w]);
    }
    __syncthreads();
  }
  TD* D = static_cast<TD*>(g.D);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int i = i0 + ty * 4 + q;
    if (i >= rows) continue;
    if constexpr (EPI == kSgDx) {
      // dx[t] = acc + sum over kept choices of the expert-side gradient rows
      const TD* dxe = static_cast<const TD*>(g.dxe);
      float add[4] = {0.f, 0.f, 0.f, 0.f};
      for (int r = 0; r < g.k; ++r) {
        const int s = R.slot[(int64_t)i * g.k + r];
        if (s < 0) continue;
        const int e = R.eidx[(int64_t)i * g.k + r];
        const TD* row = dxe + ((int64_t)e * g.Cbuf + s) * g.cols;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int j = j0 + tx * 4 + w;
          if (j < g.cols) add[w] += ldf(row, j);
        }
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int j = j0 + tx * 4 + w;
        if (j < g.cols) D[(int64_t)i * g.d_i + j] = static_cast<TD>(add[w] + acc[q][w]);
      }
    } else {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int j = j0 + tx * 4 + w;
        if (j >= g.cols) continue;
        const int64_t o = (int64_t)z * g.d_z + (int64_t)i * g.d_i + j;
        float v = acc[q][w];
        if (EPI == kSgMask) v = g.mask[o] > 0.f ? v : 0.f;
        D[o] = static_cast<TD>(v);
      }
    }
  }
}

template <typename TA, typename TB, typename TD, int EPI>
cudaError_t run_simt(const SimtGemm& g, int rows_max, int nz, const Routing& R, cudaStream_t st) {
  if (rows_max <= 0 || g.cols <= 0 || nz <= 0) return cudaSuccess;
  dim3 grid((g.cols + TN - 1) / TN, (rows_max + TM - 1) / TM, nz);
  simt_gemm_kernel<TA, TB, TD, EPI><<<grid, 256, 0, st>>>(g, R);
  return cudaGetLastError();
}

// sum of the split-K partials in split order: dWg = rows 0..M-1, dbias = row M
__global__ void __launch_bounds__(kThreads) dwg_reduce_kernel(const float* __restrict__ part, int nsplit,
                                                             int M, int E, float* dWg, float* dbias) {
  const int64_t n = (int64_t)(M + 1) * E;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kThreads) {
    float s = 0.f;
    for (int z = 0; z < nsplit; ++z) s += part[(int64_t)z * n + i];
    if (i < (int64_t)M * E) dWg[i] = s;
    else if (dbias) dbias[i - (int64_t)M * E] = s;
  }
}

int dwg_splits(int S, int M, int E, int num_sms) {
  const int tiles = ((M + 1 + TM - 1) / TM) * ((E + TN - 1) / TN);
  int ns = (2 * num_sms + tiles - 1) / tiles;
  const int maxs = (S + 255) / 256;           // at least 256 tokens per split
  if (ns > maxs) ns = maxs;
  return ns < 1 ? 1 : ns;
}

int sms_of_device() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

int gate_backward_grid(int S, int num_sms) {
  const int want = (S + (kThreads / 32) - 1) / (kThreads / 32);
  return want < num_sms * 4 ? want : num_sms * 4;
}

cudaError_t launch_gate_backward(const BwdArgs& a, const Routing& R, cudaStream_t st) {
  const int grid = gate_backward_grid(a.S, sms_of_device());
  if (a.bf16) gate_bwd_k<__nv_bfloat16>(a, R, grid, st);
  else gate_bwd_k<float>(a, R, grid, st);
  return cudaGetLastError();
}

cudaError_t launch_dx_gather(const BwdArgs& a, const Routing& R, cudaStream_t st) {
  const int grid = gate_backward_grid(a.S, sms_of_device());
  if (a.k <= 1) dx_gather_kernel<1><<<grid, kThreads, 0, st>>>(a, R);
  else if (a.k <= 2) dx_gather_kernel<2><<<grid, kThreads, 0, st>>>(a, R);
  else if (a.k <= 4) dx_gather_kernel<4><<<grid, kThreads, 0, st>>>(a, R);
  else dx_gather_kernel<8><<<grid, kThreads, 0, st>>>(a, R);
  return cudaGetLastError();
}

cudaError_t launch_dwg_tc_reduce(const BwdArgs& a, int nbpart, int num_sms, cudaStream_t st) {
  const int64_t n = (int64_t)a.M * a.E + a.E;
  int grid = (int)((n + kThreads - 1) / kThreads);
  if (grid > 4 * num_sms) grid = 4 * num_sms;
  dwg_tc_reduce_kernel<<<grid, kThreads, 0, st>>>(a.part, a.nsplit, a.M, a.E, a.EPb, a.bpart, nbpart,
                                                  a.dWg, a.dbias);
  return cudaGetLastError();
}

cudaError_t launch_pad_zero(void* const* bufs, const int* widths, int nbuf, bool bf16, int E,
                            int64_t Cbuf, const Routing& R, cudaStream_t st) {
  PadBufs b{};
  b.n = nbuf;
  for (int q = 0; q < nbuf && q < 4; ++q) {
    b.p[q] = static_cast<char*>(bufs[q]);
    b.row_bytes[q] = (int64_t)widths[q] * (bf16 ? 2 : 4);
  }
  pad_zero_kernel<<<dim3(8, E), kThreads, 0, st>>>(b, Cbuf, R);
  return cudaGetLastError();
}

cudaError_t launch_dx(const BwdArgs& a, const Routing& R, cudaStream_t st) {
  SimtGemm g{};
  g.A = a.dl;                 // A(t, e) = dl[t, e]
  g.a_i = a.E;
  g.a_k = 1;
  g.B = a.Wg;                 // B(e, m) = Wg[m, e]
  g.b_k = 1;
  g.b_j = a.E;
  g.rows = a.S;
  g.cols = a.M;
  g.K = a.E;
  g.ones_row = -1;
  g.D = a.dx;
  g.d_i = a.M;
  g.dxe = a.dybuf;
  g.Cbuf = a.Cbuf;
  g.k = a.k;
  if (a.bf16) return run_simt<float, float, __nv_bfloat16, kSgDx>(g, a.S, 1, R, st);
  return run_simt<float, float, float, kSgDx>(g, a.S, 1, R, st);
}

int dwg_tc_split_bound(int S, int M, int EPb, int num_sms) {
  const int Q = 2 * EPb;
  const int bn = Q % 256 == 0 ? 256 : (Q % 128 == 0 ? 128 : 64);
  const int tiles = ((M + 127) / 128) * (Q / bn);
  int ns = (num_sms + tiles - 1) / tiles;
  const int maxs = (S + 63) / 64;
  if (ns > maxs) ns = maxs;
  return ns < 1 ? 1 : ns;
}

void dwg_tc_split(int S, int M, int EPb, int num_sms, int& nsplit, int& kchunk) {
  const int ns = dwg_tc_split_bound(S, M, EPb, num_sms);
  kchunk = ((S + ns - 1) / ns + 63) / 64 * 64;
  if (kchunk < 64) kchunk = 64;
  nsplit = (S + kchunk - 1) / kchunk;
  if (nsplit < 1) nsplit = 1;
}

size_t dwg_partial_floats(int S, int M, int E, int num_sms) {
  return (size_t)dwg_splits(S, M, E, num_sms) * (M + 1) * E;
}

cudaError_t launch_dwg(const BwdArgs& a, int num_sms, cudaStream_t st) {
  const int ns = dwg_splits(a.S, a.M, a.E, num_sms);
  if ((size_t)ns * (a.M + 1) * a.E > a.part_floats) return cudaErrorInvalidValue;
  SimtGemm g{};
  g.A = a.x;                  // A(m, t) = x[t, m]; row M is the ones row (bias)
  g.a_i = 1;
  g.a_k = a.M;
  g.B = a.dl;                 // B(t, e) = dl[t, e]
  g.b_k = a.E;
  g.b_j = 1;
  g.rows = a.M + 1;
  g.cols = a.E;
  g.K = a.S;
  g.ones_row = a.M;
  g.kchunk = ((a.S + ns - 1) / ns + TK - 1) / TK * TK;
  g.D = a.part;
  g.d_z = (int64_t)(a.M + 1) * a.E;
  g.d_i = a.E;
  Routing none{};
  cudaError_t e = a.bf16 ? run_simt<__nv_bfloat16, float, float, kSgPartial>(g, a.M + 1, ns, none, st)
                         : run_simt<float, float, float, kSgPartial>(g, a.M + 1, ns, none, st);
  if (e != cudaSuccess) return e;
  const int64_t n = (int64_t)(a.M + 1) * a.E;
  int grid = (int)((n + kThreads - 1) / kThreads);
  if (grid > 4 * num_sms) grid = 4 * num_sms;
  dwg_reduce_kernel<<<grid, kThreads, 0, st>>>(a.part, ns, a.M, a.E, a.dWg, a.dbias);
  return cudaGetLastError();
}

cudaError_t launch_ffn_bwd_f32(const float* xbuf, const float* hbuf, float* dybuf, float* dpre,
                               const float* W1, const float* W2, float* dW1, float* dW2,
                               const int32_t* nexp, int E, int64_t Cbuf, int M, int H,
                               bool skip_empty, cudaStream_t st) {
  Routing none{};
  const int rows_cap = (int)Cbuf;
  cudaError_t e;
  // dW2[e] = h_e^T dY_e            (H x M, reduction over the kept slots)
  {
    SimtGemm g{};
    g.A = hbuf; g.a_z = Cbuf * H; g.a_i = 1; g.a_k = H;
    g.B = dybuf; g.b_z = Cbuf * M; g.b_k = M; g.b_j = 1;
    g.rows = H; g.cols = M; g.k_from_n = true; g.nexp = nexp; g.Cbuf = Cbuf; g.ones_row = -1;
    g.skip_empty = skip_empty;
    g.D = dW2; g.d_z = (int64_t)H * M; g.d_i = M;
    if ((e = run_simt<float, float, float, kSgStore>(g, H, E, none, st)) != cudaSuccess) return e;
  }
  // dP_e = (dY_e W2[e]^T) * [h_e > 0]   (n_e x H)
  {
    SimtGemm g{};
    g.A = dybuf; g.a_z = Cbuf * M; g.a_i = M; g.a_k = 1;
    g.B = W2; g.b_z = (int64_t)H * M; g.b_k = 1; g.b_j = M;
    g.cols = H; g.K = M; g.rows_from_n = true; g.nexp = nexp; g.Cbuf = Cbuf; g.ones_row = -1;
    g.D = dpre; g.d_z = Cbuf * H; g.d_i = H; g.mask = hbuf;
    if ((e = run_simt<float, float, float, kSgMask>(g, rows_cap, E, none, st)) != cudaSuccess) return e;
  }
  // dW1[e] = X_e^T dP_e            (M x H)
  {
    SimtGemm g{};
    g.A = xbuf; g.a_z = Cbuf * M; g.a_i = 1; g.a_k = M;
    g.B = dpre; g.b_z = Cbuf * H; g.b_k = H; g.b_j = 1;
    g.rows = M; g.cols = H; g.k_from_n = true; g.nexp = nexp; g.Cbuf = Cbuf; g.ones_row = -1;
    g.skip_empty = skip_empty;
    g.D = dW1; g.d_z = (int64_t)M * H; g.d_i = H;
    if ((e = run_simt<float, float, float, kSgStore>(g, M, E, none, st)) != cudaSuccess) return e;
  }
  // dX_e = dP_e W1[e]^T -> over dY_e  (n_e x M)
  {
    SimtGemm g{};
    g.A = dpre; g.a_z = Cbuf * H; g.a_i = H; g.a_k = 1;
    g.B = W1; g.b_z = (int64_t)M * H; g.b_k = 1; g.b_j = H;
    g.cols = M; g.K = H; g.rows_from_n = true; g.nexp = nexp; g.Cbuf = Cbuf; g.ones_row = -1;
    g.D = dybuf; g.d_z = Cbuf * M; g.d_i = M;
    if ((e = run_simt<float, float, float, kSgStore>(g, rows_cap, E, none, st)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace moe
