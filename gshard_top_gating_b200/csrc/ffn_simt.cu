// ffn_simt.cu -- fp32 grouped expert GEMM on CUDA cores (fp32 activations).
//
// Each expert is a two-layer ReLU feed-forward network ("GShard: Scaling Giant
// Neural Networks with Conditional Computation", "Core Components", "Expert
// Networks").  For fp32 activations the two GEMMs run here in FFMA: TF32 tensor
// cores would lose the 1e-4 output tolerance.  D[e, :n_e] = act(A[e, :n_e] B[e]),
// act = ReLU for the first layer, identity for the second.  Rows >= n_e are not
// written.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <bool RELU>
__global__ void __launch_bounds__(256) ffn_f32_kernel(const float* __restrict__ A,
                                                      const float* __restrict__ B,
                                                      float* __restrict__ D,
                                                      const int32_t* __restrict__ nexp,
                                                      int64_t Cbuf, int K, int N) {
  const int e = blockIdx.z;
  const int n_e = nexp[e];
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  if (m0 >= n_e) return;
  const float* Ae = A + (int64_t)e * Cbuf * K;
  const float* Be = B + (int64_t)e * K * N;
  float* De = D + (int64_t)e * Cbuf * N;
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  const int ar = tid >> 2, ak = (tid & 3) * 4;       // A tile loader
  const int bk = tid >> 4, bn = (tid & 15) * 4;      // B tile loader
  for (int k0 = 0; k0 < K; k0 += TK) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    if (m0 + ar < n_e) a = *reinterpret_cast<const float4*>(Ae + (int64_t)(m0 + ar) * K + k0 + ak);
    As[ak + 0][ar] = a.x;
    As[ak + 1][ar] = a.y;
    As[ak + 2][ar] = a.z;
    As[ak + 3][ar] = a.w;
    *reinterpret_cast<float4*>(&Bs[bk][bn]) =
        *reinterpret_cast<const float4*>(Be + (int64_t)(k0 + bk) * N + n0 + bn);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= n_e) continue;
    float4 o;
    o.x = RELU ? fmaxf(acc[i][0], 0.f) : acc[i][0];
    o.y = RELU ? fmaxf(acc[i][1], 0.f) : acc[i][1];
    o.z = RELU ? fmaxf(acc[i][2], 0.f) : acc[i][2];
    o.w = RELU ? fmaxf(acc[i][3], 0.f) : acc[i][3];
    *reinterpret_cast<float4*>(De + (int64_t)m * N + n0 + tx * 4) = o;
  }
}

}  // namespace

cudaError_t launch_ffn_f32(const float* A, const float* B, float* D, const int32_t* nexp, int E,
                           int64_t Cbuf, int K, int N, bool relu, cudaStream_t st) {
  dim3 grid(N / TN, (unsigned)((Cbuf + TM - 1) / TM), E);
  if (relu)
    ffn_f32_kernel<true><<<grid, 256, 0, st>>>(A, B, D, nexp, Cbuf, K, N);
  else
    ffn_f32_kernel<false><<<grid, 256, 0, st>>>(A, B, D, nexp, Cbuf, K, N);
  return cudaGetLastError();
}

}  // namespace moe
