// slots_noalloc.cu -- capacity slot assignment that allocates no device memory.
//
// Some callers cannot call cudaMalloc: for example, a serving process whose
// memory pool has already reserved nearly all of HBM, or a runtime where every
// device allocation must go through its own allocator.  In both cases an
// implicit allocation would fail or break the caller's accounting.  The layer
// handle needs one cudaMalloc at create time.  This entry point instead runs
// the capacity scan on expert ids the caller already holds, with the caller's
// own output buffers.  Its scratch (per-chunk local ranks, per-chunk histograms
// and their prefix offsets) lives in one file-scope device array of fixed size,
// which every GPU that loads this library holds until the process exits.
//
// Semantics are the layer's capacity rule: for r = 0..k-1 and tokens in order,
// an assignment (t, r) to expert e takes the next free slot of e while fewer than
// C are taken; later ones are dropped (slot -1).  cnt[e] counts every assignment
// to e (demand before capacity).
//
// Scratch use for S tokens, E experts and k choices, with nchunk = ceil(S / 64):
//   lrank [S*k] int32, hist [k*nchunk*E] int32, off [k*nchunk*E] int32,
// each region rounded up to 256 bytes.  The total must fit kNoAllocScratchBytes.
// Every scratch word a call reads is written earlier in the same call, so no
// clearing is needed between calls.  Calls whose work overlaps on the GPU
// (on different streams, or from several host threads) share the array and race.
#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "internal.h"

static constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

constexpr int kThreads = 256;
constexpr int kMaxDevices = 64;

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

// Set-up, once per device: the device address of the scratch array and the
// device's SM count.  In host code the array's name is only a host-side
// stand-in, so the real address is looked up with that device current and
// cached for later calls.  The cache belongs to the device's primary context:
// after cudaDeviceReset the library's module is loaded afresh, the cached
// address no longer names the array, and this entry point must not be called
// again in that process.
cudaError_t scratch_setup(void** out, int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    int sms = 0;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
    g_num_sms[dev] = sms > 0 ? sms : 1;
  }
  *out = g_scratch_addr[dev];
  *num_sms = g_num_sms[dev];
  return cudaSuccess;
}

size_t round256(size_t n) { return (n + 255) & ~(size_t)255; }

// Per 64-token chunk: rank of each (t, r) among same-expert rank-r choices of
// earlier tokens in the chunk, and the chunk's rank-r histogram.  Ids outside
// [0, E) are counted nowhere and get lrank -1.
__global__ void __launch_bounds__(kThreads) na_chunk_kernel(const int32_t* __restrict__ eidx, int S,
                                                            int E, int k, int nchunk,
                                                            int32_t* __restrict__ lrank,
                                                            int32_t* __restrict__ hist) {
  __shared__ int32_t sel[moe::kChunk][moe::kMaxK];
  __shared__ int32_t h[moe::kMaxK][moe::kMaxExperts];
  const int tid = threadIdx.x, chunk = blockIdx.x, tok0 = chunk * moe::kChunk;
  const int ntok = min(moe::kChunk, S - tok0);
  for (int i = tid; i < moe::kMaxK * moe::kMaxExperts; i += kThreads) (&h[0][0])[i] = 0;
  for (int i = tid; i < ntok * k; i += kThreads) {
    const int t = i / k, r = i - t * k;
    sel[t][r] = eidx[(int64_t)(tok0 + t) * k + r];
  }
  __syncthreads();
  for (int i = tid; i < ntok * k; i += kThreads) {
    const int t = i / k, r = i - t * k;
    const int e = sel[t][r];
    int c = -1;
    if (e >= 0 && e < E) {
      c = 0;
      for (int u = 0; u < t; ++u) c += (sel[u][r] == e);
      atomicAdd(&h[r][e], 1);
    }
    lrank[(int64_t)(tok0 + t) * k + r] = c;
  }
  __syncthreads();
  for (int i = tid; i < k * E; i += kThreads) {
    const int r = i / E, e = i - r * E;
    hist[((int64_t)r * nchunk + chunk) * E + e] = h[r][e];
  }
}

// One block per expert: exclusive prefix of hist over (r, chunk) in r-major
// order, and the expert's total demand.
__global__ void __launch_bounds__(kThreads) na_scan_kernel(int E, int k, int nchunk,
                                                           const int32_t* __restrict__ hist,
                                                           int32_t* __restrict__ off,
                                                           int32_t* __restrict__ cnt) {
  __shared__ int warp_sums[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, e = blockIdx.x;
  const int L = k * nchunk;
  const int seg = (L + kThreads - 1) / kThreads;
  const int a = min(L, tid * seg), b = min(L, a + seg);
  int local = 0;
  for (int q = a; q < b; ++q) local += hist[(int64_t)q * E + e];
  int x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kThreads / 32) warp_sums[lane] = w;
  }
  __syncthreads();
  int run = (warp ? warp_sums[warp - 1] : 0) + x - local;
  for (int q = a; q < b; ++q) {
    off[(int64_t)q * E + e] = run;
    run += hist[(int64_t)q * E + e];
  }
  if (tid == 0) cnt[e] = warp_sums[kThreads / 32 - 1];
}

__global__ void __launch_bounds__(kThreads) na_slot_kernel(const int32_t* __restrict__ eidx, int S,
                                                           int E, int k, int64_t C, int nchunk,
                                                           const int32_t* __restrict__ off,
                                                           const int32_t* __restrict__ lrank,
                                                           int32_t* __restrict__ slot) {
  const int64_t n = (int64_t)S * k;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * kThreads) {
    const int t = (int)(i / k), r = (int)(i - (int64_t)t * k);
    const int e = eidx[i];
    const int lr = lrank[i];
    int s = -1;
    if (e >= 0 && e < E && lr >= 0) {
      const int64_t pos = (int64_t)off[((int64_t)r * nchunk + t / moe::kChunk) * E + e] + lr;
      if (pos < C) s = (int)pos;
    }
    slot[i] = s;
  }
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

moe_status status_of(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  return MOE_ERR_CUDA;
}

}  // namespace

extern "C" MOE_API moe_status moe_assign_slots_noalloc(int64_t S, int32_t E, int32_t k, int64_t C,
                                                       const int32_t* eidx_dev, int32_t* slot_dev,
                                                       int32_t* cnt_dev, void* stream) {
  if (S < 0 || E < 1 || k < 1 || k > E || C < 0) return MOE_ERR_INVALID_ARG;
  if (E > moe::kMaxExperts || k > moe::kMaxK) return MOE_ERR_UNSUPPORTED;
  if (!cnt_dev || !aligned4(cnt_dev)) return MOE_ERR_INVALID_ARG;
  if (S > 0 && (!eidx_dev || !slot_dev || !aligned4(eidx_dev) || !aligned4(slot_dev)))
    return MOE_ERR_INVALID_ARG;
  if (S > (int64_t)1 << 30) return MOE_ERR_UNSUPPORTED;
  const int nchunk = (int)((S + moe::kChunk - 1) / moe::kChunk);
  const size_t lrank_bytes = round256((size_t)S * k * 4);
  const size_t table_bytes = round256((size_t)k * nchunk * E * 4);
  if (lrank_bytes + 2 * table_bytes > kNoAllocScratchBytes) return MOE_ERR_UNSUPPORTED;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* base = nullptr;
  int num_sms = 1;
  cudaError_t ce = scratch_setup(&base, &num_sms);
  if (ce != cudaSuccess) return status_of(ce);
  if (S == 0) return status_of(cudaMemsetAsync(cnt_dev, 0, (size_t)E * 4, st));

  char* p = static_cast<char*>(base);
  int32_t* lrank = reinterpret_cast<int32_t*>(p);
  int32_t* hist = reinterpret_cast<int32_t*>(p + lrank_bytes);
  int32_t* off = reinterpret_cast<int32_t*>(p + lrank_bytes + table_bytes);
  na_chunk_kernel<<<nchunk, kThreads, 0, st>>>(eidx_dev, (int)S, E, k, nchunk, lrank, hist);
  na_scan_kernel<<<E, kThreads, 0, st>>>(E, k, nchunk, hist, off, cnt_dev);
  // grid-stride slot pass: at most 8 blocks of 256 threads per SM
  const int64_t n = S * k, blocks = (n + kThreads - 1) / kThreads, cap = (int64_t)num_sms * 8;
  const int grid = (int)(blocks < cap ? blocks : cap);
  na_slot_kernel<<<grid, kThreads, 0, st>>>(eidx_dev, (int)S, E, k, C, nchunk, off, lrank, slot_dev);
  return status_of(cudaGetLastError());
}
