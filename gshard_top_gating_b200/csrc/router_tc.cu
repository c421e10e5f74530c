// router_tc.cu -- gate GEMM on tcgen05 tensor cores for bf16 tokens, then softmax, top-k,
// normalised gates and the per-chunk tables of the capacity scan.
//
// Gating: G(x) = Softmax(x . W_g) ("GShard: Scaling Giant Neural Networks with
// Conditional Computation", "Mixture-of-Experts Implementation"), top-k experts
// with "softmax-normalised top-2 weights" ("GShard: Scaling Giant Models with
// Conditional Computation and Automatic Sharding", paper-note summary).
//
// Precision.  The gate GEMM is fp32 in the method.  A bf16 token is exact in
// bf16, and W_g is split once, at create time, into three bf16 parts
// W_g = hi + mid + lo (about 24 significant bits, the bf16x3 scheme of Henry,
// Tang and Heinecke, "Leveraging the bfloat16 artificial intelligence datatype
// for higher-precision computations", ARITH 2019).  The three products
// x.hi, x.mid, x.lo accumulate in fp32 TMEM columns: for EP <= 64 each part has
// its own column group and one MMA of N = 3*EP covers all three, so a 16-deep K
// step is one instruction instead of three and reads the token tile from shared
// memory once; for EP >= 128 (MMAs of N >= 128, long enough on their own) the
// three parts add into one accumulator.  The tensor core's fp32 accumulation does not round to
// nearest, and over a long K its rounding error builds up coherently, so K is
// cut into segments of kSegBlocks*64: each segment accumulates from zero and the
// epilogue warps add it (lo + mid, then + hi) into a running sum with ordinary
// round-to-nearest fp32 adds.  The logits so carry fp32-level error at
// tensor-core speed.
//
// One CTA = 128 tokens (64 for small batches with E <= 64) x EP experts (E padded
// to 32/64/128/256), 16 warps; or, for 128-token CTAs with E <= 64, 8 warps and
// fewer stages so that two CTAs share an SM and one's epilogue overlaps the
// other's loads:
// warp 0 TMA producer (x tile TTx64 + three W_g parts EPx64 per stage, K-major,
// 128B swizzle), warp 1 TMEM owner and single-thread MMA issuer, four warps fold
// the K-segments (one token row per thread, as TMEM lanes dictate) and leave the
// final logits tile in shared memory.  Then all warps route (E <= 64: a thread per
// token; above: a warp per token, lanes over experts, shuffle max / sum / argmax;
// ties to the lower index) and write the same per-64-token chunk tables
// (probability sums, lse^2 sums, rank-r histograms, local ranks) as the CUDA-core
// router.
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "route_token.cuh"

namespace moe {

int router_tokens_per_cta(int E, int S);

namespace {

constexpr int BM = 128, BK = 64;
constexpr uint32_t A_BYTES = BM * BK * 2;
constexpr int kSegBlocks = 8;      // k-blocks (of 64) accumulated before each fp32 round-to-nearest add

template <int EP, int TT_, int NW_>
struct RCfg {
  // tokens per CTA: 128, or 64 when 128-token CTAs would not fill the SMs (twice
  // the CTAs stream x; the MMA keeps M=128 and its upper 64 accumulator rows are
  // ignored)
  static constexpr int TT = TT_;
  // warps: 16 (one CTA per SM), or 8 (two per SM: 128 tokens and E <= 64 only)
  static constexpr int NW = NW_;
  static constexpr int NT = NW * 32;
  static constexpr int FOLD0 = NW == 8 ? 4 : 2;       // first of the four fold warps
  static_assert(NW == 16 || (NW == 8 && TT == 128 && EP <= 64), "8-warp CTAs: 128 tokens, E <= 64");
  static constexpr int NCH = TT / kChunk;                       // 64-token chunks per CTA
  static constexpr uint32_t X_BYTES = TT * BK * 2;              // bytes TMA writes into the A tile
  static constexpr uint32_t PART_BYTES = EP * BK * 2;           // one W_g part, EP x 64 bf16
  static constexpr uint32_t STAGE_BYTES = A_BYTES + 3 * PART_BYTES;
  static constexpr uint32_t TX_BYTES = X_BYTES + 3 * PART_BYTES;
  // two 8-warp CTAs per SM must each fit in half the shared memory
  static constexpr int STAGES = NW == 8 ? (EP == 64 ? 2 : 3)
                                        : ((EP == 256) ? 2 : (EP == 128 ? 3 : (EP == 64 ? 5 : 7)));
  // L2 prefetch distance of the token tiles, in k-blocks.  With 3 or more stages in
  // flight the prefetches only queue ahead of the loads in the TMA unit (measured:
  // slower); with 2 stages (E > 128) they hide the DRAM latency of x.
  static constexpr int PREFETCH_X = STAGES <= 2 ? 12 : 0;
  // column groups of the accumulator: hi | mid | lo for EP <= 64, one shared group above
  static constexpr int NG = EP <= 64 ? 3 : 1;
  static constexpr uint32_t ACC_COLS = NG * EP;        // the running sum follows
  static constexpr uint32_t TMEM_COLS =
      ACC_COLS + EP <= 128 ? 128 : (ACC_COLS + EP <= 256 ? 256 : 512);
  // epilogue scratch reuses the stage buffers: logits L [TT][EP+1] f32 (padded row),
  // per-warp probability sums red [16][EP] f32, per-warp lse^2 [16], sel [TT][8] i32,
  // running counts / hist [NCH][8][EP] i32
  static constexpr uint32_t LD = EP + 1;
  static constexpr uint32_t L_OFF = 0;
  static constexpr uint32_t RED_OFF = L_OFF + TT * LD * 4;
  static constexpr uint32_t LSE_OFF = RED_OFF + 16 * EP * 4;
  static constexpr uint32_t SEL_OFF = LSE_OFF + 16 * 4;
  static constexpr uint32_t H_OFF = SEL_OFF + TT * kMaxK * 4;
  // E <= 64 (thread-per-token routing): probabilities P [TT][EP+1] f32, lse^2 per token [TT]
  static constexpr uint32_t P_OFF = H_OFF + NCH * kMaxK * EP * 4;
  static constexpr uint32_t LSET_OFF = P_OFF + (EP <= 64 ? TT * LD * 4 : 0);
  static constexpr uint32_t EPI_END = LSET_OFF + (EP <= 64 ? TT * 4 : 0);
  static_assert(EPI_END <= STAGES * STAGE_BYTES, "epilogue scratch must fit in the stage buffers");
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 16;
  // residency: a 16-warp CTA owns its SM; two 8-warp CTAs share one SM's 228 KB of
  // shared memory (1 KB reserved per CTA) and its 512 TMEM columns, so neither CTA's
  // allocation can wait on the other
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(NW == 16 || 2 * (SMEM + 1024) <= 228 * 1024, "two 8-warp CTAs per SM");
  static_assert(SMEM > 80 * 1024, "the GEMM kernels' residency argument assumes more than 80 KB");
  static_assert((NW == 8 ? 2 : 1) * TMEM_COLS <= 512, "TMEM columns of the CTAs on one SM");
};

__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// kind::f16, D fp32, A bf16 K-major, B bf16 K-major, M=128, N (a multiple of 16, <= 256)
template <int N>
__device__ __forceinline__ uint32_t idesc_router() {
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N out of range");
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

template <int EP, int TT, int NW>
__global__ void __launch_bounds__(NW * 32, (NW == 8) ? 2 : 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ bias, int S, int M, int E, int k, int nchunk,
                     Routing R, uint64_t limit_ns) {
  using C = RCfg<EP, TT, NW>;
  constexpr int kThreads = C::NT;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw_base);
  const uint32_t bar0 = base + C::STAGES * C::STAGE_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  const uint32_t tfull_bar = bar0 + 8u * (2 * C::STAGES);      // a K-segment is accumulated
  const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 1);
  const uint32_t tempty_bar = bar0 + 8u * (2 * C::STAGES + 2);   // the epilogue took the segment
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbase + C::STAGES * C::STAGE_BYTES + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + C::STAGES * C::STAGE_BYTES + 260);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, tok0 = tile * C::TT;
  const int KB = M / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tfull_bar, 1);
    mbar_init(done_bar, 1);
    mbar_init(tempty_bar, C::TT);            // one arrival per token row
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The scan may launch and wait while this grid runs.  Triggered after the TMEM
  // allocation, so no dependent grid is resident before every CTA of this one holds
  // its columns.
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      // x streams from DRAM once: with few stages, prefetch it into L2 ahead of the loads
      constexpr int PF = C::PREFETCH_X;
      for (int kb = 0; kb < KB && kb < PF; ++kb) tma_prefetch_l2_2d(&tmX, kb * BK, tok0);
      for (int kb = 0; kb < KB; ++kb) {
        if (PF > 0 && kb + PF < KB) tma_prefetch_l2_2d(&tmX, (kb + PF) * BK, tok0);
        if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, R.err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        const uint32_t sa = base + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(full_bar(s), C::TX_BYTES);
        tma_load_2d(sa, &tmX, full_bar(s), kb * BK, tok0);
#pragma unroll
        for (int part = 0; part < 3; ++part)
          tma_load_2d(sa + A_BYTES + part * C::PART_BYTES, &tmW, full_bar(s), kb * BK, part * EP);
        issued |= 1u << s;
        issued_par = (issued_par & ~(1u << s)) | (ph << s);
        if (++s == C::STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok)
        for (int q = 0; q < C::STAGES; ++q)
          if ((issued >> q) & 1u) mbar_wait(full_bar(q), (issued_par >> q) & 1u, R.err, limit_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int seg = kb / kSegBlocks;
        const bool seg_first = (kb % kSegBlocks) == 0;
        const bool seg_last = (kb % kSegBlocks) == kSegBlocks - 1 || kb == KB - 1;
        if (seg_first) {   // the epilogue must have taken the previous segment
          if (*abort_flag || !mbar_wait(tempty_bar, (seg & 1) ^ 1u, R.err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
        }
        if (*abort_flag || !mbar_wait(full_bar(s), ph, R.err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + s * C::STAGE_BYTES;
        if constexpr (C::NG == 3) {
          // the three parts sit back to back (1024-byte aligned), one K-major operand of 3*EP rows
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc_mma_f16(tmem_base, desc_kmajor_sw128(sa + kk * 32u), desc_kmajor_sw128(sb + kk * 32u),
                       idesc_router<3 * EP>(), !(seg_first && kk == 0));
          }
        } else {
#pragma unroll
          for (int part = 2; part >= 0; --part) {       // smallest part first
            const uint32_t sb = sa + A_BYTES + part * C::PART_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma_f16(tmem_base, desc_kmajor_sw128(sa + kk * 32u), desc_kmajor_sw128(sb + kk * 32u),
                         idesc_router<EP>(), !(seg_first && kk == 0 && part == 2));
          }
        }
        tc_commit(empty_bar(s));
        if (seg_last) tc_commit(tfull_bar);
        if (++s == C::STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        tc_commit(done_bar);
        mbar_wait(done_bar, 0, R.err, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp >= C::FOLD0 && warp < C::FOLD0 + 4 && (warp & 3) < C::TT / 32) {
    // ------------------------------------------------------------ fold K-segments (four warps)
    const int q = warp & 3;
    const int row = q * 32 + lane;              // token row within the tile (= TMEM lane)
    const uint32_t tlane = tmem_base + ((uint32_t)(q * 32) << 16);
    float* Ls = reinterpret_cast<float*>(gbase + C::L_OFF);
    const int nseg = (KB + kSegBlocks - 1) / kSegBlocks;
    bool ok = true;
    for (int seg = 0; seg < nseg; ++seg) {
      if (*abort_flag || !mbar_wait(tfull_bar, seg & 1, R.err, limit_ns)) {
        *abort_flag = 1;
        ok = false;
        break;
      }
      tc_fence_after();
      const bool last = seg == nseg - 1;
#pragma unroll 1
      for (int c = 0; c < EP / 32; ++c) {
        uint32_t a[32], b[32];
        if constexpr (C::NG == 3) {    // this segment's x.lo + x.mid, then + x.hi
          tmem_ld_32x32b_x32(tlane + 2 * EP + c * 32, a);
          tmem_ld_32x32b_x32(tlane + EP + c * 32, b);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) + __uint_as_float(b[i]));
          tmem_ld_32x32b_x32(tlane + c * 32, b);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) + __uint_as_float(b[i]));
        } else {
          tmem_ld_32x32b_x32(tlane + c * 32, a);
        }
        if (seg > 0) tmem_ld_32x32b_x32(tlane + C::ACC_COLS + c * 32, b);
        tmem_ld_wait();
        if (seg > 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) + __uint_as_float(b[i]));
        }
        if (last) {          // final logits (+ bias) into the shared tile
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int j = c * 32 + i;
            Ls[row * C::LD + j] = __uint_as_float(a[i]) + ((bias && j < E) ? __ldg(bias + j) : 0.f);
          }
        } else {
          tmem_st_32x32b_x32(tlane + C::ACC_COLS + c * 32, a);
        }
      }
      if (!last) tmem_st_wait();
      tc_fence_before();
      mbar_arrive(tempty_bar);
    }
    if (!ok)
      for (int c = 0; c < EP; ++c) Ls[row * C::LD + c] = 0.f;
  }

  // ------------------------------------------------------------ route, all warps
  __syncthreads();
  {
    float* Ls = reinterpret_cast<float*>(gbase + C::L_OFF);
    float* red = reinterpret_cast<float*>(gbase + C::RED_OFF);
    float* lse_w = reinterpret_cast<float*>(gbase + C::LSE_OFF);
    int32_t* sel = reinterpret_cast<int32_t*>(gbase + C::SEL_OFF);
    int32_t* Hs = reinterpret_cast<int32_t*>(gbase + C::H_OFF);
    constexpr int RE = EP / 32;
    const int tid = threadIdx.x;
    const bool good = !*abort_flag;
    const int ntile = good ? min(C::TT, S - tok0) : 0;
    const int chunk0 = tile * C::NCH;
    for (int i = tid; i < C::NCH * kMaxK * EP; i += kThreads) Hs[i] = 0;
    if constexpr (EP <= 64) {
      // One thread per token: the whole logit row is read from shared memory (row
      // stride EP + 1 words, so the 32 tokens of a warp hit 32 banks).  The warps
      // without tokens copy the logits tile out, coalesced.
      float* Ps = reinterpret_cast<float*>(gbase + C::P_OFF);
      float* lse_t = reinterpret_cast<float*>(gbase + C::LSET_OFF);
      if (warp < C::TT / 32) {
        const int t = warp * 32 + lane;
        if (t < ntile) {
          const float* Lr = Ls + t * C::LD;
          float* Pr = Ps + t * C::LD;
          float mx = -INFINITY;
#pragma unroll 8
          for (int j = 0; j < E; ++j) mx = fmaxf(mx, Lr[j]);
          float sum = 0.f;
#pragma unroll 8
          for (int j = 0; j < E; ++j) {
            const float ex = expf(Lr[j] - mx);
            Pr[j] = ex;
            sum += ex;
          }
          const float inv = 1.f / sum;
#pragma unroll 8
          for (int j = 0; j < E; ++j) Pr[j] *= inv;
          const float lse = mx + logf(sum);
          lse_t[t] = lse * lse;
          // top-k on the logits, ties to the lower expert index (an ascending scan
          // replaces the incumbent only on a strictly larger logit)
          uint64_t taken = 0;
          int er[kMaxK];
          float lr[kMaxK];
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            er[r] = 0;
            lr[r] = 0.f;
            if (r < k) {
              float bv = -INFINITY;
              int bj = -1;
#pragma unroll 8
              for (int j = 0; j < E; ++j) {
                const float v = Lr[j];
                if (!((taken >> j) & 1ull) && (v > bv || bj < 0)) {
                  bv = v;
                  bj = j;
                }
              }
              if (bj < 0) {                 // k > E: rejected by the host, never reached
                atomicOr(R.err, DEVERR_BOUNDS);
                bj = 0;
              }
              taken |= 1ull << bj;
              er[r] = bj;
              lr[r] = bv;
            }
          }
          float gs = 0.f, gr[kMaxK];
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            gr[r] = (r < k) ? expf(lr[r] - lr[0]) : 0.f;
            gs += gr[r];
          }
          const float ginv = 1.f / gs;
          const int64_t tok = tok0 + t;
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            if (r < k) {
              R.eidx[tok * k + r] = er[r];
              R.gate[tok * k + r] = gr[r] * ginv;
              sel[t * kMaxK + r] = er[r];
            }
          }
        }
      } else {
        const int nthr = kThreads - C::TT;
        for (int idx = tid - C::TT; idx < ntile * E; idx += nthr) {
          const int t = idx / E, j = idx - t * E;
          R.logits[(int64_t)tok0 * E + idx] = Ls[t * C::LD + j];
        }
      }
      __syncthreads();
      // per-chunk probability sums (tokens in order, four interleaved partial sums)
      // and lse^2 sums (one warp per chunk, fixed shuffle tree)
      for (int idx = tid; idx < C::NCH * E; idx += kThreads) {
        const int cc = idx / E, j = idx - cc * E;
        const int chunk = chunk0 + cc;
        if (chunk >= nchunk) continue;
        const int t0 = cc * kChunk, t1 = min(t0 + kChunk, ntile);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int t = t0;
        for (; t + 4 <= t1; t += 4) {
          a0 += Ps[t * C::LD + j];
          a1 += Ps[(t + 1) * C::LD + j];
          a2 += Ps[(t + 2) * C::LD + j];
          a3 += Ps[(t + 3) * C::LD + j];
        }
        for (; t < t1; ++t) a0 += Ps[t * C::LD + j];
        R.psum[(int64_t)chunk * E + j] = (a0 + a1) + (a2 + a3);
      }
      if (warp < C::NCH && chunk0 + warp < nchunk) {
        const int t = warp * kChunk + lane;
        float a = (t < ntile ? lse_t[t] : 0.f) + (t + 32 < ntile ? lse_t[t + 32] : 0.f);
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) R.lse2[chunk0 + warp] = a;
      }
    } else {
      // E > 64: one warp per token, lanes over experts
      static_assert(C::NW == 16, "warp-per-token routing assumes 16 warps");
      constexpr int TPW = C::TT / 16;                         // tokens per warp (4 or 8)
      constexpr int WPC = 16 / C::NCH;                        // warps per 64-token chunk
      float psum[RE];
#pragma unroll
      for (int i = 0; i < RE; ++i) psum[i] = 0.f;
      float lse2 = 0.f;
      for (int t = warp * TPW; t < warp * TPW + TPW && t < ntile; t += 2) {   // two tokens in flight
        if (t + 1 < ntile) {
          float v[2][RE];
#pragma unroll
          for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int i = 0; i < RE; ++i) {
              const int j = lane + 32 * i;
              v[n][i] = j < E ? Ls[(t + n) * C::LD + j] : -INFINITY;
            }
          const int64_t tk[2] = {tok0 + t, tok0 + t + 1};
          int32_t* const rows[2] = {sel + t * kMaxK, sel + (t + 1) * kMaxK};
          route_tokens<RE, 2>(v, tk, E, k, true, R, psum, lse2, rows);
        } else {
          float v[RE];
#pragma unroll
          for (int i = 0; i < RE; ++i) {
            const int j = lane + 32 * i;
            v[i] = j < E ? Ls[t * C::LD + j] : -INFINITY;
          }
          route_token<RE>(v, tok0 + t, E, k, true, R, psum, lse2, sel + t * kMaxK);
        }
      }
#pragma unroll
      for (int i = 0; i < RE; ++i) red[warp * EP + lane + 32 * i] = psum[i];
      if (lane == 0) lse_w[warp] = lse2;
      __syncthreads();
      // per-chunk probability and lse^2 sums, warps of a chunk added in order
      for (int cc = 0; cc < C::NCH; ++cc) {
        const int chunk = chunk0 + cc;
        if (chunk >= nchunk) break;
        for (int j = tid; j < E; j += kThreads) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < WPC; ++w) acc += red[(cc * WPC + w) * EP + j];
          R.psum[(int64_t)chunk * E + j] = acc;
        }
        if (tid == 0) {
          float acc = 0.f;
#pragma unroll
          for (int w = 0; w < WPC; ++w) acc += lse_w[cc * WPC + w];
          R.lse2[chunk] = acc;
        }
      }
    }
    // local ranks within each 64-token chunk and rank-r histograms: one warp per
    // (chunk, rank), 32 tokens at a time; tokens choosing the same expert find one
    // another with a match, and a running count per expert carries over
    for (int pi = warp; pi < C::NCH * k; pi += C::NW) {
      const int cc = pi / k, r = pi - cc * k;
      int32_t* cnt = Hs + (cc * kMaxK + r) * EP;
      for (int h = 0; h < kChunk / 32; ++h) {
        const int t = cc * kChunk + h * 32 + lane;
        const bool valid = t < ntile;
        const int e = valid ? sel[t * kMaxK + r] : EP + lane;       // unmatched when invalid
        const unsigned m = __match_any_sync(0xffffffffu, e);
        if (valid) R.lrank[(int64_t)(tok0 + t) * k + r] = cnt[e] + __popc(m & ((1u << lane) - 1u));
        __syncwarp();
        if (valid && lane == __ffs(m) - 1) cnt[e] += __popc(m);
        __syncwarp();
      }
    }
    __syncthreads();
    for (int cc = 0; cc < C::NCH; ++cc) {
      const int chunk = chunk0 + cc;
      if (chunk >= nchunk) break;
      for (int idx = tid; idx < k * E; idx += kThreads) {
        const int r = idx / E, e = idx - r * E;
        R.hist[((int64_t)r * nchunk + chunk) * E + e] = Hs[(cc * kMaxK + r) * EP + e];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------
// Persistent router (E <= 64, batches that give every SM at least four 64-token chunks).
//
// One CTA per SM owns a contiguous range of 64-token chunks (ranges differ by at most
// one chunk) and walks it in tiles of two chunks (the last tile may be one chunk,
// loaded as a 64-row box).  Unlike router_tc_kernel, a tile's routing overlaps the
// next tiles' loads and MMAs:
//   warp 0       TMA producer over every tile's k-blocks (x tile + three W_g parts)
//   warp 1       MMA issuer; K-segments alternate between two TMEM accumulators
//   warps 2..5   fold: each K-segment (lo + mid, + hi) is added into the tile's running
//                sum, one of two TMEM regions (tiles alternate), and the segment's
//                accumulator is released at once
//   warps 6..15  routing group: copies a finished tile's logits from TMEM to shared
//                memory (plus bias), releases the running-sum region, then routes the
//                tile exactly as router_tc_kernel does for E <= 64 (a thread per
//                token), writes the logits and the chunk tables
// The arithmetic of every logit, probability, gate and table entry is that of
// router_tc_kernel.  TMEM: two segment accumulators (3*EP columns each) and two
// running sums (EP each) -- 448 of 512 columns for EP = 64.
template <int EP>
struct PCfg {
  static constexpr int NT = 512;
  static constexpr int TT = 128;
  static constexpr uint32_t PART_BYTES = EP * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + 3 * PART_BYTES;
  static constexpr uint32_t ACC = 3 * EP;                 // one K-segment accumulator
  static constexpr uint32_t RUN0 = 2 * ACC;               // running sum of tile parity b at RUN0 + b*EP
  static constexpr uint32_t TMEM_COLS = (2 * ACC + 2 * EP) <= 256 ? 256 : 512;
  static constexpr uint32_t LD = EP + 1;
  static constexpr uint32_t L_OFF = 0;                    // logits, then probabilities [TT][EP+1] f32
  static constexpr uint32_t SEL_OFF = L_OFF + TT * LD * 4;    // chosen experts [TT][8]
  static constexpr uint32_t H_OFF = SEL_OFF + TT * kMaxK * 4; // running counts [2][8][EP]
  static constexpr uint32_t LSE_OFF = H_OFF + 2 * kMaxK * EP * 4;   // lse^2 per token [TT]
  static constexpr uint32_t EPI_BYTES = ((LSE_OFF + TT * 4) + 1023u) & ~1023u;
  static constexpr uint32_t BAR_BYTES = 256;
  static constexpr int STAGES_FIT = (int)((227u * 1024u - 1024u - EPI_BYTES - BAR_BYTES) / STAGE_BYTES);
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
  static_assert(EP <= 64, "the persistent router routes a thread per token (E <= 64)");
  static_assert(STAGES >= 3, "at least three stages in flight");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(2 * ACC + 2 * EP <= TMEM_COLS, "TMEM columns");
  static_assert(8u * (2 * STAGES + 9) + 12 <= BAR_BYTES, "barriers, TMEM slot and flags");
};

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int EP>
__global__ void __launch_bounds__(512, 1)
    router_tcp_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmX64,
                      const __grid_constant__ CUtensorMap tmW, const float* __restrict__ bias, int S, int M,
                      int E, int k, int nchunk, Routing R, uint64_t limit_ns) {
  using C = PCfg<EP>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw_base);
  unsigned char* gepi = gbase + C::STAGES * C::STAGE_BYTES;
  float* Ls = reinterpret_cast<float*>(gepi + C::L_OFF);
  int32_t* sel = reinterpret_cast<int32_t*>(gepi + C::SEL_OFF);
  int32_t* Hs = reinterpret_cast<int32_t*>(gepi + C::H_OFF);
  float* lse_t = reinterpret_cast<float*>(gepi + C::LSE_OFF);
  const uint32_t bar0 = base + C::STAGES * C::STAGE_BYTES + C::EPI_BYTES;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + b); };      // a K-segment is done
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 2 + b); };  // the fold took it
  auto lfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 4 + b); };   // a tile's logits are done
  auto rfree_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 6 + b); };   // its running sum is free
  const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 8);
  unsigned char* gbar = gepi + C::EPI_BYTES;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(gbar + 8u * (2 * C::STAGES + 9));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbar + 8u * (2 * C::STAGES + 9) + 4);
  volatile int* go_flag = reinterpret_cast<volatile int*>(gbar + 8u * (2 * C::STAGES + 9) + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = gridDim.x, blk = blockIdx.x;
  const int c0 = (int)((int64_t)nchunk * blk / nblk), c1 = (int)((int64_t)nchunk * (blk + 1) / nblk);
  const int ntiles = (c1 - c0 + 1) / 2;
  const int KB = M / BK;
  const int nseg = (KB + kSegBlocks - 1) / kSegBlocks;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 128);             // the four fold warps
      mbar_init(lfull_bar(b), 128);
      mbar_init(rfree_bar(b), 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmX64);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();          // after the TMEM allocation (see router_tc_kernel)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        const int ca = c0 + 2 * i;
        const bool half = ca + 1 >= c1;
        const int tok0 = ca * kChunk;
        const uint32_t tx = (half ? 64u : 128u) * BK * 2 + 3 * C::PART_BYTES;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, R.err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = base + s * C::STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(s), tx);
          tma_load_2d(sa, half ? (const void*)&tmX64 : (const void*)&tmX, full_bar(s), kb * BK, tok0);
#pragma unroll
          for (int part = 0; part < 3; ++part)
            tma_load_2d(sa + A_BYTES + part * C::PART_BYTES, &tmW, full_bar(s), kb * BK, part * EP);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok)
        for (int q = 0; q < C::STAGES; ++q)
          if ((issued >> q) & 1u) mbar_wait(full_bar(q), (issued_par >> q) & 1u, R.err, limit_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, g = 0;
      bool ok = true;
      for (int i = 0; i < ntiles && ok; ++i) {
        for (int kb = 0; kb < KB; ++kb) {
          const bool seg_first = (kb % kSegBlocks) == 0;
          const bool seg_last = (kb % kSegBlocks) == kSegBlocks - 1 || kb == KB - 1;
          const uint32_t buf = g & 1u;
          if (seg_first) {   // the fold must have taken this accumulator's previous segment
            if (*abort_flag || !mbar_wait(tempty_bar(buf), ((g >> 1) & 1u) ^ 1u, R.err, limit_ns)) {
              *abort_flag = 1;
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (*abort_flag || !mbar_wait(full_bar(s), ph, R.err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * C::STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_f16(tmem_base + buf * C::ACC, desc_kmajor_sw128(sa + kk * 32u),
                       desc_kmajor_sw128(sb + kk * 32u), idesc_router<3 * EP>(), !(seg_first && kk == 0));
          tc_commit(empty_bar(s));
          if (seg_last) {
            tc_commit(tfull_bar(buf));
            ++g;
          }
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        tc_commit(done_bar);
        mbar_wait(done_bar, 0, R.err, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ fold (warps 2..5)
    const int q = warp & 3;                           // TMEM lanes 32q .. 32q + 31 (= tile rows)
    const uint32_t tlane = tmem_base + ((uint32_t)(q * 32) << 16);
    uint32_t g = 0;
    bool ok = true;
    for (int i = 0; i < ntiles && ok; ++i) {
      const int ca = c0 + 2 * i;
      const int ntok = min((ca + 1 >= c1 ? 1 : 2) * kChunk, S - ca * kChunk);
      const bool active = q * 32 < ntok;              // warp-uniform: rows past the tile are not read
      const uint32_t run = tlane + C::RUN0 + (uint32_t)(i & 1) * EP;
      for (int seg = 0; seg < nseg; ++seg) {
        const uint32_t buf = g & 1u;
        bool w = !*abort_flag && mbar_wait(tfull_bar(buf), (g >> 1) & 1u, R.err, limit_ns);
        if (seg == 0) w = w && mbar_wait(rfree_bar(i & 1), ((i >> 1) & 1) ^ 1, R.err, limit_ns);
        if (!__all_sync(0xffffffffu, w)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        if (active) {
          const uint32_t acc = tlane + buf * C::ACC;
#pragma unroll 1
          for (int c = 0; c < EP / 32; ++c) {
            uint32_t a[32], b[32];
            tmem_ld_32x32b_x32(acc + 2 * EP + c * 32, a);       // this segment's x.lo + x.mid, then + x.hi
            tmem_ld_32x32b_x32(acc + EP + c * 32, b);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) + __uint_as_float(b[j]));
            tmem_ld_32x32b_x32(acc + c * 32, b);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) + __uint_as_float(b[j]));
            if (seg > 0) {
              tmem_ld_32x32b_x32(run + c * 32, b);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) + __uint_as_float(b[j]));
            }
            tmem_st_32x32b_x32(run + c * 32, a);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(tempty_bar(buf));
        ++g;
      }
      if (ok) mbar_arrive(lfull_bar(i & 1));          // the tile's logits (without bias) are in `run`
    }
  } else {
    // ------------------------------------------------------------ routing group (warps 6..15)
    constexpr int NR = C::NT - 192;                   // 320 threads
    const int tr = threadIdx.x - 192, wr = tr >> 5;
    for (int i = 0; i < ntiles; ++i) {
      const int ca = c0 + 2 * i;
      const int nch = ca + 1 >= c1 ? 1 : 2;
      const int tok0 = ca * kChunk;
      const int ntok = min(nch * kChunk, S - tok0);
      if (tr == 0)
        *go_flag = !*abort_flag && mbar_wait(lfull_bar(i & 1), (i >> 1) & 1, R.err, limit_ns);
      named_bar_sync(1, NR);
      if (!*go_flag) {
        if (tr == 0) *abort_flag = 1;
        break;                                        // uniform: every thread read the same flag
      }
      tc_fence_after();
      if (wr < 4) {                                   // warps 6..9 cover the four TMEM lane groups
        const int qq = warp & 3, row = qq * 32 + lane;
        const uint32_t run = tmem_base + ((uint32_t)(qq * 32) << 16) + C::RUN0 + (uint32_t)(i & 1) * EP;
#pragma unroll 1
        for (int c = 0; c < EP / 32; ++c) {
          uint32_t a[32];
          tmem_ld_32x32b_x32(run + c * 32, a);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = c * 32 + j;
            Ls[row * C::LD + col] = __uint_as_float(a[j]) + ((bias && col < E) ? __ldg(bias + col) : 0.f);
          }
        }
      } else {
        for (int idx = tr - 128; idx < 2 * kMaxK * EP; idx += NR - 128) Hs[idx] = 0;
      }
      tc_fence_before();
      named_bar_sync(1, NR);
      if (tr == 0) mbar_arrive(rfree_bar(i & 1));
      // one thread per token: softmax, lse, top-k (ties to the lower index), gates; the
      // other warps copy the logits out
      float mx = 0.f, inv = 0.f;
      if (tr < C::TT) {
        const int t = tr;
        if (t < ntok) {
          const float* Lr = Ls + t * C::LD;
          mx = -INFINITY;
#pragma unroll 8
          for (int j = 0; j < E; ++j) mx = fmaxf(mx, Lr[j]);
          float sum = 0.f;
#pragma unroll 8
          for (int j = 0; j < E; ++j) sum += expf(Lr[j] - mx);
          inv = 1.f / sum;
          const float lse = mx + logf(sum);
          lse_t[t] = lse * lse;
          uint64_t taken = 0;
          int er[kMaxK];
          float lr[kMaxK];
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            er[r] = 0;
            lr[r] = 0.f;
            if (r < k) {
              float bv = -INFINITY;
              int bj = -1;
#pragma unroll 8
              for (int j = 0; j < E; ++j) {
                const float v = Lr[j];
                if (!((taken >> j) & 1ull) && (v > bv || bj < 0)) {
                  bv = v;
                  bj = j;
                }
              }
              if (bj < 0) {
                atomicOr(R.err, DEVERR_BOUNDS);
                bj = 0;
              }
              taken |= 1ull << bj;
              er[r] = bj;
              lr[r] = bv;
            }
          }
          float gs = 0.f, gr[kMaxK];
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            gr[r] = (r < k) ? expf(lr[r] - lr[0]) : 0.f;
            gs += gr[r];
          }
          const float ginv = 1.f / gs;
          const int64_t tok = tok0 + t;
#pragma unroll
          for (int r = 0; r < kMaxK; ++r) {
            if (r < k) {
              R.eidx[tok * k + r] = er[r];
              R.gate[tok * k + r] = gr[r] * ginv;
              sel[t * kMaxK + r] = er[r];
            }
          }
        }
      } else {
        for (int idx = tr - C::TT; idx < ntok * E; idx += NR - C::TT) {
          const int t = idx / E, j = idx - t * E;
          R.logits[(int64_t)tok0 * E + idx] = Ls[t * C::LD + j];
        }
      }
      named_bar_sync(1, NR);
      // probabilities in place of the logits (the same exp and scale as the sum above)
      if (tr < C::TT && tr < ntok) {
        float* Lr = Ls + tr * C::LD;
#pragma unroll 8
        for (int j = 0; j < E; ++j) Lr[j] = expf(Lr[j] - mx) * inv;
      }
      named_bar_sync(1, NR);
      // per-chunk probability sums (tokens in order, four interleaved partial sums) and
      // lse^2 sums (one warp per chunk, fixed shuffle tree)
      for (int idx = tr; idx < nch * E; idx += NR) {
        const int cc = idx / E, j = idx - cc * E;
        const int t0 = cc * kChunk, t1 = min(t0 + kChunk, ntok);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        int t = t0;
        for (; t + 4 <= t1; t += 4) {
          a0 += Ls[t * C::LD + j];
          a1 += Ls[(t + 1) * C::LD + j];
          a2 += Ls[(t + 2) * C::LD + j];
          a3 += Ls[(t + 3) * C::LD + j];
        }
        for (; t < t1; ++t) a0 += Ls[t * C::LD + j];
        R.psum[(int64_t)(ca + cc) * E + j] = (a0 + a1) + (a2 + a3);
      }
      if (wr < nch) {
        const int t = wr * kChunk + lane;
        float a = (t < ntok ? lse_t[t] : 0.f) + (t + 32 < ntok ? lse_t[t + 32] : 0.f);
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) R.lse2[ca + wr] = a;
      }
      // local ranks within each chunk and rank-r histograms (one warp per (chunk, rank))
      for (int pi = wr; pi < nch * k; pi += NR / 32) {
        const int cc = pi / k, r = pi - cc * k;
        int32_t* cnt = Hs + (cc * kMaxK + r) * EP;
        for (int h = 0; h < kChunk / 32; ++h) {
          const int t = cc * kChunk + h * 32 + lane;
          const bool valid = t < ntok;
          const int e = valid ? sel[t * kMaxK + r] : EP + lane;
          const unsigned m = __match_any_sync(0xffffffffu, e);
          if (valid) R.lrank[(int64_t)(tok0 + t) * k + r] = cnt[e] + __popc(m & ((1u << lane) - 1u));
          __syncwarp();
          if (valid && lane == __ffs(m) - 1) cnt[e] += __popc(m);
          __syncwarp();
        }
      }
      named_bar_sync(1, NR);
      for (int cc = 0; cc < nch; ++cc)
        for (int idx = tr; idx < k * E; idx += NR) {
          const int r = idx / E, e = idx - r * E;
          R.hist[((int64_t)r * nchunk + ca + cc) * E + e] = Hs[(cc * kMaxK + r) * EP + e];
        }
      named_bar_sync(1, NR);                          // the tile's smem is reused by the next
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// W_g [M, E] fp32 -> three bf16 parts, each [EP, M] (K contiguous), rows >= E zero.
__global__ void split_gate_kernel(const float* __restrict__ Wg, int M, int E, int EP,
                                  __nv_bfloat16* __restrict__ out) {
  const int64_t n = (int64_t)EP * M;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(i / M), m = (int)(i - (int64_t)j * M);
    const float w = j < E ? Wg[(int64_t)m * E + j] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    out[i] = hi;
    out[n + i] = mid;
    out[2 * n + i] = lo;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool encode_kmajor(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_out) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_out};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EP, int TT, int NW>
cudaError_t launch_tt(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias, int S, int M,
                      int E, int k, const Routing& R, uint64_t limit_ns, cudaStream_t st) {
  using C = RCfg<EP, TT, NW>;
  auto kern = router_tc_kernel<EP, TT, NW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int nchunk = (S + kChunk - 1) / kChunk;
  kern<<<(S + TT - 1) / TT, C::NT, C::SMEM, st>>>(tmX, tmW, bias, S, M, E, k, nchunk, R, limit_ns);
  return cudaGetLastError();
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!cached[dev]) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = sms;
  }
  return cached[dev];
}

template <int EP>
cudaError_t launch_persistent(const CUtensorMap& tmX, const CUtensorMap& tmX64, const CUtensorMap& tmW,
                              const float* bias, int S, int M, int E, int k, const Routing& R,
                              uint64_t limit_ns, int grid, cudaStream_t st) {
  using C = PCfg<EP>;
  auto kern = router_tcp_kernel<EP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int nchunk = (S + kChunk - 1) / kChunk;
  kern<<<grid, C::NT, C::SMEM, st>>>(tmX, tmX64, tmW, bias, S, M, E, k, nchunk, R, limit_ns);
  return cudaGetLastError();
}

template <int EP>
cudaError_t launch_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias, int S, int M,
                     int E, int k, const Routing& R, uint64_t limit_ns, cudaStream_t st) {
  if (router_tokens_per_cta(E, S) == 128)
    return launch_tt<EP, 128, (EP <= 64 ? 8 : 16)>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
  return launch_tt<EP, 64, 16>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
}

}  // namespace

int router_tc_pad(int E) { return E <= 32 ? 32 : (E <= 64 ? 64 : (E <= 128 ? 128 : 256)); }

// 128 tokens per CTA halves the W_g bytes each token costs; 64 only for E <= 64 and
// batches too small for 128-token CTAs to fill every SM once.
int router_tokens_per_cta(int E, int S) {
  if (router_tc_pad(E) > 64) return 128;
  return (S + 127) / 128 >= sm_count() ? 128 : 64;
}

cudaError_t split_gate_weights(const float* Wg, int M, int E, void* out3, cudaStream_t st) {
  const int EP = router_tc_pad(E);
  const int64_t n = (int64_t)EP * M;
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  split_gate_kernel<<<grid, 256, 0, st>>>(Wg, M, E, EP, (__nv_bfloat16*)out3);
  return cudaGetLastError();
}

bool make_router_wmap(CUtensorMap* tm, const void* wsplit, int M, int E) {
  const int EP = router_tc_pad(E);
  return encode_kmajor(tm, wsplit, (uint64_t)M, (uint64_t)3 * EP, (uint32_t)EP);
}

bool make_router_xmap(CUtensorMap* tm, const void* x, int S, int M, int E) {
  return encode_kmajor(tm, x, (uint64_t)M, (uint64_t)S, (uint32_t)router_tokens_per_cta(E, S));
}

bool make_router_xmap64(CUtensorMap* tm, const void* x, int S, int M) {
  return encode_kmajor(tm, x, (uint64_t)M, (uint64_t)S, 64u);
}

bool router_persistent(int E, int S) {
  return router_tc_pad(E) <= 64 && (S + kChunk - 1) / kChunk >= 4 * sm_count();
}

cudaError_t launch_router_tc(const CUtensorMap& tmX, const CUtensorMap* tmX64, const void* x,
                             const CUtensorMap& tmW, const float* bias, int S, int M, int E, int k,
                             const Routing& R, uint64_t limit_ns, cudaStream_t st) {
  (void)x;
  if (tmX64 && router_persistent(E, S)) {
    if (router_tc_pad(E) == 32)
      return launch_persistent<32>(tmX, *tmX64, tmW, bias, S, M, E, k, R, limit_ns, sm_count(), st);
    return launch_persistent<64>(tmX, *tmX64, tmW, bias, S, M, E, k, R, limit_ns, sm_count(), st);
  }
  switch (router_tc_pad(E)) {
    case 32: return launch_t<32>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
    case 64: return launch_t<64>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
    case 128: return launch_t<128>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
    default: return launch_t<256>(tmX, tmW, bias, S, M, E, k, R, limit_ns, st);
  }
}

}  // namespace moe
