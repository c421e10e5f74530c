// ffn_tc.cu -- grouped expert GEMM on 5th-generation tensor cores (tcgen05), bf16 in, fp32 accumulate.
//
// Each expert is a two-layer ReLU feed-forward network ("GShard: Scaling Giant
// Neural Networks with Conditional Computation", "Core Components", "Expert
// Networks"); on one GPU all experts' GEMMs run in one persistent launch:
//
//   D[e, :n_e, :] = act( A[e, :n_e, :] . B[e] )      A [E*Cbuf, K], B [E*K, N], D [E*Cbuf, N]
//
// with n_e (kept rows of expert e) read on the device, so the host never waits
// for the routing.  FFN1: A = xbuf, B = W1 ([M, H] per expert, H contiguous),
// act = ReLU.  FFN2: A = hbuf, B = W2 ([H, M] per expert), act = identity.
//
// Design (one CTA per SM, 192 threads):
//   warp 0     TMA producer: A tile 128x64 (K-major, 128B swizzle) and B tile
//              64xBN (N contiguous = "MN-major" operand, 128B swizzle) per stage
//   warp 1     TMEM allocator + single-thread tcgen05.mma issuer (M=128, N=BN, K=16)
//   warps 2-5  epilogue: tcgen05.ld 32 lanes x 32 columns, fp32 -> bf16 (+ReLU),
//              predicated 16-byte stores of rows < n_e
// The fp32 accumulator lives in TMEM, double buffered (2*BN columns) so the
// epilogue of one tile overlaps the main loop of the next.  Tiles are ordered
// (expert, n-tile, m-tile) with m fastest, so the CTAs working at the same time
// share one weight column strip through L2.  All waits are bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 192;
constexpr uint32_t A_BYTES = BM * BK * 2;   // 16 KB

template <int BN>
struct Cfg {
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr uint32_t B_BYTES = BK * BN * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr uint32_t STAGING = 4 * 4096;   // one 32 x 64 bf16 store tile per epilogue warp
  // 1 KB alignment slack + stages + staging + 512 B of barriers + misc words and the tile tables
  static constexpr size_t SMEM =
      1024 + (size_t)STAGES * STAGE_BYTES + STAGING + 512 + 16 + 4 * (3 * kMaxExperts + 1);
  // A GEMM CTA owns its SM: beside its shared memory no other TMEM-using CTA of the
  // library fits (the smallest, an 8-warp router CTA, takes over 80 KB of the SM's
  // 228 KB), so a TMEM allocation (up to 512 columns) never waits on a co-resident CTA
  // that may itself be waiting on this kernel.
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(SMEM + 1024 + 80 * 1024 > 228 * 1024, "a GEMM CTA must own its SM");
  static_assert(TMEM_COLS <= 512, "TMEM columns");
};

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: version 1 at bit 46,
// layout type 2 = SWIZZLE_128B at bits 61-63).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, M=128, N=BN; a_mn / b_mn
// select the MN-major (transposed) operand layout (bits 15 / 16), else K-major.
template <int BN>
__device__ __forceinline__ uint32_t idesc_bf16(bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Walks this CTA's tiles in the global order (expert, n-tile, m-tile).
struct TileIter {
  const int* tile_pre;   // smem [E+1]: first tile of each expert
  const int* mtiles;     // smem [E]
  int E, NT, e;
  __device__ bool decode(int tile, int& ex, int& mt, int& nt) {
    if (tile >= tile_pre[E]) return false;
    while (tile >= tile_pre[e + 1]) ++e;
    const int local = tile - tile_pre[e];
    const int m_e = mtiles[e];
    nt = local / m_e;
    mt = local - nt * m_e;
    ex = e;
    return true;
  }
};

// Epilogue modes: plain store, ReLU, or the backward's ReLU mask (keep the
// accumulator where the first layer's saved output h is > 0, else 0).
enum { kEpiNone = 0, kEpiRelu = 1, kEpiMask = 2, kEpiF32 = 3, kEpiReluBits = 4, kEpiMaskBits = 5,
       kEpiGateY = 6 };
// kEpiGateY: g * accumulator, rounded to bf16, stored into the layer output row of the
// token that took the slot (ScatterY), instead of into D.
// kEpiReluBits: ReLU, and one bit per stored element, set when the stored bf16 value
// is > 0 (the backward's mask, 1/16 of the bytes of h).  kEpiMaskBits: keep the
// accumulator where that bit is set.  Bit j of word w of a row covers column 32w + j;
// the words are stored word-major, bits[w][row] (rows = E * Cbuf), so a warp's 32
// consecutive rows write and read one 128-byte line per word.

// 32 mask bits for 32 consecutive bf16 values of h: bit j set iff h[j] > 0
// (bit patterns 0x0001 .. 0x7f80: positive finite or +inf).
__device__ __forceinline__ uint32_t positive_bits(const uint4 (&v)[4]) {
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = w[j] & 0xFFFFu, hi = w[j] >> 16;
      bits |= (uint32_t)(lo - 1u < 0x7F80u) << (8 * q + 2 * j);
      bits |= (uint32_t)(hi - 1u < 0x7F80u) << (8 * q + 2 * j + 1);
    }
  }
  return bits;
}

// Epilogue of one warp's 32 accumulator rows x BN columns: TMEM -> bf16 (+ReLU or
// mask) -> a 4 KB staging tile in shared memory laid out as the store tensor map's
// 128-byte swizzle (row r, 16-byte chunk c at r*128 + ((c ^ (r % 8)) * 16)) -> one TMA
// store per 64 columns, under an L2 evict-first policy: a GEMM's output is far larger
// than L2 and read by the next kernel, so it should not push out the operand strips
// that this kernel's other tiles are about to read again.  Rows past n_e land in the expert's own padding rows (rows
// per expert are a multiple of 128), which nothing reads as data.  The TMA engine
// writes whole 128-byte rows, instead of each thread storing 16 bytes to 32
// different rows per instruction.  `mrow` (kEpiMask) points at this lane's row of h
// at the tile's first column; `zero` stores zeros without reading TMEM.
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

template <int BN, int EPI>
__device__ __forceinline__ void store_rows(const CUtensorMap* tmD, uint32_t tmem_rows,
                                           uint32_t stage, int row0, int col0, int lane,
                                           const uint16_t* mrow = nullptr, bool zero = false,
                                           uint32_t* brow = nullptr, const uint32_t* bw = nullptr,
                                           int64_t bstride = 0, const ScatterY* sy = nullptr,
                                           int row_end = 0) {
  if (EPI == kEpiGateY) {
    // this lane's row: its token and gate (rows at or past the expert's kept count: none)
    const int r = row0 + lane;
    const bool valid = r < row_end;
    const int tk = valid ? __ldg(sy->tok + r) : -1;
    const float g = valid ? __ldg(sy->gsc + r) : 0.f;
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(sy->y);
#pragma unroll 1
    for (int b = 0; b < BN / 64; ++b) {
      __syncwarp();                            // the previous chunk's staging reads are done
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_rows + b * 64 + h * 32, v);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          pk[j] = pack_bf16x2(g * __uint_as_float(v[2 * j]), g * __uint_as_float(v[2 * j + 1]));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t cc = h * 4 + j;
          st_shared_v4(stage + lane * 128 + ((cc ^ (lane & 7)) << 4), pk[4 * j], pk[4 * j + 1],
                       pk[4 * j + 2], pk[4 * j + 3]);
        }
      }
      __syncwarp();
      // eight lanes per row: each row's 128 bytes go out as one coalesced segment
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3), c = lane & 7;
        const int tr = __shfl_sync(0xffffffffu, tk, rr);
        if (tr >= 0) {
          const uint4 val = ld_shared_v4(stage + rr * 128 + ((c ^ (rr & 7)) << 4));
          *reinterpret_cast<uint4*>(y + (int64_t)tr * sy->ldy + col0 + b * 64 + c * 8) = val;
        }
      }
    }
    return;
  }
  if (EPI == kEpiF32) {
    // fp32 result: 32 columns (128 bytes) per row per store, same swizzled staging
#pragma unroll 1
    for (int b = 0; b < BN / 32; ++b) {
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
      uint32_t r[32];
      if (zero) {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      } else {
        tmem_ld_32x32b_x32(tmem_rows + b * 32, r);
        tmem_ld_wait();
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(stage + lane * 128 + ((j ^ (lane & 7)) << 4), r[4 * j], r[4 * j + 1], r[4 * j + 2],
                     r[4 * j + 3]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d_hint(tmD, stage, col0 + b * 32, row0, l2_policy_evict_first());
        bulk_commit();
      }
    }
    return;
  }
  // kEpiMask: the mask of 64-column chunk b + 1 is in flight while chunk b is stored
  uint4 mnext[8];
  if (EPI == kEpiMask) {
    const uint4* mp = reinterpret_cast<const uint4*>(mrow);
#pragma unroll
    for (int j = 0; j < 8; ++j) mnext[j] = ld_nc_v4(mp + j);
  }
#pragma unroll 1
  for (int b = 0; b < BN / 64; ++b) {
    uint4 mcur[8];
    if (EPI == kEpiMask) {
#pragma unroll
      for (int j = 0; j < 8; ++j) mcur[j] = mnext[j];
      if (b + 1 < BN / 64) {
        const uint4* mp = reinterpret_cast<const uint4*>(mrow + (b + 1) * 64);
#pragma unroll
        for (int j = 0; j < 8; ++j) mnext[j] = ld_nc_v4(mp + j);
      }
    }
    if (lane == 0) bulk_wait_read0();          // the previous store has read the staging tile
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t keep = 0xFFFFFFFFu;
      if (EPI == kEpiMask) {
        const uint4 mv[4] = {mcur[4 * h], mcur[4 * h + 1], mcur[4 * h + 2], mcur[4 * h + 3]};
        keep = positive_bits(mv);
      } else if (EPI == kEpiMaskBits) {
        keep = bw[2 * b + h];
      }
      uint32_t r[32];
      if (zero) {
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = 0u;
      } else {
        tmem_ld_32x32b_x32(tmem_rows + b * 64 + h * 32, r);
        tmem_ld_wait();
      }
      uint32_t pk[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float a = __uint_as_float(r[2 * j]), c = __uint_as_float(r[2 * j + 1]);
        if (EPI == kEpiRelu || EPI == kEpiReluBits) {
          a = fmaxf(a, 0.f);
          c = fmaxf(c, 0.f);
        } else if (EPI == kEpiMask || EPI == kEpiMaskBits) {
          a = ((keep >> (2 * j)) & 1u) ? a : 0.f;
          c = ((keep >> (2 * j + 1)) & 1u) ? c : 0.f;
        }
        pk[j] = pack_bf16x2(a, c);
      }
      if (EPI == kEpiReluBits) {    // positive stored values: bit patterns 0x0001 .. 0x7f80
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          word |= (uint32_t)((pk[j] & 0xFFFFu) - 1u < 0x7F80u) << (2 * j);
          word |= (uint32_t)((pk[j] >> 16) - 1u < 0x7F80u) << (2 * j + 1);
        }
        brow[(int64_t)(2 * b + h) * bstride] = word;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t cc = h * 4 + j;
        st_shared_v4(stage + lane * 128 + ((cc ^ (lane & 7)) << 4), pk[4 * j], pk[4 * j + 1],
                     pk[4 * j + 2], pk[4 * j + 3]);
      }
    }
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d_hint(tmD, stage, col0 + b * 64, row0, l2_policy_evict_first());
      bulk_commit();
    }
  }
}

// BKM = false: B[e] is [K, N] (N contiguous, the forward's weights).  BKM = true:
// B[e] is [N, K] (K contiguous): the backward's products with a transposed weight,
// dY W2[e]^T and dP W1[e]^T, read the weights in their stored layout.
template <int BN, int EPI, bool BKM>
__global__ void __launch_bounds__(kThreads, 1)
    ffn_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmD, const int32_t* __restrict__ nexp, int E,
                  int64_t Cbuf, int K, int N, const uint16_t* __restrict__ mask, int64_t row_limit,
                  uint32_t* __restrict__ bits, unsigned* err, uint64_t limit_ns, int rest_only,
                  const ScatterY sy, const int32_t* __restrict__ row_base) {
  using C = Cfg<BN>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;                 // 1024-aligned for swizzle
  unsigned char* gbase = smem_raw + (base - raw_base);
  const uint32_t staging0 = base + C::STAGES * C::STAGE_BYTES;        // 4 x 4 KB store tiles
  const uint32_t bar0 = staging0 + C::STAGING;
  // barriers: full[S], empty[S], tfull[2], tempty[2], done
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 4);
  unsigned char* misc = gbase + C::STAGES * C::STAGE_BYTES + C::STAGING + 512;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* tile_pre = reinterpret_cast<int*>(misc + 16);                 // [E+1]
  int* mtiles = tile_pre + (kMaxExperts + 1);                        // [E]
  int* rbase = mtiles + kMaxExperts;                                 // [E] first row of the tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = N / BN;
  const int KB = K / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();                          // the producing kernel's rows and counts are complete
  if (warp == 2) {
    // tile prefix over experts (warp-parallel scan, ceil(E/32) experts per lane)
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int sum = 0;
    for (int e = e0; e < min(E, e0 + per); ++e) {
      const int n = nexp[e];
      // rest_only: the rows after those the CTA-pair kernel takes (256-row tiles up to
      // 256 * ((n + 127) / 256)), at most 128 of them: one tile or none
      const int r0 = rest_only ? (n + 127) / 256 * 256 : 0;
      const int m = (n - r0 + BM - 1) / BM;
      rbase[e] = r0 + (row_base ? row_base[e] : 0);   // row_base: the tiles start at that row
      mtiles[e] = m;
      sum += m * NT;
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    int run = inc - sum;
    for (int e = e0; e < min(E, e0 + per); ++e) {
      tile_pre[e] = run;
      run += mtiles[e] * NT;
    }
    if (lane == 31) tile_pre[E] = inc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      TileIter it{tile_pre, mtiles, E, NT, 0};
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      int e, mt, nt;
      for (int tile = blockIdx.x; ok && it.decode(tile, e, mt, nt); tile += gridDim.x) {
        const int rowA = (int)(e * Cbuf + rbase[e] + mt * BM);
        const int rowB = e * K;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = base + s * C::STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
          tma_load_2d(sa, &tmA, full_bar(s), kb * BK, rowA);
          if (BKM) {
            tma_load_2d(sa + A_BYTES, &tmB, full_bar(s), kb * BK, e * N + nt * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(sa + A_BYTES + j * 8192u, &tmB, full_bar(s), nt * BN + j * 64,
                          rowB + kb * BK);
          }
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {   // let copies in flight land before the CTA exits
        for (int q = 0; q < C::STAGES; ++q)
          if ((issued >> q) & 1u) mbar_wait(full_bar(q), (issued_par >> q) & 1u, err, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      TileIter it{tile_pre, mtiles, E, NT, 0};
      const uint32_t idesc = idesc_bf16<BN>(false, !BKM);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int e, mt, nt, i = 0;
      for (int tile = blockIdx.x; ok && it.decode(tile, e, mt, nt); tile += gridDim.x, ++i) {
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (*abort_flag || !mbar_wait(tempty_bar(acc), aph ^ 1u, err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(full_bar(s), ph, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * C::STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(sa + kk * 32u, 16u, 1024u);
            const uint64_t bd = BKM ? desc_sw128(sb + kk * 32u, 16u, 1024u)
                                    : desc_sw128(sb + kk * 2048u, 8192u, 1024u);
            tc_mma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit(empty_bar(s));
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc_commit(tfull_bar(acc));
      }
      if (!ok) {   // let issued MMAs finish before TMEM is released
        tc_commit(done_bar);
        mbar_wait(done_bar, 0, err, limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                     // TMEM lane quarter this warp may access
    const uint32_t stage = staging0 + (warp - 2) * 4096u;
    TileIter it{tile_pre, mtiles, E, NT, 0};
    int e, mt, nt, i = 0;
    for (int tile = blockIdx.x; it.decode(tile, e, mt, nt); tile += gridDim.x, ++i) {
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      const int row0 = (int)(e * Cbuf + rbase[e] + mt * BM + q * 32);
      const uint16_t* mrow = EPI == kEpiMask ? mask + (int64_t)(row0 + lane) * N + nt * BN : nullptr;
      if (EPI == kEpiMask) {           // bring this row's mask into L2 while the MMAs run
#pragma unroll
        for (int c = 0; c < BN * 2 / 128; ++c) prefetch_l2(reinterpret_cast<const char*>(mrow) + c * 128);
      }
      const int64_t bstride = (int64_t)E * Cbuf;
      uint32_t* brow = (EPI == kEpiReluBits || EPI == kEpiMaskBits)
                           ? bits + (int64_t)nt * (BN / 32) * bstride + row0 + lane : nullptr;
      uint32_t bw[BN / 32];
      if (EPI == kEpiMaskBits) {       // this row's mask words, loaded while the MMAs run
#pragma unroll
        for (int w = 0; w < BN / 32; ++w) bw[w] = __ldg(brow + w * bstride);
      }
      if (*abort_flag || !mbar_wait(tfull_bar(acc), aph, err, limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      if (row0 < row_limit)           // a store box starts inside the tensor (TMA clips its tail)
        store_rows<BN, EPI>(&tmD, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN, stage, row0,
                            nt * BN, lane, mrow, false, brow, bw, bstride, &sy,
                            (int)(e * Cbuf) + (EPI == kEpiGateY ? rbase[e] + __ldg(nexp + e) : 0));
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
    }
    if (lane == 0) bulk_wait0();                // stores complete before the CTA exits
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- weight gradients
//
//   D[e] = A[e, :n_e, :]^T . B[e, :n_e, :]        A [E*Cbuf, P], B [E*Cbuf, Q], D [E*P, Q]
//
// the backward's dW2[e] = h_e^T dY_e (P = H, Q = M) and dW1[e] = X_e^T dP_e (P = M,
// Q = H).  The reduction runs over the expert's kept slots, so both operands are
// read "MN-major" (slot rows, P or Q contiguous) in 64 x 64 TMA boxes and the MMA
// takes them transposed.  The k-loop covers ceil(n_e / 64) blocks; rows n_e ..
// ceil64(n_e) - 1 of both operands must hold zeros (the caller clears them), or lie
// past the tensor maps' last row (TMA fills zeros).  An expert with no kept slot
// gets D[e] = 0 (its tiles store zeros without an MMA), or keeps D[e] untouched when
// store_zero is 0.  EPI = kEpiF32 stores the
// fp32 accumulator; the "experts" may also be consecutive row ranges of one
// operand pair (a split of a long reduction, whose partial results the caller adds).
// Tiles are (expert, p-tile, q-tile), q fastest; roles as in ffn_tc_kernel.
template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    wgrad_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmD, const int32_t* __restrict__ nexp,
                    int E, int64_t Cbuf, int P, int Q, int store_zero, unsigned* err,
                    uint64_t limit_ns) {
  using C = Cfg<BN>;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw_base);
  const uint32_t staging0 = base + C::STAGES * C::STAGE_BYTES;
  const uint32_t bar0 = staging0 + C::STAGING;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * C::STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 4);
  unsigned char* misc = gbase + C::STAGES * C::STAGE_BYTES + C::STAGING + 512;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* kblocks = reinterpret_cast<int*>(misc + 16);                  // [E]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int PT = (P + BM - 1) / BM, QT = Q / BN;
  const int per_e = PT * QT, total = E * per_e;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 128);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();                          // operands and counts complete
  if (warp == 2)
    for (int e = lane; e < E; e += 32) kblocks[e] = (min(nexp[e], (int)Cbuf) + BK - 1) / BK;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const int e = tile / per_e, r = tile - e * per_e;
        const int pt = r / QT, qt = r - pt * QT;
        const int KB = kblocks[e];
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = base + s * C::STAGE_BYTES;
          const int row = (int)(e * Cbuf + kb * BK);
          mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
          // columns of A past P (a half-filled last p-tile) read as zeros
#pragma unroll
          for (int j = 0; j < BM / 64; ++j) tma_load_2d(sa + j * 8192u, &tmA, full_bar(s), pt * BM + j * 64, row);
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sa + A_BYTES + j * 8192u, &tmB, full_bar(s), qt * BN + j * 64, row);
          issued |= 1u << s;
          issued_par = (issued_par & ~(1u << s)) | (ph << s);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        for (int q = 0; q < C::STAGES; ++q)
          if ((issued >> q) & 1u) mbar_wait(full_bar(q), (issued_par >> q) & 1u, err, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16<BN>(true, true);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int i = 0;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        const int e = tile / per_e;
        const int KB = kblocks[e];
        if (KB == 0) continue;                  // zero tile: the epilogue stores zeros
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        ++i;
        if (*abort_flag || !mbar_wait(tempty_bar(acc), aph ^ 1u, err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(full_bar(s), ph, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * C::STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(sa + kk * 2048u, 8192u, 1024u);
            const uint64_t bd = desc_sw128(sb + kk * 2048u, 8192u, 1024u);
            tc_mma_f16(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit(empty_bar(s));
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc_commit(tfull_bar(acc));
      }
      if (!ok) {
        tc_commit(done_bar);
        mbar_wait(done_bar, 0, err, limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    const uint32_t stage = staging0 + (warp - 2) * 4096u;
    int i = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int e = tile / per_e, r = tile - e * per_e;
      const int pt = r / QT, qt = r - pt * QT;
      const bool zero = kblocks[e] == 0;
      const int prow = pt * BM + q * 32;        // P is a multiple of 64: warps hold 32 rows or none
      const int row0 = e * P + prow;
      int acc = 0;
      if (!zero) {
        acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        ++i;
        if (*abort_flag || !mbar_wait(tfull_bar(acc), aph, err, limit_ns)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
      }
      if (prow < P && (!zero || store_zero))
        store_rows<BN, EPI>(&tmD, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN, stage, row0,
                            qt * BN, lane, nullptr, zero);
      if (!zero) {
        tc_fence_before();
        mbar_arrive(tempty_bar(acc));
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA-pair variant
//
// Two CTAs of a cluster compute one 256 x 256 tile with cta_group::2 MMAs: CTA r
// holds rows [128r, 128r+128) of the A tile and columns [128r, 128r+128) of the
// B tile, so each SM loads 32 KB per k-block for the same MMA work that takes
// 48 KB in the one-CTA kernel (the loads, not the tensor cores, bound that one).
// The leader (rank 0) issues the MMAs; its full barrier counts the TMA bytes of
// both CTAs; its commits arrive on both CTAs' barriers; both CTAs' epilogues
// release an accumulator by arriving on the leader's barrier.
namespace pairk {
constexpr int BN = 256;                                   // pair tile columns
constexpr int PM = 256;                                   // pair tile rows
constexpr uint32_t B_HALF_BYTES = BK * (BN / 2) * 2;      // 16 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_HALF_BYTES;  // 32 KB per CTA
constexpr int STAGES = 6;
constexpr uint32_t TMEM_COLS = 2 * BN;                    // double-buffered accumulator
constexpr uint32_t STAGING = 4 * 4096;                   // one 32 x 64 bf16 store tile per epilogue warp
constexpr size_t SMEM =
    1024 + (size_t)STAGES * STAGE_BYTES + STAGING + 512 + 16 + 4 * (4 * kMaxExperts + 1);
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;            // shared::cluster address -> rank 0
static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
static_assert(SMEM + 1024 + 80 * 1024 > 228 * 1024, "a GEMM CTA must own its SM (as Cfg)");
static_assert(TMEM_COLS <= 512, "TMEM columns");
}  // namespace pairk

// EPI and BKM as in ffn_tc_kernel; with BKM each CTA's B box is its 128 rows of
// the [N, K] weight (box {64, 128}).
template <int EPI, bool BKM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ffn_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmD, const int32_t* __restrict__ nexp, int E,
                   int64_t Cbuf, int K, int N, const uint16_t* __restrict__ mask,
                   uint32_t* __restrict__ bits, unsigned* err, uint64_t limit_ns, int leave_rest,
                   const ScatterY sy, const int32_t* __restrict__ row_base) {
  using namespace pairk;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;   // same offset in both CTAs
  unsigned char* gbase = smem_raw + (base - raw_base);
  const uint32_t staging0 = base + STAGES * STAGE_BYTES;             // 4 x 4 KB store tiles
  const uint32_t bar0 = staging0 + STAGING;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
  unsigned char* misc = gbase + STAGES * STAGE_BYTES + STAGING + 512;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* tile_pre = reinterpret_cast<int*>(misc + 16);
  int* mtiles = tile_pre + (kMaxExperts + 1);
  int* nrows = mtiles + kMaxExperts;
  int* rbase = nrows + kMaxExperts;      // [E] first row of each expert's tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int NT = N / BN;
  const int KB = K / BK;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * 128);     // epilogue threads of both CTAs
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32((const void*)tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  pdl_wait();                          // the producing kernel's rows and counts are complete
  if (warp == 2) {
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int sum = 0;
    for (int e = e0; e < min(E, e0 + per); ++e) {
      const int n = nexp[e];
      // leave_rest: a last block of at most 128 rows is left to the one-CTA kernel
      const int m = leave_rest ? (n + 127) / PM : (n + PM - 1) / PM;
      nrows[e] = n;
      rbase[e] = row_base ? row_base[e] : 0;   // row_base: the tiles start at that row
      mtiles[e] = m;
      sum += m * NT;
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    int run = inc - sum;
    for (int e = e0; e < min(E, e0 + per); ++e) {
      tile_pre[e] = run;
      run += mtiles[e] * NT;
    }
    if (lane == 31) tile_pre[E] = inc;
  }
  tc_fence_before();
  cluster_sync_all();          // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      TileIter it{tile_pre, mtiles, E, NT, 0};
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int e, mt, nt;
      for (int tile = pair; ok && it.decode(tile, e, mt, nt); tile += npairs) {
        const int rowA = (int)(e * Cbuf + rbase[e] + mt * PM + rank * (PM / 2));
        const int rowB = e * K;
        const int colB = nt * BN + rank * (BN / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t fb = full_bar(s) & kPeerBitMask;     // the leader's full barrier
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * STAGE_BYTES);
          tma_load_2d_pair(sa, &tmA, fb, kb * BK, rowA);
          if (BKM) {
            tma_load_2d_pair(sa + A_BYTES, &tmB, fb, kb * BK, e * N + colB);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tma_load_2d_pair(sa + A_BYTES + j * 8192u, &tmB, fb, colB + j * 64, rowB + kb * BK);
          }
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      TileIter it{tile_pre, mtiles, E, NT, 0};
      // kind::f16, D fp32, A bf16 K-major, B bf16 MN-major (K-major with BKM), M=256, N=256
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(!BKM) << 16) |
                             ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(PM >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int e, mt, nt, i = 0;
      for (int tile = pair; ok && it.decode(tile, e, mt, nt); tile += npairs, ++i) {
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (*abort_flag || !mbar_wait(tempty_bar(acc), aph ^ 1u, err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(full_bar(s), ph, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(sa + kk * 32u, 16u, 1024u);
            const uint64_t bd = BKM ? desc_sw128(sb + kk * 32u, 16u, 1024u)
                                    : desc_sw128(sb + kk * 2048u, 8192u, 1024u);
            tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit_pair(empty_bar(s), 0x3);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc_commit_pair(tfull_bar(acc), 0x3);
      }
      if (!ok) {
        tc_commit_pair(done_bar, 0x1);
        mbar_wait(done_bar, 0, err, limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const uint32_t stage = staging0 + (warp - 2) * 4096u;
    TileIter it{tile_pre, mtiles, E, NT, 0};
    int e, mt, nt, i = 0;
    for (int tile = pair; it.decode(tile, e, mt, nt); tile += npairs, ++i) {
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      const int row0 = (int)(e * Cbuf + rbase[e] + mt * PM + (int)rank * (PM / 2) + q * 32);
      const uint16_t* mrow = EPI == kEpiMask ? mask + (int64_t)(row0 + lane) * N + nt * BN : nullptr;
      const int64_t bstride = (int64_t)E * Cbuf;
      uint32_t* brow = (EPI == kEpiReluBits || EPI == kEpiMaskBits)
                           ? bits + (int64_t)nt * (BN / 32) * bstride + row0 + lane : nullptr;
      uint32_t bw[BN / 32];
      if (EPI == kEpiMaskBits) {       // this row's mask words, loaded while the MMAs run
#pragma unroll
        for (int w = 0; w < BN / 32; ++w) bw[w] = __ldg(brow + w * bstride);
      }
      if (*abort_flag || !mbar_wait(tfull_bar(acc), aph, err, limit_ns)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      store_rows<BN, EPI>(&tmD, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN, stage, row0,
                          nt * BN, lane, mrow, false, brow, bw, bstride, &sy,
                          (int)(e * Cbuf) + (EPI == kEpiGateY ? rbase[e] + __ldg(nexp + e) : 0));
      tc_fence_before();
      if (leader) mbar_arrive(tempty_bar(acc));
      else mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync_all();          // no CTA leaves while its pair may still use its smem or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Weight gradients on CTA pairs: D[e] tile of 256 (P) x 256 (Q) per pair, CTA r holding
// rows [128r, 128r+128) of the tile (its A columns) and columns [128r, 128r+128) of
// B.  Both operands MN-major as in wgrad_tc_kernel; the k-loop covers the expert's
// kept slots in 64-slot blocks (the caller clears the rows up to the next multiple
// of 64).  An expert with no kept slot gets zero tiles, stored by both CTAs without
// an MMA.  Same barrier and TMEM handshake as ffn_tc2_kernel.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    wgrad_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmD, const int32_t* __restrict__ nexp, int E,
                     int64_t Cbuf, int P, int Q, int store_zero, unsigned* err, uint64_t limit_ns) {
  using namespace pairk;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;   // same offset in both CTAs
  unsigned char* gbase = smem_raw + (base - raw_base);
  const uint32_t staging0 = base + STAGES * STAGE_BYTES;
  const uint32_t bar0 = staging0 + STAGING;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
  unsigned char* misc = gbase + STAGES * STAGE_BYTES + STAGING + 512;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  int* kblocks = reinterpret_cast<int*>(misc + 16);                  // [E]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int PT = (P + PM - 1) / PM, QT = Q / BN;
  const int per_e = PT * QT, total = E * per_e;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * 128);     // epilogue threads of both CTAs
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32((const void*)tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  pdl_wait();                          // operands and counts complete
  if (warp == 2)
    for (int e = lane; e < E; e += 32) kblocks[e] = (min(nexp[e], (int)Cbuf) + BK - 1) / BK;
  tc_fence_before();
  cluster_sync_all();          // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const int e = tile / per_e, r = tile - e * per_e;
        const int pt = r / QT, qt = r - pt * QT;
        const int KB = kblocks[e];
        const int colA = pt * PM + (int)rank * (PM / 2), colB = qt * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(empty_bar(s), ph ^ 1u, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t fb = full_bar(s) & kPeerBitMask;     // the leader's full barrier
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * STAGE_BYTES);
          const int row = (int)(e * Cbuf + kb * BK);
          // columns of A past P (the second CTA of a half-filled last p-tile) read as zeros
#pragma unroll
          for (int j = 0; j < 2; ++j) tma_load_2d_pair(sa + j * 8192u, &tmA, fb, colA + j * 64, row);
#pragma unroll
          for (int j = 0; j < 2; ++j)
            tma_load_2d_pair(sa + A_BYTES + j * 8192u, &tmB, fb, colB + j * 64, row);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && leader) {
      // kind::f16, D fp32, A and B bf16 MN-major, M=256, N=256
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                             ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(PM >> 4) << 24);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int i = 0;
      for (int tile = pair; ok && tile < total; tile += npairs) {
        const int KB = kblocks[tile / per_e];
        if (KB == 0) continue;                  // zero tile: the epilogues store zeros
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        ++i;
        if (*abort_flag || !mbar_wait(tempty_bar(acc), aph ^ 1u, err, limit_ns)) {
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (*abort_flag || !mbar_wait(full_bar(s), ph, err, limit_ns)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_sw128(sa + kk * 2048u, 8192u, 1024u);
            const uint64_t bd = desc_sw128(sb + kk * 2048u, 8192u, 1024u);
            tc_mma_f16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          tc_commit_pair(empty_bar(s), 0x3);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) tc_commit_pair(tfull_bar(acc), 0x3);
      }
      if (!ok) {
        tc_commit_pair(done_bar, 0x1);
        mbar_wait(done_bar, 0, err, limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const uint32_t stage = staging0 + (warp - 2) * 4096u;
    int i = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const int e = tile / per_e, r = tile - e * per_e;
      const int pt = r / QT, qt = r - pt * QT;
      const bool zero = kblocks[e] == 0;
      const int prow = pt * PM + (int)rank * (PM / 2) + q * 32;   // P is a multiple of 64
      int acc = 0;
      if (!zero) {
        acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        ++i;
        if (*abort_flag || !mbar_wait(tfull_bar(acc), aph, err, limit_ns)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
      }
      if (prow < P && (!zero || store_zero))
        store_rows<BN, kEpiNone>(&tmD, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN, stage,
                                 e * P + prow, qt * BN, lane, nullptr, zero);
      if (!zero) {
        tc_fence_before();
        if (leader) mbar_arrive(tempty_bar(acc));
        else mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync_all();          // no CTA leaves while its pair may still use its smem or TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
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

// 2-D row-major tensor of `outer` rows x `inner` elements (row pitch `pitch` bytes,
// 0 = dense), 128-byte swizzle.
bool encode_2d(CUtensorMap* tm, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_in,
               uint32_t box_out, bool f32 = false, uint64_t pitch = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch ? pitch : inner * es};
  cuuint32_t box[2] = {box_in, box_out};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI, bool BKM>
cudaError_t launch_pair(const GemmPlan& p, const int32_t* nexp, unsigned* err, uint64_t limit_ns,
                        int num_sms, cudaStream_t st, int leave_rest = 0) {
  auto kern = ffn_tc2_kernel<EPI, BKM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)pairk::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(num_sms & ~1), dim3(kThreads), pairk::SMEM, st, p.tmA,
                    BKM ? p.tmB2 : p.tmB, p.tmD, nexp, p.E, p.Cbuf, p.K, p.N,
                    static_cast<const uint16_t*>(p.mask), p.bits, err, limit_ns, leave_rest, p.sy, p.row_base);
}

template <int BN, int EPI, bool BKM>
cudaError_t launch_t(const GemmPlan& p, const int32_t* nexp, unsigned* err, uint64_t limit_ns,
                     int num_sms, cudaStream_t st, int rest_only = 0) {
  auto kern = ffn_tc_kernel<BN, EPI, BKM>;
  const size_t smem = Cfg<BN>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t row_limit = p.row_limit > 0 ? p.row_limit : (int64_t)p.E * p.Cbuf;
  return launch_pdl(kern, dim3(num_sms), dim3(kThreads), smem, st, p.tmA, p.tmB, p.tmD, nexp, p.E,
                    p.Cbuf, p.K, p.N, static_cast<const uint16_t*>(p.mask), row_limit, p.bits, err,
                    limit_ns, rest_only, p.sy, p.row_base);
}

template <int BN, int EPI>
cudaError_t launch_w(const GemmPlan& p, const int32_t* nexp, unsigned* err, uint64_t limit_ns,
                     int num_sms, cudaStream_t st) {
  auto kern = wgrad_tc_kernel<BN, EPI>;
  const size_t smem = Cfg<BN>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(num_sms), dim3(kThreads), smem, st, p.tmA, p.tmB, p.tmD, nexp, p.E,
                    p.Cbuf, p.K, p.N, p.skip_zero ? 0 : 1, err, limit_ns);
}

cudaError_t launch_w2(const GemmPlan& p, const int32_t* nexp, unsigned* err, uint64_t limit_ns,
                      int num_sms, cudaStream_t st) {
  auto kern = wgrad_tc2_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)pairk::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(num_sms & ~1), dim3(kThreads), pairk::SMEM, st, p.tmA, p.tmB, p.tmD,
                    nexp, p.E, p.Cbuf, p.K, p.N, p.skip_zero ? 0 : 1, err, limit_ns);
}

int pick_bn(int N) { return (N % 256 == 0) ? 256 : (N % 128 == 0 ? 128 : 64); }

}  // namespace

bool make_gemm_plan(GemmPlan& p, const void* A, const void* B, void* D, int E, int64_t Cbuf, int K,
                    int N, bool relu) {
  p = GemmPlan{};
  p.kind = kGemmFwd;
  p.E = E;
  p.Cbuf = Cbuf;
  p.K = K;
  p.N = N;
  p.D = D;
  p.relu = relu;
  p.BN = pick_bn(N);
  p.pair = (N % pairk::BN) == 0;      // CTA-pair kernel whenever the 256-wide tile divides N
  if (K % BK || N % 64) return false;
  if (!encode_2d(&p.tmA, A, (uint64_t)K, (uint64_t)E * Cbuf, BK, BM)) return false;
  if (!encode_2d(&p.tmB, B, (uint64_t)N, (uint64_t)E * K, 64, BK)) return false;
  if (!encode_2d(&p.tmD, D, (uint64_t)N, (uint64_t)E * Cbuf, 64, 32)) return false;
  return true;
}

bool make_dgrad_plan(GemmPlan& p, const void* A, const void* Bt, void* D, const void* mask, int E,
                     int64_t Cbuf, int K, int N) {
  p = GemmPlan{};
  p.kind = kGemmDgrad;
  p.E = E;
  p.Cbuf = Cbuf;
  p.K = K;
  p.N = N;
  p.D = D;
  p.mask = mask;
  p.BN = pick_bn(N);
  p.pair = (N % pairk::BN) == 0;
  if (K % BK || N % 64) return false;
  if (!encode_2d(&p.tmA, A, (uint64_t)K, (uint64_t)E * Cbuf, BK, BM)) return false;
  if (!encode_2d(&p.tmB, Bt, (uint64_t)K, (uint64_t)E * N, BK, (uint32_t)p.BN)) return false;
  if (p.pair && !encode_2d(&p.tmB2, Bt, (uint64_t)K, (uint64_t)E * N, BK, pairk::BN / 2)) return false;
  if (!encode_2d(&p.tmD, D, (uint64_t)N, (uint64_t)E * Cbuf, 64, 32)) return false;
  return true;
}

bool make_wgrad_plan(GemmPlan& p, const void* A, const void* B, void* D, int E, int64_t Cbuf, int P,
                     int Q, bool f32out, int64_t rows_ab) {
  p = GemmPlan{};
  p.kind = kGemmWgrad;
  p.E = E;
  p.Cbuf = Cbuf;
  p.K = P;                             // rows of each expert's result
  p.N = Q;
  p.D = D;
  p.f32out = f32out;
  p.BN = pick_bn(Q);
  p.pair = !f32out && (Q % pairk::BN) == 0;   // wgrad_tc2_kernel: 256 x 256 tiles on CTA pairs
  if (P % 64 || Q % 64 || Cbuf % BK) return false;
  const uint64_t rows = rows_ab > 0 ? (uint64_t)rows_ab : (uint64_t)E * Cbuf;
  if (!encode_2d(&p.tmA, A, (uint64_t)P, rows, 64, BK)) return false;
  if (!encode_2d(&p.tmB, B, (uint64_t)Q, rows, 64, BK)) return false;
  if (!encode_2d(&p.tmD, D, (uint64_t)Q, (uint64_t)E * P, f32out ? 32 : 64, 32, f32out)) return false;
  return true;
}

bool make_gate_dx_plan(GemmPlan& p, const void* dlb, int64_t S, int EPb, const void* wsplit,
                       int EPr, void* dx, int M) {
  p = GemmPlan{};
  p.kind = kGemmFwd;
  p.E = 1;
  p.Cbuf = S;
  p.K = EPb;
  p.N = M;
  p.D = dx;
  p.BN = pick_bn(M);
  if (EPb % BK || M % 64 || 3 * EPr < EPb) return false;
  // A: the hi half of dl's bf16 split, rows of 2*EPb elements
  if (!encode_2d(&p.tmA, dlb, (uint64_t)EPb, (uint64_t)S, BK, BM, false, (uint64_t)EPb * 4)) return false;
  // B: W_g's hi part [EPr, M] (E contiguous rows past E are zero; rows EPr.. of the
  // next part only meet zero columns of A)
  if (!encode_2d(&p.tmB, wsplit, (uint64_t)M, (uint64_t)3 * EPr, 64, BK)) return false;
  if (!encode_2d(&p.tmD, dx, (uint64_t)M, (uint64_t)S, 64, 32)) return false;
  p.row_limit = S;
  return true;
}

template <int EPI>
cudaError_t launch_mixed(const GemmPlan& p, const int32_t* nexp, unsigned* err, uint64_t limit_ns,
                         int num_sms, cudaStream_t st) {
  cudaError_t e = launch_pair<EPI, false>(p, nexp, err, limit_ns, num_sms, st, 1);
  if (e != cudaSuccess) return e;
  switch (p.BN) {
    case 256: return launch_t<256, EPI, false>(p, nexp, err, limit_ns, num_sms, st, 1);
    case 128: return launch_t<128, EPI, false>(p, nexp, err, limit_ns, num_sms, st, 1);
    default: return launch_t<64, EPI, false>(p, nexp, err, limit_ns, num_sms, st, 1);
  }
}

cudaError_t launch_ffn_bf16(const GemmPlan& p, const int32_t* nexp, unsigned* err,
                            uint64_t wait_limit_ns, int num_sms, bool want_pair, cudaStream_t st,
                            bool mixed) {
  if (p.kind == kGemmWgrad) {
    if (!p.f32out && p.pair && want_pair) return launch_w2(p, nexp, err, wait_limit_ns, num_sms, st);
    if (p.f32out) {
      switch (p.BN) {
        case 256: return launch_w<256, kEpiF32>(p, nexp, err, wait_limit_ns, num_sms, st);
        case 128: return launch_w<128, kEpiF32>(p, nexp, err, wait_limit_ns, num_sms, st);
        default: return launch_w<64, kEpiF32>(p, nexp, err, wait_limit_ns, num_sms, st);
      }
    }
    switch (p.BN) {
      case 256: return launch_w<256, kEpiNone>(p, nexp, err, wait_limit_ns, num_sms, st);
      case 128: return launch_w<128, kEpiNone>(p, nexp, err, wait_limit_ns, num_sms, st);
      default: return launch_w<64, kEpiNone>(p, nexp, err, wait_limit_ns, num_sms, st);
    }
  }
  if (p.kind == kGemmDgrad) {
    const int epi = (p.bits && p.use_bits) ? kEpiMaskBits : (p.mask ? kEpiMask : kEpiNone);
    if (p.pair && want_pair && (p.Cbuf % pairk::PM) == 0) {
      if (epi == kEpiMaskBits) return launch_pair<kEpiMaskBits, true>(p, nexp, err, wait_limit_ns, num_sms, st);
      if (epi == kEpiMask) return launch_pair<kEpiMask, true>(p, nexp, err, wait_limit_ns, num_sms, st);
      return launch_pair<kEpiNone, true>(p, nexp, err, wait_limit_ns, num_sms, st);
    }
    switch (p.BN) {
      case 256:
        if (epi == kEpiMaskBits) return launch_t<256, kEpiMaskBits, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        if (epi == kEpiMask) return launch_t<256, kEpiMask, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        return launch_t<256, kEpiNone, true>(p, nexp, err, wait_limit_ns, num_sms, st);
      case 128:
        if (epi == kEpiMaskBits) return launch_t<128, kEpiMaskBits, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        if (epi == kEpiMask) return launch_t<128, kEpiMask, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        return launch_t<128, kEpiNone, true>(p, nexp, err, wait_limit_ns, num_sms, st);
      default:
        if (epi == kEpiMaskBits) return launch_t<64, kEpiMaskBits, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        if (epi == kEpiMask) return launch_t<64, kEpiMask, true>(p, nexp, err, wait_limit_ns, num_sms, st);
        return launch_t<64, kEpiNone, true>(p, nexp, err, wait_limit_ns, num_sms, st);
    }
  }
  // forward: ReLU (and the backward's mask bits when a bit buffer is set), none, or the
  // gate-scaled stores into the layer output
  const int epi = p.sy.y ? kEpiGateY : (p.relu ? (p.bits ? kEpiReluBits : kEpiRelu) : kEpiNone);
  if (epi == kEpiGateY) {
    if (p.pair && mixed && !want_pair && (p.Cbuf % pairk::PM) == 0)
      return launch_mixed<kEpiGateY>(p, nexp, err, wait_limit_ns, num_sms, st);
    if (p.pair && want_pair && (p.Cbuf % pairk::PM) == 0)
      return launch_pair<kEpiGateY, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    switch (p.BN) {
      case 256: return launch_t<256, kEpiGateY, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      case 128: return launch_t<128, kEpiGateY, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      default: return launch_t<64, kEpiGateY, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    }
  }
  if (p.pair && mixed && !want_pair && (p.Cbuf % pairk::PM) == 0) {
    // each expert's 256-row blocks on CTA pairs, a last block of at most 128 rows on
    // one-CTA tiles: as little padding as 128-row tiles, most rows at the pair rate
    if (epi == kEpiReluBits) return launch_mixed<kEpiReluBits>(p, nexp, err, wait_limit_ns, num_sms, st);
    if (epi == kEpiRelu) return launch_mixed<kEpiRelu>(p, nexp, err, wait_limit_ns, num_sms, st);
    return launch_mixed<kEpiNone>(p, nexp, err, wait_limit_ns, num_sms, st);
  }
  if (p.pair && want_pair && (p.Cbuf % pairk::PM) == 0) {
    if (epi == kEpiReluBits) return launch_pair<kEpiReluBits, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    if (epi == kEpiRelu) return launch_pair<kEpiRelu, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    return launch_pair<kEpiNone, false>(p, nexp, err, wait_limit_ns, num_sms, st);
  }
  switch (p.BN) {
    case 256:
      if (epi == kEpiReluBits) return launch_t<256, kEpiReluBits, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      if (epi == kEpiRelu) return launch_t<256, kEpiRelu, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      return launch_t<256, kEpiNone, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    case 128:
      if (epi == kEpiReluBits) return launch_t<128, kEpiReluBits, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      if (epi == kEpiRelu) return launch_t<128, kEpiRelu, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      return launch_t<128, kEpiNone, false>(p, nexp, err, wait_limit_ns, num_sms, st);
    default:
      if (epi == kEpiReluBits) return launch_t<64, kEpiReluBits, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      if (epi == kEpiRelu) return launch_t<64, kEpiRelu, false>(p, nexp, err, wait_limit_ns, num_sms, st);
      return launch_t<64, kEpiNone, false>(p, nexp, err, wait_limit_ns, num_sms, st);
  }
}

}  // namespace moe
