// apply_tc.cuh -- apply step on the 5th-generation tensor cores (bf16, d = 128).
//
//   O_n = (RoPE(ReLU(Q_n)) S) / (ReLU(Q_n) . z + eps) * sigmoid(G_n)
// (SANA-Video 2.0, Eq. (1); SANA-Video Sec. 3.2: rotated numerator, un-rotated denominator).
//
// Per 128-token tile one tcgen05 MMA chain computes the numerator D[128 tok x 128] =
// A[128 tok x 128 ch] * S[128 x 128].  A = RoPE(ReLU(Q)) is built on the CUDA cores and written
// to tensor memory (thread n owns token n and TMEM lane n), so a staged Q tile is released as
// soon as its rows are in registers; S is the unit's state as a bf16 operand (N-major) in shared
// memory.  The denominator, the divide and the gate run on the CUDA cores.  The rotation reads
// cos/sin from per-band tables (fp64-accurate, built by the prep kernel).
//
// Warps (one CTA per SM, persistent over a contiguous range of tiles):
//   warpgroup 0   warp 0: TMA producer of Q tiles (and the state operand once per unit)
//                 warp 1: MMA issuer (and TMEM owner); warp 2: TMA store of finished O tiles
//                 warp 3: TMA producer of G tiles
//   warpgroups 1-4  two math groups of two warpgroups each; group m takes local tiles
//                 i = m (mod 2) and its warpgroup h handles channels [64h, 64h+64) of every row
//                 (thread = token, as TMEM lanes require).  Software-pipelined: the group builds
//                 the A operand of its tile k in TMEM, then runs the epilogue of its tile k-1:
//                 its accumulator half is pulled into registers and released at once (so the MMA
//                 of tile k overlaps the rest of the epilogue), then scaled by 1/den and
//                 sigmoid(g) and rounded to bf16 in place over the staged G tile.  The two halves
//                 of a row swap their partial denominators through tensor memory.
// TMEM: group m owns accumulator columns [256m, 256m+128), A columns [256m+128, 256m+192) and
// partial-denominator columns [256m+192, 256m+196).  (Shared memory stays within the 196 KB
// configuration, so that L1 keeps room for the cos/sin table.)
// The control warpgroup hands registers to the math groups (setmaxnreg); the host checks the
// launch's register budget before launching.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

#ifndef LA_AP_QST
#define LA_AP_QST 2
#endif
#ifndef LA_AP_GST
#define LA_AP_GST 2
#endif
#ifndef LA_AP_NSB
#define LA_AP_NSB 2
#endif

namespace la {
namespace ap {

constexpr int TILE = 128;
constexpr int D = 128;
constexpr int QST = LA_AP_QST;  // Q stages (freed once the math group has read them)
constexpr int GST = LA_AP_GST;  // G / O stages (freed when the O tile has been stored)
constexpr int NSB = LA_AP_NSB;  // state operand buffers
constexpr int NWG = 2;          // math groups (two warpgroups each, one per channel half)
constexpr int MATH_WGS = 2 * NWG;
constexpr int THREADS = 128 * (1 + MATH_WGS);
constexpr uint32_t HALF = 128 * 128;
constexpr uint32_t BUF = 2 * HALF;  // 32 KB: a 128 x 128 bf16 tile
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_G = OFF_Q + QST * BUF;
constexpr uint32_t OFF_S = OFF_G + GST * BUF;
constexpr uint32_t OFF_BAR = OFF_S + NSB * BUF;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t GROUP_COLS = 256, ACC_COL = 0, A_COL = 128;
constexpr uint32_t DEN_COL = 192;  // + 2 * slot + half: partial denominators (fp32, lane = row)
constexpr uint32_t RMS_COL = 196;  // + 2 * slot + half: partial sums of squares (RMSNorm)
constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/true);
// Register split: the launch grants REGS_LAUNCH per thread (the largest multiple of 8 that fits
// 65536 / THREADS); the control warpgroup shrinks to REGS_CTRL and the math groups grow to
// REGS_MATH, never asking for more than the launch granted.
constexpr uint32_t REGS_LAUNCH = (65536 / THREADS) / 8 * 8;
constexpr uint32_t REGS_CTRL = 56;  // the single-lane control loops (the MMA issuer keeps per-group state)
constexpr uint32_t REGS_MATH_FIT = ((THREADS * REGS_LAUNCH - 128 * REGS_CTRL) / (128 * MATH_WGS)) / 8 * 8;
constexpr uint32_t REGS_MATH = REGS_MATH_FIT > 232 ? 232 : REGS_MATH_FIT;
constexpr bool SPLIT_REGS = true;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// Tile i uses Q stage i mod QST, G stage i mod GST and math group i mod 2, so each stage always
// serves the same group and no group polls a stage's barrier more than one phase ahead (which
// would alias the parity test).
static_assert(QST % NWG == 0 && GST % NWG == 0, "stages must be a multiple of the math groups");
static_assert(NWG * GROUP_COLS <= TMEM_COLS && A_COL + 64 <= DEN_COL && DEN_COL + 4 <= RMS_COL &&
                  RMS_COL + 4 <= GROUP_COLS,
              "TMEM columns");
static_assert(128 * REGS_CTRL + 128 * MATH_WGS * REGS_MATH <= THREADS * REGS_LAUNCH, "register split");
static_assert(REGS_CTRL <= REGS_LAUNCH && REGS_LAUNCH <= REGS_MATH, "register split");

struct Bars {
  uint64_t qfull[QST], qempty[QST];
  uint64_t gfull[GST], gempty[GST], ostaged[GST];
  uint64_t sfull[NSB], sfree[NSB];
  uint64_t aready[NWG], afree[NWG], accfull[NWG], accempty[NWG];
  uint64_t denx[NWG][4];  // the two warps holding the halves of rows 32q .. 32q+31 of group m
  uint64_t rmsx[NWG][4];  // the same pairs, for the RMSNorm sums of squares
  uint64_t final_;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block too large");

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <uint32_t R>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

// In place over half a row held in registers (channels [64 HF, 64 HF + 64) as 32 bf16 pairs,
// already ReLU'd): a <- RoPE(a).  Returns the half's share of ReLU(q) . z (un-rotated).
// (pt, ph, pw) is the token's grid position.
//   Band split fixed at compile time: `tab2` holds two consecutive pairs of a band per 16-byte
//   entry, t and h bands position-major and the w band [pair / 2][x], so a half row takes 16
//   vector loads, most of them at constant offsets from one per-band base.
//   Run-time split: pair i of band b at coordinate x reads `tab` at (band offset) +
//   i_in_band * extent_b + x.
template <int DT, int DH, int HF>
__device__ __forceinline__ float transform_half(uint32_t (&a)[32], const float* __restrict__ zg,
                                                const float2* __restrict__ tab, const float4* __restrict__ tab2,
                                                const Rope& rope, int pt, int ph, int pw, int ext_t, int ext_h,
                                                int ext_w) {
  uint64_t den2[4] = {0, 0, 0, 0};  // packed fp32 pairs: (even, odd) channel partial sums
  if constexpr (DT >= 0 && DH >= 0) {
    constexpr int DW = 128 - DT - DH;
    static_assert(DT % 4 == 0 && DH % 4 == 0 && DW % 4 == 0, "bands of whole 16-byte entries");
    const float4* bt = tab2 + pt * (DT / 4);
    const float4* bh = tab2 + rope.tab_off_h / 2 + ph * (DH / 4);
    const float4* bw = tab2 + rope.tab_off_w / 2 + pw;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int pi = 32 * HF + 2 * j;  // pairs pi, pi + 1 (same band: band edges are even)
      const int bnd = band_of<DT, DH>(pi, rope);
      const int e = pair_in_band<DT, DH>(pi, rope) / 2;
      const float4 cs = __ldg(bnd == 0 ? bt + e : (bnd == 1 ? bh + e : bw + e * ext_w));
      const ulonglong2 z4 = __ldg(reinterpret_cast<const ulonglong2*>(zg + 4 * j));
      const float x0 = bf16lo(a[2 * j]), x1 = bf16hi(a[2 * j]);
      const float y0 = bf16lo(a[2 * j + 1]), y1 = bf16hi(a[2 * j + 1]);
      den2[(2 * j) & 3] = fma2(pk(x0, x1), z4.x, den2[(2 * j) & 3]);
      den2[(2 * j + 1) & 3] = fma2(pk(y0, y1), z4.y, den2[(2 * j + 1) & 3]);
      a[2 * j] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
      a[2 * j + 1] = pack_bf16(y0 * cs.z - y1 * cs.w, y0 * cs.w + y1 * cs.z);
    }
  } else {
    const int it = pt, ih = static_cast<int>(rope.tab_off_h) + ph, iw = static_cast<int>(rope.tab_off_w) + pw;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      const ulonglong2 za = __ldg(reinterpret_cast<const ulonglong2*>(zg + c8 * 8));
      const ulonglong2 zc = __ldg(reinterpret_cast<const ulonglong2*>(zg + c8 * 8 + 4));
      const uint64_t zz[4] = {za.x, za.y, zc.x, zc.y};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = 4 * c8 + q;
        const int pi = 32 * HF + j;
        const int bnd = band_of<DT, DH>(pi, rope);
        const int loc = pair_in_band<DT, DH>(pi, rope);
        const int idx = bnd == 0 ? it + loc * ext_t : (bnd == 1 ? ih + loc * ext_h : iw + loc * ext_w);
        const float2 cs = __ldg(tab + idx);
        const float x0 = bf16lo(a[j]);
        const float x1 = bf16hi(a[j]);
        den2[q] = fma2(pk(x0, x1), zz[q], den2[q]);
        a[j] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
      }
    }
  }
  const float2 d0 = upk(den2[0]), d1 = upk(den2[1]), d2 = upk(den2[2]), d3 = upk(den2[3]);
  return ((d0.x + d0.y) + (d1.x + d1.y)) + ((d2.x + d2.y) + (d3.x + d3.y));
}

// RMS: RMSNorm of y = num / den over the row's 128 channels before the gate (SANA-Video 2.0,
// Eq. (1)), y / sqrt(mean(y^2) + norm_eps) * gamma (gamma may be null: 1).
template <int DT, int DH, bool RMS>
__global__ void __launch_bounds__(THREADS, 1)
apply_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                const __grid_constant__ CUtensorMap tmO, const Plan p, const __grid_constant__ Rope rope,
                const uint8_t* __restrict__ simg, const float* __restrict__ zimg,
                const float2* __restrict__ tab, const float4* __restrict__ tab2, const float* __restrict__ gamma,
                float norm_eps, __nv_bfloat16* __restrict__ O) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  const uint32_t sbase = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c);
  const int64_t g1 = cta_start(p, c + 1);
  const int64_t u_first = unit_of_tile(p, g0);
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QST; ++s) {
      mbar_init(&bars->qfull[s], 1);
      mbar_init(&bars->qempty[s], 8);
    }
    for (int s = 0; s < GST; ++s) {
      mbar_init(&bars->gfull[s], 1);
      mbar_init(&bars->gempty[s], 1);
      mbar_init(&bars->ostaged[s], 8);
    }
    for (int s = 0; s < NSB; ++s) {
      mbar_init(&bars->sfull[s], 1);
      mbar_init(&bars->sfree[s], 1);
    }
    for (int m = 0; m < NWG; ++m) {
      mbar_init(&bars->aready[m], 8);
      mbar_init(&bars->afree[m], 1);
      mbar_init(&bars->accfull[m], 1);
      mbar_init(&bars->accempty[m], 8);
      for (int q = 0; q < 4; ++q) {
        mbar_init(&bars->denx[m][q], 2);
        mbar_init(&bars->rmsx[m][q], 2);
      }
    }
    mbar_init(&bars->final_, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmG);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // The state image, z and the cos/sin tables come from the kernels before this one: the threads
  // that read them wait for those kernels; the G loads start at once.
  pdl_trigger();

  if (warp < 4) {
    regs_dec<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer: Q, state
      // A tile's Q is requested before its unit's state image, and only the image waits for the
      // kernels before (the first Q tiles land while they finish).
      int64_t issued_q = 0, issued_s = 0;
      int64_t prev_unit = -1;
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const TileInfo ti = tile_info(p, g);
        in_bounds(ti.unit < p.BH * p.nblk && ti.bh < p.BH && ti.n0 < ti.n_end && ti.n_end <= p.N);
        const int qs = static_cast<int>(i % QST);
        if (!mbar_wait(&bars->qempty[qs], static_cast<uint32_t>(((i / QST) & 1) ^ 1), abort_flag, LA_SLEEP_PROD)) break;
        mbar_arrive_expect_tx(&bars->qfull[qs], BUF);
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        tma_load_3d(smem + OFF_Q + qs * BUF, &tmQ, 0, n0, bh, &bars->qfull[qs]);
        tma_load_3d(smem + OFF_Q + qs * BUF + HALF, &tmQ, 64, n0, bh, &bars->qfull[qs]);
        ++issued_q;
        if (ti.unit != prev_unit) {
          if (prev_unit < 0) pdl_wait();
          const int64_t ku = ti.unit - u_first;
          const int b = static_cast<int>(ku % NSB);
          if (!mbar_wait(&bars->sfree[b], static_cast<uint32_t>(((ku / NSB) & 1) ^ 1), abort_flag, LA_SLEEP_PROD)) break;
          mbar_arrive_expect_tx(&bars->sfull[b], BUF);
          bulk_load(smem + OFF_S + b * BUF, simg + ti.unit * static_cast<int64_t>(BUF), BUF, &bars->sfull[b]);
          prev_unit = ti.unit;
          ++issued_s;
        }
      }
      if (*abort_flag) {
        // Let every copy still in flight land before the CTA's shared memory goes away.
        for (int64_t j = (issued_q > QST ? issued_q - QST : 0); j < issued_q; ++j)
          mbar_wait_drain(&bars->qfull[j % QST], static_cast<uint32_t>((j / QST) & 1));
        for (int64_t j = (issued_s > NSB ? issued_s - NSB : 0); j < issued_s; ++j)
          mbar_wait_drain(&bars->sfull[j % NSB], static_cast<uint32_t>((j / NSB) & 1));
      }
    } else if (warp == 3 && lane == 0) {
      // ---------------------------------------------------------- TMA producer: G
      // (separate from the Q producer so that a G stage still busy with an epilogue never
      // holds back the next Q tile)
      int64_t issued_g = 0;
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const int gs = static_cast<int>(i % GST);
        if (!mbar_wait(&bars->gempty[gs], static_cast<uint32_t>(((i / GST) & 1) ^ 1), abort_flag, LA_SLEEP_PROD)) break;
        const TileInfo ti = tile_info(p, g);
        mbar_arrive_expect_tx(&bars->gfull[gs], BUF);
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        tma_load_3d(smem + OFF_G + gs * BUF, &tmG, 0, n0, bh, &bars->gfull[gs]);
        tma_load_3d(smem + OFF_G + gs * BUF + HALF, &tmG, 64, n0, bh, &bars->gfull[gs]);
        ++issued_g;
      }
      if (*abort_flag) {
        for (int64_t j = (issued_g > GST ? issued_g - GST : 0); j < issued_g; ++j)
          mbar_wait_drain(&bars->gfull[j % GST], static_cast<uint32_t>((j / GST) & 1));
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // The math groups are served independently, each in its own tile order, so a group that is
      // ahead never waits behind the other group's tile.  A state buffer is freed after the last
      // of its unit's tiles in this CTA's range has been issued (by either group).
      int64_t next[NWG];
      uint32_t kdone[NWG];
      for (int mm = 0; mm < NWG; ++mm) {
        next[mm] = g0 + mm;
        kdone[mm] = 0;
      }
      int64_t buf_unit[NSB], buf_issued[NSB];
      for (int bb = 0; bb < NSB; ++bb) {
        buf_unit[bb] = -1;
        buf_issued[bb] = 0;
      }
      uint64_t t_progress = globaltimer_ns();
      uint32_t idle = 0;
      bool ok = true;
      while (ok) {
        bool pending = false, progressed = false;
        for (int mm = 0; mm < NWG; ++mm) {
          const int64_t g = next[mm];
          if (g >= g1) continue;
          pending = true;
          const int64_t u = unit_of_tile(p, g);
          const int64_t ku = u - u_first;
          const int b = static_cast<int>(ku % NSB);
          const uint32_t kph = kdone[mm] & 1u;
          if (!mbar_test_wait(&bars->accempty[mm], kph ^ 1u) || !mbar_test_wait(&bars->aready[mm], kph) ||
              !mbar_test_wait(&bars->sfull[b], static_cast<uint32_t>((ku / NSB) & 1)))
            continue;
          tc_fence_after();
          const uint32_t acc = tmem + static_cast<uint32_t>(mm) * GROUP_COLS + ACC_COL;
          const uint32_t at = tmem + static_cast<uint32_t>(mm) * GROUP_COLS + A_COL;
          const uint32_t sa = sbase + OFF_S + b * BUF;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            // K step kk: A columns 8kk .. 8kk+7 (16 bf16), B rows 16kk .. 16kk+15 (two 8-row groups).
            const uint64_t bd = smem_desc_sw128(sa + kk * 2048, HALF, 1024);
            mma_bf16_ts(acc, at + 8 * kk, bd, IDESC, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->accfull[mm]);
          mma_commit(&bars->afree[mm]);
          if (buf_unit[b] != u) {
            buf_unit[b] = u;
            buf_issued[b] = 0;
          }
          int64_t first = 0, count = 0;
          unit_tiles(p, u, &first, &count);
          const int64_t in_range = (first + count < g1 ? first + count : g1) - (first > g0 ? first : g0);
          if (++buf_issued[b] == in_range) mma_commit(&bars->sfree[b]);
          next[mm] += NWG;
          ++kdone[mm];
          progressed = true;
        }
        if (!pending) break;
        if (progressed) {
          t_progress = globaltimer_ns();
          idle = 0;
          continue;
        }
        // Nothing ready: back off briefly instead of spinning on the issue slots the math warps use.
        __nanosleep(32);
        if ((++idle & 255u) == 0u) {
          if (*abort_flag) break;
          if (globaltimer_ns() - t_progress > LA_WAIT_LIMIT_NS) {
            *abort_flag = 1;
            atomicOr(&g_la_error, ERR_WAIT_TIMEOUT);
            ok = false;
          }
        }
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------------------- TMA store of O
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const int gs = static_cast<int>(i % GST);
        if (!mbar_wait(&bars->ostaged[gs], static_cast<uint32_t>((i / GST) & 1), abort_flag, LA_SLEEP_PROD)) break;
        const TileInfo ti = tile_info(p, g);
        if ((ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N)) {
          const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
          tma_store_3d(&tmO, smem + OFF_G + gs * BUF, 0, n0, bh);
          tma_store_3d(&tmO, smem + OFF_G + gs * BUF + HALF, 64, n0, bh);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        mbar_arrive(&bars->gempty[gs]);
      }
      bulk_wait_group0();
    }
  } else {
    // ------------------------------------------------------------ math groups
    regs_inc<REGS_MATH>();
    const int wgi = (warp >> 2) - 1;
    const int m = wgi & 1;   // math group
    const int hf = wgi >> 1;  // channel half
    const int quarter = warp & 3;  // a warp reaches TMEM lanes 32*quarter .. +31 only
    const int row = quarter * 32 + lane;
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    const uint32_t row_off = static_cast<uint32_t>(row) * 128u + static_cast<uint32_t>(hf) * HALF;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_grp = tmem + static_cast<uint32_t>(m) * GROUP_COLS + lane_bits;
    const uint32_t t_acc = t_grp + ACC_COL + 64u * hf;
    const uint32_t t_a = t_grp + A_COL + 32u * hf;
    const int ext_t = static_cast<int>(p.T), ext_h = static_cast<int>(p.Hh), ext_w = static_cast<int>(p.W);
    uint64_t* denx = &bars->denx[m][quarter];
    uint64_t* rmsx = &bars->rmsx[m][quarter];
    const bool use_gamma = RMS && gamma != nullptr;
    const float* gm = use_gamma ? gamma + 64 * hf : nullptr;
    pdl_wait();
    int64_t g_prev = -1;
    uint32_t k_prev = 0;
    float hinv_prev = 0.f;
    for (int64_t g = g0 + m, k = 0;; g += NWG, ++k) {
      const bool have = g < g1;
      float hinv = 0.f;
      if (have) {
        // -- tile k: half row of Q -> registers (stage released), RoPE(ReLU(q)) -> TMEM A buffer
        const int64_t i = g - g0;
        const TileInfo ti = tile_info(p, g);
        const int qs = static_cast<int>(i % QST);
        if (!warp_wait(&bars->qfull[qs], static_cast<uint32_t>((i / QST) & 1), abort_flag)) break;
        uint32_t a[32];
        const uint32_t qrow = sbase + OFF_Q + qs * BUF + row_off;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 raw = lds128(qrow + ((static_cast<uint32_t>(c8) ^ swz) << 4));
          a[4 * c8 + 0] = relu_bf16x2(raw.x);
          a[4 * c8 + 1] = relu_bf16x2(raw.y);
          a[4 * c8 + 2] = relu_bf16x2(raw.z);
          a[4 * c8 + 3] = relu_bf16x2(raw.w);
        }
        // Every lane's loads have been consumed (by the ReLU above): the stage can be refilled.
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->qempty[qs]);

        const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
        uint32_t pt = 0, ph = 0, pw = 0;
        // Rows past the end of the head keep position 0 (their output is dropped).
        if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph, pw);
        in_bounds(pt < static_cast<uint32_t>(p.T) && ph < static_cast<uint32_t>(p.Hh) &&
                  pw < static_cast<uint32_t>(p.W));
        const float* zg = zimg + ti.unit * D + 64 * hf;
        const int ipt = static_cast<int>(pt), iph = static_cast<int>(ph), ipw = static_cast<int>(pw);
        const float dpart =
            hf == 0 ? transform_half<DT, DH, 0>(a, zg, tab, tab2, rope, ipt, iph, ipw, ext_t, ext_h, ext_w)
                    : transform_half<DT, DH, 1>(a, zg, tab, tab2, rope, ipt, iph, ipw, ext_t, ext_h, ext_w);
        // Swap partial denominators with the warp holding the other half of these rows (two
        // slots: a slot is rewritten only after the partner's next arrival, which follows its read).
        const uint32_t t_den = t_grp + DEN_COL + 2u * static_cast<uint32_t>(k & 1);
        tmem_st_x1(t_den + hf, __float_as_uint(dpart));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(denx);
        if (!warp_wait(denx, static_cast<uint32_t>(k & 1), abort_flag)) break;
        tc_fence_after();
        const float other = __uint_as_float(tmem_ld_x1(t_den + (hf ^ 1)));
        tmem_ld_wait();
        const float d0 = hf == 0 ? dpart : other, d1 = hf == 0 ? other : dpart;
        // o = acc / den * sigmoid(g) = h + h * tanh(g / 2) with h = acc * 0.5 / den.
        hinv = 0.5f / ((d0 + d1) + p.eps);
        // This group's previous MMA must have finished reading the A buffer.
        if (!warp_wait(&bars->afree[m], static_cast<uint32_t>((k & 1) ^ 1), abort_flag)) break;
        tc_fence_after();
        tmem_st_x16(t_a, &a[0]);
        tmem_st_x16(t_a + 16, &a[16]);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->aready[m]);
      }

      if (g_prev >= 0) {
        // -- epilogue of tile k-1 (this warp's channel half), in place over its G tile
        const int64_t i = g_prev - g0;
        const TileInfo ti = tile_info(p, g_prev);
        const int gs = static_cast<int>(i % GST);
        if (!warp_wait(&bars->accfull[m], k_prev & 1u, abort_flag)) break;
        tc_fence_after();
        uint32_t r[64];
        tmem_ld_x32(t_acc, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld_x32(t_acc + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld_wait();
        // The accumulator is free for this group's next MMA.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->accempty[m]);
        float scale = hinv_prev;  // h = acc * scale (* gamma)
        if constexpr (RMS) {
          // Sum of squares of this half of the row, swapped with the other half through TMEM
          // (two slots, as for the denominators).  y = acc / den = 2 h, so mean(y^2) =
          // 4 hinv^2 ss / 128 and the normalised h = acc * hinv / sqrt(mean(y^2) + norm_eps).
          uint64_t s2[4] = {0, 0, 0, 0};
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const uint64_t a2 = pk(__uint_as_float(r[2 * c]), __uint_as_float(r[2 * c + 1]));
            s2[c & 3] = fma2(a2, a2, s2[c & 3]);
          }
          const float2 e0 = upk(s2[0]), e1 = upk(s2[1]), e2 = upk(s2[2]), e3 = upk(s2[3]);
          const float ss_half = ((e0.x + e0.y) + (e1.x + e1.y)) + ((e2.x + e2.y) + (e3.x + e3.y));
          const uint32_t t_rms = t_grp + RMS_COL + 2u * (k_prev & 1u);
          tmem_st_x1(t_rms + hf, __float_as_uint(ss_half));
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(rmsx);
          if (!warp_wait(rmsx, k_prev & 1u, abort_flag)) break;
          tc_fence_after();
          const float other = __uint_as_float(tmem_ld_x1(t_rms + (hf ^ 1)));
          tmem_ld_wait();
          const float ss = hf == 0 ? ss_half + other : other + ss_half;
          scale = hinv_prev * rsqrtf(4.f * hinv_prev * hinv_prev * ss * (1.f / D) + norm_eps);
        }
        if (!warp_wait(&bars->gfull[gs], static_cast<uint32_t>((i / GST) & 1), abort_flag)) break;
        const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
        const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
        const bool valid = static_cast<int64_t>(n) < ti.n_end;
        const uint32_t grow = sbase + OFF_G + gs * BUF + row_off;
        __nv_bfloat16* orow = O + (ti.bh * p.N + static_cast<int64_t>(n)) * D + 64 * hf;
        const uint64_t hh = pk(scale, scale);
        // The G row is read and overwritten in place, four chunks at a time: the loads of a batch
        // are all issued before its first store, so their latency is paid once per batch.
#pragma unroll
        for (int b4 = 0; b4 < 2; ++b4) {
          uint4 graw[4];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            graw[c4] = lds128(grow + ((static_cast<uint32_t>(4 * b4 + c4) ^ swz) << 4));
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c8 = 4 * b4 + c4;
            // g/2 is exact in bf16, so halve the packed words before unpacking.
            const uint32_t gw[4] = {half_bf16x2(graw[c4].x), half_bf16x2(graw[c4].y), half_bf16x2(graw[c4].z),
                                    half_bf16x2(graw[c4].w)};
            uint32_t ov[4];
            ulonglong2 gw01 = make_ulonglong2(0, 0), gw23 = make_ulonglong2(0, 0);
            if (use_gamma) {
              gw01 = __ldg(reinterpret_cast<const ulonglong2*>(gm + 8 * c8));
              gw23 = __ldg(reinterpret_cast<const ulonglong2*>(gm + 8 * c8 + 4));
            }
            const uint64_t gpair[4] = {gw01.x, gw01.y, gw23.x, gw23.y};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint64_t h = mul2(pk(__uint_as_float(r[c8 * 8 + 2 * q]), __uint_as_float(r[c8 * 8 + 2 * q + 1])), hh);
              if (use_gamma) h = mul2(h, gpair[q]);
              const uint64_t t = pk(tanh_approx(bf16lo(gw[q])), tanh_approx(bf16hi(gw[q])));
              const float2 o2 = upk(fma2(h, t, h));
              ov[q] = pack_bf16(o2.x, o2.y);
            }
            const uint4 o4 = make_uint4(ov[0], ov[1], ov[2], ov[3]);
            if (tma_out) {
              sts128(grow + ((static_cast<uint32_t>(c8) ^ swz) << 4), o4);
            } else if (valid) {
              *reinterpret_cast<uint4*>(orow + c8 * 8) = o4;
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ostaged[gs]);
      }
      if (!have) break;
      g_prev = g;
      k_prev = static_cast<uint32_t>(k);
      hinv_prev = hinv;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace ap
}  // namespace la
