// apply_tc.cuh -- apply step on the 5th-generation tensor cores (bf16, d = 128).
//
//   O_n = (RoPE(ReLU(Q_n)) S) / (ReLU(Q_n) . z + eps) * sigmoid(G_n)
// (SANA-Video 2.0, Eq. (1); SANA-Video Sec. 3.2: rotated numerator, un-rotated denominator).
//
// Per 128-token tile one tcgen05 MMA chain computes the numerator D[128 tok x 128] =
// A[128 tok x 128 ch] * S[128 x 128], with A = RoPE(ReLU(Q)) written in place over the staged
// Q tile (K-major, 128B swizzle) and S the unit's state as a bf16 operand (N-major).  The
// denominator, the divide and the gate run on the CUDA cores around it: the thread that
// transforms row n of Q also owns TMEM lane n, so the denominator never leaves its register.
// The rotation reads cos/sin from a per-band table (fp64-accurate, built by the prep kernel),
// indexed [pair][position] so the 32 rows of a warp read consecutive entries.
//
// Warps (one CTA per SM, persistent over a contiguous range of tiles):
//   warpgroup 0   warp 0: TMA producer (Q and G tiles; the state operand once per unit)
//                 warp 1: MMA issuer (and TMEM owner); warp 2: TMA store of finished O tiles
//   warpgroups 1..NWG  math: group w takes local tiles i = w-1 (mod NWG): transform Q, then the
//                 epilogue (TMEM -> registers, divide, gate, bf16) in place over the staged G tile
// With three math groups the control warpgroup hands registers to the math groups
// (setmaxnreg); the host checks the launch's register budget before launching.
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
#ifndef LA_AP_NWG
#define LA_AP_NWG 2
#endif

namespace la {
namespace ap {

constexpr int TILE = 128;
constexpr int D = 128;
constexpr int QST = LA_AP_QST;  // Q stages (freed when the MMA has read them)
constexpr int GST = LA_AP_GST;  // G / O stages (freed when the O tile has been stored)
constexpr int NSB = LA_AP_NSB;  // state operand buffers
constexpr int NWG = LA_AP_NWG;  // math warpgroups
constexpr int THREADS = 128 * (1 + NWG);
constexpr uint32_t HALF = 128 * 128;
constexpr uint32_t BUF = 2 * HALF;  // 32 KB: a 128 x 128 bf16 tile
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_G = OFF_Q + QST * BUF;
constexpr uint32_t OFF_S = OFF_G + GST * BUF;
constexpr uint32_t OFF_BAR = OFF_S + NSB * BUF;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = NWG <= 2 ? 256 : 512;   // one 128-column accumulator per math group
constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/true);
// Register split (used only with three or more math groups).  The launch grants REGS_LAUNCH per
// thread (the largest multiple of 8 that fits 65536 / THREADS); the control warpgroup shrinks to
// REGS_CTRL and the math groups grow to REGS_MATH, never asking for more than the launch granted.
constexpr bool SPLIT_REGS = NWG >= 3;
constexpr uint32_t REGS_LAUNCH = (65536 / THREADS) / 8 * 8;
constexpr uint32_t REGS_CTRL = 56;
constexpr uint32_t REGS_MATH = ((THREADS * REGS_LAUNCH - 128 * REGS_CTRL) / (128 * NWG)) / 8 * 8;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
// Each Q / G stage must always serve the same math group: a group then never polls a stage's
// barrier more than one phase ahead of it, so the parity test cannot alias.
static_assert(QST % NWG == 0 && GST % NWG == 0, "stages must be a multiple of the math groups");
static_assert(!SPLIT_REGS || 128 * REGS_CTRL + 128 * NWG * REGS_MATH <= THREADS * REGS_LAUNCH, "register split");
static_assert(!SPLIT_REGS || (REGS_CTRL <= REGS_LAUNCH && REGS_LAUNCH <= REGS_MATH), "register split");

struct Bars {
  uint64_t qfull[QST], aready[QST], qempty[QST];
  uint64_t gfull[GST], gempty[GST], ostaged[GST];
  uint64_t sfull[NSB], sfree[NSB];
  uint64_t accfull[NWG], accempty[NWG];
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

// Transform of chunks [CK0, CK1) of one row, all in one RoPE band: q <- RoPE(ReLU(q)) in place,
// den += ReLU(q) . z.  `tp` walks the band's [pair][position] table column of this row.
template <int CK0, int CK1>
__device__ __forceinline__ void transform_band(uint32_t qrow, uint32_t swz, const float* __restrict__ zg,
                                               const float2* __restrict__ tp, int ext, float (&den4)[4]) {
#pragma unroll 2
  for (int ck = CK0; ck < CK1; ++ck) {
    const uint32_t addr = qrow + (ck >> 3) * HALF + (((static_cast<uint32_t>(ck) & 7u) ^ swz) << 4);
    const uint4 raw = lds128(addr);
    const float4 za = __ldg(reinterpret_cast<const float4*>(zg + ck * 8));
    const float4 zc = __ldg(reinterpret_cast<const float4*>(zg + ck * 8 + 4));
    const float zz[8] = {za.x, za.y, za.z, za.w, zc.x, zc.y, zc.z, zc.w};
    const uint32_t w[4] = {relu_bf16x2(raw.x), relu_bf16x2(raw.y), relu_bf16x2(raw.z), relu_bf16x2(raw.w)};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 cs = __ldg(tp + (4 * (ck - CK0) + q) * ext);
      const float x0 = bf16lo(w[q]);
      const float x1 = bf16hi(w[q]);
      den4[q] = fmaf(x0, zz[2 * q], den4[q]);
      den4[q] = fmaf(x1, zz[2 * q + 1], den4[q]);
      o[q] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
    }
    sts128(addr, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

template <int DT, int DH>
__global__ void __launch_bounds__(THREADS, 1)
apply_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
                const __grid_constant__ CUtensorMap tmO, const Plan p, const __grid_constant__ Rope rope,
                const uint8_t* __restrict__ simg, const float* __restrict__ zimg,
                const float2* __restrict__ tab, __nv_bfloat16* __restrict__ O) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
      mbar_init(&bars->aready[s], 4);
      mbar_init(&bars->qempty[s], 1);
    }
    for (int s = 0; s < GST; ++s) {
      mbar_init(&bars->gfull[s], 1);
      mbar_init(&bars->gempty[s], 1);
      mbar_init(&bars->ostaged[s], 4);
    }
    for (int s = 0; s < NSB; ++s) {
      mbar_init(&bars->sfull[s], 1);
      mbar_init(&bars->sfree[s], 1);
    }
    for (int a = 0; a < NWG; ++a) {
      mbar_init(&bars->accfull[a], 1);
      mbar_init(&bars->accempty[a], 4);
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

  if (warp < 4) {
    if constexpr (SPLIT_REGS) regs_dec<REGS_CTRL>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      int64_t issued_q = 0, issued_g = 0, issued_s = 0;
      int64_t prev_unit = -1;
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const TileInfo ti = tile_info(p, g);
        if (ti.unit != prev_unit) {
          const int64_t ku = ti.unit - u_first;
          const int b = static_cast<int>(ku % NSB);
          if (!mbar_wait(&bars->sfree[b], static_cast<uint32_t>(((ku / NSB) & 1) ^ 1), abort_flag)) break;
          mbar_arrive_expect_tx(&bars->sfull[b], BUF);
          bulk_load(smem + OFF_S + b * BUF, simg + ti.unit * static_cast<int64_t>(BUF), BUF, &bars->sfull[b]);
          prev_unit = ti.unit;
          ++issued_s;
        }
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        const int qs = static_cast<int>(i % QST);
        if (!mbar_wait(&bars->qempty[qs], static_cast<uint32_t>(((i / QST) & 1) ^ 1), abort_flag)) break;
        mbar_arrive_expect_tx(&bars->qfull[qs], BUF);
        tma_load_3d(smem + OFF_Q + qs * BUF, &tmQ, 0, n0, bh, &bars->qfull[qs]);
        tma_load_3d(smem + OFF_Q + qs * BUF + HALF, &tmQ, 64, n0, bh, &bars->qfull[qs]);
        ++issued_q;
        const int gs = static_cast<int>(i % GST);
        if (!mbar_wait(&bars->gempty[gs], static_cast<uint32_t>(((i / GST) & 1) ^ 1), abort_flag)) break;
        mbar_arrive_expect_tx(&bars->gfull[gs], BUF);
        tma_load_3d(smem + OFF_G + gs * BUF, &tmG, 0, n0, bh, &bars->gfull[gs]);
        tma_load_3d(smem + OFF_G + gs * BUF + HALF, &tmG, 64, n0, bh, &bars->gfull[gs]);
        ++issued_g;
      }
      if (*abort_flag) {
        // Let every copy still in flight land before the CTA's shared memory goes away.
        for (int64_t j = (issued_q > QST ? issued_q - QST : 0); j < issued_q; ++j)
          mbar_wait_drain(&bars->qfull[j % QST], static_cast<uint32_t>((j / QST) & 1));
        for (int64_t j = (issued_g > GST ? issued_g - GST : 0); j < issued_g; ++j)
          mbar_wait_drain(&bars->gfull[j % GST], static_cast<uint32_t>((j / GST) & 1));
        for (int64_t j = (issued_s > NSB ? issued_s - NSB : 0); j < issued_s; ++j)
          mbar_wait_drain(&bars->sfull[j % NSB], static_cast<uint32_t>((j / NSB) & 1));
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const int64_t u = unit_of_tile(p, g);
        const int64_t ku = u - u_first;
        const int b = static_cast<int>(ku % NSB);
        const int wg = static_cast<int>(i % NWG);
        const int qs = static_cast<int>(i % QST);
        const uint32_t qph = static_cast<uint32_t>((i / QST) & 1);
        if (!mbar_wait(&bars->accempty[wg], static_cast<uint32_t>(((i / NWG) & 1) ^ 1), abort_flag)) break;
        if (!mbar_wait(&bars->sfull[b], static_cast<uint32_t>((ku / NSB) & 1), abort_flag)) break;
        if (!mbar_wait(&bars->qfull[qs], qph, abort_flag)) break;
        if (!mbar_wait(&bars->aready[qs], qph, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(wg) * 128u;
        const uint32_t qa = sbase + OFF_Q + qs * BUF;
        const uint32_t sa = sbase + OFF_S + b * BUF;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(qa + (kk >> 2) * HALF + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sa + kk * 2048, HALF, 1024);
          mma_bf16(acc, ad, bd, IDESC, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->accfull[wg]);
        mma_commit(&bars->qempty[qs]);
        const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != u);
        if (last) mma_commit(&bars->sfree[b]);
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    } else if (warp == 2 && lane == 0) {
      // ---------------------------------------------------------- TMA store of O
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const int gs = static_cast<int>(i % GST);
        if (!mbar_wait(&bars->ostaged[gs], static_cast<uint32_t>((i / GST) & 1), abort_flag)) break;
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
    if constexpr (SPLIT_REGS) regs_inc<REGS_MATH>();
    const int wg = (warp >> 2) - 1;
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t swz = static_cast<uint32_t>(row & 7);
    const uint32_t row_off = static_cast<uint32_t>(row) * 128u;
    const int ext_t = static_cast<int>(p.T), ext_h = static_cast<int>(p.Hh), ext_w = static_cast<int>(p.W);
    for (int64_t g = g0 + wg; g < g1; g += NWG) {
      const int64_t i = g - g0;
      const TileInfo ti = tile_info(p, g);
      const int qs = static_cast<int>(i % QST);
      const int gs = static_cast<int>(i % GST);
      // z is read straight from the combine kernel's output (read-only here), so the math groups
      // never wait on the state buffer's barrier; only the MMA issuer does.
      if (!warp_wait(&bars->qfull[qs], static_cast<uint32_t>((i / QST) & 1), abort_flag)) break;

      // -- transform: A = RoPE(ReLU(q)) in place, den = ReLU(q) . z
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      uint32_t pt = 0, ph = 0, pw = 0;
      // Rows past the end of the head keep position 0 (their output is dropped).
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph, pw);
      const uint32_t qrow = sbase + OFF_Q + qs * BUF + row_off;
      const float* zg = zimg + ti.unit * D;
      float den4[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (DT >= 0 && DH >= 0 && DT % 8 == 0 && DH % 8 == 0) {
        transform_band<0, DT / 8>(qrow, swz, zg, tab + pt, ext_t, den4);
        transform_band<DT / 8, (DT + DH) / 8>(qrow, swz, zg, tab + rope.tab_off_h + ph, ext_h, den4);
        transform_band<(DT + DH) / 8, 16>(qrow, swz, zg, tab + rope.tab_off_w + pw, ext_w, den4);
      } else {
        const int it = static_cast<int>(pt);
        const int ih = static_cast<int>(rope.tab_off_h + ph);
        const int iw = static_cast<int>(rope.tab_off_w + pw);
#pragma unroll 2
        for (int ck = 0; ck < 16; ++ck) {
          const uint32_t addr = qrow + (ck >> 3) * HALF + (((static_cast<uint32_t>(ck) & 7u) ^ swz) << 4);
          const uint4 raw = lds128(addr);
          const float4 za = __ldg(reinterpret_cast<const float4*>(zg + ck * 8));
          const float4 zc = __ldg(reinterpret_cast<const float4*>(zg + ck * 8 + 4));
          const float zz[8] = {za.x, za.y, za.z, za.w, zc.x, zc.y, zc.z, zc.w};
          const uint32_t w[4] = {relu_bf16x2(raw.x), relu_bf16x2(raw.y), relu_bf16x2(raw.z), relu_bf16x2(raw.w)};
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int pi = 4 * ck + q;
            const int bnd = band_of<DT, DH>(pi, rope);
            const int loc = pair_in_band<DT, DH>(pi, rope);
            const int idx = bnd == 0 ? it + loc * ext_t : (bnd == 1 ? ih + loc * ext_h : iw + loc * ext_w);
            const float2 cs = __ldg(tab + idx);
            const float x0 = bf16lo(w[q]);
            const float x1 = bf16hi(w[q]);
            den4[q] = fmaf(x0, zz[2 * q], den4[q]);
            den4[q] = fmaf(x1, zz[2 * q + 1], den4[q]);
            o[q] = pack_bf16(x0 * cs.x - x1 * cs.y, x0 * cs.y + x1 * cs.x);
          }
          sts128(addr, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->aready[qs]);
      // o = acc / den * sigmoid(g) = a + a * tanh(g / 2) with a = acc * 0.5 / den.
      const float hinv = 0.5f / ((den4[0] + den4[1]) + (den4[2] + den4[3]) + p.eps);

      // -- epilogue, in place over the G tile
      if (!warp_wait(&bars->accfull[wg], static_cast<uint32_t>((i / NWG) & 1), abort_flag)) break;
      if (!warp_wait(&bars->gfull[gs], static_cast<uint32_t>((i / GST) & 1), abort_flag)) break;
      tc_fence_after();
      const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
      const bool valid = static_cast<int64_t>(n) < ti.n_end;
      const uint32_t grow = sbase + OFF_G + gs * BUF + row_off;
      __nv_bfloat16* orow = O + (ti.bh * p.N + static_cast<int64_t>(n)) * D;
      const uint32_t taddr = tmem + static_cast<uint32_t>(wg) * 128u + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld_x32(taddr + ch * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ck = ch * 4 + cc;
          const uint32_t addr = grow + (ck >> 3) * HALF + (((static_cast<uint32_t>(ck) & 7u) ^ swz) << 4);
          const uint4 graw = lds128(addr);
          // g/2 is exact in bf16, so halve the packed words before unpacking.
          const uint32_t gw[4] = {half_bf16x2(graw.x), half_bf16x2(graw.y), half_bf16x2(graw.z), half_bf16x2(graw.w)};
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float a0 = __uint_as_float(r[cc * 8 + 2 * q]) * hinv;
            const float a1 = __uint_as_float(r[cc * 8 + 2 * q + 1]) * hinv;
            const float t0 = tanh_approx(bf16lo(gw[q]));
            const float t1 = tanh_approx(bf16hi(gw[q]));
            o[q] = pack_bf16(fmaf(a0, t0, a0), fmaf(a1, t1, a1));
          }
          const uint4 ov = make_uint4(o[0], o[1], o[2], o[3]);
          if (tma_out) {
            sts128(addr, ov);
          } else if (valid) {
            *reinterpret_cast<uint4*>(orow + ck * 8) = ov;
          }
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->accempty[wg]);
        mbar_arrive(&bars->ostaged[gs]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace ap
}  // namespace la
