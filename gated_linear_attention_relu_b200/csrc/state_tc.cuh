// state_tc.cuh -- state reduction on the 5th-generation tensor cores (bf16, d = 128).
//
// Computes, per unit (a head, or one block of a head), the partial sums over the tiles a CTA
// owns of
//   S[k][v] = sum_n RoPE(ReLU(K_n))[k] V_n[v]     (SANA-Video 2.0, Eq. (1), the state)
//   z[k]    = sum_n ReLU(K_n)[k]                  (the un-rotated normaliser, SANA-Video Sec. 3.2)
// as one tcgen05 MMA per 16 tokens: D[128 x 128] += A[128 x 16] * B[16 x 128], where
// A = RoPE(ReLU(K))^T (channels x tokens, M-major) and B = V (tokens x channels, N-major).
//
// Pipeline (one CTA per SM, persistent over a contiguous range of 128-token tiles):
//   warp 0       TMA producer of K tiles (two 64-channel, 128-row, 128B-swizzled boxes each)
//   warp 14      TMA producer of V tiles, on a ring of its own: a V tile is only read by the MMA,
//                so it need not sit in shared memory while its K tile is being transformed, and
//                the K ring gets the deeper pipeline
//   warp 1       MMA issuer: 8 x tcgen05.mma per tile into one of two TMEM accumulators
//   warps 2-9    transform, two groups of four warps splitting each tile's rows: ReLU + RoPE of
//                K in place (bf16; cos/sin from the fp64-accurate table the prep kernel builds),
//                z accumulated in registers
//   warps 10-13  drain: TMEM accumulator -> fp32 partial S in global memory, once per unit
// The staged K tile is already in the canonical 128B-swizzled MN-major operand layout, so the
// transform rewrites it in place.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

#ifndef LA_ST_TILE
#define LA_ST_TILE 128
#endif
#ifndef LA_ST_KSTAGES
#define LA_ST_KSTAGES 4
#endif
#ifndef LA_ST_VSTAGES
#define LA_ST_VSTAGES 2
#endif
#ifndef LA_ST_TGROUPS
#define LA_ST_TGROUPS 2
#endif

namespace la {
namespace st {

constexpr int TILE = LA_ST_TILE;              // tokens per stage (the MMA K extent of one stage)
constexpr int D = 128;
constexpr int KST = LA_ST_KSTAGES;           // K stages (held through transform and MMA)
constexpr int VST = LA_ST_VSTAGES;           // V stages (held through the MMA only)
constexpr int TGROUPS = LA_ST_TGROUPS;        // transform warpgroups, each owning TILE/TGROUPS rows
constexpr int GROUP_ROWS = TILE / TGROUPS;
constexpr int THREADS = 32 * (2 + 4 * TGROUPS + 4 + 1);
constexpr uint32_t HALF = TILE * 128;         // one 64-channel box of TILE rows x 128 B
constexpr uint32_t BUF = 2 * HALF;            // TILE tokens x 128 channels bf16
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = KST * BUF;
constexpr uint32_t OFF_BAR = (KST + VST) * BUF;  // barriers after the stages
constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // + alignment slack
constexpr int ZPARTS = TGROUPS;               // z is written as one partial sum per transform group
constexpr int64_t SLOT = D * D + ZPARTS * D;  // floats per partial slot: S, then ZPARTS x z
constexpr uint32_t TMEM_COLS = 256;           // two 128-column fp32 accumulators
constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, /*a_mn=*/true, /*b_mn=*/true);
constexpr int DRAIN_WARP0 = 2 + 4 * TGROUPS;
constexpr int VPROD_WARP = DRAIN_WARP0 + 4;

struct Bars {
  uint64_t kfull[KST];       // TMA landed K                  (1 arrival + tx bytes)
  uint64_t aready[KST];      // transform wrote the A operand  (one arrival per transform warp)
  uint64_t kempty[KST];      // MMAs of the K stage completed  (tcgen05.commit)
  uint64_t vfull[VST];       // TMA landed V
  uint64_t vempty[VST];      // MMAs of the V stage completed
  uint64_t accfull[2];       // accumulator holds a finished unit (tcgen05.commit)
  uint64_t accempty[2];      // drain finished reading it     (4 warps)
  uint64_t final_;           // all MMAs completed (teardown)
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block too large");
static_assert(TILE % 16 == 0 && TILE <= 256 && GROUP_ROWS % 8 == 0 && GROUP_ROWS * TGROUPS == TILE, "tile shape");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// BETA: each token's rotated key is scaled by its write gate beta_n before the contraction
// (SANA-Video 2.0, Eq. (1): S = sum_n v_n (beta_n k_n^r)^T); z stays un-gated.
template <int DT, int DH, bool BETA>
__global__ void __launch_bounds__(THREADS, 1)
state_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const Plan p, const __grid_constant__ Rope rope, const float2* __restrict__ tab,
                const float4* __restrict__ tab2, const __nv_bfloat16* __restrict__ beta,
                float* __restrict__ partial) {
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
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->aready[s], 4 * TGROUPS);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
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
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // Only the transform warps read what the kernel before this one wrote (the cos/sin tables);
  // the K and V loads start at once.
  pdl_trigger();

  if (warp == 0 || warp == VPROD_WARP) {
    // ------------------------------------------------------------ TMA producers (K; V)
    if (lane == 0) {
      const bool is_k = warp == 0;
      const int nst = is_k ? KST : VST;
      uint64_t* fullb = is_k ? bars->kfull : bars->vfull;
      uint64_t* emptyb = is_k ? bars->kempty : bars->vempty;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      uint8_t* ring = smem + (is_k ? OFF_K : OFF_V);
      int64_t issued = 0;
      for (int64_t g = g0; g < g1; ++g, ++issued) {
        const int64_t i = g - g0;
        const int s = static_cast<int>(i % nst);
        const uint32_t ph = static_cast<uint32_t>((i / nst) & 1);
        if (!mbar_wait(&emptyb[s], ph ^ 1u, abort_flag, LA_SLEEP_PROD)) break;
        const TileInfo ti = tile_info(p, g);
        in_bounds(ti.bh < p.BH && ti.n0 < ti.n_end && ti.n_end <= p.N);
#ifdef LA_TEST_HOOKS
        if (is_k && g == g_la_skip_tile) continue;  // (counted as issued: the drain below waits for it)
#endif
        uint8_t* buf = ring + s * BUF;
        mbar_arrive_expect_tx(&fullb[s], BUF);
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        tma_load_3d(buf, tm, 0, n0, bh, &fullb[s]);
        tma_load_3d(buf + HALF, tm, 64, n0, bh, &fullb[s]);
      }
      if (*abort_flag) {
        // Let every copy still in flight land before the CTA's shared memory goes away.
        for (int64_t j = (issued > nst ? issued - nst : 0); j < issued; ++j)
          mbar_wait_drain(&fullb[j % nst], static_cast<uint32_t>((j / nst) & 1));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t seg = -1;
      int64_t prev_unit = -1;
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const int s = static_cast<int>(i % KST);
        const uint32_t ph = static_cast<uint32_t>((i / KST) & 1);
        const int sv = static_cast<int>(i % VST);
        const uint32_t phv = static_cast<uint32_t>((i / VST) & 1);
        const int64_t u = unit_of_tile(p, g);
        const bool first = (u != prev_unit);
        const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != u);
        prev_unit = u;
        if (first) {
          ++seg;
          if (!mbar_wait(&bars->accempty[seg & 1], static_cast<uint32_t>(((seg >> 1) & 1) ^ 1), abort_flag, LA_SLEEP_PROD)) break;
        }
        if (!mbar_wait(&bars->aready[s], ph, abort_flag)) break;
        if (!mbar_wait(&bars->vfull[sv], phv, abort_flag)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(seg & 1) * 128u;
        const uint32_t ka = sbase + OFF_K + s * BUF;
        const uint32_t va = sbase + OFF_V + sv * BUF;
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(ka + kk * 2048, HALF, 1024);
          const uint64_t bd = smem_desc_sw128(va + kk * 2048, HALF, 1024);
          mma_bf16(acc, ad, bd, IDESC, (kk > 0 || !first) ? 1u : 0u);
        }
        mma_commit(&bars->kempty[s]);
        mma_commit(&bars->vempty[sv]);
        if (last) mma_commit(&bars->accfull[seg & 1]);
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else if (warp < DRAIN_WARP0) {
    // ------------------------------------------------------------ transform: ReLU + RoPE of K
    // Group tg owns rows GROUP_ROWS*tg .. GROUP_ROWS*(tg+1)-1 of each tile.  Warp k of the group
    // owns the 8-channel chunks 4k .. 4k+3; each lane walks rows GROUP_ROWS*tg + rg + 8j, so the
    // 32 lanes of a load touch 8 consecutive tokens and the cos/sin table reads coalesce.
    const int tg = (warp - 2) >> 2;
    const int wk = (warp - 2) & 3;
    const int ck = 4 * wk + (lane & 3);           // channels 8ck .. 8ck+7
    // Each 8-lane phase of a 16-byte shared access covers rows r and r+4 (r = rg mod 4) and the
    // 4 chunks: the swizzled positions (chunk ^ row) % 8 are then all distinct (no bank conflict).
    const int rg = ((lane >> 2) & 1) * 4 + (lane >> 3);  // row % 8
    const uint32_t chunk_off = static_cast<uint32_t>((ck >> 3) * HALF + (((ck & 7) ^ rg) << 4));
    // With the band split fixed at compile time (a multiple of 8 channels per band), the 4 pairs
    // of a chunk share one band, so the position is selected once per row, and the packed table
    // (two pairs per 16-byte entry; t and h bands position-major, the w band [pair / 2][x])
    // gives the chunk's 4 cos/sin pairs in two loads: entries e and e + step2, e = off2 + x * mul2.
    constexpr bool UNIFORM = DT >= 0 && DH >= 0 && DT % 8 == 0 && DH % 8 == 0;
    const int bnd0 = band_of<DT, DH>(4 * ck, rope);
    const int loc0 = pair_in_band<DT, DH>(4 * ck, rope);
    const int off2 = bnd0 == 0 ? loc0 / 2
                               : (bnd0 == 1 ? static_cast<int>(rope.tab_off_h / 2) + loc0 / 2
                                            : static_cast<int>(rope.tab_off_w / 2) + (loc0 / 2) * static_cast<int>(p.W));
    const int mul2 = bnd0 == 0 ? rope.dt / 4 : (bnd0 == 1 ? rope.dh / 4 : 1);
    const int step2 = bnd0 == 2 ? static_cast<int>(p.W) : 1;
    int bd[4], tix[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int pi = 4 * ck + q;
      bd[q] = band_of<DT, DH>(pi, rope);
      const int loc = pair_in_band<DT, DH>(pi, rope);
      tix[q] = bd[q] == 0 ? loc * static_cast<int>(p.T)
                          : (bd[q] == 1 ? static_cast<int>(rope.tab_off_h) + loc * static_cast<int>(p.Hh)
                                        : static_cast<int>(rope.tab_off_w) + loc * static_cast<int>(p.W));
    }
    uint64_t zacc[4] = {0, 0, 0, 0};  // packed fp32 pairs: z of channels (8ck + 2q, 8ck + 2q + 1)
    pdl_wait();
    const uint32_t N = static_cast<uint32_t>(p.N);
    const uint32_t Wd = static_cast<uint32_t>(p.W), Hd = static_cast<uint32_t>(p.Hh);
    const bool step_ok = Wd >= 8;  // incremental positions need at most one wrap per 8 rows
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const int s = static_cast<int>(i % KST);
      const uint32_t ph = static_cast<uint32_t>((i / KST) & 1);
      const TileInfo ti = tile_info(p, g);
      const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != ti.unit);
      if (!warp_wait(&bars->kfull[s], ph, abort_flag, LA_SLEEP_MATH)) break;
      const int row0 = GROUP_ROWS * tg + rg;
      const uint32_t base = sbase + OFF_K + s * BUF + chunk_off + static_cast<uint32_t>(row0 * 128);
      const uint32_t n0 = static_cast<uint32_t>(ti.n0) + row0;
      const uint32_t n_end = static_cast<uint32_t>(ti.n_end);
      // One 8-channel chunk of one row: ReLU (rows past the unit's end zeroed by `keep`), RoPE with
      // the chunk's cos/sin, z, written back in place.
      const __nv_bfloat16* beta_h = BETA ? beta + ti.bh * p.N : nullptr;
      auto item = [&](uint32_t addr, uint32_t keep, uint32_t n, uint32_t pt, uint32_t ph_, uint32_t pw) {
        in_bounds(n < N && pt < static_cast<uint32_t>(p.T) && ph_ < Hd && pw < Wd);
        const uint4 raw = lds128(addr);
        float2 cs[4];
        if constexpr (UNIFORM) {
          const int x = static_cast<int>(bnd0 == 0 ? pt : (bnd0 == 1 ? ph_ : pw));
          const float4* tp = tab2 + off2 + x * mul2;
          const float4 c01 = __ldg(tp), c23 = __ldg(tp + step2);
          cs[0] = make_float2(c01.x, c01.y);
          cs[1] = make_float2(c01.z, c01.w);
          cs[2] = make_float2(c23.x, c23.y);
          cs[3] = make_float2(c23.z, c23.w);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t pos = bd[q] == 0 ? pt : (bd[q] == 1 ? ph_ : pw);
            cs[q] = __ldg(tab + tix[q] + pos);
          }
        }
        if constexpr (BETA) {
          // The gate scales the rotated key: fold it into this row's cos/sin.
          const float b = __bfloat162float(beta_h[n]);
#pragma unroll
          for (int q = 0; q < 4; ++q) cs[q] = make_float2(cs[q].x * b, cs[q].y * b);
        }
        const uint32_t w[4] = {relu_bf16x2(raw.x) & keep, relu_bf16x2(raw.y) & keep,
                               relu_bf16x2(raw.z) & keep, relu_bf16x2(raw.w) & keep};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x0 = bf16lo(w[q]);
          const float x1 = bf16hi(w[q]);
          zacc[q] = add2(zacc[q], pk(x0, x1));
          o[q] = pack_bf16(x0 * cs[q].x - x1 * cs[q].y, x0 * cs[q].y + x1 * cs[q].x);
        }
        sts128(addr, make_uint4(o[0], o[1], o[2], o[3]));
      };
      if (ti.n0 + TILE <= ti.n_end && step_ok) {
        // Whole tile inside the unit (warp-uniform): no masking, and the position of row n + 8
        // follows from that of row n with at most one wrap of w (W >= 8).
        uint32_t pt, ph_, pw;
        token_pos(p, n0, pt, ph_, pw);
#pragma unroll 4
        for (int j = 0; j < GROUP_ROWS / 8; ++j) {
          item(base + static_cast<uint32_t>(j * 8 * 128), 0xffffffffu, n0 + 8 * j, pt, ph_, pw);
          pw += 8;
          const bool wrap = pw >= Wd;
          pw = wrap ? pw - Wd : pw;
          ph_ += wrap ? 1u : 0u;
          const bool wrap2 = ph_ >= Hd;
          ph_ = wrap2 ? 0u : ph_;
          pt += wrap2 ? 1u : 0u;
        }
      } else {
        // Branch-free over rows so the unrolled iterations' load chains overlap: rows past the
        // end of the unit are zeroed with a select, and their (unused) position is clamped.
#pragma unroll 4
        for (int j = 0; j < GROUP_ROWS / 8; ++j) {
          const uint32_t n = n0 + 8 * j;
          const uint32_t nc = n < N ? n : N - 1;
          uint32_t pt, ph_, pw;
          token_pos(p, nc, pt, ph_, pw);
          item(base + static_cast<uint32_t>(j * 8 * 128), n < n_end ? 0xffffffffu : 0u, nc, pt, ph_, pw);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->aready[s]);
      if (last) {
        // z of this unit: the 8 lanes holding chunk ck (lane bits 2-4 = the row group) add their
        // sums with a butterfly (every lane ends with the same bits), and lanes 0-3 write one
        // partial row per transform group; the combine kernel adds those in order.
        float zs[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 v = upk(zacc[q]);
          zs[2 * q] = v.x;
          zs[2 * q + 1] = v.y;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          zs[e] += __shfl_xor_sync(0xffffffffu, zs[e], 4);
          zs[e] += __shfl_xor_sync(0xffffffffu, zs[e], 8);
          zs[e] += __shfl_xor_sync(0xffffffffu, zs[e], 16);
        }
        const int64_t slot = c * p.maxseg + (ti.unit - u_first);
        if (lane < 4 && in_bounds(ti.unit - u_first < p.maxseg && slot < int64_t(p.grid) * p.maxseg)) {
          float4* zd = reinterpret_cast<float4*>(partial + slot * SLOT + D * D + tg * D + 8 * ck);
          zd[0] = make_float4(zs[0], zs[1], zs[2], zs[3]);
          zd[1] = make_float4(zs[4], zs[5], zs[6], zs[7]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) zacc[q] = 0;
      }
    }
  } else if (warp < VPROD_WARP) {
    // ------------------------------------------------------------ drain TMEM -> partial S
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const int64_t nseg = (g1 > g0) ? unit_of_tile(p, g1 - 1) - u_first + 1 : 0;
    for (int64_t k = 0; k < nseg; ++k) {
      if (!warp_wait(&bars->accfull[k & 1], static_cast<uint32_t>((k >> 1) & 1), abort_flag, LA_SLEEP_LONG)) break;
      tc_fence_after();
      if (!in_bounds(k < p.maxseg)) break;
      float* dst = partial + (c * p.maxseg + k) * SLOT + static_cast<int64_t>(row) * D;
      const uint32_t taddr = tmem + static_cast<uint32_t>(k & 1) * 128u + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        tmem_ld_x32(taddr + ch * 32, r);
        tmem_ld_wait();
        float4* d4 = reinterpret_cast<float4*>(dst + ch * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          d4[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]),
                              __uint_as_float(r[4 * e + 2]), __uint_as_float(r[4 * e + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->accempty[k & 1]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace st
}  // namespace la
