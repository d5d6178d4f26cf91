// causal_tc.cuh -- token-causal operator on the 5th-generation tensor cores (bf16, d = 128).
//
// Token n reads the states of tokens 0..n of its head in the flattened order (the causal form
// of "SANA-Video: Efficient Video Generation with Block Linear Diffusion Transformer", Sec. 3.4,
// taken token by token):
//   O_n = (phi(q_n) S_{<=n}) / (q_n^+ . z_{<=n} + eps) * sigmoid(g_n),
//   S_{<=n} = sum_{m<=n} phi(k_m)^T v_m,  z_{<=n} = sum_{m<=n} k_m^+,  phi = RoPE3D(ReLU(.)).
//
// Chunkwise form.  The tiles of every head are split into contiguous segments, one per
// persistent CTA (the same split as the state kernel's, whose per-segment sums the start
// kernel prefix-sums into each CTA's starting state).  A CTA walks its 128-token chunks in order
// carrying S (fp32, in TMEM) and z (fp32, in shared memory); for chunk c with rows n, m:
//   C   = M K^+,                        M_nm = [m <= n]  (C_n = sum_{m<=n} k_m^+ over the chunk)
//   num = phi(Q) S_prev + (P o M) V,    P = phi(Q) phi(K)^T
//   den = q_n^+ . (z_prev + C_n) + eps
//   S  += phi(K)^T V,  z += C_127 (the chunk's last row: its column sums of K^+)
// M is a constant bf16 operand in TMEM, so C is one product of the same form as (P o M) V; P o M
// goes back to TMEM as bf16 and is the A operand of that product; S_prev is the bf16 image of
// the carried state in shared memory (rewritten after every chunk).
//
// Warps: 0-15 own the chunk's rows, four per row (channel quarters; thread = token = TMEM lane,
// warp w reaching lanes 32 (w mod 4) ..); warp 16 issues the TMA copies and the MMAs.  Only K^+
// goes back to shared memory before the first product; the rotation of Q runs while C is
// computed (into the columns P takes later), phi(Q) S_prev starts as soon as phi(Q) is written,
// K is rotated from registers, the mask of P starts once P alone is done (the state update runs
// under it), and the new state image is written while P V runs.  The next chunk's tiles are
// loaded as soon as their buffers are free (Q and K once the products reading them are done, V
// after P V, G after this chunk's O has been stored), each on its own barrier and waited for only
// by its first reader (Q and K: the ReLU pass; V: the state update; G: the epilogue), so their
// latency overlaps the chunk's work.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "tile_ops.cuh"

namespace la {
namespace ca {

using namespace la::tile;

constexpr int TILE = 128;
constexpr int D = 128;
constexpr int MATH_WARPS = 16;  // four per TMEM lane quarter: channel quarters of a row
constexpr int PARTS = MATH_WARPS / 4;
constexpr int CTRL_WARP = MATH_WARPS;
constexpr int THREADS = 32 * (MATH_WARPS + 1);
constexpr uint32_t HALF = 128 * 128;
constexpr uint32_t BUF = 2 * HALF;
constexpr uint32_t OFF_Q = 0, OFF_K = BUF, OFF_V = 2 * BUF, OFF_G = 3 * BUF, OFF_S = 4 * BUF;
constexpr uint32_t OFF_Z = 5 * BUF;              // z of the tokens before the chunk, [2 slots][128] fp32
constexpr uint32_t OFF_ZC = OFF_Z + 1024;        // the chunk's column sums of K^+, [128] fp32
constexpr uint32_t OFF_DX = OFF_ZC + 512;        // partial denominators, [2 slots][4 parts][128]
constexpr uint32_t OFF_BAR = OFF_DX + 2 * 4 * 512;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
// carried S; num; C then P (fp32); the masked P as bf16 (the A operand of P V); the mask M as
// bf16 (the A operand of C)
constexpr uint32_t COL_S = 0, COL_ND = 128, COL_P = 256, COL_PB = 384, COL_M = 448;
constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/false);
constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/true);
constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128, /*a_mn=*/true, /*b_mn=*/true);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Bars {
  uint64_t full_qk;   // Q and K of the chunk landed
  uint64_t full_v;    // V landed
  uint64_t full_g;    // G landed
  uint64_t relu;      // math: K^+ written in place (and, before the first chunk, M into TMEM)
  uint64_t qready;    // math: phi(Q) written in place
  uint64_t zready;    // math: z before chunk i published in slot i mod 2 (phase i; 16 warps)
  uint64_t dready;    // MMA: C = M K^+ done (and its operand reads)
  uint64_t rot;       // math: phi(K) written in place, C read
  uint64_t pdone;     // MMA: P done (num = phi(Q) S_prev too)
  uint64_t pready;    // MMA: the S update done too (the last reader of Q and K)
  uint64_t pw;        // math: masked P written to TMEM as bf16 (4 warps)
  uint64_t numready;  // MMA: num += P V done
  uint64_t out;       // math: O staged over G, S image rewritten (8 warps)
  uint64_t denx[4];   // the four warps holding the quarters of rows 32q .. 32q+31 (4 arrivals)
  uint64_t final_;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block too large");

template <int DT, int DH>
__global__ void __launch_bounds__(THREADS, 1)
causal_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                 const __grid_constant__ CUtensorMap tmO, const Plan p, const __grid_constant__ Rope rope,
                 const float* __restrict__ start, const float2* __restrict__ tab,
                 const float4* __restrict__ tab2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  float* zs = reinterpret_cast<float*>(smem + OFF_Z);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c);
  const int64_t g1 = cta_start(p, c + 1);
  volatile int* abort_flag = &bars->abort_flag;

  // Does this CTA's first unit start in an earlier CTA (then the start kernel summed its state)?
  bool has_start = false;
  if (g0 < g1) {
    int64_t first = 0, count = 0;
    unit_tiles(p, unit_of_tile(p, g0), &first, &count);
    has_start = cta_of(p, first) != c;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->full_qk, 1);
    mbar_init(&bars->full_v, 1);
    mbar_init(&bars->full_g, 1);
    mbar_init(&bars->relu, MATH_WARPS);
    mbar_init(&bars->qready, MATH_WARPS);
    mbar_init(&bars->zready, MATH_WARPS);
    mbar_init(&bars->pdone, 1);
    mbar_init(&bars->dready, 1);
    mbar_init(&bars->rot, MATH_WARPS);
    mbar_init(&bars->pready, 1);
    mbar_init(&bars->pw, MATH_WARPS);
    mbar_init(&bars->numready, 1);
    mbar_init(&bars->out, MATH_WARPS);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->denx[q], PARTS);
    mbar_init(&bars->final_, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CTRL_WARP) {
    tmem_alloc(&bars->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_trigger();

  if (warp == CTRL_WARP) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA + MMA issue
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmG);
      tma_prefetch_desc(&tmO);
      int64_t prev_unit = -1;
      // chunks whose loads have been armed on full_qk, full_v, full_g
      int64_t issued_qk = 0, issued_v = 0, issued_g = 0;
      auto load2 = [&](uint32_t off, const CUtensorMap* tm, const TileInfo& t, uint64_t* bar) {
        const int32_t n0 = static_cast<int32_t>(t.n0), bh = static_cast<int32_t>(t.bh);
        tma_load_3d(smem + off, tm, 0, n0, bh, bar);
        tma_load_3d(smem + off + HALF, tm, 64, n0, bh, bar);
      };
      if (g0 < g1) {
        const TileInfo t0 = tile_info(p, g0);
        mbar_arrive_expect_tx(&bars->full_qk, 2 * BUF);
        load2(OFF_Q, &tmQ, t0, &bars->full_qk);
        load2(OFF_K, &tmK, t0, &bars->full_qk);
        mbar_arrive_expect_tx(&bars->full_v, BUF);
        load2(OFF_V, &tmV, t0, &bars->full_v);
        mbar_arrive_expect_tx(&bars->full_g, BUF);
        load2(OFF_G, &tmG, t0, &bars->full_g);
        issued_qk = issued_v = issued_g = 1;
      }
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        const TileInfo ti = tile_info(p, g);
        const bool first = ti.unit != prev_unit;
        const bool zero_start = first && !(g == g0 && has_start);
        prev_unit = ti.unit;
        const bool has_next = g + 1 < g1;
        const TileInfo tn = has_next ? tile_info(p, g + 1) : ti;
        // C = M K^+ (into the P columns)
        if (!mbar_wait(&bars->relu, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + COL_P, tmem + COL_M + 8u * kk, desc_mn(sbase + OFF_K, kk), IDESC_QS, kk > 0 ? 1u : 0u);
        mma_commit(&bars->dready);
        // num = phi(Q) S_prev
        if (!mbar_wait(&bars->qready, ph, abort_flag)) break;
        tc_fence_after();
        if (!zero_start) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16(tmem + COL_ND, desc_k(sbase + OFF_Q, kk), desc_mn(sbase + OFF_S, kk), IDESC_QS,
                     kk > 0 ? 1u : 0u);
        }
        // P = phi(Q) phi(K)^T over C (read by then);  S += phi(K)^T V
        if (!mbar_wait(&bars->rot, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + COL_P, desc_k(sbase + OFF_Q, kk), desc_k(sbase + OFF_K, kk), IDESC_QK, kk > 0 ? 1u : 0u);
        mma_commit(&bars->pdone);
        if (!mbar_wait(&bars->full_v, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + COL_S, desc_mn(sbase + OFF_K, kk), desc_mn(sbase + OFF_V, kk), IDESC_KV,
                   (kk > 0 || !zero_start) ? 1u : 0u);
        mma_commit(&bars->pready);
        // Those products were the last readers of Q and K: the next chunk's Q and K can land
        // while this chunk's P V product and epilogue run.
        if (has_next) {
          if (!mbar_wait(&bars->pready, ph, abort_flag)) break;
          mbar_arrive_expect_tx(&bars->full_qk, 2 * BUF);
          load2(OFF_Q, &tmQ, tn, &bars->full_qk);
          load2(OFF_K, &tmK, tn, &bars->full_qk);
          ++issued_qk;
        }
        // num += (P o M) V
        if (!mbar_wait(&bars->pw, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + COL_ND, tmem + COL_PB + 8u * kk, desc_mn(sbase + OFF_V, kk), IDESC_QS,
                      (kk > 0 || !zero_start) ? 1u : 0u);
        mma_commit(&bars->numready);
        if (has_next) {
          if (!mbar_wait(&bars->numready, ph, abort_flag)) break;
          mbar_arrive_expect_tx(&bars->full_v, BUF);
          load2(OFF_V, &tmV, tn, &bars->full_v);
          ++issued_v;
        }
        // O of this chunk (staged over G) out, then the next chunk's G in.
        if (!mbar_wait(&bars->out, ph, abort_flag)) break;
        {
          const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
          tma_store_3d(&tmO, smem + OFF_G, 0, n0, bh);
          tma_store_3d(&tmO, smem + OFF_G + HALF, 64, n0, bh);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        if (has_next) {
          mbar_arrive_expect_tx(&bars->full_g, BUF);
          load2(OFF_G, &tmG, tn, &bars->full_g);
          ++issued_g;
        }
      }
      bulk_wait_group0();
      if (*abort_flag) {
        if (issued_qk > 0) mbar_wait_drain(&bars->full_qk, static_cast<uint32_t>((issued_qk - 1) & 1));
        if (issued_v > 0) mbar_wait_drain(&bars->full_v, static_cast<uint32_t>((issued_v - 1) & 1));
        if (issued_g > 0) mbar_wait_drain(&bars->full_g, static_cast<uint32_t>((issued_g - 1) & 1));
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else {
    // ------------------------------------------------------------ rows (warps 0-15)
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;  // token row of the chunk = TMEM lane
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t cpart = 32u * static_cast<uint32_t>(part);  // this warp's channels (and P columns)
    const uint32_t t_s = tmem + COL_S + lane_bits + cpart, t_nd = tmem + COL_ND + lane_bits + cpart;
    const uint32_t t_p = tmem + COL_P + lane_bits + cpart, t_pb = tmem + COL_PB + lane_bits + cpart / 2;
    float* zc = reinterpret_cast<float*>(smem + OFF_ZC);
    float* dx = reinterpret_cast<float*>(smem + OFF_DX);
    uint64_t* denx = &bars->denx[quarter];
    // The mask M: row `row`, this quarter's columns m = cpart .. cpart + 31 as bf16 pairs.
    {
      uint32_t mk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int m0 = static_cast<int>(cpart) + 2 * e;
        mk[e] = (m0 <= row ? 0x3F80u : 0u) | (m0 + 1 <= row ? 0x3F800000u : 0u);
      }
      tmem_st_x16(tmem + COL_M + lane_bits + cpart / 2, mk);
      tmem_st_wait();
    }
    pdl_wait();  // the start states and the cos/sin tables come from the kernels before
    if (g0 < g1 && has_start) {
      // Carried state at the segment start: this quarter of fp32 row `row` of S into TMEM, its
      // bf16 image, and z.
      const float* src = start + c * (D * D + D);
      uint32_t r[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(src[row * D + cpart + e]);
      tmem_st_x16(t_s, &r[0]);
      tmem_st_x16(t_s + 16, &r[16]);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        sts128(row_chunk(sbase + OFF_S, row, 4 * part + e),
               make_uint4(pack_bf16(__uint_as_float(r[8 * e]), __uint_as_float(r[8 * e + 1])),
                          pack_bf16(__uint_as_float(r[8 * e + 2]), __uint_as_float(r[8 * e + 3])),
                          pack_bf16(__uint_as_float(r[8 * e + 4]), __uint_as_float(r[8 * e + 5])),
                          pack_bf16(__uint_as_float(r[8 * e + 6]), __uint_as_float(r[8 * e + 7]))));
      tmem_st_wait();
      fence_proxy_async_smem();
    }
    // z before the first chunk (slot 0, phase 0 of zready).
    if (part == 0) zs[row] = (g0 < g1 && has_start) ? start[c * (D * D + D) + D * D + row] : 0.f;
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->zready);
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const TileInfo ti = tile_info(p, g);
      // Does the next chunk start a head (then its z starts from zero)?
      const bool next_new = g + 1 < g1 && unit_of_tile(p, g + 1) != ti.unit;
      if (!warp_wait(&bars->full_qk, ph, abort_flag)) break;
      // ReLU of this quarter of the Q and K rows; K^+ back in place, both kept in registers.
      uint32_t qa[16], ka[16];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint4 rq = lds128(row_chunk(sbase + OFF_Q, row, 4 * part + c4));
        qa[4 * c4] = relu_bf16x2(rq.x);
        qa[4 * c4 + 1] = relu_bf16x2(rq.y);
        qa[4 * c4 + 2] = relu_bf16x2(rq.z);
        qa[4 * c4 + 3] = relu_bf16x2(rq.w);
        const uint32_t ak = row_chunk(sbase + OFF_K, row, 4 * part + c4);
        const uint4 rk = lds128(ak);
        ka[4 * c4] = relu_bf16x2(rk.x);
        ka[4 * c4 + 1] = relu_bf16x2(rk.y);
        ka[4 * c4 + 2] = relu_bf16x2(rk.z);
        ka[4 * c4 + 3] = relu_bf16x2(rk.w);
        sts128(ak, make_uint4(ka[4 * c4], ka[4 * c4 + 1], ka[4 * c4 + 2], ka[4 * c4 + 3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->relu);
      // RoPE of this quarter of Q^+ over Q (no product reads Q before phi(Q)), while C runs.
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      uint32_t pt = 0, ph_ = 0, pw = 0;
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph_, pw);
      auto rot = [&](uint32_t (&a)[16]) {
        const int ipt = static_cast<int>(pt), iph = static_cast<int>(ph_), ipw = static_cast<int>(pw);
        switch (part) {
          case 0: rotate_span<DT, DH, 0, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 1: rotate_span<DT, DH, 16, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 2: rotate_span<DT, DH, 32, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          default: rotate_span<DT, DH, 48, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
        }
      };
      {
        uint32_t a[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) a[e] = qa[e];
        rot(a);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          sts128(row_chunk(sbase + OFF_Q, row, 4 * part + c4), make_uint4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qready);
      // This quarter's share of the denominator, q^+ . (z_prev + C_n) over its channels; the
      // last row's C is the chunk's column sums, which advance z for the next chunk.
      float dpart;
      if (!warp_wait(&bars->zready, ph, abort_flag)) break;
      {
        const float* zcur = zs + (i & 1) * 128;
        if (!warp_wait(&bars->dready, ph, abort_flag)) break;
        tc_fence_after();
        uint32_t r[32];
        tmem_ld_x32(t_p, r);
        tmem_ld_wait();
        float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
          const float4 z4 = *reinterpret_cast<const float4*>(zcur + cpart + 4 * k4);
          d4[0] = fmaf(bf16lo(qa[2 * k4]), z4.x + __uint_as_float(r[4 * k4]), d4[0]);
          d4[1] = fmaf(bf16hi(qa[2 * k4]), z4.y + __uint_as_float(r[4 * k4 + 1]), d4[1]);
          d4[2] = fmaf(bf16lo(qa[2 * k4 + 1]), z4.z + __uint_as_float(r[4 * k4 + 2]), d4[2]);
          d4[3] = fmaf(bf16hi(qa[2 * k4 + 1]), z4.w + __uint_as_float(r[4 * k4 + 3]), d4[3]);
        }
        dpart = (d4[0] + d4[1]) + (d4[2] + d4[3]);
        if (quarter == 3) {
          if (lane == 31) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              *reinterpret_cast<float4*>(zc + cpart + 4 * e) =
                  make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]), __uint_as_float(r[4 * e + 2]),
                              __uint_as_float(r[4 * e + 3]));
          }
          __syncwarp();
          const int k = static_cast<int>(cpart) + lane;
          zs[((i + 1) & 1) * 128 + k] = next_new ? 0.f : zcur[k] + zc[k];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->zready);
      // RoPE of this quarter of K^+ over K^+ (C, its last reader, is done).
      rot(ka);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        sts128(row_chunk(sbase + OFF_K, row, 4 * part + c4), make_uint4(ka[4 * c4], ka[4 * c4 + 1], ka[4 * c4 + 2], ka[4 * c4 + 3]));
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rot);
      float hinv;
      {
        float* slot = dx + static_cast<int>(i & 1) * (PARTS * 128);
        slot[part * 128 + row] = dpart;
        __syncwarp();
        if (lane == 0) mbar_arrive(denx);
        if (!warp_wait(denx, ph, abort_flag)) break;
        const float den = (slot[row] + slot[128 + row]) + (slot[256 + row] + slot[384 + row]);
        hinv = 1.0f / (den + p.eps);
      }
      // Causal mask on this quarter of P (columns m in [32 part, 32 part + 32), kept where m <= n),
      // written as bf16 to the A operand of P V (columns 16 part .. 16 part + 15 of that region).
      if (!warp_wait(&bars->pdone, ph, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t pb[16];
        uint32_t r[32];
        tmem_ld_x32(t_p, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int m0 = static_cast<int>(cpart) + 2 * e;
          const float p0 = m0 <= row ? __uint_as_float(r[2 * e]) : 0.f;
          const float p1 = m0 + 1 <= row ? __uint_as_float(r[2 * e + 1]) : 0.f;
          pb[e] = pack_bf16(p0, p1);
        }
        tmem_st_x16(t_pb, &pb[0]);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pw);
      // This quarter of the updated state's bf16 image, while P V runs (phi(Q) S_prev, the old
      // image's reader, finished before P).
      if (!warp_wait(&bars->pready, ph, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld_x32(t_s, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 4; ++e)
          sts128(row_chunk(sbase + OFF_S, row, 4 * part + e),
                 make_uint4(pack_bf16(__uint_as_float(r[8 * e]), __uint_as_float(r[8 * e + 1])),
                            pack_bf16(__uint_as_float(r[8 * e + 2]), __uint_as_float(r[8 * e + 3])),
                            pack_bf16(__uint_as_float(r[8 * e + 4]), __uint_as_float(r[8 * e + 5])),
                            pack_bf16(__uint_as_float(r[8 * e + 6]), __uint_as_float(r[8 * e + 7]))));
      }
      // O = num / den * sigmoid(g) for this quarter, in place over G.
      if (!warp_wait(&bars->numready, ph, abort_flag)) break;
      if (!warp_wait(&bars->full_g, ph, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t r[32];
        tmem_ld_x32(t_nd, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t ag = row_chunk(sbase + OFF_G, row, 4 * part + e);
          const uint4 gr = lds128(ag);
          const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
          uint32_t ov[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float o0 = __uint_as_float(r[8 * e + 2 * q]) * hinv * sigmoid_tanh(bf16lo(gw[q]));
            const float o1 = __uint_as_float(r[8 * e + 2 * q + 1]) * hinv * sigmoid_tanh(bf16hi(gw[q]));
            ov[q] = pack_bf16(o0, o1);
          }
          sts128(ag, make_uint4(ov[0], ov[1], ov[2], ov[3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->out);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == CTRL_WARP) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace ca
}  // namespace la
