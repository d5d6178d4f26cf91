// bwd_tc.cuh -- gradients of the bidirectional operator on the 5th-generation tensor cores
// (bf16, d = 128).
//
// Forward (SANA-Video 2.0, Eq. (1); SANA-Video Sec. 3.2): phi = RoPE(ReLU), S = sum phi(k)^T v,
// z = sum ReLU(k), num = phi(q) S, den = ReLU(q) . z + eps, y = num / den, o = y * sigmoid(g).
// Given dO, per token (ReLU'(x) = [x > 0], s = sigmoid(g)):
//   dg = dO y s (1 - s),  dy = dO s,  dnum = dy / den,  dden = -(dy . y) / den
//   dS = sum_n phi(q_n)^T dnum_n,  dz = sum_n dden_n ReLU(q_n)
//   dq = [q > 0] (RoPE^T(dnum S^T) + dden z)
//   dv = phi(k) dS,  dk = [k > 0] (RoPE^T(v dS^T) + dz)
//
// Two kernels, both walking the same persistent tile ranges as the forward state kernel, one
// 128-token tile at a time (warps 0-15: four per row, by channel quarters; thread = token = TMEM
// lane; warp 16: TMA and MMA issue).  Outputs are staged in buffers of their own, so the next
// tile's inputs load as soon as the products reading them are done; every input lands on a
// barrier of its own, waited for only by its first reader (the first kernel: Q with the state
// image and z, then dO, then G; the second: K with the dS image and dz, then V), and the two
// products of a tile are committed apart so each epilogue waits only for the one it reads:
//   bwdq_tc_kernel: num = phi(Q) S and dphi(q) = dnum S^T (the state's bf16 image serves as S,
//     read N-major, and as S^T, read K-major), dS += phi(Q)^T dnum (TMEM accumulator drained to
//     the CTA's partial slot at the end of each unit, like the state kernel); dQ, dG out.
//   bwdk_tc_kernel: dV = phi(K) dS and dphi(k) = V dS^T (the bf16 image of dS that the combine
//     kernel builds from those partial slots); dK, dV out.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "tile_ops.cuh"

namespace la {
namespace bw {

using namespace la::tile;

constexpr int TILE = 128;
constexpr int D = 128;
constexpr int MATH_WARPS = 16;  // four per TMEM lane quarter: channel quarters of a row
constexpr int PARTS = MATH_WARPS / 4;
constexpr int CTRL_WARP = MATH_WARPS;
constexpr int THREADS = 32 * (MATH_WARPS + 1);
constexpr uint32_t BUF = 2 * HALF;
constexpr int ZPARTS = 4;  // dz partial rows per slot: one per lane quarter (the channel quarters
                           // fill disjoint channels of a row)
constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/true);   // X S
constexpr uint32_t IDESC_QST = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/false); // X S^T
constexpr uint32_t IDESC_TD = idesc_bf16_f32(128, 128, /*a_mn=*/true, /*b_mn=*/true);    // X^T Y

// ---- bwdq smem: Q (-> phi(Q)), G (-> dG), dO (-> dnum), S image, dQ staging, exchanges
constexpr uint32_t QO_Q = 0, QO_G = BUF, QO_DO = 2 * BUF, QO_S = 3 * BUF, QO_DQ = 4 * BUF;
constexpr uint32_t QO_X = 5 * BUF;  // [3 values][4 parts][128] fp32: partial den, dy.y (RMSNorm: sum y^2, sum y du gamma)
constexpr uint32_t QO_Z = QO_X + 3 * PARTS * 512;  // z of the unit, [2 slots by unit parity][128] fp32
constexpr uint32_t QO_BAR = QO_Z + 1024;
constexpr uint32_t SMEM_Q = QO_BAR + 256 + 1024;
constexpr uint32_t QCOL_NUM = 0, QCOL_DPQ = 128, QCOL_DS = 256;
// ---- bwdk smem: K (-> phi(K)), V, dS image, dK and dV staging
constexpr uint32_t KO_K = 0, KO_V = BUF, KO_S = 2 * BUF, KO_DK = 3 * BUF, KO_DV = 4 * BUF;
constexpr uint32_t KO_Z = 5 * BUF;  // dz of the unit, [2 slots by unit parity][128] fp32
constexpr uint32_t KO_X = KO_Z + 1024;  // [2 slots by tile parity][4 parts][128] fp32: partial dbeta
constexpr uint32_t KO_BAR = KO_X + 2 * PARTS * 512;
constexpr uint32_t SMEM_K = KO_BAR + 256 + 1024;
constexpr uint32_t KCOL_DV = 0, KCOL_DPK = 128;
static_assert(SMEM_Q <= 232448 && SMEM_K <= 232448, "shared memory budget");

struct BarsQ {
  uint64_t full;     // Q (and the state image and z at a unit's first tile) landed
  uint64_t full_do;  // dO landed
  uint64_t full_g;   // G landed
  uint64_t rot, numready, dn;
  uint64_t dpqready;  // MMA: dphi(q) = dnum S^T done (the last reader of the state image)
  uint64_t qfree;     // MMA: dS += phi(Q)^T dnum done too (the last reader of Q and dnum)
  uint64_t out, final_;
  uint64_t pair[4];  // the four warps of rows 32q .. 32q+31: two meetings per tile (den, then dy.y)
  uint32_t tmem_base;
  int abort_flag;
};
struct BarsK {
  uint64_t pair[4];  // the four warps of rows 32q .. 32q+31 (write gate: partial dbeta)
  uint64_t full;    // K (and the dS image at a unit's first tile) landed
  uint64_t full_v;  // V landed
  uint64_t rot;
  uint64_t dvready;  // MMA: dV = phi(K) dS done
  uint64_t ready;    // MMA: dphi(k) = V dS^T done too (the last reader of K, V, the dS image)
  uint64_t out, final_;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(BarsQ) <= 256 && sizeof(BarsK) <= 256, "barrier block too large");

__device__ __forceinline__ float tanh_f(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

// RMS: RMSNorm before the output gate (SANA-Video 2.0, Eq. (1)); its gradient is formed from two
// row sums, sum y^2 and sum y du gamma, which the four quarters of a row swap once, and dgamma's
// column sums are kept per warp and written to dgamma_part[(CTA * 4 + lane quarter) * D + channel].
template <int DT, int DH, bool RMS>
__global__ void __launch_bounds__(THREADS, 1)
bwdq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
               const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmDQ,
               const __grid_constant__ CUtensorMap tmDG, const Plan p, const __grid_constant__ Rope rope,
               const uint8_t* __restrict__ simg, const float* __restrict__ zimg, const float2* __restrict__ tab,
               const float4* __restrict__ tab2, float* __restrict__ partial, __nv_bfloat16* __restrict__ dQg,
               __nv_bfloat16* __restrict__ dGg, const float* __restrict__ gamma, float norm_eps,
               float* __restrict__ dgamma_part) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  BarsQ* bars = reinterpret_cast<BarsQ*>(smem + QO_BAR);
  float* xch = reinterpret_cast<float*>(smem + QO_X);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c);
  const int64_t g1 = cta_start(p, c + 1);
  const int64_t u_first = unit_of_tile(p, g0);
  volatile int* abort_flag = &bars->abort_flag;
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(ZPARTS) * D;

  if (threadIdx.x == 0) {
    mbar_init(&bars->full, 1);
    mbar_init(&bars->full_do, 1);
    mbar_init(&bars->full_g, 1);
    mbar_init(&bars->rot, MATH_WARPS);
    mbar_init(&bars->numready, 1);
    mbar_init(&bars->dn, MATH_WARPS);
    mbar_init(&bars->qfree, 1);
    mbar_init(&bars->dpqready, 1);
    mbar_init(&bars->out, MATH_WARPS);
    mbar_init(&bars->final_, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], PARTS);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CTRL_WARP) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_trigger();
  // Everything below reads what the kernels before wrote (state image, z, tables) or writes the
  // partial slots the combine kernel before read: wait for them first.
  pdl_wait();

  if (warp == CTRL_WARP) {
    if (lane == 0) {
      auto load2 = [&](uint32_t off, const CUtensorMap* tm, const TileInfo& t, uint64_t* bar) {
        const int32_t n0 = static_cast<int32_t>(t.n0), bh = static_cast<int32_t>(t.bh);
        tma_load_3d(smem + off, tm, 0, n0, bh, bar);
        tma_load_3d(smem + off + HALF, tm, 64, n0, bh, bar);
      };
      int64_t issued = 0, issued_do = 0, issued_g = 0;
      int64_t zslot = 0;  // z slot of the unit being loaded (unit parity within the CTA)
      if (g0 < g1) {
        const TileInfo t0 = tile_info(p, g0);
        mbar_arrive_expect_tx(&bars->full, 2 * BUF + 512);
        bulk_load(smem + QO_S, simg + t0.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
        bulk_load(smem + QO_Z, zimg + t0.unit * D, 512, &bars->full);
        load2(QO_Q, &tmQ, t0, &bars->full);
        mbar_arrive_expect_tx(&bars->full_do, BUF);
        load2(QO_DO, &tmDO, t0, &bars->full_do);
        mbar_arrive_expect_tx(&bars->full_g, BUF);
        load2(QO_G, &tmG, t0, &bars->full_g);
        issued = issued_do = issued_g = 1;
      }
      int64_t prev_unit = -1;
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        const TileInfo ti = tile_info(p, g);
        const bool first = ti.unit != prev_unit;
        prev_unit = ti.unit;
        const bool has_next = g + 1 < g1;
        const TileInfo tn = has_next ? tile_info(p, g + 1) : ti;
        const bool next_new_unit = has_next && tn.unit != ti.unit;
        // num = phi(Q) S
        if (!mbar_wait(&bars->rot, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_NUM, desc_k(sbase + QO_Q, kk), desc_mn(sbase + QO_S, kk), IDESC_QS, kk > 0 ? 1u : 0u);
        mma_commit(&bars->numready);
        // dS += phi(Q)^T dnum (frees Q first);  dphi(q) = dnum S^T
        if (!mbar_wait(&bars->dn, ph, abort_flag)) break;
        tc_fence_after();
        // The gate pass has written this tile's dG over G: it goes out now (one bulk group), so
        // that G's buffer can take the next tile's G while this tile's dq epilogue runs.  A tile
        // that ends inside a head's block (block-causal units) is written out row by row by the
        // math warps; its groups stay (empty) so the group accounting is the same.
        const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
        const int32_t tn0 = static_cast<int32_t>(ti.n0), tbh = static_cast<int32_t>(ti.bh);
        if (tma_out) {
          tma_store_3d(&tmDG, smem + QO_G, 0, tn0, tbh);
          tma_store_3d(&tmDG, smem + QO_G + HALF, 64, tn0, tbh);
        }
        bulk_commit_group();
        // dphi(q) first: the math warps wait for it (dq epilogue); dS is read only at the end of a
        // unit, and its completion frees Q for the next tile.
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_DPQ, desc_k(sbase + QO_DO, kk), desc_k(sbase + QO_S, kk), IDESC_QST, kk > 0 ? 1u : 0u);
        // The previous tile's dQ (the older of the two groups in flight) has left the staging
        // buffer the dq epilogue reuses.
        bulk_wait_group_read1();
        mma_commit(&bars->dpqready);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_DS, desc_mn(sbase + QO_Q, kk), desc_mn(sbase + QO_DO, kk), IDESC_TD,
                   (kk > 0 || !first) ? 1u : 0u);
        mma_commit(&bars->qfree);
        // The next tile's Q and dO once dS, the last product, has read this tile's (and, at a new
        // unit, the state image and z with them); its G once this tile's dG has been read out.
        if (has_next) {
          if (!mbar_wait(&bars->qfree, ph, abort_flag)) break;
          mbar_arrive_expect_tx(&bars->full, BUF + (next_new_unit ? BUF + 512u : 0u));
          if (next_new_unit) {
            zslot ^= 1;
            bulk_load(smem + QO_S, simg + tn.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
            bulk_load(smem + QO_Z + 512u * static_cast<uint32_t>(zslot), zimg + tn.unit * D, 512, &bars->full);
          }
          load2(QO_Q, &tmQ, tn, &bars->full);
          ++issued;
          mbar_arrive_expect_tx(&bars->full_do, BUF);
          load2(QO_DO, &tmDO, tn, &bars->full_do);
          ++issued_do;
          bulk_wait_group_read0();
          mbar_arrive_expect_tx(&bars->full_g, BUF);
          load2(QO_G, &tmG, tn, &bars->full_g);
          ++issued_g;
        }
        // dQ (staged) of this tile out.
        if (!mbar_wait(&bars->out, ph, abort_flag)) break;
        if (tma_out) {
          tma_store_3d(&tmDQ, smem + QO_DQ, 0, tn0, tbh);
          tma_store_3d(&tmDQ, smem + QO_DQ + HALF, 64, tn0, tbh);
        }
        bulk_commit_group();
      }
      bulk_wait_group0();
      if (*abort_flag) {
        if (issued > 0) mbar_wait_drain(&bars->full, static_cast<uint32_t>((issued - 1) & 1));
        if (issued_do > 0) mbar_wait_drain(&bars->full_do, static_cast<uint32_t>((issued_do - 1) & 1));
        if (issued_g > 0) mbar_wait_drain(&bars->full_g, static_cast<uint32_t>((issued_g - 1) & 1));
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else {
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const int cpart = 32 * part;  // this warp's channels
    uint64_t* pr = &bars->pair[quarter];
    float dzacc = 0.f;  // dz of channel 32 part + lane over this warp's rows
    float dgacc = 0.f;  // RMSNorm: dgamma of channel 32 part + lane over this warp's rows
    int zslot = 0;      // z slot of the current unit
    int64_t prev_unit = -1;
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const TileInfo ti = tile_info(p, g);
      const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != ti.unit);
      if (prev_unit >= 0 && ti.unit != prev_unit) zslot ^= 1;
      prev_unit = ti.unit;
      if (!warp_wait(&bars->full, ph, abort_flag)) break;
      // q^+ of this quarter kept packed; phi(q) written in place.
      uint32_t qa[16];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint4 rq = lds128(row_chunk(sbase + QO_Q, row, 4 * part + c4));
        qa[4 * c4] = relu_bf16x2(rq.x);
        qa[4 * c4 + 1] = relu_bf16x2(rq.y);
        qa[4 * c4 + 2] = relu_bf16x2(rq.z);
        qa[4 * c4 + 3] = relu_bf16x2(rq.w);
      }
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      // Rows past the end of the unit (the next block of the head) take no part: a zero query
      // adds nothing to dS or dz, and their outputs are not written.
      const bool valid = static_cast<int64_t>(n) < ti.n_end;
      const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
      if (!valid) {
#pragma unroll
        for (int e = 0; e < 16; ++e) qa[e] = 0u;
      }
      __nv_bfloat16* dq_row = dQg + (ti.bh * p.N + static_cast<int64_t>(n)) * D + cpart;
      __nv_bfloat16* dg_row = dGg + (ti.bh * p.N + static_cast<int64_t>(n)) * D + cpart;
      uint32_t pt = 0, ph_ = 0, pw = 0;
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph_, pw);
      const int ipt = static_cast<int>(pt), iph = static_cast<int>(ph_), ipw = static_cast<int>(pw);
      {
        uint32_t a[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) a[e] = qa[e];
        switch (part) {
          case 0: rotate_span<DT, DH, 0, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 1: rotate_span<DT, DH, 16, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 2: rotate_span<DT, DH, 32, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          default: rotate_span<DT, DH, 48, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          sts128(row_chunk(sbase + QO_Q, row, 4 * part + c4), make_uint4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rot);
      // den = q^+ . z + eps: each quarter's share, then the four add them in a fixed order.
      const float* zg = reinterpret_cast<const float*>(smem + QO_Z) + zslot * D + cpart;
      float dpart = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        const float4 z4 = *reinterpret_cast<const float4*>(zg + 4 * k4);
        dpart = fmaf(bf16lo(qa[2 * k4]), z4.x, dpart);
        dpart = fmaf(bf16hi(qa[2 * k4]), z4.y, dpart);
        dpart = fmaf(bf16lo(qa[2 * k4 + 1]), z4.z, dpart);
        dpart = fmaf(bf16hi(qa[2 * k4 + 1]), z4.w, dpart);
      }
      xch[part * 128 + row] = dpart;
      __syncwarp();
      if (lane == 0) mbar_arrive(pr);
      if (!warp_wait(pr, 0u, abort_flag)) break;
      const float den = ((xch[row] + xch[128 + row]) + (xch[256 + row] + xch[384 + row])) + p.eps;
      const float rden = 1.0f / den;
      // num -> y; with G and dO: dG (over G), dnum (over dO), this quarter's dy . y.
      if (!warp_wait(&bars->numready, ph, abort_flag)) break;
      if (!warp_wait(&bars->full_g, ph, abort_flag)) break;
      if (!warp_wait(&bars->full_do, ph, abort_flag)) break;
      tc_fence_after();
      float dden;
      if constexpr (!RMS) {
      // Channel pairs in packed fp32 (sigmoid(g) = 1/2 + tanh(g/2)/2, with g/2 exact in bf16):
      //   y = num / den, dy = dO s, dG = dy y (1 - s), dnum = dy / den, dy . y accumulated.
      const uint64_t rden2 = pk(rden, rden), half2 = pk(0.5f, 0.5f), mhalf2 = pk(-0.5f, -0.5f);
      uint64_t dyy2 = 0;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // num of 16 channels at a time (fewer live registers)
        uint32_t r[16];
        tmem_ld_x16(tmem + QCOL_NUM + lane_bits + static_cast<uint32_t>(cpart) + 16u * static_cast<uint32_t>(hh), r);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ck = 4 * part + 2 * hh + cc;
          const uint32_t ag = row_chunk(sbase + QO_G, row, ck);
          const uint4 gr = lds128(ag);
          const uint32_t ad = row_chunk(sbase + QO_DO, row, ck);
          const uint4 dr = lds128(ad);
          const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w}, dw[4] = {dr.x, dr.y, dr.z, dr.w};
          uint32_t dgw[4], dnw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = 8 * cc + 2 * q;
            const uint32_t gh = half_bf16x2(gw[q]);
            const uint64_t t2 = pk(tanh_f(bf16lo(gh)), tanh_f(bf16hi(gh)));
            const uint64_t sg2 = fma2(t2, half2, half2), om2 = fma2(t2, mhalf2, half2);
            const uint64_t y2 = mul2(pk(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), rden2);
            const uint64_t dy2 = mul2(pk(bf16lo(dw[q]), bf16hi(dw[q])), sg2);
            const float2 dg = upk(mul2(mul2(dy2, y2), om2));
            const float2 dn = upk(mul2(dy2, rden2));
            dyy2 = fma2(dy2, y2, dyy2);
            dgw[q] = pack_bf16(dg.x, dg.y);
            dnw[q] = pack_bf16(dn.x, dn.y);
          }
          if (tma_out) sts128(ag, make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]));
          else if (valid) *reinterpret_cast<uint4*>(dg_row + 8 * (2 * hh + cc)) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
          sts128(ad, make_uint4(dnw[0], dnw[1], dnw[2], dnw[3]));
        }
      }
      float dyy;
      {
        const float2 d = upk(dyy2);
        dyy = d.x + d.y;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dn);
      xch[PARTS * 128 + part * 128 + row] = dyy;
      __syncwarp();
      if (lane == 0) mbar_arrive(pr);
      if (!warp_wait(pr, 1u, abort_flag)) break;
      const float* yx = xch + PARTS * 128;
      dden = -((yx[row] + yx[128 + row]) + (yx[256 + row] + yx[384 + row])) * rden;
      } else {
      // RMSNorm before the gate: with y = num / den, r = sqrt(mean(y^2) + norm_eps), yh = y / r,
      // u = yh gamma, s = sigmoid(g), du = dO s:
      //   dG = dO u s (1 - s),  dy = (du gamma - yh (yh . du gamma) / d) / r,  dnum = dy / den,
      //   dy . y = (1/r) T (1 - SS / (d r^2)) with SS = sum y^2, T = sum y du gamma,
      // so the row needs only SS and T from the other quarters (pass 1), then pass 2 forms every
      // output.  dgamma += du yh per channel.
      float ssp = 0.f, ttp = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[16];
        tmem_ld_x16(tmem + QCOL_NUM + lane_bits + static_cast<uint32_t>(cpart) + 16u * static_cast<uint32_t>(hh), r);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ck = 4 * part + 2 * hh + cc;
          const uint4 gr = lds128(row_chunk(sbase + QO_G, row, ck));
          const uint4 dr = lds128(row_chunk(sbase + QO_DO, row, ck));
          const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w}, dw[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = 8 * cc + 2 * q;
            const int ch = 8 * ck + 2 * q;
            const uint32_t gh = half_bf16x2(gw[q]);
            const float s0 = 0.5f + 0.5f * tanh_f(bf16lo(gh)), s1 = 0.5f + 0.5f * tanh_f(bf16hi(gh));
            const float y0 = __uint_as_float(r[e]) * rden, y1 = __uint_as_float(r[e + 1]) * rden;
            const float g0 = gamma ? __ldg(gamma + ch) : 1.f, g1 = gamma ? __ldg(gamma + ch + 1) : 1.f;
            ssp = fmaf(y0, y0, fmaf(y1, y1, ssp));
            ttp = fmaf(y0 * g0, bf16lo(dw[q]) * s0, fmaf(y1 * g1, bf16hi(dw[q]) * s1, ttp));
          }
        }
      }
      xch[PARTS * 128 + part * 128 + row] = ssp;
      xch[2 * PARTS * 128 + part * 128 + row] = ttp;
      __syncwarp();
      if (lane == 0) mbar_arrive(pr);
      if (!warp_wait(pr, 1u, abort_flag)) break;
      const float* sx = xch + PARTS * 128;
      const float* tx = xch + 2 * PARTS * 128;
      const float SS = (sx[row] + sx[128 + row]) + (sx[256 + row] + sx[384 + row]);
      const float TT = (tx[row] + tx[128 + row]) + (tx[256 + row] + tx[384 + row]);
      const float rinv = rsqrtf(SS * (1.f / D) + norm_eps);
      const float dotd = rinv * TT * (1.f / D);  // (yh . dyh) / d
      dden = -(rinv * TT * (1.f - rinv * rinv * SS * (1.f / D))) * rden;
      float gv[32];  // du yh of this quarter's 32 channels (dgamma)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t r[16];
        tmem_ld_x16(tmem + QCOL_NUM + lane_bits + static_cast<uint32_t>(cpart) + 16u * static_cast<uint32_t>(hh), r);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int ck = 4 * part + 2 * hh + cc;
          const uint32_t ag = row_chunk(sbase + QO_G, row, ck);
          const uint4 gr = lds128(ag);
          const uint32_t ad = row_chunk(sbase + QO_DO, row, ck);
          const uint4 dr = lds128(ad);
          const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w}, dw[4] = {dr.x, dr.y, dr.z, dr.w};
          uint32_t dgw[4], dnw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = 8 * cc + 2 * q;
            const int ch = 8 * ck + 2 * q;
            const uint32_t gh = half_bf16x2(gw[q]);
            float o_g[2], o_n[2];
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const float sgm = 0.5f + 0.5f * tanh_f(h2 ? bf16hi(gh) : bf16lo(gh));
              const float y = __uint_as_float(r[e + h2]) * rden;
              const float yh = y * rinv;
              const float gmv = gamma ? __ldg(gamma + ch + h2) : 1.f;
              const float dov = h2 ? bf16hi(dw[q]) : bf16lo(dw[q]);
              const float du = dov * sgm;
              o_g[h2] = dov * yh * gmv * sgm * (1.f - sgm);
              o_n[h2] = (du * gmv - yh * dotd) * rinv * rden;
              gv[16 * hh + e + h2] = du * yh;
            }
            dgw[q] = pack_bf16(o_g[0], o_g[1]);
            dnw[q] = pack_bf16(o_n[0], o_n[1]);
          }
          if (tma_out) sts128(ag, make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]));
          else if (valid) *reinterpret_cast<uint4*>(dg_row + 8 * (2 * hh + cc)) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
          sts128(ad, make_uint4(dnw[0], dnw[1], dnw[2], dnw[3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dn);
      // dgamma over this warp's 32 rows for this quarter's 32 channels (rows past the unit's end
      // have yh = 0): lane L ends with channel 32 part + L, as for dz below.
#pragma unroll
      for (int off = 16, size = 32; off >= 1; off >>= 1, size >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int e = 0; e < size / 2; ++e) {
          const float keep = up ? gv[e + size / 2] : gv[e];
          const float send = up ? gv[e] : gv[e + size / 2];
          const float other = __shfl_xor_sync(0xffffffffu, send, off);
          gv[e] = keep + other;  // (IEEE addition commutes: both lanes form the same sum)
        }
      }
      dgacc += gv[0];
      }
      // dz over this warp's 32 rows for this quarter's 32 channels: lane L ends with channel
      // 32 part + L (a butterfly that halves the range per step, each sum formed once).
      {
        float v[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          v[2 * e] = dden * bf16lo(qa[e]);
          v[2 * e + 1] = dden * bf16hi(qa[e]);
        }
#pragma unroll
        for (int off = 16, size = 32; off >= 1; off >>= 1, size >>= 1) {
          const bool up = (lane & off) != 0;
#pragma unroll
          for (int e = 0; e < size / 2; ++e) {
            const float keep = up ? v[e + size / 2] : v[e];
            const float send = up ? v[e] : v[e + size / 2];
            const float other = __shfl_xor_sync(0xffffffffu, send, off);
            v[e] = keep + other;  // (IEEE addition commutes: both lanes form the same sum)
          }
        }
        dzacc += v[0];
      }
      // dq = [q > 0] (RoPE^T(dnum S^T) + dden z) for this quarter, into the dQ staging buffer.
      if (!warp_wait(&bars->dpqready, ph, abort_flag)) break;
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // 16 channels at a time (fewer live registers)
        float x[16];
        {
          uint32_t r[16];
          tmem_ld_x16(tmem + QCOL_DPQ + lane_bits + static_cast<uint32_t>(cpart) + 16u * static_cast<uint32_t>(hh), r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(r[e]);
        }
        switch (2 * part + hh) {
          case 0: rotate_span_t<DT, DH, 0, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 1: rotate_span_t<DT, DH, 8, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 2: rotate_span_t<DT, DH, 16, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 3: rotate_span_t<DT, DH, 24, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 4: rotate_span_t<DT, DH, 32, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 5: rotate_span_t<DT, DH, 40, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 6: rotate_span_t<DT, DH, 48, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
          default: rotate_span_t<DT, DH, 56, 8>(x, tab, tab2, rope, p, ipt, iph, ipw); break;
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c4 = 2 * hh + cc;
          const float4 za = *reinterpret_cast<const float4*>(zg + 8 * c4);
          const float4 zb = *reinterpret_cast<const float4*>(zg + 8 * c4 + 4);
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t w = qa[4 * c4 + e / 2];
            const float qv = (e & 1) ? bf16hi(w) : bf16lo(w);
            o8[e] = qv > 0.f ? x[8 * cc + e] + dden * zz[e] : 0.f;
          }
          if (tma_out) sts128(row_chunk(sbase + QO_DQ, row, 4 * part + c4), pack8(o8));
          else if (valid) *reinterpret_cast<uint4*>(dq_row + 8 * c4) = pack8(o8);
        }
      }
      if (last) {
        // dS of this unit (TMEM lane = channel k of phi(Q); this quarter's 32 columns) and dz ->
        // the CTA's partial slot.
        if (!warp_wait(&bars->qfree, ph, abort_flag)) break;
        tc_fence_after();
        if (!in_bounds(ti.unit - u_first < p.maxseg)) break;
        float* dst = partial + (c * p.maxseg + (ti.unit - u_first)) * slot_floats;
        uint32_t r[32];
        tmem_ld_x32(tmem + QCOL_DS + lane_bits + static_cast<uint32_t>(cpart), r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 8; ++e)
          reinterpret_cast<float4*>(dst + row * D + cpart)[e] =
              make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]), __uint_as_float(r[4 * e + 2]),
                          __uint_as_float(r[4 * e + 3]));
        dst[D * D + quarter * D + cpart + lane] = dzacc;
        dzacc = 0.f;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->out);
    }
    // This warp's dgamma column sums (rows 32 quarter .. +31 of every tile of the CTA).
    if (RMS && dgamma_part) dgamma_part[(c * 4 + quarter) * D + cpart + lane] = dgacc;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == CTRL_WARP) tmem_dealloc(tmem, 512);
}

// BETA: the write gate of SANA-Video 2.0, Eq. (1), which scales each key's term of S:
// dV = beta phi(K) dS, dphi(k) = beta V dS^T, and dbeta = phi(k) . (V dS^T) per row (the four
// quarters of a row add their shares through shared memory).
template <int DT, int DH, bool BETA>
__global__ void __launch_bounds__(THREADS, 1)
bwdk_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV, const Plan p,
               const __grid_constant__ Rope rope, const uint8_t* __restrict__ dsimg, const float* __restrict__ dzimg,
               const float2* __restrict__ tab, const float4* __restrict__ tab2, __nv_bfloat16* __restrict__ dKg,
               __nv_bfloat16* __restrict__ dVg, const __nv_bfloat16* __restrict__ beta,
               __nv_bfloat16* __restrict__ dbeta) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  BarsK* bars = reinterpret_cast<BarsK*>(smem + KO_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c);
  const int64_t g1 = cta_start(p, c + 1);
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars->full, 1);
    mbar_init(&bars->full_v, 1);
    mbar_init(&bars->rot, MATH_WARPS);
    mbar_init(&bars->dvready, 1);
    mbar_init(&bars->ready, 1);
    mbar_init(&bars->out, MATH_WARPS);
    mbar_init(&bars->final_, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bars->pair[q], PARTS);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == CTRL_WARP) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_trigger();
  pdl_wait();

  if (warp == CTRL_WARP) {
    if (lane == 0) {
      auto load2 = [&](uint32_t off, const CUtensorMap* tm, const TileInfo& t, uint64_t* bar) {
        const int32_t n0 = static_cast<int32_t>(t.n0), bh = static_cast<int32_t>(t.bh);
        tma_load_3d(smem + off, tm, 0, n0, bh, bar);
        tma_load_3d(smem + off + HALF, tm, 64, n0, bh, bar);
      };
      int64_t issued = 0, issued_v = 0;
      int64_t zslot = 0;  // dz slot of the unit being loaded (unit parity within the CTA)
      if (g0 < g1) {
        const TileInfo t0 = tile_info(p, g0);
        mbar_arrive_expect_tx(&bars->full, 2 * BUF + 512);
        bulk_load(smem + KO_S, dsimg + t0.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
        bulk_load(smem + KO_Z, dzimg + t0.unit * D, 512, &bars->full);
        load2(KO_K, &tmK, t0, &bars->full);
        mbar_arrive_expect_tx(&bars->full_v, BUF);
        load2(KO_V, &tmV, t0, &bars->full_v);
        issued = issued_v = 1;
      }
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        const TileInfo ti = tile_info(p, g);
        const bool has_next = g + 1 < g1;
        const TileInfo tn = has_next ? tile_info(p, g + 1) : ti;
        const bool next_new_unit = has_next && tn.unit != ti.unit;
        if (!mbar_wait(&bars->rot, ph, abort_flag)) break;
        tc_fence_after();
        // dV = phi(K) dS;  dphi(k) = V dS^T
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + KCOL_DV, desc_k(sbase + KO_K, kk), desc_mn(sbase + KO_S, kk), IDESC_QS, kk > 0 ? 1u : 0u);
        bulk_wait_group_read1();  // the previous tile's dV has left its staging buffer
        mma_commit(&bars->dvready);
        if (!mbar_wait(&bars->full_v, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + KCOL_DPK, desc_k(sbase + KO_V, kk), desc_k(sbase + KO_S, kk), IDESC_QST, kk > 0 ? 1u : 0u);
        bulk_wait_group_read0();  // and its dK
        mma_commit(&bars->ready);
        // The products were the last readers of K, V and the dS image: the next tile's land now.
        if (has_next) {
          if (!mbar_wait(&bars->ready, ph, abort_flag)) break;
          mbar_arrive_expect_tx(&bars->full, BUF + (next_new_unit ? BUF + 512u : 0u));
          if (next_new_unit) {
            zslot ^= 1;
            bulk_load(smem + KO_S, dsimg + tn.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
            bulk_load(smem + KO_Z + 512u * static_cast<uint32_t>(zslot), dzimg + tn.unit * D, 512, &bars->full);
          }
          load2(KO_K, &tmK, tn, &bars->full);
          mbar_arrive_expect_tx(&bars->full_v, BUF);
          load2(KO_V, &tmV, tn, &bars->full_v);
          ++issued;
          ++issued_v;
        }
        // dV and dK of this tile out, as two groups; their reads are waited for before the next
        // tile's products are committed to the epilogues that rewrite the staging buffers.
        if (!mbar_wait(&bars->out, ph, abort_flag)) break;
        {
          // (a tile that ends inside a head's block was written out row by row by the math warps)
          const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
          const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
          if (tma_out) {
            tma_store_3d(&tmDV, smem + KO_DV, 0, n0, bh);
            tma_store_3d(&tmDV, smem + KO_DV + HALF, 64, n0, bh);
          }
          bulk_commit_group();
          if (tma_out) {
            tma_store_3d(&tmDK, smem + KO_DK, 0, n0, bh);
            tma_store_3d(&tmDK, smem + KO_DK + HALF, 64, n0, bh);
          }
          bulk_commit_group();
        }
      }
      bulk_wait_group0();
      if (*abort_flag) {
        if (issued > 0) mbar_wait_drain(&bars->full, static_cast<uint32_t>((issued - 1) & 1));
        if (issued_v > 0) mbar_wait_drain(&bars->full_v, static_cast<uint32_t>((issued_v - 1) & 1));
      }
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else {
    const int quarter = warp & 3, part = warp >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const int cpart = 32 * part;  // this warp's channels
    int zslot = 0;                // dz slot of the current unit
    int64_t prev_unit = -1;
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const TileInfo ti = tile_info(p, g);
      if (prev_unit >= 0 && ti.unit != prev_unit) zslot ^= 1;
      prev_unit = ti.unit;
      if (!warp_wait(&bars->full, ph, abort_flag)) break;
      uint32_t ka[16];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint4 rk = lds128(row_chunk(sbase + KO_K, row, 4 * part + c4));
        ka[4 * c4] = rk.x;
        ka[4 * c4 + 1] = rk.y;
        ka[4 * c4 + 2] = rk.z;
        ka[4 * c4 + 3] = rk.w;
      }
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      // Rows past the end of the unit (the next block of the head) are not written.
      const bool valid = static_cast<int64_t>(n) < ti.n_end;
      const bool tma_out = (ti.n0 + TILE <= ti.n_end) || (ti.n_end == p.N);
      __nv_bfloat16* dk_row = dKg + (ti.bh * p.N + static_cast<int64_t>(n)) * D + cpart;
      __nv_bfloat16* dv_row = dVg + (ti.bh * p.N + static_cast<int64_t>(n)) * D + cpart;
      uint32_t pt = 0, ph_ = 0, pw = 0;
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph_, pw);
      const int ipt = static_cast<int>(pt), iph = static_cast<int>(ph_), ipw = static_cast<int>(pw);
      // The row's write gate (1 without one).
      const float bt = (BETA && valid) ? __bfloat162float(beta[ti.bh * p.N + n]) : 1.f;
      uint32_t kr[16];  // phi(k) of this quarter, kept for dbeta
      {
        uint32_t a[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) a[e] = relu_bf16x2(ka[e]);
        switch (part) {
          case 0: rotate_span<DT, DH, 0, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 1: rotate_span<DT, DH, 16, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 2: rotate_span<DT, DH, 32, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
          default: rotate_span<DT, DH, 48, 16>(a, tab, tab2, rope, p, ipt, iph, ipw); break;
        }
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          sts128(row_chunk(sbase + KO_K, row, 4 * part + c4), make_uint4(a[4 * c4], a[4 * c4 + 1], a[4 * c4 + 2], a[4 * c4 + 3]));
#pragma unroll
        for (int e = 0; e < 16; ++e) kr[e] = BETA ? a[e] : 0u;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rot);
      if (!warp_wait(&bars->dvready, ph, abort_flag)) break;
      tc_fence_after();
      float x[32];
      {
        uint32_t r[32];
        tmem_ld_x32(tmem + KCOL_DV + lane_bits + static_cast<uint32_t>(cpart), r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]) * bt;
      }
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        if (tma_out) sts128(row_chunk(sbase + KO_DV, row, 4 * part + c4), pack8(&x[8 * c4]));
        else if (valid) *reinterpret_cast<uint4*>(dv_row + 8 * c4) = pack8(&x[8 * c4]);
      }
      if (!warp_wait(&bars->ready, ph, abort_flag)) break;
      tc_fence_after();
      const float* zg = reinterpret_cast<const float*>(smem + KO_Z) + zslot * D + cpart;
      float dbp = 0.f;  // this quarter's share of phi(k) . (V dS^T)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // 16 channels at a time (fewer live registers)
        float y[16];
        {
          uint32_t r[16];
          tmem_ld_x16(tmem + KCOL_DPK + lane_bits + static_cast<uint32_t>(cpart) + 16u * static_cast<uint32_t>(hh), r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = __uint_as_float(r[e]);
        }
        if constexpr (BETA) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t w = kr[8 * hh + e / 2];
            dbp = fmaf((e & 1) ? bf16hi(w) : bf16lo(w), y[e], dbp);
            y[e] *= bt;
          }
        }
        switch (2 * part + hh) {
          case 0: rotate_span_t<DT, DH, 0, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 1: rotate_span_t<DT, DH, 8, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 2: rotate_span_t<DT, DH, 16, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 3: rotate_span_t<DT, DH, 24, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 4: rotate_span_t<DT, DH, 32, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 5: rotate_span_t<DT, DH, 40, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          case 6: rotate_span_t<DT, DH, 48, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
          default: rotate_span_t<DT, DH, 56, 8>(y, tab, tab2, rope, p, ipt, iph, ipw); break;
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c4 = 2 * hh + cc;
          const float4 za = *reinterpret_cast<const float4*>(zg + 8 * c4);
          const float4 zb = *reinterpret_cast<const float4*>(zg + 8 * c4 + 4);
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t w = ka[4 * c4 + e / 2];
            const float kv = (e & 1) ? bf16hi(w) : bf16lo(w);
            o8[e] = kv > 0.f ? y[8 * cc + e] + zz[e] : 0.f;
          }
          if (tma_out) sts128(row_chunk(sbase + KO_DK, row, 4 * part + c4), pack8(o8));
          else if (valid) *reinterpret_cast<uint4*>(dk_row + 8 * c4) = pack8(o8);
        }
      }
      if constexpr (BETA) {
        // dbeta of the row: the four quarters' shares added in a fixed order by quarter 0 (two
        // slots by tile parity: a quarter reaching the next tile's write has met the others on
        // this one, but quarter 0 may not have read yet).
        float* xk = reinterpret_cast<float*>(smem + KO_X) + ph * (PARTS * 128);
        xk[part * 128 + row] = dbp;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->pair[quarter]);
        if (!warp_wait(&bars->pair[quarter], ph, abort_flag)) break;
        if (part == 0 && valid)
          dbeta[ti.bh * p.N + n] = __float2bfloat16_rn((xk[row] + xk[128 + row]) + (xk[256 + row] + xk[384 + row]));
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
  if (warp == CTRL_WARP) tmem_dealloc(tmem, 256);
}

}  // namespace bw
}  // namespace la
