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
// 128-token tile at a time (warps 0-3: thread = token = TMEM lane; warp 4: TMA and MMA issue):
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
constexpr int THREADS = 160;
constexpr uint32_t BUF = 2 * HALF;
constexpr int ZPARTS = 4;  // dz partial rows per slot: one per math warp
constexpr uint32_t IDESC_QS = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/true);   // X S
constexpr uint32_t IDESC_QST = idesc_bf16_f32(128, 128, /*a_mn=*/false, /*b_mn=*/false); // X S^T
constexpr uint32_t IDESC_TD = idesc_bf16_f32(128, 128, /*a_mn=*/true, /*b_mn=*/true);    // X^T Y

// ---- bwdq smem: Q (-> phi(Q) -> dQ), G (-> dG), dO (-> dnum), S image
constexpr uint32_t QO_Q = 0, QO_G = BUF, QO_DO = 2 * BUF, QO_S = 3 * BUF, QO_BAR = 4 * BUF;
constexpr uint32_t SMEM_Q = QO_BAR + 256 + 1024;
constexpr uint32_t QCOL_NUM = 0, QCOL_DPQ = 128, QCOL_DS = 256;
// ---- bwdk smem: K (-> phi(K) -> dK), V (-> dV), dS image
constexpr uint32_t KO_K = 0, KO_V = BUF, KO_S = 2 * BUF, KO_BAR = 3 * BUF;
constexpr uint32_t SMEM_K = KO_BAR + 256 + 1024;
constexpr uint32_t KCOL_DV = 0, KCOL_DPK = 128;
static_assert(SMEM_Q <= 232448 && SMEM_K <= 232448, "shared memory budget");

struct BarsQ {
  uint64_t full, rot, numready, dn, dpqready, out, final_;
  uint32_t tmem_base;
  int abort_flag;
};
struct BarsK {
  uint64_t full, rot, ready, out, final_;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(BarsQ) <= 256 && sizeof(BarsK) <= 256, "barrier block too large");

__device__ __forceinline__ float sigmoid_f(float g) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(0.5f * g));
  return 0.5f + 0.5f * y;
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

// Pulls 128 fp32 columns of the calling thread's TMEM lane.
__device__ __forceinline__ void pull128(uint32_t taddr, float (&x)[128]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t r[32];
    tmem_ld_x32(taddr + 32 * j, r);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) x[32 * j + e] = __uint_as_float(r[e]);
  }
}

template <int DT, int DH>
__global__ void __launch_bounds__(THREADS, 1)
bwdq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmG,
               const __grid_constant__ CUtensorMap tmDO, const __grid_constant__ CUtensorMap tmDQ,
               const __grid_constant__ CUtensorMap tmDG, const Plan p, const __grid_constant__ Rope rope,
               const uint8_t* __restrict__ simg, const float* __restrict__ zimg, const float2* __restrict__ tab,
               const float4* __restrict__ tab2, float* __restrict__ partial) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  BarsQ* bars = reinterpret_cast<BarsQ*>(smem + QO_BAR);
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
    mbar_init(&bars->rot, 4);
    mbar_init(&bars->numready, 1);
    mbar_init(&bars->dn, 4);
    mbar_init(&bars->dpqready, 1);
    mbar_init(&bars->out, 4);
    mbar_init(&bars->final_, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
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

  if (warp == 4) {
    if (lane == 0) {
      int64_t prev_unit = -1;
      int64_t issued = 0;
      TileInfo tprev{};
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        const TileInfo ti = tile_info(p, g);
        const bool first = ti.unit != prev_unit;
        prev_unit = ti.unit;
        if (i > 0) {
          if (!mbar_wait(&bars->out, static_cast<uint32_t>((i - 1) & 1), abort_flag)) break;
          const int32_t pn0 = static_cast<int32_t>(tprev.n0), pbh = static_cast<int32_t>(tprev.bh);
          tma_store_3d(&tmDQ, smem + QO_Q, 0, pn0, pbh);
          tma_store_3d(&tmDQ, smem + QO_Q + HALF, 64, pn0, pbh);
          tma_store_3d(&tmDG, smem + QO_G, 0, pn0, pbh);
          tma_store_3d(&tmDG, smem + QO_G + HALF, 64, pn0, pbh);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        tprev = ti;
        mbar_arrive_expect_tx(&bars->full, 3 * BUF + (first ? BUF : 0u));
        if (first) bulk_load(smem + QO_S, simg + ti.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        tma_load_3d(smem + QO_Q, &tmQ, 0, n0, bh, &bars->full);
        tma_load_3d(smem + QO_Q + HALF, &tmQ, 64, n0, bh, &bars->full);
        tma_load_3d(smem + QO_G, &tmG, 0, n0, bh, &bars->full);
        tma_load_3d(smem + QO_G + HALF, &tmG, 64, n0, bh, &bars->full);
        tma_load_3d(smem + QO_DO, &tmDO, 0, n0, bh, &bars->full);
        tma_load_3d(smem + QO_DO + HALF, &tmDO, 64, n0, bh, &bars->full);
        ++issued;
        // num = phi(Q) S
        if (!mbar_wait(&bars->rot, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_NUM, desc_k(sbase + QO_Q, kk), desc_mn(sbase + QO_S, kk), IDESC_QS, kk > 0 ? 1u : 0u);
        mma_commit(&bars->numready);
        // dphi(q) = dnum S^T;  dS += phi(Q)^T dnum
        if (!mbar_wait(&bars->dn, ph, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_DPQ, desc_k(sbase + QO_DO, kk), desc_k(sbase + QO_S, kk), IDESC_QST, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + QCOL_DS, desc_mn(sbase + QO_Q, kk), desc_mn(sbase + QO_DO, kk), IDESC_TD,
                   (kk > 0 || !first) ? 1u : 0u);
        mma_commit(&bars->dpqready);
      }
      if (issued > 0 && !*abort_flag &&
          mbar_wait(&bars->out, static_cast<uint32_t>((issued - 1) & 1), abort_flag)) {
        const int32_t pn0 = static_cast<int32_t>(tprev.n0), pbh = static_cast<int32_t>(tprev.bh);
        tma_store_3d(&tmDQ, smem + QO_Q, 0, pn0, pbh);
        tma_store_3d(&tmDQ, smem + QO_Q + HALF, 64, pn0, pbh);
        tma_store_3d(&tmDG, smem + QO_G, 0, pn0, pbh);
        tma_store_3d(&tmDG, smem + QO_G + HALF, 64, pn0, pbh);
        bulk_commit_group();
      }
      bulk_wait_group0();
      if (*abort_flag && issued > 0) mbar_wait_drain(&bars->full, static_cast<uint32_t>((issued - 1) & 1));
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else {
    const int row = threadIdx.x;
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    float dzacc[4] = {0.f, 0.f, 0.f, 0.f};  // dz of channels 4*lane .. 4*lane+3 over this warp's rows
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const TileInfo ti = tile_info(p, g);
      const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != ti.unit);
      if (!warp_wait(&bars->full, ph, abort_flag)) break;
      // q^+ kept packed; phi(q) written in place (the A operand of num and of the dS update).
      uint32_t qa[64];
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) {
        const uint4 rq = lds128(row_chunk(sbase + QO_Q, row, ck));
        qa[4 * ck] = relu_bf16x2(rq.x);
        qa[4 * ck + 1] = relu_bf16x2(rq.y);
        qa[4 * ck + 2] = relu_bf16x2(rq.z);
        qa[4 * ck + 3] = relu_bf16x2(rq.w);
      }
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      uint32_t pt = 0, ph_ = 0, pw = 0;
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph_, pw);
      {
        uint32_t a[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) a[e] = qa[e];
        rotate_row<DT, DH>(a, tab, tab2, rope, p, static_cast<int>(pt), static_cast<int>(ph_), static_cast<int>(pw));
#pragma unroll
        for (int ck = 0; ck < 16; ++ck)
          sts128(row_chunk(sbase + QO_Q, row, ck), make_uint4(a[4 * ck], a[4 * ck + 1], a[4 * ck + 2], a[4 * ck + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rot);
      // den = q^+ . z + eps
      const float* zg = zimg + ti.unit * D;
      float den = 0.f;
#pragma unroll
      for (int k4 = 0; k4 < 32; ++k4) {
        const float4 z4 = __ldg(reinterpret_cast<const float4*>(zg + 4 * k4));
        den = fmaf(bf16lo(qa[2 * k4]), z4.x, den);
        den = fmaf(bf16hi(qa[2 * k4]), z4.y, den);
        den = fmaf(bf16lo(qa[2 * k4 + 1]), z4.z, den);
        den = fmaf(bf16hi(qa[2 * k4 + 1]), z4.w, den);
      }
      den += p.eps;
      const float rden = 1.0f / den;
      // num -> y; with G and dO: dG (over G), dnum (over dO), dden.
      if (!warp_wait(&bars->numready, ph, abort_flag)) break;
      tc_fence_after();
      float x[128];
      pull128(tmem + QCOL_NUM + lane_bits, x);  // num
      float dyy = 0.f;
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) {
        const uint32_t ag = row_chunk(sbase + QO_G, row, ck), ad = row_chunk(sbase + QO_DO, row, ck);
        const uint4 gr = lds128(ag), dr = lds128(ad);
        const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w}, dw[4] = {dr.x, dr.y, dr.z, dr.w};
        float dg8[8], dy8[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int e = 8 * ck + 2 * q + h;
            const float gv = h ? bf16hi(gw[q]) : bf16lo(gw[q]);
            const float dov = h ? bf16hi(dw[q]) : bf16lo(dw[q]);
            const float y = x[e] * rden;
            const float s = sigmoid_f(gv);
            dg8[2 * q + h] = dov * y * s * (1.f - s);
            const float dy = dov * s;
            dy8[2 * q + h] = dy * rden;  // dnum
            dyy = fmaf(dy, y, dyy);
          }
        }
        sts128(ag, pack8(dg8));
        sts128(ad, pack8(dy8));
      }
      const float dden = -dyy * rden;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dn);
      // dz over this warp's rows: every lane ends with channels 4*lane .. 4*lane+3 (a butterfly
      // that halves the channel range per step; each sum is formed once, lower lane first).
      {
        float v[128];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          v[2 * e] = dden * bf16lo(qa[e]);
          v[2 * e + 1] = dden * bf16hi(qa[e]);
        }
#pragma unroll
        for (int off = 16, size = 128; off >= 1; off >>= 1, size >>= 1) {
          const bool up = (lane & off) != 0;
#pragma unroll
          for (int e = 0; e < size / 2; ++e) {
            const float keep = up ? v[e + size / 2] : v[e];
            const float send = up ? v[e] : v[e + size / 2];
            const float other = __shfl_xor_sync(0xffffffffu, send, off);
            v[e] = up ? other + keep : keep + other;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) dzacc[e] += v[e];
      }
      // dq = [q > 0] (RoPE^T(dnum S^T) + dden z), over phi(Q) (the MMAs are done with it).
      if (!warp_wait(&bars->dpqready, ph, abort_flag)) break;
      tc_fence_after();
      pull128(tmem + QCOL_DPQ + lane_bits, x);
      rotate_row_t<DT, DH>(x, tab, tab2, rope, p, static_cast<int>(pt), static_cast<int>(ph_), static_cast<int>(pw));
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) {
        const float4 za = __ldg(reinterpret_cast<const float4*>(zg + 8 * ck));
        const float4 zb = __ldg(reinterpret_cast<const float4*>(zg + 8 * ck + 4));
        const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
        float o8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t w = qa[4 * ck + e / 2];
          const float qv = (e & 1) ? bf16hi(w) : bf16lo(w);
          o8[e] = qv > 0.f ? x[8 * ck + e] + dden * zz[e] : 0.f;
        }
        sts128(row_chunk(sbase + QO_Q, row, ck), pack8(o8));
      }
      if (last) {
        // dS of this unit (TMEM lane = channel k of phi(Q)) and dz -> the CTA's partial slot.
        pull128(tmem + QCOL_DS + lane_bits, x);
        float* dst = partial + (c * p.maxseg + (ti.unit - u_first)) * slot_floats;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          reinterpret_cast<float4*>(dst + row * D)[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        reinterpret_cast<float4*>(dst + D * D + warp * D)[lane] = make_float4(dzacc[0], dzacc[1], dzacc[2], dzacc[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) dzacc[e] = 0.f;
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
  if (warp == 4) tmem_dealloc(tmem, 512);
}

template <int DT, int DH>
__global__ void __launch_bounds__(THREADS, 1)
bwdk_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV, const Plan p,
               const __grid_constant__ Rope rope, const uint8_t* __restrict__ dsimg, const float* __restrict__ dzimg,
               const float2* __restrict__ tab, const float4* __restrict__ tab2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
    mbar_init(&bars->rot, 4);
    mbar_init(&bars->ready, 1);
    mbar_init(&bars->out, 4);
    mbar_init(&bars->final_, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  pdl_trigger();
  pdl_wait();

  if (warp == 4) {
    if (lane == 0) {
      int64_t prev_unit = -1;
      int64_t issued = 0;
      TileInfo tprev{};
      for (int64_t g = g0; g < g1; ++g) {
        const int64_t i = g - g0;
        const uint32_t ph = static_cast<uint32_t>(i & 1);
        const TileInfo ti = tile_info(p, g);
        const bool first = ti.unit != prev_unit;
        prev_unit = ti.unit;
        if (i > 0) {
          if (!mbar_wait(&bars->out, static_cast<uint32_t>((i - 1) & 1), abort_flag)) break;
          const int32_t pn0 = static_cast<int32_t>(tprev.n0), pbh = static_cast<int32_t>(tprev.bh);
          tma_store_3d(&tmDK, smem + KO_K, 0, pn0, pbh);
          tma_store_3d(&tmDK, smem + KO_K + HALF, 64, pn0, pbh);
          tma_store_3d(&tmDV, smem + KO_V, 0, pn0, pbh);
          tma_store_3d(&tmDV, smem + KO_V + HALF, 64, pn0, pbh);
          bulk_commit_group();
          bulk_wait_group_read0();
        }
        tprev = ti;
        mbar_arrive_expect_tx(&bars->full, 2 * BUF + (first ? BUF : 0u));
        if (first) bulk_load(smem + KO_S, dsimg + ti.unit * static_cast<int64_t>(BUF), BUF, &bars->full);
        const int32_t n0 = static_cast<int32_t>(ti.n0), bh = static_cast<int32_t>(ti.bh);
        tma_load_3d(smem + KO_K, &tmK, 0, n0, bh, &bars->full);
        tma_load_3d(smem + KO_K + HALF, &tmK, 64, n0, bh, &bars->full);
        tma_load_3d(smem + KO_V, &tmV, 0, n0, bh, &bars->full);
        tma_load_3d(smem + KO_V + HALF, &tmV, 64, n0, bh, &bars->full);
        ++issued;
        if (!mbar_wait(&bars->rot, ph, abort_flag)) break;
        tc_fence_after();
        // dV = phi(K) dS;  dphi(k) = V dS^T
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + KCOL_DV, desc_k(sbase + KO_K, kk), desc_mn(sbase + KO_S, kk), IDESC_QS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + KCOL_DPK, desc_k(sbase + KO_V, kk), desc_k(sbase + KO_S, kk), IDESC_QST, kk > 0 ? 1u : 0u);
        mma_commit(&bars->ready);
      }
      if (issued > 0 && !*abort_flag &&
          mbar_wait(&bars->out, static_cast<uint32_t>((issued - 1) & 1), abort_flag)) {
        const int32_t pn0 = static_cast<int32_t>(tprev.n0), pbh = static_cast<int32_t>(tprev.bh);
        tma_store_3d(&tmDK, smem + KO_K, 0, pn0, pbh);
        tma_store_3d(&tmDK, smem + KO_K + HALF, 64, pn0, pbh);
        tma_store_3d(&tmDV, smem + KO_V, 0, pn0, pbh);
        tma_store_3d(&tmDV, smem + KO_V + HALF, 64, pn0, pbh);
        bulk_commit_group();
      }
      bulk_wait_group0();
      if (*abort_flag && issued > 0) mbar_wait_drain(&bars->full, static_cast<uint32_t>((issued - 1) & 1));
      mma_commit(&bars->final_);
      mbar_wait_drain(&bars->final_, 0);
    }
  } else {
    const int row = threadIdx.x;
    const uint32_t lane_bits = static_cast<uint32_t>(warp * 32) << 16;
    for (int64_t g = g0; g < g1; ++g) {
      const int64_t i = g - g0;
      const uint32_t ph = static_cast<uint32_t>(i & 1);
      const TileInfo ti = tile_info(p, g);
      if (!warp_wait(&bars->full, ph, abort_flag)) break;
      uint32_t ka[64];
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) {
        const uint4 rk = lds128(row_chunk(sbase + KO_K, row, ck));
        ka[4 * ck] = rk.x;
        ka[4 * ck + 1] = rk.y;
        ka[4 * ck + 2] = rk.z;
        ka[4 * ck + 3] = rk.w;
      }
      const uint32_t n = static_cast<uint32_t>(ti.n0) + static_cast<uint32_t>(row);
      uint32_t pt = 0, ph_ = 0, pw = 0;
      if (static_cast<int64_t>(n) < p.N) token_pos(p, n, pt, ph_, pw);
      {
        uint32_t a[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) a[e] = relu_bf16x2(ka[e]);
        rotate_row<DT, DH>(a, tab, tab2, rope, p, static_cast<int>(pt), static_cast<int>(ph_), static_cast<int>(pw));
#pragma unroll
        for (int ck = 0; ck < 16; ++ck)
          sts128(row_chunk(sbase + KO_K, row, ck), make_uint4(a[4 * ck], a[4 * ck + 1], a[4 * ck + 2], a[4 * ck + 3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->rot);
      if (!warp_wait(&bars->ready, ph, abort_flag)) break;
      tc_fence_after();
      float x[128];
      pull128(tmem + KCOL_DV + lane_bits, x);
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) sts128(row_chunk(sbase + KO_V, row, ck), pack8(&x[8 * ck]));
      pull128(tmem + KCOL_DPK + lane_bits, x);
      rotate_row_t<DT, DH>(x, tab, tab2, rope, p, static_cast<int>(pt), static_cast<int>(ph_), static_cast<int>(pw));
      const float* zg = dzimg + ti.unit * D;
#pragma unroll
      for (int ck = 0; ck < 16; ++ck) {
        const float4 za = __ldg(reinterpret_cast<const float4*>(zg + 8 * ck));
        const float4 zb = __ldg(reinterpret_cast<const float4*>(zg + 8 * ck + 4));
        const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
        float o8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t w = ka[4 * ck + e / 2];
          const float kv = (e & 1) ? bf16hi(w) : bf16lo(w);
          o8[e] = kv > 0.f ? x[8 * ck + e] + zz[e] : 0.f;
        }
        sts128(row_chunk(sbase + KO_K, row, ck), pack8(o8));
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
  if (warp == 4) tmem_dealloc(tmem, 256);
}

}  // namespace bw
}  // namespace la
