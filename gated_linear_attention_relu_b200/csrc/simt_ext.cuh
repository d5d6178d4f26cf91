// simt_ext.cuh -- CUDA-core kernels of the token-causal operator and of the gradients, for every
// dtype and head dimension (fp32, d = 32 / 64, and LA_FLAG_FORCE_SIMT), and for the forms the
// tensor-core backward does not take (the write gate beta and RMSNorm of SANA-Video 2.0, Eq. (1)).
//
// They walk the same persistent tile ranges as the CUDA-core state kernel (32-token tiles, units
// never crossing a tile), accumulate in fp32 and keep a unit's d x d state in shared memory.
#pragma once
#include "common.cuh"
#include "sm100.cuh"
#include "simt.cuh"

namespace la {
namespace simt {

// Shared-memory bytes of causal_simt_kernel / bwdq_simt_kernel / bwdk_simt_kernel for head dim d.
__host__ __device__ constexpr size_t causal_simt_smem(int d) {
  return (size_t(d) * d + d + 5 * size_t(TS) * (d + 1) + 2 * size_t(TS) * (TS + 1) + TS) * sizeof(float);
}
__host__ __device__ constexpr size_t bwdq_simt_smem(int d) {
  return (size_t(d) * d + d + 5 * size_t(TS) * (d + 1) + 4 * size_t(TS)) * sizeof(float);
}
__host__ __device__ constexpr size_t bwdk_simt_smem(int d) {
  return (size_t(d) * d + d + 4 * size_t(TS) * (d + 1) + size_t(TS)) * sizeof(float);
}

// ReLU'd and rotated features of one channel pair of token n (zero past the unit's end).
template <typename T>
__device__ __forceinline__ void load_pair(const T* __restrict__ x, const Plan& p, const Rope& rope, int64_t n,
                                          int64_t n_end, int pi, float& p0, float& p1, float& r0, float& r1,
                                          float& cs, float& sn) {
  p0 = p1 = 0.f;
  uint32_t pt = 0, ph = 0, pw = 0;
  if (n < n_end) {
    p0 = fmaxf(to_f(x[2 * pi]), 0.f);
    p1 = fmaxf(to_f(x[2 * pi + 1]), 0.f);
    token_pos(p, static_cast<uint32_t>(n), pt, ph, pw);
  }
  rope_cs(static_cast<double>(axis_pos(rope.band[pi], pt, ph, pw)) +
              (rope.band[pi] == 0 ? static_cast<double>(rope.t_offset) : 0.0),
          rope.theta_d[pi], cs, sn);
  r0 = p0 * cs - p1 * sn;
  r1 = p0 * sn + p1 * cs;
}

// ---------------------------------------------------------------------------------------------
// Token-causal operator (token n reads tokens 0..n of its head):
//   O_n = (phi(q_n) S_{<=n}) / (q_n^+ . z_{<=n} + eps) * sigmoid(g_n).
// Each CTA walks its tile range carrying (S, z): from `start` (the sum of the earlier CTAs' parts
// of its first unit), reset to zero when a new unit begins.  Per 32-token tile:
//   num_r = phi(q_r) S + sum_{m <= r} (phi(q_r) . phi(k_m)) v_m,
//   den_r = q_r^+ . z + sum_{m <= r} q_r^+ . k_m^+ + eps,
// then S += phi(K)^T V and z += sum k^+ over the tile.
template <int D, typename T>
__global__ void __launch_bounds__(THREADS)
causal_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                   const T* __restrict__ G, T* __restrict__ O, const Plan p, const __grid_constant__ Rope rope,
                   const float* __restrict__ start) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1;
  float* Ss = sm;                  // [D][D] carried state
  float* zs = Ss + D * D;          // [D]
  float* qr = zs + D;              // [TS][LD]
  float* qp = qr + TS * LD;
  float* kr = qp + TS * LD;
  float* kp = kr + TS * LD;
  float* vs = kp + TS * LD;
  float* P = vs + TS * LD;         // [TS][TS + 1] rotated scores (masked)
  float* Pd = P + TS * (TS + 1);   // [TS][TS + 1] un-rotated scores (masked)
  float* inv = Pd + TS * (TS + 1); // [TS]
  constexpr int R = D / 16;        // the S update: each thread owns an R x R block
  constexpr int CW = D / 8;        // the numerator: each thread owns CW columns of one row
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int r_own = tid % TS, cg = tid / TS;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c), g1 = cta_start(p, c + 1);
  int64_t cur_unit = -1;
  for (int64_t g = g0; g < g1; ++g) {
    const TileInfo ti = tile_info(p, g);
    __syncthreads();
    if (ti.unit != cur_unit) {
      // The carried state: the earlier CTAs' share of this unit at the CTA's first tile, zero at a
      // unit that begins inside the range.
      const bool carry = cur_unit < 0;
      cur_unit = ti.unit;
      const float* st = start + c * (static_cast<int64_t>(D) * D + D);
      for (int e = tid; e < D * D + D; e += THREADS) sm[e] = carry ? st[e] : 0.f;
    }
    const int64_t base = ti.bh * p.N;
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      float a0, a1, b0, b1, cs, sn;
      load_pair(Q + (base + n) * D, p, rope, n, ti.n_end, pi, a0, a1, b0, b1, cs, sn);
      qp[r * LD + 2 * pi] = a0;
      qp[r * LD + 2 * pi + 1] = a1;
      qr[r * LD + 2 * pi] = b0;
      qr[r * LD + 2 * pi + 1] = b1;
      float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
      if (n < ti.n_end) {
        k0 = fmaxf(to_f(K[(base + n) * D + 2 * pi]), 0.f);
        k1 = fmaxf(to_f(K[(base + n) * D + 2 * pi + 1]), 0.f);
        v0 = to_f(V[(base + n) * D + 2 * pi]);
        v1 = to_f(V[(base + n) * D + 2 * pi + 1]);
      }
      kp[r * LD + 2 * pi] = k0;
      kp[r * LD + 2 * pi + 1] = k1;
      kr[r * LD + 2 * pi] = k0 * cs - k1 * sn;
      kr[r * LD + 2 * pi + 1] = k0 * sn + k1 * cs;
      vs[r * LD + 2 * pi] = v0;
      vs[r * LD + 2 * pi + 1] = v1;
    }
    __syncthreads();
    // Intra-tile scores, lower triangle (m <= r).
    for (int e = tid; e < TS * TS; e += THREADS) {
      const int r = e / TS, m = e % TS;
      float a = 0.f, b = 0.f;
      if (m <= r) {
        for (int k = 0; k < D; ++k) {
          a = fmaf(qr[r * LD + k], kr[m * LD + k], a);
          b = fmaf(qp[r * LD + k], kp[m * LD + k], b);
        }
      }
      P[r * (TS + 1) + m] = a;
      Pd[r * (TS + 1) + m] = b;
    }
    __syncthreads();
    if (tid < TS) {
      float den = 0.f;
      for (int k = 0; k < D; ++k) den = fmaf(qp[tid * LD + k], zs[k], den);
      for (int m = 0; m <= tid; ++m) den += Pd[tid * (TS + 1) + m];
      inv[tid] = 1.0f / (den + p.eps);
    }
    float acc[CW];
#pragma unroll
    for (int j = 0; j < CW; ++j) acc[j] = 0.f;
    for (int k = 0; k < D; ++k) {
      const float a = qr[r_own * LD + k];
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = fmaf(a, Ss[k * D + cg * CW + j], acc[j]);
    }
    for (int m = 0; m <= r_own; ++m) {
      const float a = P[r_own * (TS + 1) + m];
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = fmaf(a, vs[m * LD + cg * CW + j], acc[j]);
    }
    __syncthreads();  // inv ready; every read of S and z for this tile done
    {
      const int64_t n = ti.n0 + r_own;
      if (n < ti.n_end) {
        const float iv = inv[r_own];
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int v = cg * CW + j;
          const float gv = to_f(G[(base + n) * D + v]);
          const float sig = 1.0f / (1.0f + expf(-gv));
          O[(base + n) * D + v] = from_f<T>(acc[j] * iv * sig);
        }
      }
    }
    // S += phi(K)^T V, z += sum k^+ over the tile (rows past the unit's end are zero).
#pragma unroll
    for (int i = 0; i < R; ++i) {
      float s[R];
#pragma unroll
      for (int j = 0; j < R; ++j) s[j] = Ss[(ty * R + i) * D + tx * R + j];
      for (int r = 0; r < TS; ++r) {
        const float a = kr[r * LD + ty * R + i];
#pragma unroll
        for (int j = 0; j < R; ++j) s[j] = fmaf(a, vs[r * LD + tx * R + j], s[j]);
      }
#pragma unroll
      for (int j = 0; j < R; ++j) Ss[(ty * R + i) * D + tx * R + j] = s[j];
    }
    if (tid < D) {
      float zz = zs[tid];
      for (int r = 0; r < TS; ++r) zz += kp[r * LD + tid];
      zs[tid] = zz;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Gradients, query side, of the full form (block-causal, RMSNorm optional):
//   y = num / den with num = phi(q) S_b, den = q^+ . z_b + eps (S_b, z_b: the inclusive state the
//   token's block reads); u = RMSNorm(y) (y without it); o = u * sigmoid(g).
//   dg = do u s (1 - s), du = do s, dgamma += du * y / r, dy = (dyh - yh (yh . dyh) / d) / r with
//   yh = y / r, dyh = du gamma (dy = du without RMSNorm), dnum = dy / den, dden = -(dy . y) / den,
//   dq = [q > 0] (RoPE^T(dnum S_b^T) + dden z_b); and per unit the partial sums
//   dS_b = sum phi(q)^T dnum, dz_b = sum dden q^+ into the CTA's slot, dgamma into the CTA's row.
template <int D, typename T>
__global__ void __launch_bounds__(THREADS)
bwdq_simt_kernel(const T* __restrict__ Q, const T* __restrict__ G, const T* __restrict__ dO,
                 const float* __restrict__ S, const float* __restrict__ z, T* __restrict__ dQ, T* __restrict__ dG,
                 const Plan p, const __grid_constant__ Rope rope, int rms, const float* __restrict__ gamma,
                 float norm_eps, float* __restrict__ partial, float* __restrict__ dgamma_part) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1;
  float* Ss = sm;                 // [D][D] the unit's state
  float* zs = Ss + D * D;         // [D]
  float* qr = zs + D;             // [TS][LD] phi(q)
  float* qp = qr + TS * LD;       // [TS][LD] q^+
  float* yv = qp + TS * LD;       // [TS][LD] y
  float* dn = yv + TS * LD;       // [TS][LD] du, then dnum
  float* dq = dn + TS * LD;       // [TS][LD] dnum S^T
  float* rden = dq + TS * LD;     // [TS] 1 / den
  float* rinv = rden + TS;        // [TS] 1 / r (RMSNorm)
  float* dot = rinv + TS;         // [TS] yh . dyh
  float* dden = dot + TS;         // [TS]
  constexpr int R = D / 16;
  constexpr int CW = D / 8;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int r_own = tid % TS, cg = tid / TS;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c), g1 = cta_start(p, c + 1);
  const int64_t u_first = unit_of_tile(p, g0);
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(p.zparts) * D;
  float acc[R][R];
  float dzacc = 0.f, dgacc = 0.f;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;
  int64_t cur_unit = -1;
  for (int64_t g = g0; g < g1; ++g) {
    const TileInfo ti = tile_info(p, g);
    const int64_t base = ti.bh * p.N;
    __syncthreads();
    if (ti.unit != cur_unit) {
      cur_unit = ti.unit;
      for (int e = tid; e < D * D; e += THREADS) Ss[e] = S[ti.unit * D * D + e];
      for (int e = tid; e < D; e += THREADS) zs[e] = z[ti.unit * D + e];
    }
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      float a0, a1, b0, b1, cs, sn;
      load_pair(Q + (base + n) * D, p, rope, n, ti.n_end, pi, a0, a1, b0, b1, cs, sn);
      qp[r * LD + 2 * pi] = a0;
      qp[r * LD + 2 * pi + 1] = a1;
      qr[r * LD + 2 * pi] = b0;
      qr[r * LD + 2 * pi + 1] = b1;
    }
    __syncthreads();
    if (tid < TS) {
      float den = 0.f;
      for (int k = 0; k < D; ++k) den = fmaf(qp[tid * LD + k], zs[k], den);
      rden[tid] = 1.0f / (den + p.eps);
    }
    __syncthreads();
    {  // y = num / den
      float a[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) a[j] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float x = qr[r_own * LD + k];
#pragma unroll
        for (int j = 0; j < CW; ++j) a[j] = fmaf(x, Ss[k * D + cg * CW + j], a[j]);
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) yv[r_own * LD + cg * CW + j] = a[j] * rden[r_own];
    }
    __syncthreads();
    if (tid < TS) {
      float ss = 0.f;
      for (int v = 0; v < D; ++v) ss = fmaf(yv[tid * LD + v], yv[tid * LD + v], ss);
      rinv[tid] = rms ? rsqrtf(ss / static_cast<float>(D) + norm_eps) : 1.f;
    }
    __syncthreads();
    // dG and du (= do * s); with RMSNorm: dgamma, then dyh = du * gamma into dn.
    for (int e = tid; e < TS * D; e += THREADS) {
      const int r = e / D, v = e % D;
      const int64_t n = ti.n0 + r;
      float du = 0.f;
      if (n < ti.n_end) {
        const float gv = to_f(G[(base + n) * D + v]);
        const float s = 1.0f / (1.0f + expf(-gv));
        const float dov = to_f(dO[(base + n) * D + v]);
        const float y = yv[r * LD + v];
        const float yh = y * rinv[r];
        const float gm = (rms && gamma) ? gamma[v] : 1.f;
        const float u = rms ? yh * gm : y;
        dG[(base + n) * D + v] = from_f<T>(dov * u * s * (1.f - s));
        du = dov * s;
        dn[r * LD + v] = rms ? du * gm : du;
      } else {
        dn[r * LD + v] = 0.f;
      }
      (void)du;
    }
    __syncthreads();
    if (rms) {
      if (tid < TS) {
        float d2 = 0.f;
        for (int v = 0; v < D; ++v) d2 = fmaf(yv[tid * LD + v] * rinv[tid], dn[tid * LD + v], d2);
        dot[tid] = d2;
      }
      if (gamma && tid < D) {
        // dgamma_v += sum_r du_rv * yh_rv, with du = dyh / gamma_v recomputed from dO and G.
        for (int r = 0; r < TS; ++r) {
          const int64_t n = ti.n0 + r;
          if (n < ti.n_end) {
            const float gv = to_f(G[(base + n) * D + tid]);
            const float s = 1.0f / (1.0f + expf(-gv));
            dgacc = fmaf(to_f(dO[(base + n) * D + tid]) * s, yv[r * LD + tid] * rinv[r], dgacc);
          }
        }
      }
      __syncthreads();
      // dy = (dyh - yh (yh . dyh) / D) / r, in place of dyh.
      for (int e = tid; e < TS * D; e += THREADS) {
        const int r = e / D, v = e % D;
        const float yh = yv[r * LD + v] * rinv[r];
        dn[r * LD + v] = (dn[r * LD + v] - yh * dot[r] / static_cast<float>(D)) * rinv[r];
      }
      __syncthreads();
    }
    // dden = -(dy . y) / den; dnum = dy / den.
    if (tid < TS) {
      float d2 = 0.f;
      for (int v = 0; v < D; ++v) d2 = fmaf(dn[tid * LD + v], yv[tid * LD + v], d2);
      dden[tid] = -d2 * rden[tid];
    }
    __syncthreads();
    for (int e = tid; e < TS * D; e += THREADS) {
      const int r = e / D, v = e % D;
      dn[r * LD + v] *= rden[r];
    }
    __syncthreads();
    {  // dphi(q) = dnum S^T
      float a[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) a[j] = 0.f;
      for (int v = 0; v < D; ++v) {
        const float x = dn[r_own * LD + v];
#pragma unroll
        for (int j = 0; j < CW; ++j) a[j] = fmaf(x, Ss[(cg * CW + j) * D + v], a[j]);
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) dq[r_own * LD + cg * CW + j] = a[j];
    }
    __syncthreads();
    // dq = [q > 0] (RoPE^T(dphi(q)) + dden z), one channel pair per item.
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      if (n < ti.n_end) {
        uint32_t pt = 0, ph = 0, pw = 0;
        token_pos(p, static_cast<uint32_t>(n), pt, ph, pw);
        float cs, sn;
        rope_cs(static_cast<double>(axis_pos(rope.band[pi], pt, ph, pw)) +
                    (rope.band[pi] == 0 ? static_cast<double>(rope.t_offset) : 0.0),
                rope.theta_d[pi], cs, sn);
        const float x0 = dq[r * LD + 2 * pi], x1 = dq[r * LD + 2 * pi + 1];
        const float q0 = to_f(Q[(base + n) * D + 2 * pi]), q1 = to_f(Q[(base + n) * D + 2 * pi + 1]);
        const float d0 = x0 * cs + x1 * sn + dden[r] * zs[2 * pi];
        const float d1 = -x0 * sn + x1 * cs + dden[r] * zs[2 * pi + 1];
        dQ[(base + n) * D + 2 * pi] = from_f<T>(q0 > 0.f ? d0 : 0.f);
        dQ[(base + n) * D + 2 * pi + 1] = from_f<T>(q1 > 0.f ? d1 : 0.f);
      }
    }
    // dS += phi(q)^T dnum, dz += sum dden q^+ (rows past the unit's end are zero).
    for (int r = 0; r < TS; ++r) {
      float a[R], b[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        a[i] = qr[r * LD + ty * R + i];
        b[i] = dn[r * LD + tx * R + i];
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (tid < D)
      for (int r = 0; r < TS; ++r) dzacc = fmaf(dden[r], qp[r * LD + tid], dzacc);
    const bool last = (g + 1 == g1) || (unit_of_tile(p, g + 1) != ti.unit);
    if (last && in_bounds(ti.unit - u_first < p.maxseg)) {
      float* dst = partial + (c * p.maxseg + (ti.unit - u_first)) * slot_floats;
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) {
          dst[(ty * R + i) * D + tx * R + j] = acc[i][j];
          acc[i][j] = 0.f;
        }
      if (tid < D) {
        dst[D * D + tid] = dzacc;
        dzacc = 0.f;
      }
    }
  }
  if (dgamma_part && tid < D) dgamma_part[c * D + tid] = dgacc;
}

// ---------------------------------------------------------------------------------------------
// Gradients, key side: with dS, dz the suffix sums (over blocks at and after the key's own) of
// the query side's per-unit sums, P = v dS^T (per token):
//   dv = beta phi(k) dS,  dk = [k > 0] (RoPE^T(beta P) + dz),  dbeta = phi(k) . P.
template <int D, typename T>
__global__ void __launch_bounds__(THREADS)
bwdk_simt_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ beta,
                 const float* __restrict__ dS, const float* __restrict__ dz, T* __restrict__ dK,
                 T* __restrict__ dV, T* __restrict__ dbeta, const Plan p, const __grid_constant__ Rope rope) {
  extern __shared__ float sm[];
  constexpr int LD = D + 1;
  float* Ss = sm;                 // [D][D] dS of the unit
  float* zs = Ss + D * D;         // [D] dz of the unit
  float* kr = zs + D;             // [TS][LD] phi(k)
  float* vs = kr + TS * LD;       // [TS][LD] v
  float* pv = vs + TS * LD;       // [TS][LD] v dS^T
  float* dv = pv + TS * LD;       // [TS][LD] phi(k) dS
  float* bt = dv + TS * LD;       // [TS] beta
  constexpr int CW = D / 8;
  const int tid = threadIdx.x;
  const int r_own = tid % TS, cg = tid / TS;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c), g1 = cta_start(p, c + 1);
  int64_t cur_unit = -1;
  for (int64_t g = g0; g < g1; ++g) {
    const TileInfo ti = tile_info(p, g);
    const int64_t base = ti.bh * p.N;
    __syncthreads();
    if (ti.unit != cur_unit) {
      cur_unit = ti.unit;
      for (int e = tid; e < D * D; e += THREADS) Ss[e] = dS[ti.unit * D * D + e];
      for (int e = tid; e < D; e += THREADS) zs[e] = dz[ti.unit * D + e];
    }
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      float a0, a1, b0, b1, cs, sn;
      load_pair(K + (base + n) * D, p, rope, n, ti.n_end, pi, a0, a1, b0, b1, cs, sn);
      kr[r * LD + 2 * pi] = b0;
      kr[r * LD + 2 * pi + 1] = b1;
      vs[r * LD + 2 * pi] = n < ti.n_end ? to_f(V[(base + n) * D + 2 * pi]) : 0.f;
      vs[r * LD + 2 * pi + 1] = n < ti.n_end ? to_f(V[(base + n) * D + 2 * pi + 1]) : 0.f;
    }
    if (tid < TS) {
      const int64_t n = ti.n0 + tid;
      bt[tid] = (beta && n < ti.n_end) ? to_f(beta[base + n]) : 1.f;
    }
    __syncthreads();
    {
      float a[CW], b[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) a[j] = b[j] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float x = kr[r_own * LD + k], y = vs[r_own * LD + k];
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          a[j] = fmaf(x, Ss[k * D + cg * CW + j], a[j]);   // (phi(k) dS)_j
          b[j] = fmaf(y, Ss[(cg * CW + j) * D + k], b[j]); // (v dS^T)_j
        }
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        dv[r_own * LD + cg * CW + j] = a[j];
        pv[r_own * LD + cg * CW + j] = b[j];
      }
    }
    __syncthreads();
    if (dbeta && tid < TS) {
      const int64_t n = ti.n0 + tid;
      if (n < ti.n_end) {
        float s = 0.f;
        for (int k = 0; k < D; ++k) s = fmaf(kr[tid * LD + k], pv[tid * LD + k], s);
        dbeta[base + n] = from_f<T>(s);
      }
    }
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      if (n < ti.n_end) {
        uint32_t pt = 0, ph = 0, pw = 0;
        token_pos(p, static_cast<uint32_t>(n), pt, ph, pw);
        float cs, sn;
        rope_cs(static_cast<double>(axis_pos(rope.band[pi], pt, ph, pw)) +
                    (rope.band[pi] == 0 ? static_cast<double>(rope.t_offset) : 0.0),
                rope.theta_d[pi], cs, sn);
        const float b = bt[r];
        const float x0 = b * pv[r * LD + 2 * pi], x1 = b * pv[r * LD + 2 * pi + 1];
        const float k0 = to_f(K[(base + n) * D + 2 * pi]), k1 = to_f(K[(base + n) * D + 2 * pi + 1]);
        const float d0 = x0 * cs + x1 * sn + zs[2 * pi];
        const float d1 = -x0 * sn + x1 * cs + zs[2 * pi + 1];
        dK[(base + n) * D + 2 * pi] = from_f<T>(k0 > 0.f ? d0 : 0.f);
        dK[(base + n) * D + 2 * pi + 1] = from_f<T>(k1 > 0.f ? d1 : 0.f);
        dV[(base + n) * D + 2 * pi] = from_f<T>(b * dv[r * LD + 2 * pi]);
        dV[(base + n) * D + 2 * pi + 1] = from_f<T>(b * dv[r * LD + 2 * pi + 1]);
      }
    }
  }
}

// dgamma = the per-CTA rows summed in CTA order (one thread per channel).
__global__ void __launch_bounds__(THREADS)
dgamma_sum_kernel(int grid, int D, const float* __restrict__ part, float* __restrict__ dgamma) {
  const int v = blockIdx.x * THREADS + threadIdx.x;
  if (v >= D) return;
  float s = 0.f;
  for (int c = 0; c < grid; ++c) s += part[static_cast<int64_t>(c) * D + v];
  dgamma[v] = s;
}

}  // namespace simt
}  // namespace la
