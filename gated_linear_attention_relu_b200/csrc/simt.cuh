// simt.cuh -- CUDA-core kernels: the fp32 dtype path, head dimensions 32 and 64, and the
// reference point the tensor-core kernels are measured against (LA_FLAG_FORCE_SIMT).
//
// Same operator and the same work decomposition as the tensor-core kernels (common.cuh), with
// fp32 FFMA accumulation.  RoPE angles are formed and reduced modulo 2*pi in fp64 before the
// fp32 sincos, so the rotation is accurate to a few ulp even at large grid positions.
#pragma once
#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace simt {

constexpr int THREADS = 256;
constexpr int TS = 32;  // tokens per tile (state and apply)

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ void rope_cs(double pos, double theta, float& c, float& s) {
  const double two_pi = 6.283185307179586476925286766559;
  double a = pos * theta;
  a -= two_pi * rint(a / two_pi);
  sincosf(static_cast<float>(a), &s, &c);
}

__device__ __forceinline__ uint32_t axis_pos(int band, uint32_t t, uint32_t h, uint32_t w) {
  return band == 0 ? t : (band == 1 ? h : w);
}

// ---------------------------------------------------------------------------------------------
// State: per CTA, partial S (D x D) and z (D) for every unit it touches, into partial slots.
template <int D, typename T>
__global__ void __launch_bounds__(THREADS)
state_simt_kernel(const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ beta, const Plan p,
                  const __grid_constant__ Rope rope, float* __restrict__ partial) {
  constexpr int R = D / 16;  // each thread owns an R x R block of S
  __shared__ float kr[TS][D];
  __shared__ float vs[TS][D];
  __shared__ float kp[TS][D];
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c), g1 = cta_start(p, c + 1);
  const int64_t u_first = unit_of_tile(p, g0);
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(p.zparts) * D;
  float acc[R][R];
  float zacc = 0.f;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int b = 0; b < R; ++b) acc[a][b] = 0.f;

  for (int64_t g = g0; g < g1; ++g) {
    const TileInfo ti = tile_info(p, g);
    const T* kb = K + (ti.bh * p.N) * D;
    const T* vb = V + (ti.bh * p.N) * D;
    __syncthreads();
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      float x0 = 0.f, x1 = 0.f, v0 = 0.f, v1 = 0.f;
      uint32_t pt = 0, ph = 0, pw = 0;
      if (n < ti.n_end) {
        x0 = fmaxf(to_f(kb[n * D + 2 * pi]), 0.f);
        x1 = fmaxf(to_f(kb[n * D + 2 * pi + 1]), 0.f);
        v0 = to_f(vb[n * D + 2 * pi]);
        v1 = to_f(vb[n * D + 2 * pi + 1]);
        token_pos(p, static_cast<uint32_t>(n), pt, ph, pw);
      }
      float cs, sn;
      rope_cs(static_cast<double>(axis_pos(rope.band[pi], pt, ph, pw)) +
                  (rope.band[pi] == 0 ? static_cast<double>(rope.t_offset) : 0.0),
              rope.theta_d[pi], cs, sn);
      // Write gate (optional): scales the rotated key only; z keeps ReLU(k).
      const float b = (beta && n < ti.n_end) ? to_f(beta[ti.bh * p.N + n]) : 1.f;
      kp[r][2 * pi] = x0;
      kp[r][2 * pi + 1] = x1;
      kr[r][2 * pi] = (x0 * cs - x1 * sn) * b;
      kr[r][2 * pi + 1] = (x0 * sn + x1 * cs) * b;
      vs[r][2 * pi] = v0;
      vs[r][2 * pi + 1] = v1;
    }
    __syncthreads();
    for (int r = 0; r < TS; ++r) {
      float a[R], b[R];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        a[i] = kr[r][ty * R + i];
        b[i] = vs[r][tx * R + i];
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < R; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (tid < D)
      for (int r = 0; r < TS; ++r) zacc += kp[r][tid];

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
        dst[D * D + tid] = zacc;
        zacc = 0.f;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Apply: O_n = (RoPE(ReLU(q_n)) S) / (ReLU(q_n) . z + eps) * sigmoid(g_n), state fp32 in smem.
template <int D, typename T>
__global__ void __launch_bounds__(THREADS)
apply_simt_kernel(const T* __restrict__ Q, const T* __restrict__ G, const float* __restrict__ S,
                  const float* __restrict__ z, T* __restrict__ O, const Plan p,
                  const __grid_constant__ Rope rope, int rms, const float* __restrict__ gamma, float norm_eps) {
  extern __shared__ float sm[];
  float* Ss = sm;                   // [D][D]
  float* zs = Ss + D * D;           // [D]
  float* qr = zs + D;               // [TS][D+1] rotated features
  float* qp = qr + TS * (D + 1);    // [TS][D+1] un-rotated ReLU features
  float* inv = qp + TS * (D + 1);   // [TS]
  float* ot = inv + TS;             // [TS][D+1] numerators
  constexpr int CW = D / 8;         // columns per thread
  const int tid = threadIdx.x;
  const int r_own = tid % TS, cg = tid / TS;
  const int64_t c = blockIdx.x;
  const int64_t g0 = cta_start(p, c), g1 = cta_start(p, c + 1);
  int64_t cur_unit = -1;
  for (int64_t g = g0; g < g1; ++g) {
    const TileInfo ti = tile_info(p, g);
    __syncthreads();
    if (ti.unit != cur_unit) {
      cur_unit = ti.unit;
      const float* Su = S + ti.unit * D * D;
      for (int e = tid; e < D * D; e += THREADS) Ss[e] = Su[e];
      for (int e = tid; e < D; e += THREADS) zs[e] = z[ti.unit * D + e];
    }
    const T* qb = Q + (ti.bh * p.N) * D;
    for (int e = tid; e < TS * D / 2; e += THREADS) {
      const int r = e / (D / 2), pi = e % (D / 2);
      const int64_t n = ti.n0 + r;
      float x0 = 0.f, x1 = 0.f;
      uint32_t pt = 0, ph = 0, pw = 0;
      if (n < ti.n_end) {
        x0 = fmaxf(to_f(qb[n * D + 2 * pi]), 0.f);
        x1 = fmaxf(to_f(qb[n * D + 2 * pi + 1]), 0.f);
        token_pos(p, static_cast<uint32_t>(n), pt, ph, pw);
      }
      float cs, sn;
      rope_cs(static_cast<double>(axis_pos(rope.band[pi], pt, ph, pw)) +
                  (rope.band[pi] == 0 ? static_cast<double>(rope.t_offset) : 0.0),
              rope.theta_d[pi], cs, sn);
      qp[r * (D + 1) + 2 * pi] = x0;
      qp[r * (D + 1) + 2 * pi + 1] = x1;
      qr[r * (D + 1) + 2 * pi] = x0 * cs - x1 * sn;
      qr[r * (D + 1) + 2 * pi + 1] = x0 * sn + x1 * cs;
    }
    __syncthreads();
    if (tid < TS) {
      float den = 0.f;
      for (int k = 0; k < D; ++k) den = fmaf(qp[tid * (D + 1) + k], zs[k], den);
      inv[tid] = 1.0f / (den + p.eps);
    }
    {
      float acc[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = 0.f;
      for (int k = 0; k < D; ++k) {
        const float a = qr[r_own * (D + 1) + k];
#pragma unroll
        for (int j = 0; j < CW; ++j) acc[j] = fmaf(a, Ss[k * D + cg * CW + j], acc[j]);
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) ot[r_own * (D + 1) + cg * CW + j] = acc[j];
    }
    __syncthreads();
    if (rms) {
      // RMSNorm of y = num / den over the row's D channels, before the gate: fold
      // 1 / sqrt(mean(y^2) + norm_eps) into the row's scale.
      if (tid < TS) {
        float ss = 0.f;
        for (int v = 0; v < D; ++v) ss = fmaf(ot[tid * (D + 1) + v], ot[tid * (D + 1) + v], ss);
        const float iv = inv[tid];
        inv[tid] = iv * rsqrtf(iv * iv * ss / static_cast<float>(D) + norm_eps);
      }
      __syncthreads();
    }
    const T* gb = G + (ti.bh * p.N) * D;
    T* ob = O + (ti.bh * p.N) * D;
    for (int e = tid; e < TS * D; e += THREADS) {
      const int r = e / D, v = e % D;
      const int64_t n = ti.n0 + r;
      if (n < ti.n_end) {
        const float gv = to_f(gb[n * D + v]);
        const float sig = 1.0f / (1.0f + expf(-gv));
        const float gm = (rms && gamma) ? gamma[v] : 1.f;
        ob[n * D + v] = from_f<T>(ot[r * (D + 1) + v] * inv[r] * gm * sig);
      }
    }
  }
}

}  // namespace simt

// ---------------------------------------------------------------------------------------------
// Combine: sum the partial slots of every unit in a fixed order; optionally the per-block states,
// the inclusive prefix over blocks, and the bf16 operand image the tensor-core apply reads.
// One thread per (head, group of 8 consecutive elements of [S | z]).
namespace cmb {

constexpr int THREADS = 256;

// Byte offset of S[k][v] (bf16) in the 128B-swizzled, N-major operand image of a 128 x 128 state:
// two 64-column halves of 128 rows x 128 B; 16-byte chunk j of row k sits at chunk j ^ (k % 8).
__device__ __forceinline__ uint32_t img_offset(int k, int v) {
  const int half = v >> 6, chunk = (v & 63) >> 3;
  return static_cast<uint32_t>(half * 16384 + k * 128 + ((chunk ^ (k & 7)) << 4) + (v & 7) * 2);
}

__device__ __forceinline__ void write_image(uint8_t* img, float* zimg, int64_t unit, int D, int e0,
                                            const float (&x)[8]) {
  if (e0 < D * D) {
    const int k = e0 / D, v = e0 % D;
    uint4 pk = make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]),
                          pack_bf16(x[6], x[7]));
    *reinterpret_cast<uint4*>(img + unit * 32768 + img_offset(k, v)) = pk;
  } else {
    float4* zd = reinterpret_cast<float4*>(zimg + unit * D + (e0 - D * D));
    zd[0] = make_float4(x[0], x[1], x[2], x[3]);
    zd[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
}

__device__ __forceinline__ void store8(float* S, float* z, int64_t unit, int D, int e0, const float (&x)[8]) {
  float* dst = (e0 < D * D) ? S + unit * D * D + e0 : z + unit * D + (e0 - D * D);
  float4* d4 = reinterpret_cast<float4*>(dst);
  d4[0] = make_float4(x[0], x[1], x[2], x[3]);
  d4[1] = make_float4(x[4], x[5], x[6], x[7]);
}

// cos/sin of every (band, pair, position) the tensor-core apply reads, computed in fp64:
// entry e of band b holds (cos, sin)(x * theta) for pair i = (e - off_b) / extent_b and
// position x = (e - off_b) % extent_b.
// Layout [band][pair][position]: the lanes of a warp, which hold consecutive tokens, read
// consecutive positions of one pair.
__device__ __forceinline__ void rope_table_entry(const Plan& p, const Rope& r, int64_t e, float2* tab,
                                                 float2* tab2) {
  int64_t i, x;
  int pair, band;
  if (e < r.tab_off_h) {
    i = e / p.T; x = e - i * p.T; pair = static_cast<int>(i); band = 0;
  } else if (e < r.tab_off_w) {
    i = (e - r.tab_off_h) / p.Hh; x = (e - r.tab_off_h) - i * p.Hh; pair = r.dt / 2 + static_cast<int>(i); band = 1;
  } else {
    i = (e - r.tab_off_w) / p.W; x = (e - r.tab_off_w) - i * p.W; pair = (r.dt + r.dh) / 2 + static_cast<int>(i);
    band = 2;
  }
  double s, c;
  const int64_t xg = band == 0 ? x + r.t_offset : x;  // t rotates at its global frame index
  sincos(static_cast<double>(xg) * r.theta_d[pair], &s, &c);
  const float2 v = make_float2(static_cast<float>(c), static_cast<float>(s));
  tab[e] = v;
  if (tab2) {
    // Second layout (even pair counts per band only): two consecutive pairs of a band per
    // 16-byte entry; t and h bands position-major ([x][pair]), w band [pair / 2][x].
    int64_t e2;
    if (band == 0) e2 = x * (r.dt / 2) + i;
    else if (band == 1) e2 = r.tab_off_h + x * (r.dh / 2) + i;
    else e2 = r.tab_off_w + ((i >> 1) * p.W + x) * 2 + (i & 1);
    tab2[e2] = v;
  }
}

// Builds the cos/sin table of the tensor-core kernels (one thread per entry).
__global__ void __launch_bounds__(THREADS)
rope_table_kernel(const Plan p, const __grid_constant__ Rope rope, float2* tab, float2* tab2) {
  pdl_trigger();
  const int64_t e = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  if (e < rope.tab_entries) rope_table_entry(p, rope, e, tab, tab2);
}

// Thread blocks per unit of the combine kernels: each block covers THREADS groups of 8 elements
// of one unit's [S | z], so all of its threads read the same partial slots.
__host__ __device__ constexpr int blocks_per_unit(int D) { return ((D * D + D) / 8 + THREADS - 1) / THREADS; }

constexpr int MAXC = THREADS;  // slot offsets staged in shared memory per pass

// Shared per-block bookkeeping of the slots of unit u: thread 0 finds the unit's CTA range, then
// the block's threads compute the float offsets of the slots of up to MAXC CTAs at a time (a
// negative offset marks a slot that failed its bounds check).  `fn(m)` is called by every thread
// for each pass, with the offsets of the pass's m CTAs in off[0 .. m), in increasing CTA order,
// between two block-wide barriers.
template <typename Fn>
__device__ __forceinline__ void for_unit_slots(const Plan& p, int64_t u, int64_t slot_floats, int64_t* off,
                                               int64_t* rng, Fn&& fn) {
  if (threadIdx.x == 0) {
    int64_t first = 0, count = 0, c0 = 0, n = 0;
    if (p.total > 0) unit_tiles(p, u, &first, &count);
    if (count > 0) {
      c0 = cta_of(p, first);
      n = cta_of(p, first + count - 1) - c0 + 1;
    }
    rng[0] = c0;
    rng[1] = n;
  }
  __syncthreads();
  const int64_t c0 = rng[0], n = rng[1];
  __syncthreads();  // every thread holds the range before thread 0 may write the next unit's
  for (int64_t j = 0; j < n; j += MAXC) {
    const int m = static_cast<int>(n - j < MAXC ? n - j : MAXC);
    if (static_cast<int>(threadIdx.x) < m) {
      const int64_t cc = c0 + j + threadIdx.x;
      const int64_t k = u - unit_of_tile(p, cta_start(p, cc));
      off[threadIdx.x] = in_bounds(k >= 0 && k < p.maxseg && cc < p.grid) ? (cc * p.maxseg + k) * slot_floats : -1;
    }
    __syncthreads();
    fn(m);
    __syncthreads();
  }
}

// Adds 8 consecutive elements (from e0) of the given slots in order: S part, or the z rows of a
// slot one after another.
__device__ __forceinline__ void add_slots(const float* __restrict__ partial, const int64_t* off, int m, int D,
                                          int zparts, int e0, float (&acc)[8]) {
  if (e0 < D * D) {
#pragma unroll 4
    for (int j = 0; j < m; ++j) {
      const int64_t o = off[j];
      if (o < 0) continue;
      const float4* s4 = reinterpret_cast<const float4*>(partial + o + e0);
      const float4 a = s4[0], b = s4[1];
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
  } else {
    for (int j = 0; j < m; ++j) {
      const int64_t o = off[j];
      if (o < 0) continue;
      for (int zp = 0; zp < zparts; ++zp) {
        const float4* s4 = reinterpret_cast<const float4*>(partial + o + D * D + zp * D + (e0 - D * D));
        const float4 a = s4[0], b = s4[1];
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
      }
    }
  }
}

// Grid: BH * blocks_per_unit(d) blocks; block (bh, chunk) walks the units of head bh in order.
__global__ void __launch_bounds__(THREADS)
combine_kernel(const Plan p, const float* __restrict__ partial, float* S_blk, float* z_blk, float* S_inc,
               float* z_inc, uint8_t* img, float* zimg, int accumulate) {
  __shared__ int64_t off[MAXC];
  __shared__ int64_t rng[2];
  pdl_trigger();
  const int D = p.d;
  const int groups = (D * D + D) / 8;
  const int bpu = blocks_per_unit(D);
  const int64_t bh = blockIdx.x / static_cast<uint32_t>(bpu);
  const int gi = static_cast<int>(blockIdx.x - bh * bpu) * THREADS + static_cast<int>(threadIdx.x);
  if (bh >= p.BH) return;  // (whole blocks only)
  const bool active = gi < groups;
  const int e0 = 8 * (active ? gi : 0);
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(p.zparts) * D;
  // Every thread reads the state kernel's partial sums: wait for that kernel first.
  pdl_wait();
  float run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0.f;
  if (accumulate && active) {
    // Cache update: the running sum starts from the carried state in S_inc / z_inc (one unit per
    // head), which is then overwritten with carried + this call's sum.
    const float* src = (e0 < D * D) ? S_inc + bh * D * D + e0 : z_inc + bh * D + (e0 - D * D);
    const float4 a = reinterpret_cast<const float4*>(src)[0], b = reinterpret_cast<const float4*>(src)[1];
    run[0] = a.x; run[1] = a.y; run[2] = a.z; run[3] = a.w;
    run[4] = b.x; run[5] = b.y; run[6] = b.z; run[7] = b.w;
  }
  for (int64_t blk = 0; blk < p.nblk; ++blk) {
    const int64_t u = bh * p.nblk + blk;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for_unit_slots(p, u, slot_floats, off, rng, [&](int m) {
      if (active) add_slots(partial, off, m, D, p.zparts, e0, acc);
    });
    if (!active) continue;
    if (S_blk) store8(S_blk, z_blk, u, D, e0, acc);
#pragma unroll
    for (int e = 0; e < 8; ++e) run[e] += acc[e];
    if (S_inc) store8(S_inc, z_inc, u, D, e0, run);
    if (img) write_image(img, zimg, u, D, e0, run);
  }
}

// Block-causal combine, first pass: the state of every (head, block) unit alone, summed over its
// CTAs' partial slots in increasing CTA order.  Grid: units * blocks_per_unit(d) blocks, so all
// units run in parallel.
__global__ void __launch_bounds__(THREADS)
blocksum_kernel(const Plan p, const float* __restrict__ partial, float* __restrict__ S_blk, float* __restrict__ z_blk) {
  __shared__ int64_t off[MAXC];
  __shared__ int64_t rng[2];
  pdl_trigger();
  const int D = p.d;
  const int groups = (D * D + D) / 8;
  const int bpu = blocks_per_unit(D);
  const int64_t u = blockIdx.x / static_cast<uint32_t>(bpu);
  const int gi = static_cast<int>(blockIdx.x - u * bpu) * THREADS + static_cast<int>(threadIdx.x);
  if (u >= p.BH * p.nblk) return;  // (whole blocks only)
  const bool active = gi < groups;
  const int e0 = 8 * (active ? gi : 0);
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(p.zparts) * D;
  pdl_wait();
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for_unit_slots(p, u, slot_floats, off, rng, [&](int m) {
    if (active) add_slots(partial, off, m, D, p.zparts, e0, acc);
  });
  if (active) store8(S_blk, z_blk, u, D, e0, acc);
}

// Block-causal combine, second pass: inclusive prefix over the blocks of every head, from the
// per-block states of the first pass (with `reverse`, the suffix sums over blocks b' >= b, which
// the key side of the gradients reads); writes the resulting states and/or the operand image.
// One thread per (head, group of 8 elements); the loads of different blocks are independent, so
// they overlap.
__global__ void __launch_bounds__(THREADS)
prefix_kernel(const Plan p, const float* __restrict__ S_blk, const float* __restrict__ z_blk, float* S_inc,
              float* z_inc, uint8_t* img, float* zimg, int reverse) {
  pdl_trigger();
  pdl_wait();
  const int D = p.d;
  const int groups = (D * D + D) / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  const int64_t bh = idx / groups;
  if (bh >= p.BH) return;
  const int e0 = static_cast<int>(idx - bh * groups) * 8;
  float run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0.f;
#pragma unroll 4
  for (int64_t i = 0; i < p.nblk; ++i) {
    const int64_t blk = reverse ? p.nblk - 1 - i : i;  // reverse: suffix sums over blocks >= blk
    const int64_t u = bh * p.nblk + blk;
    const float* src = (e0 < D * D) ? S_blk + u * D * D + e0 : z_blk + u * D + (e0 - D * D);
    const float4 a = reinterpret_cast<const float4*>(src)[0], b = reinterpret_cast<const float4*>(src)[1];
    run[0] += a.x; run[1] += a.y; run[2] += a.z; run[3] += a.w;
    run[4] += b.x; run[5] += b.y; run[6] += b.z; run[7] += b.w;
    if (S_inc) store8(S_inc, z_inc, u, D, e0, run);
    if (img) write_image(img, zimg, u, D, e0, run);
  }
}

// Token-causal: the state each CTA's first unit carries into the CTA's tile range, i.e. the sum,
// in CTA order, of that unit's partial states from the CTAs before it (zero when the unit starts
// in the CTA itself).  One thread per (CTA, group of 8 consecutive elements of [S | z]).
__global__ void __launch_bounds__(THREADS)
start_kernel(const Plan p, const float* __restrict__ partial, float* __restrict__ start) {
  pdl_trigger();
  pdl_wait();
  const int D = p.d;
  const int groups = (D * D + D) / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  const int64_t c = idx / groups;
  if (c >= p.grid) return;
  const int e0 = static_cast<int>(idx - c * groups) * 8;
  const int64_t slot_floats = static_cast<int64_t>(D) * D + static_cast<int64_t>(p.zparts) * D;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const int64_t g0 = cta_start(p, c);
  if (g0 < cta_start(p, c + 1)) {
    const int64_t u = unit_of_tile(p, g0);
    int64_t first = 0, count = 0;
    unit_tiles(p, u, &first, &count);
    for (int64_t cc = cta_of(p, first); cc < c; ++cc) {
      const int64_t k = u - unit_of_tile(p, cta_start(p, cc));
      if (!in_bounds(k >= 0 && k < p.maxseg)) continue;
      const float* src = partial + (cc * p.maxseg + k) * slot_floats;
      for (int zp = 0; zp < (e0 < D * D ? 1 : p.zparts); ++zp) {
        const float4* s4 = reinterpret_cast<const float4*>(e0 < D * D ? src + e0 : src + D * D + zp * D + (e0 - D * D));
        const float4 a = s4[0], b = s4[1];
        acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
        acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
      }
    }
  }
  float4* d4 = reinterpret_cast<float4*>(start + c * (static_cast<int64_t>(D) * D + D) + e0);
  d4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  d4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// In-place inclusive prefix over blocks of [B*H][nblk][D*D] and [B*H][nblk][D] (with `reverse`,
// the suffix sums over blocks b' >= b).
__global__ void __launch_bounds__(THREADS)
scan_kernel(int64_t BH, int64_t nblk, int D, float* S, float* z, int reverse = 0) {
  const int groups = (D * D + D) / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  const int64_t bh = idx / groups;
  if (bh >= BH) return;
  const int e0 = static_cast<int>(idx - bh * groups) * 8;
  float run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0.f;
  for (int64_t i = 0; i < nblk; ++i) {
    const int64_t blk = reverse ? nblk - 1 - i : i;
    const int64_t u = bh * nblk + blk;
    float* src = (e0 < D * D) ? S + u * D * D + e0 : z + u * D + (e0 - D * D);
    float4* s4 = reinterpret_cast<float4*>(src);
    const float4 a = s4[0], b = s4[1];
    run[0] += a.x; run[1] += a.y; run[2] += a.z; run[3] += a.w;
    run[4] += b.x; run[5] += b.y; run[6] += b.z; run[7] += b.w;
    s4[0] = make_float4(run[0], run[1], run[2], run[3]);
    s4[1] = make_float4(run[4], run[5], run[6], run[7]);
  }
}

// bf16 operand image of given fp32 states (for the tensor-core apply called on its own).
__global__ void __launch_bounds__(THREADS)
pack_kernel(int64_t units, int D, const float* __restrict__ S, const float* __restrict__ z, uint8_t* img,
            float* zimg, const Plan p, const __grid_constant__ Rope rope, float2* tab, float2* tab2,
            int64_t pack_blocks) {
  if (static_cast<int64_t>(blockIdx.x) >= pack_blocks) {
    const int64_t e = (static_cast<int64_t>(blockIdx.x) - pack_blocks) * THREADS + threadIdx.x;
    if (tab && e < rope.tab_entries) rope_table_entry(p, rope, e, tab, tab2);
    return;
  }
  const int groups = (D * D + D) / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * THREADS + threadIdx.x;
  const int64_t u = idx / groups;
  if (u >= units) return;
  const int e0 = static_cast<int>(idx - u * groups) * 8;
  const float* src = (e0 < D * D) ? S + u * D * D + e0 : z + u * D + (e0 - D * D);
  const float4 a = reinterpret_cast<const float4*>(src)[0], b = reinterpret_cast<const float4*>(src)[1];
  const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  write_image(img, zimg, u, D, e0, x);
}

}  // namespace cmb
}  // namespace la
