// common.cuh -- work decomposition shared by the kernels.
//
// Tokens are grouped in "units": one unit is the token range one state is reduced over
// (a whole head in bidirectional mode, one block of latent frames of a head in block-causal
// mode).  Each unit is cut into tiles of `tile` tokens; the last tile of a unit may be
// ragged.  Tiles are numbered globally, head-major then block then tile, and a persistent
// grid of `grid` CTAs splits that sequence into contiguous, nearly equal ranges:
// CTA c owns tiles [c*total/grid, (c+1)*total/grid).  A CTA whose range crosses a unit
// boundary emits one partial state per unit it touches ("segment" k = 0, 1, ...), into slot
// c*maxseg + k.  The combine kernel sums the slots of a unit in increasing c, so the result
// is the same bit for bit on every run.
#pragma once
#include <cstdint>

namespace la {

// Division by a run-time constant 1 <= d < 2^31, exact for every dividend n < 2^31:
// with s = ceil(log2 d), mul = ceil(2^(31+s) / d) < 2^32 and q = floor(n * mul / 2^(31+s)).
// (n * mul / 2^(31+s) = n/d + n*e/2^(31+s) with 0 <= e < 1, and the excess is below 2^-s <= 1/d,
// so it never carries the quotient past the next integer.)
struct FastDiv {
  uint32_t d, mul, shift;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.mul = 0;
  f.shift = 0;
  if (d <= 1) return f;
  uint32_t s = 0;
  while ((uint64_t(1) << s) < d) ++s;
  f.mul = static_cast<uint32_t>(((uint64_t(1) << (31 + s)) + d - 1) / d);
  f.shift = s - 1;
  return f;
}

__host__ __device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  if (f.d == 1) return n;
#ifdef __CUDA_ARCH__
  return __umulhi(n, f.mul) >> f.shift;
#else
  return static_cast<uint32_t>((uint64_t(n) * f.mul) >> 32) >> f.shift;
#endif
}

struct Plan {
  int64_t BH;              // B * H
  int64_t N;               // tokens per head
  int64_t T, Hh, W, HW;    // latent grid
  int64_t nblk;            // units per head (1 when bidirectional)
  int64_t blk_tokens;      // tokens of a full unit
  int64_t tile;            // tokens per tile
  int64_t tiles_full;      // tiles of a full unit
  int64_t tiles_last;      // tiles of the last unit of a head
  int64_t tiles_per_head;
  int64_t total;           // total tiles
  int32_t grid;            // persistent CTAs (each owns >= 1 tile when total > 0)
  int32_t maxseg;          // partial slots per CTA
  int32_t d;
  int32_t zparts;          // partial z rows per slot (summed in order by the combine kernel)
  float eps;
  FastDiv fd_tph, fd_tfull, fd_HW, fd_W;  // tiles_per_head, tiles_full, Hh*W, W
  // CTA ranges without 64-bit division: total = cta_q * grid + cta_r, so
  // c * total / grid = c * cta_q + (c * cta_r) / grid, and c * cta_r < grid^2 < 2^31.
  int64_t cta_q;
  uint32_t cta_r;
  FastDiv fd_grid;
};

// Rotation parameters of the d/2 channel pairs (at most 64 for d = 128).
struct Rope {
  float theta[64];      // base^(-2i/D) of the pair's band, fp32
  double theta_d[64];   // same in fp64
  int32_t band[64];     // 0: t, 1: h, 2: w
  int32_t dt, dh, dw;   // band widths in channels
  // cos/sin table (float2 entries), band-major then pair then position:
  //   t band: [dt/2][T] at 0, h band: [dh/2][Hh] at off_h, w band: [dw/2][W] at off_w.
  int64_t tab_off_h, tab_off_w, tab_entries;
  int64_t t_offset;     // global index of frame 0: the t band rotates at t_offset + t
};

// Band (0: t, 1: h, 2: w) of channel pair `pair`.  DT/DH >= 0 fix the split at compile time.
template <int DT, int DH>
__host__ __device__ __forceinline__ int band_of(int pair, const Rope& r) {
  const int dt = DT >= 0 ? DT : r.dt;
  const int dh = DH >= 0 ? DH : r.dh;
  return (2 * pair < dt) ? 0 : (2 * pair < dt + dh ? 1 : 2);
}
// Index of `pair` within its band.
template <int DT, int DH>
__host__ __device__ __forceinline__ int pair_in_band(int pair, const Rope& r) {
  const int dt = DT >= 0 ? DT : r.dt;
  const int dh = DH >= 0 ? DH : r.dh;
  const int b = band_of<DT, DH>(pair, r);
  return b == 0 ? pair : (b == 1 ? pair - dt / 2 : pair - (dt + dh) / 2);
}

struct TileInfo {
  int64_t bh;      // flat head index b*H + h
  int64_t unit;    // bh * nblk + blk
  int64_t n0;      // first token of the tile (within the head)
  int64_t n_end;   // one past the last token of the tile's unit
};

// Tile indices, token indices and tile counts all stay below 2^31 (checked on the host), so the
// per-tile bookkeeping uses 32-bit multiply-high division.
__host__ __device__ inline TileInfo tile_info(const Plan& p, int64_t g) {
  TileInfo t;
  const uint32_t gg = static_cast<uint32_t>(g);
  const uint32_t bh = fdiv(gg, p.fd_tph);
  const uint32_t r = gg - bh * static_cast<uint32_t>(p.tiles_per_head);
  uint32_t blk = fdiv(r, p.fd_tfull);
  if (blk > static_cast<uint32_t>(p.nblk - 1)) blk = static_cast<uint32_t>(p.nblk - 1);
  const uint32_t tib = r - blk * static_cast<uint32_t>(p.tiles_full);
  const int64_t start = int64_t(blk) * p.blk_tokens;
  int64_t end = start + p.blk_tokens;
  if (end > p.N) end = p.N;
  t.bh = bh;
  t.unit = int64_t(bh) * p.nblk + blk;
  t.n0 = start + int64_t(tib) * p.tile;
  t.n_end = end;
  return t;
}

__host__ __device__ inline int64_t unit_of_tile(const Plan& p, int64_t g) {
  const uint32_t gg = static_cast<uint32_t>(g);
  const uint32_t bh = fdiv(gg, p.fd_tph);
  uint32_t blk = fdiv(gg - bh * static_cast<uint32_t>(p.tiles_per_head), p.fd_tfull);
  if (blk > static_cast<uint32_t>(p.nblk - 1)) blk = static_cast<uint32_t>(p.nblk - 1);
  return int64_t(bh) * p.nblk + blk;
}

// First tile of CTA c, floor(c * total / grid) (c <= grid < 46341, checked on the host).
__host__ __device__ inline int64_t cta_start(const Plan& p, int64_t c) {
  return c * p.cta_q + static_cast<int64_t>(fdiv(static_cast<uint32_t>(c) * p.cta_r, p.fd_grid));
}

// The CTA whose range holds tile g: the largest c with cta_start(c) <= g.  Estimated in double
// precision (error well below one CTA), then settled exactly against cta_start.
__host__ __device__ inline int64_t cta_of(const Plan& p, int64_t g) {
  int64_t c = static_cast<int64_t>(static_cast<double>(g) * static_cast<double>(p.grid) / static_cast<double>(p.total));
  if (c >= p.grid) c = p.grid - 1;
  if (c < 0) c = 0;
  while (c + 1 < p.grid && cta_start(p, c + 1) <= g) ++c;
  while (c > 0 && cta_start(p, c) > g) --c;
  return c;
}

// Global tile range [first, first + count) of unit u.
__host__ __device__ inline void unit_tiles(const Plan& p, int64_t u, int64_t* first, int64_t* count) {
  int64_t bh = u / p.nblk;
  int64_t blk = u - bh * p.nblk;
  *first = bh * p.tiles_per_head + blk * p.tiles_full;
  *count = (blk == p.nblk - 1) ? p.tiles_last : p.tiles_full;
}

// Grid position of token n, row-major over (T, Hh, W) with t slowest.
__device__ __forceinline__ void token_pos(const Plan& p, uint32_t n, uint32_t& t, uint32_t& h, uint32_t& w) {
  t = fdiv(n, p.fd_HW);
  const uint32_t rem = n - t * static_cast<uint32_t>(p.HW);
  h = fdiv(rem, p.fd_W);
  w = rem - h * static_cast<uint32_t>(p.W);
}

// Advance a grid position by `step` tokens.
__device__ __forceinline__ void token_pos_advance(const Plan& p, uint32_t step, uint32_t& t, uint32_t& h,
                                                  uint32_t& w) {
  uint32_t W = static_cast<uint32_t>(p.W), Hh = static_cast<uint32_t>(p.Hh);
  w += step;
  while (w >= W) {
    w -= W;
    if (++h >= Hh) {
      h = 0;
      ++t;
    }
  }
}

}  // namespace la
