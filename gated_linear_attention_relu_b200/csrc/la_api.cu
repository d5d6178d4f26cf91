// la_api.cu -- the C ABI declared in include/la.h: argument checks, work planning, TMA
// descriptors and kernel launches.  Single translation unit: the kernels are included here.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "la.h"
#include "common.cuh"
#include "sm100.cuh"
#include "state_tc.cuh"
#include "apply_tc.cuh"
#include "causal_tc.cuh"
#include "bwd_tc.cuh"
#include "simt.cuh"
#include "simt_ext.cuh"

namespace {

using la::Plan;
using la::Rope;

thread_local int g_last_launches = 0;

constexpr int64_t kMaxTokens = (int64_t(1) << 31) - 1024;  // token indices stay in 32 bits

// ------------------------------------------------------------------------------- validation
bool is_pow2_dim(int32_t d) { return d == 32 || d == 64 || d == 128; }

int validate(const la_problem* p) {
  if (!p) return LA_ERR_NULL;
  if (p->B < 0 || p->H < 0 || p->T < 0 || p->Hh < 0 || p->W < 0 || p->block_frames < 0) return LA_ERR_SHAPE;
  if (p->dtype != LA_BF16 && p->dtype != LA_F32) return LA_ERR_UNSUPPORTED;
  if ((p->flags & ~(LA_FLAG_FORCE_SIMT | LA_FLAG_TOKEN_CAUSAL)) != 0u) return LA_ERR_UNSUPPORTED;
  if (!is_pow2_dim(p->d)) return LA_ERR_UNSUPPORTED;
  if (p->dt < 0 || p->dh < 0 || p->dw < 0 || (p->dt & 1) || (p->dh & 1) || (p->dw & 1) ||
      p->dt + p->dh + p->dw != p->d)
    return LA_ERR_BANDS;
  if (!(p->rope_base > 0.0) || !std::isfinite(p->rope_base)) return LA_ERR_SHAPE;
  if (!std::isfinite(p->eps) || p->eps < 0.f) return LA_ERR_SHAPE;
  // Overflow-safe size checks.
  const int64_t lim = int64_t(1) << 31;
  if (p->T >= lim || p->Hh >= lim || p->W >= lim || p->B >= lim || p->H >= lim) return LA_ERR_SHAPE;
  if (p->t0 < 0 || p->t0 + p->T >= lim) return LA_ERR_SHAPE;
  const double n = double(p->T) * double(p->Hh) * double(p->W);
  if (n > double(kMaxTokens)) return LA_ERR_SHAPE;
  if (double(p->B) * double(p->H) > double(lim - 1)) return LA_ERR_SHAPE;
  if (double(p->B) * double(p->H) * n * double(p->d) > 4.0e18) return LA_ERR_SHAPE;
  // Tile and token indices are 32-bit on the device: at most 2^31 - 1 tiles of >= 32 tokens.
  if (double(p->B) * double(p->H) * (n / 32.0 + double(p->T) + 1.0) >= double(lim - 1)) return LA_ERR_SHAPE;
  return LA_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Checks a tensor pointer that must be present whenever the problem has elements.
int check_ptr(const void* ptr, bool needed) {
  if (!needed) return LA_OK;
  if (!ptr) return LA_ERR_NULL;
  if (!aligned16(ptr)) return LA_ERR_ALIGN;
  return LA_OK;
}

// ------------------------------------------------------------------------------- planning
void set_fastdiv(Plan& p) {
  const int64_t g = p.grid > 0 ? p.grid : 1;
  p.cta_q = p.total / g;
  p.cta_r = static_cast<uint32_t>(p.total % g);
  p.fd_grid = la::make_fastdiv(static_cast<uint32_t>(g));
  p.fd_tph = la::make_fastdiv(static_cast<uint32_t>(p.tiles_per_head > 0 ? p.tiles_per_head : 1));
  p.fd_tfull = la::make_fastdiv(static_cast<uint32_t>(p.tiles_full > 0 ? p.tiles_full : 1));
  p.fd_HW = la::make_fastdiv(static_cast<uint32_t>(p.HW > 0 ? p.HW : 1));
  p.fd_W = la::make_fastdiv(static_cast<uint32_t>(p.W > 0 ? p.W : 1));
}

Plan build_plan(const la_problem& q, int64_t tile, int64_t grid_cap, int zparts) {
  Plan p;
  std::memset(&p, 0, sizeof p);
  p.BH = q.B * q.H;
  p.T = q.T;
  p.Hh = q.Hh;
  p.W = q.W;
  p.HW = q.Hh * q.W;
  p.N = q.T * p.HW;
  p.d = q.d;
  p.zparts = zparts;
  p.eps = q.eps;
  p.tile = tile;
  if (q.block_frames > 0) {
    p.nblk = (q.T + q.block_frames - 1) / q.block_frames;
    p.blk_tokens = int64_t(q.block_frames) * p.HW;
  } else {
    p.nblk = 1;
    p.blk_tokens = p.N;
  }
  if (p.N == 0 || p.BH == 0 || p.nblk == 0) {
    p.total = 0;
    p.grid = 0;
    p.maxseg = 0;
    p.tiles_full = p.tiles_last = p.tiles_per_head = 0;
    set_fastdiv(p);
    return p;
  }
  const int64_t full_len = p.blk_tokens < p.N ? p.blk_tokens : p.N;
  const int64_t last_len = p.N - (p.nblk - 1) * p.blk_tokens;
  p.tiles_full = (full_len + tile - 1) / tile;
  p.tiles_last = (last_len + tile - 1) / tile;
  p.tiles_per_head = (p.nblk - 1) * p.tiles_full + p.tiles_last;
  p.total = p.BH * p.tiles_per_head;
  // (at most 46340 CTAs, so that the CTA-range arithmetic of common.cuh stays within 32 bits)
  if (grid_cap > 46340) grid_cap = 46340;
  p.grid = static_cast<int32_t>(p.total < grid_cap ? p.total : grid_cap);
  set_fastdiv(p);
  int64_t maxseg = 0;
  for (int64_t c = 0; c < p.grid; ++c) {
    const int64_t a = la::cta_start(p, c), b = la::cta_start(p, c + 1);
    const int64_t segs = la::unit_of_tile(p, b - 1) - la::unit_of_tile(p, a) + 1;
    if (segs > maxseg) maxseg = segs;
  }
  p.maxseg = static_cast<int32_t>(maxseg);
  return p;
}

// The band split of the production head (d = 128: t/h/w = 32/48/48) gets kernels with the split
// fixed at compile time; any other split uses the run-time variant.
bool standard_bands(const la_problem& q) { return q.d == 128 && q.dt == 32 && q.dh == 48 && q.dw == 48; }

struct PlanSet {
  bool tc;            // tensor-core kernels (bf16, d = 128)
  Plan ps;            // state reduction
  Plan pa;            // apply
  int64_t units;      // B*H*nblk
  size_t off_partial, off_states, off_img, off_zimg, off_tab, off_tab2, off_start, off_states2, off_dgamma, total;
  int64_t tab_entries;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

PlanSet make_plans(const la_problem& q, int sm_count) {
  PlanSet s;
  s.tc = q.dtype == LA_BF16 && q.d == 128 && !(q.flags & LA_FLAG_FORCE_SIMT);
  if (s.tc) {
    s.ps = build_plan(q, la::st::TILE, sm_count, la::st::ZPARTS);
    s.pa = build_plan(q, la::ap::TILE, sm_count, 1);
  } else {
    s.ps = build_plan(q, la::simt::TS, int64_t(sm_count) * 2, 1);
    s.pa = build_plan(q, la::simt::TS, sm_count, 1);
  }
  const int64_t D = q.d;
  s.units = s.ps.BH * s.ps.nblk;
  // (the backward kernel writes up to bw::ZPARTS dz rows per slot)
  const size_t slot_bytes = size_t(D * D + int64_t(s.tc ? std::max(s.ps.zparts, la::bw::ZPARTS) : s.ps.zparts) * D) * 4;
  size_t off = 0;
  s.off_partial = off;
  off = align256(off + size_t(s.ps.grid) * size_t(s.ps.maxseg) * slot_bytes);
  s.off_states = off;
  off = align256(off + size_t(s.units) * size_t(D * D + D) * 4);
  s.off_img = off;
  off = align256(off + (s.tc ? size_t(s.units) * 32768 : 0));
  s.off_zimg = off;
  off = align256(off + (s.tc ? size_t(s.units) * 512 : 0));
  s.tab_entries = (s.tc && s.pa.total > 0) ? (q.dt / 2) * q.T + (q.dh / 2) * q.Hh + (q.dw / 2) * q.W : 0;
  s.off_tab = off;
  off = align256(off + size_t(s.tab_entries) * 8);
  s.off_tab2 = off;  // the same entries in the apply kernel's layout (standard band split only)
  off = align256(off + (standard_bands(q) ? size_t(s.tab_entries) * 8 : 0));
  s.off_start = off;  // token-causal: state carried into each CTA's range
  off = align256(off + size_t(s.ps.grid) * size_t(D * D + D) * 4);
  s.off_states2 = off;  // gradients on the CUDA cores: per-unit dS, dz (suffix sums over blocks)
  off = align256(off + (s.tc ? 0 : size_t(s.units) * size_t(D * D + D) * 4));
  s.off_dgamma = off;   // gradients: the query side's dgamma rows (4 per CTA on the tensor cores)
  off = align256(off + size_t(s.ps.grid) * size_t(D) * 4 * (s.tc ? 4 : 1));
  s.total = off;
  return s;
}

// Bytes a workspace needs for every entry point: the gradients of the gated forms run on the
// CUDA-core kernels even where the other calls take the tensor-core ones, so both layouts fit.
size_t workspace_need(const la_problem& q, int sm_count) {
  const PlanSet s = make_plans(q, sm_count);
  if (!s.tc) return s.total;
  la_problem qs = q;
  qs.flags |= LA_FLAG_FORCE_SIMT;
  return std::max(s.total, make_plans(qs, sm_count).total);
}

// Bytes the forward paths use: everything before the token-causal start states, which (with the
// gradients' regions after them) sit last in the layout and are read by no forward path.
size_t forward_bytes(const PlanSet& s) { return s.off_start; }

Rope make_rope(const la_problem& q) {
  Rope r;
  std::memset(&r, 0, sizeof r);
  const int bands[3] = {q.dt, q.dh, q.dw};
  int pi = 0;
  for (int axis = 0; axis < 3; ++axis) {
    for (int i = 0; i < bands[axis] / 2; ++i, ++pi) {
      const double th = std::pow(q.rope_base, -2.0 * double(i) / double(bands[axis]));
      r.theta_d[pi] = th;
      r.theta[pi] = static_cast<float>(th);
      r.band[pi] = axis;
    }
  }
  r.dt = q.dt;
  r.dh = q.dh;
  r.dw = q.dw;
  r.tab_off_h = int64_t(q.dt / 2) * q.T;
  r.tab_off_w = r.tab_off_h + int64_t(q.dh / 2) * q.Hh;
  r.tab_entries = r.tab_off_w + int64_t(q.dw / 2) * q.W;
  r.t_offset = q.t0;
  return r;
}


// ------------------------------------------------------------------------------- CUDA helpers
int current_sm_count(int* sm) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
  if (cudaDeviceGetAttribute(sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LA_ERR_CUDA;
  return LA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [BH, N, 128] bf16 viewed as a 3D tensor {128, N, BH}; boxes of 64 channels x 128 tokens,
// 128-byte swizzle (the canonical UMMA operand layout).
bool make_tmap(CUtensorMap* m, const void* base, int64_t BH, int64_t N, uint32_t box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, cuuint64_t(N), cuuint64_t(BH)};
  cuuint64_t strides[2] = {128 * 2, cuuint64_t(N) * 128 * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int launched_ok() { return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

// Launches `kern`; with `pdl` it may start while the previous kernel in the stream is still
// running (programmatic stream serialization).  Only kernels whose predecessor in the stream is
// one of this library's own kernels get `pdl`, and each of them calls pdl_wait() before reading
// anything produced before it; what they read earlier (K, V, G) was produced before the first
// kernel of the call, which is launched normally.
template <typename... KArgs, typename... Args>
int launch_k(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st, bool pdl,
             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

template <typename F>
int set_smem(F* kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) == cudaSuccess
             ? LA_OK
             : LA_ERR_CUDA;
}

// Optional terms of the full gated form (la_gates), as the launchers see them.
struct Gates {
  const void* beta = nullptr;   // [B,H,N] write gate, problem dtype; null: 1
  const float* gamma = nullptr; // [d] RMSNorm weight; null: 1
  float norm_eps = 0.f;
  bool rms = false;
};

// ------------------------------------------------------------------------------- launchers
// cos/sin table shared by the tensor-core state and apply kernels, one entry per thread.
int launch_table(const PlanSet& s, const la_problem& q, void* ws, cudaStream_t st, int* nl) {
  if (!s.tc || s.tab_entries == 0) return LA_OK;
  float2* tab = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + s.off_tab);
  const Rope rope = make_rope(q);
  const int64_t tblocks = (s.tab_entries + la::cmb::THREADS - 1) / la::cmb::THREADS;
  float2* tab2 = standard_bands(q) ? reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + s.off_tab2) : nullptr;
  la::cmb::rope_table_kernel<<<unsigned(tblocks), la::cmb::THREADS, 0, st>>>(s.ps, rope, tab, tab2);
  ++*nl;
  return launched_ok();
}

// The bf16 operand image (and z) of given fp32 unit states, with the cos/sin tables, in one launch:
// what the tensor-core apply and query-side gradient kernels read when the states come from the
// caller instead of the state kernel.
int launch_pack(const PlanSet& s, const la_problem& q, const float* S, const float* z, void* ws, cudaStream_t st,
                int* nl) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int64_t threads = s.units * ((128 * 128 + 128) / 8);
  const int64_t pblocks = (threads + la::cmb::THREADS - 1) / la::cmb::THREADS;
  const int64_t tblocks = (s.tab_entries + la::cmb::THREADS - 1) / la::cmb::THREADS;
  const Rope rope = make_rope(q);
  la::cmb::pack_kernel<<<unsigned(pblocks + tblocks), la::cmb::THREADS, 0, st>>>(
      s.units, 128, S, z, w + s.off_img, reinterpret_cast<float*>(w + s.off_zimg), s.pa, rope,
      reinterpret_cast<float2*>(w + s.off_tab), standard_bands(q) ? reinterpret_cast<float2*>(w + s.off_tab2) : nullptr,
      pblocks);
  ++*nl;
  return launched_ok();
}

int launch_state(const PlanSet& s, const la_problem& q, const void* K, const void* V, void* ws,
                 cudaStream_t st, int* nl, const void* beta = nullptr) {
  if (s.ps.total == 0) return LA_OK;
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + s.off_partial);
  const Rope rope = make_rope(q);
  if (s.tc) {
    CUtensorMap tk, tv;
    if (!make_tmap(&tk, K, s.ps.BH, s.ps.N, la::st::TILE) || !make_tmap(&tv, V, s.ps.BH, s.ps.N, la::st::TILE))
      return LA_ERR_CUDA;
    const float2* tab = reinterpret_cast<const float2*>(static_cast<uint8_t*>(ws) + s.off_tab);
    auto kern = standard_bands(q) ? (beta ? la::st::state_tc_kernel<32, 48, true> : la::st::state_tc_kernel<32, 48, false>)
                                  : (beta ? la::st::state_tc_kernel<-1, -1, true> : la::st::state_tc_kernel<-1, -1, false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, la::st::SMEM_BYTES) != cudaSuccess)
      return LA_ERR_CUDA;
    const float4* tab2 =
        standard_bands(q) ? reinterpret_cast<const float4*>(static_cast<uint8_t*>(ws) + s.off_tab2) : nullptr;
    // The cos/sin table kernel runs just before (same condition: tensor-core path, tokens > 0).
    if (launch_k(kern, unsigned(s.ps.grid), la::st::THREADS, la::st::SMEM_BYTES, st, true, tk, tv, s.ps, rope,
                 tab, tab2, static_cast<const __nv_bfloat16*>(beta), partial))
      return LA_ERR_CUDA;
  } else {
#define LA_STATE_SIMT(DD, TT)                                                                         \
  la::simt::state_simt_kernel<DD, TT><<<s.ps.grid, la::simt::THREADS, 0, st>>>(                      \
      static_cast<const TT*>(K), static_cast<const TT*>(V), static_cast<const TT*>(beta), s.ps, rope, partial)
    if (q.dtype == LA_BF16) {
      if (q.d == 32) LA_STATE_SIMT(32, __nv_bfloat16);
      else if (q.d == 64) LA_STATE_SIMT(64, __nv_bfloat16);
      else LA_STATE_SIMT(128, __nv_bfloat16);
    } else {
      if (q.d == 32) LA_STATE_SIMT(32, float);
      else if (q.d == 64) LA_STATE_SIMT(64, float);
      else LA_STATE_SIMT(128, float);
    }
#undef LA_STATE_SIMT
  }
  ++*nl;
  return launched_ok();
}

// `after` (optional) is called with the launch count after each kernel this queues (timing marks).
// `reverse` (block-causal only): the image holds suffix sums over blocks instead of prefixes.
int launch_combine(const PlanSet& s, const la_problem& q, void* ws, float* S_blk, float* z_blk, float* S_inc,
                   float* z_inc, bool img, cudaStream_t st, int* nl, bool accumulate = false,
                   const std::function<void(int)>& after = nullptr, bool reverse = false) {
  const int64_t groups = (int64_t(s.ps.d) * s.ps.d + s.ps.d) / 8;
  const int64_t threads = s.ps.BH * groups;
  if (threads == 0 || s.ps.nblk == 0) return LA_OK;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const float* partial = reinterpret_cast<const float*>(w + s.off_partial);
  uint8_t* im = img ? w + s.off_img : nullptr;
  float* zim = img ? reinterpret_cast<float*>(w + s.off_zimg) : nullptr;
  (void)q;
  const int64_t cblocks = (threads + la::cmb::THREADS - 1) / la::cmb::THREADS;       // prefix: one thread per group
  const int64_t hblocks = s.ps.BH * la::cmb::blocks_per_unit(s.ps.d);               // combine: per head
  const int64_t ublocks = s.units * la::cmb::blocks_per_unit(s.ps.d);               // blocksum: per unit
  // Block-causal, tensor-core path (several blocks, no accumulation): per-block sums of all units
  // in parallel, then the prefix over blocks.  The per-block states go to the caller's S_blk if it
  // wants them, else to the workspace's state area (on this path the inclusive states go only to
  // the caller's buffer and the operand image, never to that area, so nothing aliases).
  if (s.tc && s.ps.nblk > 1 && !accumulate) {
    float* sb = S_blk ? S_blk : reinterpret_cast<float*>(w + s.off_states);
    float* zb = S_blk ? z_blk : reinterpret_cast<float*>(w + s.off_states) + s.units * q.d * q.d;
    if (launch_k(la::cmb::blocksum_kernel, unsigned(ublocks), la::cmb::THREADS, 0, st, s.tc && s.ps.total > 0, s.ps,
                 partial, sb, zb))
      return LA_ERR_CUDA;
    ++*nl;
    if (after) after(*nl);
    if (S_inc || im) {
      if (launch_k(la::cmb::prefix_kernel, unsigned(cblocks), la::cmb::THREADS, 0, st, true, s.ps,
                   static_cast<const float*>(sb), static_cast<const float*>(zb), S_inc, z_inc, im, zim,
                   reverse ? 1 : 0))
        return LA_ERR_CUDA;
      ++*nl;
      if (after) after(*nl);
    }
    return LA_OK;
  }
  // After the tensor-core state kernel (if it ran) the combine kernel may launch early; it waits
  // for that kernel before its first read.
  if (launch_k(la::cmb::combine_kernel, unsigned(hblocks), la::cmb::THREADS, 0, st, s.tc && s.ps.total > 0,
               s.ps, partial, S_blk, z_blk, S_inc, z_inc, im, zim, accumulate ? 1 : 0))
    return LA_ERR_CUDA;
  ++*nl;
  if (after) after(*nl);
  return launched_ok();
}

size_t apply_simt_smem(int d) {
  const size_t D = size_t(d), TS = la::simt::TS;
  return (D * D + D + 3 * TS * (D + 1) + TS) * sizeof(float);
}

int launch_apply(const PlanSet& s, const la_problem& q, const void* Q, const void* G, const float* S,
                 const float* z, void* O, void* ws, cudaStream_t st, int* nl, const Gates& gt = Gates()) {
  if (s.pa.total == 0) return LA_OK;
  const Rope rope = make_rope(q);
  if (s.tc) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    CUtensorMap tq, tg, to;
    if (!make_tmap(&tq, Q, s.pa.BH, s.pa.N) || !make_tmap(&tg, G, s.pa.BH, s.pa.N) ||
        !make_tmap(&to, O, s.pa.BH, s.pa.N))
      return LA_ERR_CUDA;
    auto kern = standard_bands(q) ? (gt.rms ? la::ap::apply_tc_kernel<32, 48, true> : la::ap::apply_tc_kernel<32, 48, false>)
                                  : (gt.rms ? la::ap::apply_tc_kernel<-1, -1, true> : la::ap::apply_tc_kernel<-1, -1, false>);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, la::ap::SMEM_BYTES) != cudaSuccess)
      return LA_ERR_CUDA;
    if (la::ap::SPLIT_REGS) {
      // The math warpgroups grow their register files out of what the launch granted; refuse to
      // launch unless the kernel really starts with the per-thread count the split assumes.
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != int(la::ap::REGS_LAUNCH) ||
          int64_t(fa.numRegs) * la::ap::THREADS <
              128 * (int64_t(la::ap::REGS_CTRL) + int64_t(la::ap::MATH_WGS) * la::ap::REGS_MATH))
        return LA_ERR_CUDA;
    }
    // Called right after the combine kernel (forward) or the pack kernel (apply on its own).
    if (launch_k(kern, unsigned(s.pa.grid), la::ap::THREADS, la::ap::SMEM_BYTES, st, true, tq, tg, to, s.pa, rope,
                 static_cast<const uint8_t*>(w + s.off_img), reinterpret_cast<const float*>(w + s.off_zimg),
                 reinterpret_cast<const float2*>(w + s.off_tab), reinterpret_cast<const float4*>(w + s.off_tab2),
                 gt.gamma, gt.norm_eps, static_cast<__nv_bfloat16*>(O)))
      return LA_ERR_CUDA;
  } else {
    const size_t smem = apply_simt_smem(q.d);
#define LA_APPLY_SIMT(DD, TT)                                                                              \
  do {                                                                                                     \
    if (cudaFuncSetAttribute(la::simt::apply_simt_kernel<DD, TT>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             int(smem)) != cudaSuccess)                                                    \
      return LA_ERR_CUDA;                                                                                  \
    la::simt::apply_simt_kernel<DD, TT><<<s.pa.grid, la::simt::THREADS, smem, st>>>(                       \
        static_cast<const TT*>(Q), static_cast<const TT*>(G), S, z, static_cast<TT*>(O), s.pa, rope,       \
        gt.rms ? 1 : 0, gt.gamma, gt.norm_eps);                                                            \
  } while (0)
    if (q.dtype == LA_BF16) {
      if (q.d == 32) LA_APPLY_SIMT(32, __nv_bfloat16);
      else if (q.d == 64) LA_APPLY_SIMT(64, __nv_bfloat16);
      else LA_APPLY_SIMT(128, __nv_bfloat16);
    } else {
      if (q.d == 32) LA_APPLY_SIMT(32, float);
      else if (q.d == 64) LA_APPLY_SIMT(64, float);
      else LA_APPLY_SIMT(128, float);
    }
#undef LA_APPLY_SIMT
  }
  ++*nl;
  return launched_ok();
}

// `need`: the bytes the calling path uses (the whole layout unless given).
int check_ws(const PlanSet& s, const void* ws, size_t ws_bytes, size_t need = size_t(-1)) {
  if (need == size_t(-1)) need = s.total;
  if (need == 0) return LA_OK;
  if (!ws || ws_bytes < need) return LA_ERR_WORKSPACE;
  if (!aligned16(ws)) return LA_ERR_ALIGN;
  return LA_OK;
}

int64_t elems(const la_problem& q) { return q.B * q.H * q.T * q.Hh * q.W * int64_t(q.d); }
int64_t state_units(const la_problem& q) {
  const int64_t nblk = q.block_frames > 0 ? (q.T + q.block_frames - 1) / q.block_frames : 1;
  return q.B * q.H * nblk;
}

}  // namespace

// ================================================================================= C ABI
extern "C" {

size_t la_workspace_bytes_for(const la_problem* p, int sm_count) {
  if (validate(p) != LA_OK || sm_count <= 0) return 0;
  return workspace_need(*p, sm_count);
}

size_t la_workspace_bytes(const la_problem* p) {
  if (validate(p) != LA_OK) return 0;
  int sm = 0;
  if (current_sm_count(&sm) != LA_OK) return 0;
  return workspace_need(*p, sm);
}

int la_state_reduce(const la_problem* p, const void* K, const void* V, float* S, float* z, void* ws,
                    size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  const bool has_tok = elems(*p) > 0;
  const bool has_state = state_units(*p) > 0;
  if ((rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) || (rc = check_ptr(S, has_state)) ||
      (rc = check_ptr(z, has_state)))
    return rc;
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes))) return rc;
  int nl = 0;
  if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
  if ((rc = launch_state(s, *p, K, V, ws, stream, &nl))) return rc;
  if ((rc = launch_combine(s, *p, ws, S, z, nullptr, nullptr, false, stream, &nl))) return rc;
  g_last_launches = nl;
  return LA_OK;
}

int la_state_update(const la_problem* p, const void* K, const void* V, float* S, float* z, void* ws,
                    size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  const bool has_tok = elems(*p) > 0;
  const bool has_state = state_units(*p) > 0;
  if ((rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) || (rc = check_ptr(S, has_state)) ||
      (rc = check_ptr(z, has_state)))
    return rc;
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes))) return rc;
  int nl = 0;
  if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
  if ((rc = launch_state(s, *p, K, V, ws, stream, &nl))) return rc;
  // No tokens: the state reduction queues nothing and the carried state stays as it is.
  if (has_tok && (rc = launch_combine(s, *p, ws, nullptr, nullptr, S, z, false, stream, &nl, true))) return rc;
  g_last_launches = nl;
  return LA_OK;
}

int la_block_step(const la_problem* p, const void* Q, const void* K, const void* V, const void* G, void* O,
                  float* S, float* z, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  const bool has_tok = elems(*p) > 0;
  const bool has_state = state_units(*p) > 0;
  if ((rc = check_ptr(Q, has_tok)) || (rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) ||
      (rc = check_ptr(G, has_tok)) || (rc = check_ptr(O, has_tok)) || (rc = check_ptr(S, has_state)) ||
      (rc = check_ptr(z, has_state)))
    return rc;
  if (!has_tok) {
    g_last_launches = 0;
    return LA_OK;
  }
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes))) return rc;
  int nl = 0;
  if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
  if ((rc = launch_state(s, *p, K, V, ws, stream, &nl))) return rc;
  // carried + this block -> S, z (and the tensor-core apply's operand image)
  if ((rc = launch_combine(s, *p, ws, nullptr, nullptr, S, z, s.tc, stream, &nl, true))) return rc;
  if ((rc = launch_apply(s, *p, Q, G, S, z, O, ws, stream, &nl))) return rc;
  g_last_launches = nl;
  return LA_OK;
}

// Dispatches a CUDA-core kernel template over the head dimension and dtype of the problem.
#define LA_SIMT_DISPATCH(q, ...)                                           \
  do {                                                                     \
    if ((q).dtype == LA_BF16) {                                            \
      using TT = __nv_bfloat16;                                            \
      if ((q).d == 32) { constexpr int DD = 32; __VA_ARGS__; }             \
      else if ((q).d == 64) { constexpr int DD = 64; __VA_ARGS__; }        \
      else { constexpr int DD = 128; __VA_ARGS__; }                        \
    } else {                                                               \
      using TT = float;                                                    \
      if ((q).d == 32) { constexpr int DD = 32; __VA_ARGS__; }             \
      else if ((q).d == 64) { constexpr int DD = 64; __VA_ARGS__; }        \
      else { constexpr int DD = 128; __VA_ARGS__; }                        \
    }                                                                      \
  } while (0)

static int tokencausal_common(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                              void* O, void* ws, size_t ws_bytes, cudaStream_t stream, cudaEvent_t* marks = nullptr,
                              int nmarks = 0) {
  static_assert(la::st::TILE == la::ca::TILE, "the causal kernel walks the state kernel's tile ranges");
  int rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  const bool has_tok = elems(*p) > 0;
  if ((rc = check_ptr(Q, has_tok)) || (rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) ||
      (rc = check_ptr(G, has_tok)) || (rc = check_ptr(O, has_tok)))
    return rc;
  if (!has_tok) {
    g_last_launches = 0;
    return LA_OK;
  }
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes))) return rc;
  int nl = 0;
  auto mark = [&](int i) {
    if (i < nmarks && marks && marks[i]) cudaEventRecord(marks[i], stream);
  };
  mark(0);
  if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
  mark(nl);
  // Per-segment state sums (the state kernel's partial slots), then each CTA's carried state.
  if ((rc = launch_state(s, *p, K, V, ws, stream, &nl))) return rc;
  mark(nl);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* start = reinterpret_cast<float*>(w + s.off_start);
  const int64_t threads = int64_t(s.ps.grid) * ((int64_t(p->d) * p->d + p->d) / 8);
  if (launch_k(la::cmb::start_kernel, unsigned((threads + la::cmb::THREADS - 1) / la::cmb::THREADS),
               la::cmb::THREADS, 0, stream, s.tc, s.ps, reinterpret_cast<const float*>(w + s.off_partial), start))
    return LA_ERR_CUDA;
  ++nl;
  mark(nl);
  const Rope rope = make_rope(*p);
  if (!s.tc) {
    // CUDA-core path: every dtype and head dimension.
    const size_t smem = la::simt::causal_simt_smem(p->d);
    LA_SIMT_DISPATCH(*p, {
      if ((rc = set_smem(la::simt::causal_simt_kernel<DD, TT>, smem))) return rc;
      la::simt::causal_simt_kernel<DD, TT><<<unsigned(s.ps.grid), la::simt::THREADS, smem, stream>>>(
          static_cast<const TT*>(Q), static_cast<const TT*>(K), static_cast<const TT*>(V), static_cast<const TT*>(G),
          static_cast<TT*>(O), s.ps, rope, static_cast<const float*>(start));
    });
    if ((rc = launched_ok())) return rc;
    ++nl;
    mark(nl);
    g_last_launches = nl;
    return LA_OK;
  }
  CUtensorMap tq, tk, tv, tg, to;
  if (!make_tmap(&tq, Q, s.ps.BH, s.ps.N) || !make_tmap(&tk, K, s.ps.BH, s.ps.N) ||
      !make_tmap(&tv, V, s.ps.BH, s.ps.N) || !make_tmap(&tg, G, s.ps.BH, s.ps.N) ||
      !make_tmap(&to, O, s.ps.BH, s.ps.N))
    return LA_ERR_CUDA;
  auto kern = standard_bands(*p) ? la::ca::causal_tc_kernel<32, 48> : la::ca::causal_tc_kernel<-1, -1>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, la::ca::SMEM_BYTES) != cudaSuccess)
    return LA_ERR_CUDA;
  if (launch_k(kern, unsigned(s.ps.grid), la::ca::THREADS, la::ca::SMEM_BYTES, stream, true, tq, tk, tv, tg, to,
               s.ps, rope, static_cast<const float*>(start), reinterpret_cast<const float2*>(w + s.off_tab),
               reinterpret_cast<const float4*>(w + s.off_tab2)))
    return LA_ERR_CUDA;
  ++nl;
  mark(nl);
  g_last_launches = nl;
  return LA_OK;
}

int la_forward_tokencausal(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                           void* O, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  return tokencausal_common(p, Q, K, V, G, O, ws, ws_bytes, stream);
}

// Gradients of the operator in every form: bidirectional or block-causal (p->block_frames), with
// the optional write gate and RMSNorm.  bf16 with d = 128 takes the tensor-core kernels; fp32,
// d = 32 / 64 and LA_FLAG_FORCE_SIMT the CUDA-core kernels.
// S_saved / z_saved (both or neither): the unit states token n reads, as the forward computed them
// (the head's state, or each block's inclusive prefix); given, the forward state is not recomputed.
static int backward_common(const la_problem* p, const Gates& gt, const void* Q, const void* K, const void* V,
                           const void* G, const void* dO, void* dQ, void* dK, void* dV, void* dG, void* dbeta,
                           float* dgamma, void* ws, size_t ws_bytes, cudaStream_t stream,
                           const float* S_saved = nullptr, const float* z_saved = nullptr) {
  static_assert(la::st::TILE == la::bw::TILE, "the backward kernels walk the state kernel's tile ranges");
  int rc;
  const bool has_tok = elems(*p) > 0;
  const void* ins[5] = {Q, K, V, G, dO};
  void* outs[4] = {dQ, dK, dV, dG};
  for (const void* x : ins)
    if ((rc = check_ptr(x, has_tok))) return rc;
  for (void* x : outs)
    if ((rc = check_ptr(x, has_tok))) return rc;
  if (gt.beta && (rc = check_ptr(dbeta, has_tok))) return rc;
  if (gt.rms && gt.gamma && (rc = check_ptr(dgamma, true))) return rc;
  if (gt.beta && !aligned16(gt.beta)) return LA_ERR_ALIGN;
  if (gt.gamma && !aligned16(gt.gamma)) return LA_ERR_ALIGN;
  if (S_saved || z_saved) {
    if ((rc = check_ptr(S_saved, has_tok)) || (rc = check_ptr(z_saved, has_tok))) return rc;
  }
  if (!has_tok) {
    g_last_launches = 0;
    if (gt.rms && gt.gamma) {  // no tokens: dgamma is zero
      if (cudaMemsetAsync(dgamma, 0, size_t(p->d) * sizeof(float), stream) != cudaSuccess) return LA_ERR_CUDA;
    }
    return LA_OK;
  }
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes))) return rc;
  int nl = 0;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const Rope rope = make_rope(*p);
  if (s.tc) {
    // Forward state (per unit: a head, or a block's inclusive prefix) and its operand image: from
    // the caller's states, or reduced again from K and V.
    if (S_saved) {
      if ((rc = launch_pack(s, *p, S_saved, z_saved, ws, stream, &nl))) return rc;
    } else {
      if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
      if ((rc = launch_state(s, *p, K, V, ws, stream, &nl, gt.beta))) return rc;
      if ((rc = launch_combine(s, *p, ws, nullptr, nullptr, nullptr, nullptr, true, stream, &nl))) return rc;
    }
    const bool sb = standard_bands(*p);
    float* dgp = reinterpret_cast<float*>(w + s.off_dgamma);
    CUtensorMap tq, tg, tdo, tdq, tdg, tk, tv, tdk, tdv;
    if (!make_tmap(&tq, Q, s.ps.BH, s.ps.N) || !make_tmap(&tg, G, s.ps.BH, s.ps.N) ||
        !make_tmap(&tdo, dO, s.ps.BH, s.ps.N) || !make_tmap(&tdq, dQ, s.ps.BH, s.ps.N) ||
        !make_tmap(&tdg, dG, s.ps.BH, s.ps.N) || !make_tmap(&tk, K, s.ps.BH, s.ps.N) ||
        !make_tmap(&tv, V, s.ps.BH, s.ps.N) || !make_tmap(&tdk, dK, s.ps.BH, s.ps.N) ||
        !make_tmap(&tdv, dV, s.ps.BH, s.ps.N))
      return LA_ERR_CUDA;
    // Q side: dQ, dG and the partial sums of dS, dz.
    auto kq = sb ? (gt.rms ? la::bw::bwdq_tc_kernel<32, 48, true> : la::bw::bwdq_tc_kernel<32, 48, false>)
                 : (gt.rms ? la::bw::bwdq_tc_kernel<-1, -1, true> : la::bw::bwdq_tc_kernel<-1, -1, false>);
    if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, la::bw::SMEM_Q) != cudaSuccess)
      return LA_ERR_CUDA;
    if (launch_k(kq, unsigned(s.ps.grid), la::bw::THREADS, la::bw::SMEM_Q, stream, true, tq, tg, tdo, tdq, tdg,
                 s.ps, rope, static_cast<const uint8_t*>(w + s.off_img), reinterpret_cast<const float*>(w + s.off_zimg),
                 reinterpret_cast<const float2*>(w + s.off_tab), reinterpret_cast<const float4*>(w + s.off_tab2),
                 reinterpret_cast<float*>(w + s.off_partial), static_cast<__nv_bfloat16*>(dQ),
                 static_cast<__nv_bfloat16*>(dG), gt.gamma, gt.norm_eps, gt.rms ? dgp : nullptr))
      return LA_ERR_CUDA;
    ++nl;
    // dS, dz summed in fixed order into the operand image (reusing the state image's space); in
    // block-causal mode a key of block b feeds the states of blocks b' >= b, so its image holds
    // the suffix sums over blocks.
    PlanSet s2 = s;
    s2.ps.zparts = la::bw::ZPARTS;
    if ((rc = launch_combine(s2, *p, ws, nullptr, nullptr, nullptr, nullptr, true, stream, &nl, false, nullptr,
                             /*reverse=*/true)))
      return rc;
    // K side: dK, dV.
    auto kk = sb ? (gt.beta ? la::bw::bwdk_tc_kernel<32, 48, true> : la::bw::bwdk_tc_kernel<32, 48, false>)
                 : (gt.beta ? la::bw::bwdk_tc_kernel<-1, -1, true> : la::bw::bwdk_tc_kernel<-1, -1, false>);
    if (cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, la::bw::SMEM_K) != cudaSuccess)
      return LA_ERR_CUDA;
    if (launch_k(kk, unsigned(s.ps.grid), la::bw::THREADS, la::bw::SMEM_K, stream, true, tk, tv, tdk, tdv, s.ps,
                 rope, static_cast<const uint8_t*>(w + s.off_img), reinterpret_cast<const float*>(w + s.off_zimg),
                 reinterpret_cast<const float2*>(w + s.off_tab), reinterpret_cast<const float4*>(w + s.off_tab2),
                 static_cast<__nv_bfloat16*>(dK), static_cast<__nv_bfloat16*>(dV),
                 static_cast<const __nv_bfloat16*>(gt.beta), static_cast<__nv_bfloat16*>(dbeta)))
      return LA_ERR_CUDA;
    ++nl;
    if (gt.rms && gt.gamma) {  // dgamma: the query side's per-warp column sums, in a fixed order
      la::simt::dgamma_sum_kernel<<<unsigned((p->d + la::simt::THREADS - 1) / la::simt::THREADS),
                                    la::simt::THREADS, 0, stream>>>(s.ps.grid * 4, p->d, dgp, dgamma);
      ++nl;
      if ((rc = launched_ok())) return rc;
    }
    g_last_launches = nl;
    return LA_OK;
  }
  // CUDA-core path (fp32 states throughout).
  la_problem qs = *p;
  qs.flags |= LA_FLAG_FORCE_SIMT;
  const PlanSet sp = make_plans(qs, sm);  // the CUDA-core kernels' tile ranges (32-token tiles)
  if ((rc = check_ws(sp, ws, ws_bytes))) return rc;
  float* partial = reinterpret_cast<float*>(w + sp.off_partial);
  float* Sw = reinterpret_cast<float*>(w + sp.off_states);
  float* zw = Sw + sp.units * p->d * p->d;
  const float* Sf = S_saved ? S_saved : Sw;
  const float* zf = S_saved ? z_saved : zw;
  float* dSf = reinterpret_cast<float*>(w + sp.off_states2);
  float* dzf = dSf + sp.units * p->d * p->d;
  float* dgp = reinterpret_cast<float*>(w + sp.off_dgamma);
  const int64_t groups = (int64_t(p->d) * p->d + p->d) / 8;
  const unsigned ublocks = unsigned(sp.units * la::cmb::blocks_per_unit(p->d));
  const unsigned hblocks = unsigned((sp.ps.BH * groups + la::cmb::THREADS - 1) / la::cmb::THREADS);
  // Forward states (unless given): per-unit sums, then (block-causal) the inclusive prefix over blocks.
  if (!S_saved) {
    if ((rc = launch_state(sp, qs, K, V, ws, stream, &nl, gt.beta))) return rc;
    la::cmb::blocksum_kernel<<<ublocks, la::cmb::THREADS, 0, stream>>>(sp.ps, partial, Sw, zw);
    ++nl;
    if (sp.ps.nblk > 1) {
      la::cmb::scan_kernel<<<hblocks, la::cmb::THREADS, 0, stream>>>(sp.ps.BH, sp.ps.nblk, p->d, Sw, zw, 0);
      ++nl;
    }
    if ((rc = launched_ok())) return rc;
  }
  // Query side.
  const size_t smq = la::simt::bwdq_simt_smem(p->d);
  LA_SIMT_DISPATCH(*p, {
    if ((rc = set_smem(la::simt::bwdq_simt_kernel<DD, TT>, smq))) return rc;
    la::simt::bwdq_simt_kernel<DD, TT><<<unsigned(sp.ps.grid), la::simt::THREADS, smq, stream>>>(
        static_cast<const TT*>(Q), static_cast<const TT*>(G), static_cast<const TT*>(dO), Sf, zf,
        static_cast<TT*>(dQ), static_cast<TT*>(dG), sp.ps, rope, gt.rms ? 1 : 0, gt.gamma, gt.norm_eps, partial,
        dgp);
  });
  ++nl;
  // dS, dz per unit, then (block-causal) the suffix sums over blocks.
  la::cmb::blocksum_kernel<<<ublocks, la::cmb::THREADS, 0, stream>>>(sp.ps, partial, dSf, dzf);
  ++nl;
  if (sp.ps.nblk > 1) {
    la::cmb::scan_kernel<<<hblocks, la::cmb::THREADS, 0, stream>>>(sp.ps.BH, sp.ps.nblk, p->d, dSf, dzf, 1);
    ++nl;
  }
  if ((rc = launched_ok())) return rc;
  // Key side.
  const size_t smk = la::simt::bwdk_simt_smem(p->d);
  LA_SIMT_DISPATCH(*p, {
    if ((rc = set_smem(la::simt::bwdk_simt_kernel<DD, TT>, smk))) return rc;
    la::simt::bwdk_simt_kernel<DD, TT><<<unsigned(sp.ps.grid), la::simt::THREADS, smk, stream>>>(
        static_cast<const TT*>(K), static_cast<const TT*>(V), static_cast<const TT*>(gt.beta), dSf, dzf,
        static_cast<TT*>(dK), static_cast<TT*>(dV), static_cast<TT*>(dbeta), sp.ps, rope);
  });
  ++nl;
  if (gt.rms && gt.gamma) {
    la::simt::dgamma_sum_kernel<<<unsigned((p->d + la::simt::THREADS - 1) / la::simt::THREADS), la::simt::THREADS, 0,
                                  stream>>>(sp.ps.grid, p->d, dgp, dgamma);
    ++nl;
  }
  if ((rc = launched_ok())) return rc;
  g_last_launches = nl;
  return LA_OK;
}

int la_backward_bidir(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                      const void* dO, void* dQ, void* dK, void* dV, void* dG, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  return backward_common(p, Gates(), Q, K, V, G, dO, dQ, dK, dV, dG, nullptr, nullptr, ws, ws_bytes, stream);
}

int la_state_scan(const la_problem* p, float* S, float* z, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames == 0) {
    g_last_launches = 0;
    return LA_OK;
  }
  const int64_t BH = p->B * p->H;
  const int64_t nblk = (p->T + p->block_frames - 1) / p->block_frames;
  const bool has_state = BH * nblk > 0;
  if ((rc = check_ptr(S, has_state)) || (rc = check_ptr(z, has_state))) return rc;
  if (!has_state) {
    g_last_launches = 0;
    return LA_OK;
  }
  const int64_t threads = BH * ((int64_t(p->d) * p->d + p->d) / 8);
  const unsigned blocks = unsigned((threads + la::cmb::THREADS - 1) / la::cmb::THREADS);
  la::cmb::scan_kernel<<<blocks, la::cmb::THREADS, 0, stream>>>(BH, nblk, p->d, S, z);
  if ((rc = launched_ok())) return rc;
  g_last_launches = 1;
  return LA_OK;
}

int la_apply(const la_problem* p, const void* Q, const void* G, const float* S, const float* z, void* O,
             void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  const bool has_tok = elems(*p) > 0;
  if ((rc = check_ptr(Q, has_tok)) || (rc = check_ptr(G, has_tok)) || (rc = check_ptr(O, has_tok)) ||
      (rc = check_ptr(S, has_tok)) || (rc = check_ptr(z, has_tok)))
    return rc;
  if (!has_tok) {
    g_last_launches = 0;
    return LA_OK;
  }
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  int nl = 0;
  if (s.tc) {
    if ((rc = check_ws(s, ws, ws_bytes))) return rc;
    if ((rc = launch_pack(s, *p, S, z, ws, stream, &nl))) return rc;
  }
  if ((rc = launch_apply(s, *p, Q, G, S, z, O, ws, stream, &nl))) return rc;
  g_last_launches = nl;
  return LA_OK;
}

static int forward_common(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                          void* O, float* S_incl, float* z_incl, void* ws, size_t ws_bytes, cudaStream_t stream,
                          cudaEvent_t* marks = nullptr, int nmarks = 0, const Gates& gt = Gates()) {
  int rc;
  const bool has_tok = elems(*p) > 0;
  if ((rc = check_ptr(Q, has_tok)) || (rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) ||
      (rc = check_ptr(G, has_tok)) || (rc = check_ptr(O, has_tok)))
    return rc;
  if (gt.beta && !aligned16(gt.beta)) return LA_ERR_ALIGN;
  if (gt.gamma && !aligned16(gt.gamma)) return LA_ERR_ALIGN;
  if (S_incl && !aligned16(S_incl)) return LA_ERR_ALIGN;
  if (z_incl && !aligned16(z_incl)) return LA_ERR_ALIGN;
  if ((S_incl == nullptr) != (z_incl == nullptr)) return LA_ERR_NULL;
  const bool want_states = S_incl != nullptr && state_units(*p) > 0;
  if (!has_tok && !want_states) {
    g_last_launches = 0;
    return LA_OK;
  }
  int sm = 0;
  if ((rc = current_sm_count(&sm))) return rc;
  const PlanSet s = make_plans(*p, sm);
  if ((rc = check_ws(s, ws, ws_bytes, forward_bytes(s)))) return rc;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* st_S = S_incl ? S_incl : reinterpret_cast<float*>(w + s.off_states);
  float* st_z = z_incl ? z_incl : reinterpret_cast<float*>(w + s.off_states) + s.units * p->d * p->d;
  // The tensor-core apply reads the bf16 operand image; the CUDA-core apply reads fp32 states.
  const bool need_fp32 = !s.tc || S_incl != nullptr;
  int nl = 0;
  auto mark = [&](int i) {
    if (i < nmarks && marks && marks[i]) cudaEventRecord(marks[i], stream);
  };
  mark(0);
  if ((rc = launch_table(s, *p, ws, stream, &nl))) return rc;
  if (nl) mark(nl);
  const int b0 = nl;
  if ((rc = launch_state(s, *p, K, V, ws, stream, &nl, gt.beta))) return rc;
  if (nl != b0) mark(nl);
  if ((rc = launch_combine(s, *p, ws, nullptr, nullptr, need_fp32 ? st_S : nullptr, need_fp32 ? st_z : nullptr,
                           s.tc, stream, &nl, false, mark)))
    return rc;
  if (has_tok) {
    const int b2 = nl;
    if ((rc = launch_apply(s, *p, Q, G, st_S, st_z, O, ws, stream, &nl, gt))) return rc;
    if (nl != b2) mark(nl);
  }
  g_last_launches = nl;
  return LA_OK;
}

int la_forward_bidir(const la_problem* p, const void* Q, const void* K, const void* V, const void* G, void* O,
                     void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  return forward_common(p, Q, K, V, G, O, nullptr, nullptr, ws, ws_bytes, stream);
}

int la_forward_blockcausal(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                           void* O, float* S_incl, float* z_incl, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames <= 0) return LA_ERR_SHAPE;
  return forward_common(p, Q, K, V, G, O, S_incl, z_incl, ws, ws_bytes, stream);
}

// Checks and converts la_gates (NULL: no optional terms).
static int read_gates(const la_gates* gates, Gates* gt) {
  *gt = Gates();
  if (!gates) return LA_OK;
  if (gates->rms_norm != 0 && gates->rms_norm != 1) return LA_ERR_UNSUPPORTED;
  if (gates->rms_norm && (!std::isfinite(gates->norm_eps) || gates->norm_eps < 0.f)) return LA_ERR_SHAPE;
  gt->beta = gates->beta;
  gt->rms = gates->rms_norm == 1;
  gt->gamma = gt->rms ? gates->gamma : nullptr;
  gt->norm_eps = gates->norm_eps;
  return LA_OK;
}

int la_forward_gated(const la_problem* p, const la_gates* gates, const void* Q, const void* K, const void* V,
                     const void* G, void* O, float* S_incl, float* z_incl, void* ws, size_t ws_bytes,
                     cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  Gates gt;
  if ((rc = read_gates(gates, &gt))) return rc;
  return forward_common(p, Q, K, V, G, O, S_incl, z_incl, ws, ws_bytes, stream, nullptr, 0, gt);
}

int la_backward(const la_problem* p, const la_gates* gates, const void* Q, const void* K, const void* V,
                const void* G, const void* dO, void* dQ, void* dK, void* dV, void* dG, void* dbeta, float* dgamma,
                void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  Gates gt;
  if ((rc = read_gates(gates, &gt))) return rc;
  return backward_common(p, gt, Q, K, V, G, dO, dQ, dK, dV, dG, dbeta, dgamma, ws, ws_bytes, stream);
}

int la_backward_saved(const la_problem* p, const la_gates* gates, const float* S, const float* z, const void* Q,
                      const void* K, const void* V, const void* G, const void* dO, void* dQ, void* dK, void* dV,
                      void* dG, void* dbeta, float* dgamma, void* ws, size_t ws_bytes, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (!S || !z) return LA_ERR_NULL;
  if (!aligned16(S) || !aligned16(z)) return LA_ERR_ALIGN;
  Gates gt;
  if ((rc = read_gates(gates, &gt))) return rc;
  return backward_common(p, gt, Q, K, V, G, dO, dQ, dK, dV, dG, dbeta, dgamma, ws, ws_bytes, stream, S, z);
}

int la_forward_marked(const la_problem* p, const la_gates* gates, const void* Q, const void* K, const void* V,
                      const void* G, void* O, float* S_incl, float* z_incl, void* ws, size_t ws_bytes,
                      cudaStream_t stream, cudaEvent_t* marks, int nmarks) {
  int rc = validate(p);
  if (rc) return rc;
  if (nmarks < 0 || (nmarks > 0 && !marks)) return LA_ERR_NULL;
  if (p->flags & LA_FLAG_TOKEN_CAUSAL) {
    if (gates || S_incl || z_incl) return LA_ERR_UNSUPPORTED;
    return tokencausal_common(p, Q, K, V, G, O, ws, ws_bytes, stream, marks, nmarks);
  }
  Gates gt;
  if ((rc = read_gates(gates, &gt))) return rc;
  return forward_common(p, Q, K, V, G, O, S_incl, z_incl, ws, ws_bytes, stream, marks, nmarks, gt);
}

const char* la_status_string(int status) {
  switch (status) {
    case LA_OK: return "ok";
    case LA_ERR_NULL: return "a required pointer is NULL";
    case LA_ERR_SHAPE: return "invalid or inconsistent sizes";
    case LA_ERR_BANDS: return "RoPE bands must be even, non-negative and add up to d";
    case LA_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case LA_ERR_UNSUPPORTED: return "unsupported head dimension, dtype or flag";
    case LA_ERR_WORKSPACE: return "workspace missing or smaller than la_workspace_bytes()";
    case LA_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case LA_ERR_DEVICE: return "a kernel reported a device-side failure (a bounded wait ran out)";
    default: return "unknown status";
  }
}

int la_device_error(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return LA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, la::g_la_error, sizeof v) != cudaSuccess) return LA_ERR_CUDA;
  if (v == 0) return LA_OK;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(la::g_la_error, &zero, sizeof zero) != cudaSuccess) return LA_ERR_CUDA;
  return LA_ERR_DEVICE;
}

int la_last_launch_count(void) { return g_last_launches; }

#ifdef LA_TEST_HOOKS
// Hooks build only (not part of the regular library): from the next launch on, the state kernel
// does not issue the K load of global tile `tile` (-1: load every tile), so the bounded waits for
// it run out and the kernel winds down with the error word set.  Used to test that path.
int la_test_skip_tile(long long tile) {
  return cudaMemcpyToSymbol(la::g_la_skip_tile, &tile, sizeof tile) == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
#endif

}  // extern "C"

// Fixed scratch for callers that cannot allocate (la_forward_bidir_static).  In host code the
// symbol is only a handle: its device address is looked up per device with
// cudaGetSymbolAddress, with that device current, and cached.
static __device__ __align__(256) uint8_t g_la_static_ws[LA_STATIC_WORKSPACE_BYTES];

namespace {
std::mutex g_static_mu;
constexpr int kMaxDevices = 256;
void* g_static_ptr[kMaxDevices] = {};

int static_workspace(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return LA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_la_static_ws) != cudaSuccess || !ptr) return LA_ERR_CUDA;
    g_static_ptr[dev] = ptr;
  }
  *out = g_static_ptr[dev];
  return LA_OK;
}
}  // namespace

extern "C" {

int la_forward_bidir_static(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                            void* O, cudaStream_t stream) {
  int rc = validate(p);
  if (rc) return rc;
  if (p->block_frames != 0) return LA_ERR_SHAPE;
  // Argument errors are reported before any CUDA call, as for every other entry point.
  const bool has_tok = elems(*p) > 0;
  if ((rc = check_ptr(Q, has_tok)) || (rc = check_ptr(K, has_tok)) || (rc = check_ptr(V, has_tok)) ||
      (rc = check_ptr(G, has_tok)) || (rc = check_ptr(O, has_tok)))
    return rc;
  int dev = 0, sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
  if ((rc = current_sm_count(&sm))) return rc;
  if (forward_bytes(make_plans(*p, sm)) > LA_STATIC_WORKSPACE_BYTES) return LA_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((rc = static_workspace(dev, &ws))) return rc;
  return forward_common(p, Q, K, V, G, O, nullptr, nullptr, ws, LA_STATIC_WORKSPACE_BYTES, stream);
}

// Host-side self-check of the work decomposition: exact fast division, and every tile of a set
// of problems owned by exactly one CTA with its partial slot in range.  Returns 0 on success.
int la_selftest_host(void) {
  // Fast division against exact division.
  const uint32_t divs[] = {1, 2, 3, 5, 7, 12, 80, 127, 128, 129, 3600, 3601, 65535, 65536, 75600, 1000003,
                           (1u << 30) + 1, (1u << 31) - 1};
  uint64_t x = 88172645463325252ull;
  for (uint32_t d : divs) {
    const la::FastDiv f = la::make_fastdiv(d);
    const uint32_t edge[] = {0, 1, d - 1, d, d + 1, 2 * d - 1, (1u << 31) - 1, (1u << 31) - 2};
    for (uint32_t n : edge)
      if (n < (1u << 31) && la::fdiv(n, f) != n / d) return 1;
    for (int k = 0; k < 20000; ++k) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      const uint32_t n = static_cast<uint32_t>(x) & 0x7fffffffu;
      if (la::fdiv(n, f) != n / d) return 2;
    }
  }
  // CTA ranges (32-bit arithmetic) against exact 64-bit division, and cta_of against its definition.
  for (int trial = 0; trial < 4000; ++trial) {
    x ^= x << 13; x ^= x >> 7; x ^= x << 17;
    Plan p;
    std::memset(&p, 0, sizeof p);
    p.total = static_cast<int64_t>(x & 0x7fffffffu) + 1;
    const int64_t gcap = trial % 3 == 0 ? 46340 : static_cast<int64_t>((x >> 33) % 1000) + 1;
    p.grid = static_cast<int32_t>(p.total < gcap ? p.total : gcap);
    set_fastdiv(p);
    for (int k = 0; k < 8; ++k) {
      x ^= x << 13; x ^= x >> 7; x ^= x << 17;
      const int64_t c = static_cast<int64_t>(x % static_cast<uint64_t>(p.grid + 1));
      if (la::cta_start(p, c) != c * p.total / p.grid) return 11;
      const int64_t g = static_cast<int64_t>((x >> 20) % static_cast<uint64_t>(p.total));
      const int64_t o = la::cta_of(p, g);
      if (!(la::cta_start(p, o) <= g && g < la::cta_start(p, o + 1))) return 12;
    }
  }
  // Decomposition invariants on assorted problems and SM counts.
  struct Shape { int64_t B, H, T, Hh, W; int32_t bf; };
  const Shape shapes[] = {{1, 32, 21, 45, 80, 0}, {1, 32, 81, 45, 80, 3}, {3, 70, 1, 2, 64, 0},
                          {1, 2, 7, 6, 10, 2}, {2, 1, 3, 5, 30, 10}, {1, 1, 1, 1, 1, 0}, {1, 3, 6, 4, 33, 1}};
  const int sms[] = {1, 7, 148, 1000, 46340, 60000};
  for (const Shape& sh : shapes)
    for (int sm : sms)
      for (int64_t tile : {int64_t(32), int64_t(128)}) {
        la_problem q;
        std::memset(&q, 0, sizeof q);
        q.B = sh.B; q.H = sh.H; q.T = sh.T; q.Hh = sh.Hh; q.W = sh.W; q.d = 128; q.dt = 32; q.dh = 48;
        q.dw = 48; q.rope_base = 10000.0; q.eps = 1e-6f; q.block_frames = sh.bf; q.dtype = LA_BF16;
        const Plan p = build_plan(q, tile, sm, 1);
        int64_t covered = 0;
        for (int64_t c = 0; c < p.grid; ++c) {
          const int64_t a = la::cta_start(p, c), b = la::cta_start(p, c + 1);
          if (b <= a) return 3;                       // every CTA owns at least one tile
          for (int64_t g = a; g < b; ++g) {
            if (la::cta_of(p, g) != c) return 4;      // ownership is consistent
            const la::TileInfo ti = la::tile_info(p, g);
            if (ti.unit - la::unit_of_tile(p, a) >= p.maxseg) return 5;
            if (ti.n0 < 0 || ti.n0 >= ti.n_end || ti.n_end > p.N) return 6;
            // the tile starts on its unit's 'tile' grid
            const int64_t blk = ti.unit % p.nblk;
            if ((ti.n0 - blk * p.blk_tokens) % p.tile != 0) return 7;
            ++covered;
          }
        }
        if (covered != p.total) return 8;
        // Tiles of a unit are contiguous and cover its tokens.
        for (int64_t u = 0; u < p.BH * p.nblk; ++u) {
          int64_t first, count;
          la::unit_tiles(p, u, &first, &count);
          int64_t tok = 0;
          for (int64_t g = first; g < first + count; ++g) {
            const la::TileInfo ti = la::tile_info(p, g);
            if (ti.unit != u) return 9;
            tok += std::min<int64_t>(p.tile, ti.n_end - ti.n0);
          }
          const int64_t blk = u % p.nblk;
          const int64_t len = std::min<int64_t>(p.blk_tokens, p.N - blk * p.blk_tokens);
          if (tok != len) return 10;
        }
      }
  return 0;
}

}  // extern "C"
