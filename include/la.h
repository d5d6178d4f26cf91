/*
 * la.h -- C ABI of the gated ReLU linear-attention token mixer for NVIDIA B200 (sm_100a).
 *
 * The operator, per (batch b, head h), on tokens n of a (T, Hh, W) latent grid:
 *
 *   phi(x) = RoPE3D(ReLU(x))                        (RoPE applied after ReLU)
 *   S      = sum_n phi(K_n)^T V_n                   (d x d state)
 *   z      = sum_n ReLU(K_n)                        (d normaliser, NOT rotated)
 *   O_n    = (phi(Q_n) S) / (ReLU(Q_n) . z + eps) * sigmoid(G_n)
 *
 * Sources: "SANA-Video 2.0: Hybrid Linear Attention with Attention Residuals for
 * Efficient Video Generation", Sec. 2, Eq. (1) (state, normaliser, sigmoid output
 * gate; the write gate beta is 1 and RMSNorm / W_o are outside this operator), and
 * "SANA-Video: Efficient Video Generation with Block Linear Diffusion Transformer",
 * Sec. 3.2 (RoPE after ReLU, un-rotated denominator) and Sec. 3.4 (block-causal
 * constant-memory cache: a block reads the summed states of all earlier blocks plus
 * its own; Algorithm 1 updates the cache once per block).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Q, K, V, G, O are dense, contiguous [B, H, N, d] tensors in device memory, of
 *    the dtype given in la_problem.dtype (bf16 or fp32).  N = T * Hh * W.  Token n of a
 *    head sits at grid position (t, h, w) with n = (t * Hh + h) * W + w.
 *  - 3D RoPE: channels [0, dt) rotate with t, [dt, dt+dh) with h, [dt+dh, d) with w.
 *    Pair i of a band of width D rotates channels (2i, 2i+1) of the band by the angle
 *    pos * rope_base^(-2i/D), counter-clockwise: (x0, x1) -> (x0 c - x1 s, x0 s + x1 c).
 *  - States are fp32: S is [B, H, nblk, d, d] with S[k][v] = sum_n phi(K_n)[k] V_n[v],
 *    z is [B, H, nblk, d].  nblk = 1 in bidirectional mode, ceil(T / block_frames) in
 *    block-causal mode; block j holds latent frames [j*block_frames, (j+1)*block_frames)
 *    (the last block may be shorter).
 *  - Every device pointer must be 16-byte aligned.  Inputs must be finite.
 *  - Ownership: the caller allocates and frees every buffer, including the workspace.
 *    The library never allocates, frees or synchronises; all work is queued on the
 *    given stream, in stream order, and the call returns before it finishes.
 *  - Errors: every entry point returns an la_status.  Invalid arguments are detected
 *    on the host before anything is launched; LA_ERR_CUDA reports a launch failure.
 *    No exception crosses the ABI.  A device-side failure (a bounded wait that ran
 *    out) sets a per-device error word that la_device_error() reads and clears.
 *  - Results are deterministic: the same problem, inputs and device give bitwise the
 *    same outputs (no floating-point atomics; every reduction has a fixed order).
 *  - Concurrent calls on different streams must use different workspaces.
 */
#ifndef LA_H_
#define LA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LA_OK = 0,
  LA_ERR_NULL = 1,        /* a required pointer is NULL */
  LA_ERR_SHAPE = 2,       /* negative / inconsistent sizes, or sizes beyond the limits */
  LA_ERR_BANDS = 3,       /* dt + dh + dw != d, or a band width is odd or negative */
  LA_ERR_ALIGN = 4,       /* a device pointer is not 16-byte aligned */
  LA_ERR_UNSUPPORTED = 5, /* d not in {32, 64, 128}, unknown dtype or flag */
  LA_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than la_workspace_bytes() */
  LA_ERR_CUDA = 7,        /* a CUDA runtime call or kernel launch failed */
  LA_ERR_DEVICE = 8       /* la_device_error(): a kernel reported a device-side failure */
} la_status;

typedef enum { LA_BF16 = 0, LA_F32 = 1 } la_dtype;

/* la_problem.flags */
#define LA_FLAG_FORCE_SIMT 1u   /* use the CUDA-core kernels even where tcgen05 kernels exist */
#define LA_FLAG_TOKEN_CAUSAL 2u /* la_forward_marked: the token-causal operator (block_frames 0) */

typedef struct {
  int64_t B, H;          /* batch and heads */
  int64_t T, Hh, W;      /* latent grid; N = T * Hh * W tokens per head */
  int32_t d;             /* head dimension: 32, 64 or 128 */
  int32_t dt, dh, dw;    /* RoPE band widths along t, h, w; even, dt + dh + dw == d */
  double rope_base;      /* RoPE base (> 0), e.g. 10000 */
  float eps;             /* added to the denominator after the dot product, e.g. 1e-6 */
  int32_t block_frames;  /* 0: bidirectional; > 0: latent frames per causal block */
  int32_t dtype;         /* la_dtype of Q, K, V, G and O */
  uint32_t flags;        /* LA_FLAG_* */
  int64_t t0;            /* global index of latent frame 0 (>= 0): the t band rotates at t0 + t.
                            0 for a whole video; the first frame of the block when a
                            block-autoregressive generator processes one block per call. */
} la_problem;

/* Bytes of device workspace the calls below need for this problem on the CURRENT
 * device (the split of the token range over SMs depends on the device's SM count).
 * Returns 0 for an invalid problem.  One workspace serves every entry point. */
size_t la_workspace_bytes(const la_problem* p);

/* The same for an explicit SM count (pure host computation, no CUDA call). */
size_t la_workspace_bytes_for(const la_problem* p, int sm_count);

/* State reduction (SANA-Video 2.0, Eq. (1), the sum defining S; SANA-Video Sec. 3.4,
 * per-block states): writes S [B,H,nblk,d,d] and z [B,H,nblk,d], fp32.  In block-causal
 * mode these are the states of each block alone (not prefixed).  K, V: [B,H,N,d]. */
int la_state_reduce(const la_problem* p, const void* K, const void* V, float* S, float* z,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Constant-memory cache update for block-autoregressive generation (SANA-Video Sec. 3.4,
 * Algorithm 1: after a block is generated, its keys and values are folded into the cache):
 *   S += sum_n phi(K_n)^T V_n,   z += sum_n ReLU(K_n)   over all N tokens of the call, in place.
 * S: [B,H,d,d], z: [B,H,d], fp32, the carried cache (zeros before the first block).  The call's
 * frames form one block: p->block_frames must be 0; set p->t0 to the block's first global frame
 * so its keys rotate at their global t.  Then la_apply with the same problem and the updated
 * cache gives the block's outputs (a block sees itself and every earlier block), matching
 * la_forward_blockcausal on the whole video up to rounding.  K, V: [B,H,N,d]. */
int la_state_update(const la_problem* p, const void* K, const void* V, float* S, float* z,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* One step of block-autoregressive generation in one call (SANA-Video Sec. 3.4, Algorithm 1):
 * folds the block into the carried cache exactly like la_state_update, then computes the
 * block's outputs against the updated cache exactly like la_apply, with one cos/sin table and
 * one state image for both (4 kernels).  Same arguments and rules as those two calls:
 * p->block_frames == 0, p->t0 = the block's first global frame, S [B,H,d,d] and z [B,H,d]
 * read-modified-written.  Q, K, V, G, O: [B,H,N,d] of the block. */
int la_block_step(const la_problem* p, const void* Q, const void* K, const void* V, const void* G,
                  void* O, float* S, float* z, void* workspace, size_t workspace_bytes,
                  cudaStream_t stream);

/* In-place inclusive prefix over blocks (SANA-Video Sec. 3.4: the cache after block j
 * is the sum of the states of blocks 0..j).  S: [B,H,nblk,d,d], z: [B,H,nblk,d].
 * A no-op in bidirectional mode. */
int la_state_scan(const la_problem* p, float* S, float* z, cudaStream_t stream);

/* Apply (SANA-Video 2.0, Eq. (1) output; SANA-Video Sec. 3.2 numerator/denominator):
 * O_n = (phi(Q_n) S_j) / (ReLU(Q_n) . z_j + eps) * sigmoid(G_n), where j is the block of
 * token n (j = 0 in bidirectional mode) and S, z are the states each block READS, i.e.
 * the inclusive prefixes in block-causal mode.  Q, G, O: [B,H,N,d]. */
int la_apply(const la_problem* p, const void* Q, const void* G, const float* S, const float* z,
             void* O, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Whole bidirectional operator: state reduction then apply.  p->block_frames must be 0. */
int la_forward_bidir(const la_problem* p, const void* Q, const void* K, const void* V,
                     const void* G, void* O, void* workspace, size_t workspace_bytes,
                     cudaStream_t stream);

/* Whole block-causal operator: per-block states, inclusive scan over blocks, apply.
 * p->block_frames must be > 0.  S_incl [B,H,nblk,d,d] and z_incl [B,H,nblk,d] receive the
 * inclusive states (the constant-memory cache after each block) when non-NULL. */
int la_forward_blockcausal(const la_problem* p, const void* Q, const void* K, const void* V,
                           const void* G, void* O, float* S_incl, float* z_incl,
                           void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Token-causal operator (the causal form of SANA-Video Sec. 3.4 taken token by token): token n
 * of a head reads the states of tokens 0..n in the flattened order n = (t*Hh + h)*W + w:
 *   O_n = (phi(Q_n) S_{<=n}) / (ReLU(Q_n) . z_{<=n} + eps) * sigmoid(G_n),
 *   S_{<=n} = sum_{m<=n} phi(K_m)^T V_m,  z_{<=n} = sum_{m<=n} ReLU(K_m).
 * p->block_frames must be 0.  bf16 with d = 128 runs on the tensor cores; fp32, d = 32 / 64 and
 * LA_FLAG_FORCE_SIMT on the CUDA cores (4 kernels either way).  Q, K, V, G, O: [B,H,N,d]. */
int la_forward_tokencausal(const la_problem* p, const void* Q, const void* K, const void* V,
                           const void* G, void* O, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream);

/* Gradients of the bidirectional operator (la_forward_bidir) for training: given the output
 * gradient dO, writes dQ, dK, dV, dG (same layout and dtype as the inputs).  With
 * s = sigmoid(G), y = num / den the pre-gate output and ReLU'(x) = [x > 0]:
 *   dG = dO y s (1 - s),  dnum = dO s / den,  dden = -(dO s . y) / den,
 *   dS = sum_n phi(Q_n)^T dnum_n,  dz = sum_n dden_n ReLU(Q_n),
 *   dQ = [Q > 0] (RoPE^T(dnum S^T) + dden z),  dV = phi(K) dS,  dK = [K > 0] (RoPE^T(V dS^T) + dz)
 * (the chain rule through SANA-Video 2.0, Eq. (1)).  p->block_frames must be 0.  bf16 with
 * d = 128 runs on the tensor cores (6 kernels); fp32, d = 32 / 64 and LA_FLAG_FORCE_SIMT on the
 * CUDA cores.  Recomputes the forward state. */
int la_backward_bidir(const la_problem* p, const void* Q, const void* K, const void* V,
                      const void* G, const void* dO, void* dQ, void* dK, void* dV, void* dG,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Optional terms of the full gated form (SANA-Video 2.0, Sec. 2, Eq. (1)):
 *   S = sum_n beta_n phi(K_n)^T V_n            (write gate; z keeps the un-gated ReLU(K_n):
 *                                               Eq. (1)'s denominator has no beta)
 *   O_n = RMSNorm((phi(Q_n) S) / (ReLU(Q_n) . z + eps)) * sigmoid(G_n)
 *   RMSNorm(y) = y / sqrt(mean_c(y_c^2) + norm_eps) * gamma   (over the d channels of a row)
 * RMSNorm sits before the output gate as in Eq. (1); W_o stays outside the operator. */
typedef struct {
  const void* beta;   /* [B,H,N] write gate per token, in the problem's dtype; NULL: beta = 1 */
  const float* gamma; /* [d] fp32 RMSNorm weight (shared by all heads); NULL: gamma = 1 */
  float norm_eps;     /* RMSNorm epsilon (finite, >= 0), e.g. 1e-6; used when rms_norm = 1 */
  int32_t rms_norm;   /* 1: apply RMSNorm before the gate; 0: no RMSNorm */
} la_gates;

/* The whole operator with the optional terms of la_gates: bidirectional if p->block_frames
 * == 0, else block-causal with the same arguments as la_forward_blockcausal.  S_incl / z_incl
 * (both or neither; fp32, 16-byte aligned) receive, when non-NULL, the states the outputs read:
 * [B,H,d,d] / [B,H,d] bidirectional (each head's state, beta included), [B,H,nblk,d,d] /
 * [B,H,nblk,d] block-causal (each block's inclusive prefix) -- what la_backward_saved takes.
 * gates == NULL, or beta == NULL with rms_norm == 0, computes exactly what la_forward_bidir /
 * la_forward_blockcausal compute.  beta and gamma must be 16-byte aligned when given. */
int la_forward_gated(const la_problem* p, const la_gates* gates, const void* Q, const void* K,
                     const void* V, const void* G, void* O, float* S_incl, float* z_incl,
                     void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Gradients of the operator in every form la_forward_gated computes: bidirectional
 * (p->block_frames == 0) or block-causal, with the optional write gate beta and RMSNorm of
 * `gates` (NULL: none).  Given dO, writes dQ, dK, dV, dG ([B,H,N,d], problem dtype) and
 *   dbeta  [B,H,N] (problem dtype): required when gates->beta is given, else ignored;
 *   dgamma [d] fp32, summed over all tokens and heads: required when gates->rms_norm is set and
 *          gates->gamma is given, else ignored.
 * Chain rule (the reading of SANA-Video 2.0, Eq. (1) and SANA-Video Sec. 3.4): with s = sigmoid(G),
 * y = num / den, u = RMSNorm(y) (u = y without), r = sqrt(mean(y^2) + norm_eps), yh = y / r:
 *   dG = dO u s (1 - s),  du = dO s,  dgamma = sum du yh,
 *   dy = (dyh - yh (yh . dyh) / d) / r with dyh = du gamma   (dy = du without RMSNorm),
 *   dnum = dy / den,  dden = -(dy . y) / den,
 *   dS_b = sum_{n in block b} phi(Q_n)^T dnum_n,  dz_b = sum_{n in block b} dden_n ReLU(Q_n),
 *   dQ = [Q > 0] (RoPE^T(dnum S_b^T) + dden z_b)   (S_b, z_b: the inclusive state token n reads),
 *   and with the suffix sums dS^c = sum_{b >= c} dS_b, dz^c likewise (a key of block c feeds
 *   the states of blocks c and later), for a key of block c:
 *   dV = beta phi(K) dS^c,  dK = [K > 0] (RoPE^T(beta V dS^cT) + dz^c),  dbeta = phi(K) . (dS^c V).
 * bf16 with d = 128 runs on the tensor cores (every form); fp32, d = 32 / 64 and
 * LA_FLAG_FORCE_SIMT on the CUDA cores.  The workspace is la_workspace_bytes(). */
int la_backward(const la_problem* p, const la_gates* gates, const void* Q, const void* K, const void* V,
                const void* G, const void* dO, void* dQ, void* dK, void* dV, void* dG, void* dbeta,
                float* dgamma, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* la_backward given the states the forward pass computed, so that the forward state is not
 * reduced again from K and V (a training step keeps them from its forward: 64 KB per head and
 * block at d = 128).  S [B,H,nblk,d,d] and z [B,H,nblk,d] fp32 (nblk = 1 bidirectional), 16-byte
 * aligned, exactly as la_forward_gated returns them in S_incl / z_incl for the same problem and
 * gates (with beta, the gated state; z is never gated).  Results are those of la_backward up to
 * the rounding of the states the caller passes: with the forward's own states, bit for bit on
 * the tensor cores.  Errors: LA_ERR_NULL if S or z is NULL, LA_ERR_ALIGN if either is not
 * 16-byte aligned; otherwise as la_backward.  Nothing is written to S or z. */
int la_backward_saved(const la_problem* p, const la_gates* gates, const float* S, const float* z,
                      const void* Q, const void* K, const void* V, const void* G, const void* dO, void* dQ,
                      void* dK, void* dV, void* dG, void* dbeta, float* dgamma, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/* The whole operator (bidirectional if p->block_frames == 0, else block-causal, with the
 * same arguments as la_forward_gated; gates may be NULL; token-causal, as la_forward_tokencausal,
 * when p->flags has LA_FLAG_TOKEN_CAUSAL, with gates, S_incl and z_incl NULL) with timing marks: records marks[0]
 * on `stream` before the first kernel and marks[i] right after the i-th kernel it queues, for
 * every i < nmarks.  The events are created and owned by the caller.  Used to time the
 * individual kernels of one forward pass with CUDA events. */
int la_forward_marked(const la_problem* p, const la_gates* gates, const void* Q, const void* K,
                      const void* V, const void* G, void* O, float* S_incl, float* z_incl,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream,
                      cudaEvent_t* marks, int nmarks);

/* Bytes of the library's fixed device scratch used by la_forward_bidir_static(). */
#define LA_STATIC_WORKSPACE_BYTES (32u << 20)

/* la_forward_bidir() for callers that must not allocate device memory themselves: for example
 * a plugin whose host framework owns every device allocation and forbids new ones while it
 * executes, or a latency-critical service that fixes all of its memory at start-up.  This
 * entry point takes no workspace and allocates nothing; it uses a scratch array of
 * LA_STATIC_WORKSPACE_BYTES that is part of the library's device code.  (The pages describe no
 * such call; it exists only for those callers.)
 *  - The caller still passes Q, K, V, G and O (same rules as la_forward_bidir).
 *  - The scratch lives in every GPU that loads the library, until the process exits.
 *  - The first call on a device looks up the scratch's device address (a host-side query that
 *    allocates nothing); make that first call before any stream capture.
 *  - It needs la_workspace_bytes() less the token-causal start states that sit last in that
 *    layout (sm_count x (d*d + d) x 4 bytes on the tensor-core path), which only
 *    la_forward_tokencausal reads.  Problems needing more than LA_STATIC_WORKSPACE_BYTES are
 *    rejected with LA_ERR_WORKSPACE before anything is launched.  The need grows with the SM
 *    count: B = 1, H = 32 at the 720p/5s or 720p/60s latent grid takes about 22 MiB on a
 *    148-SM B200 and fits up to about 200 SMs.
 *  - NULL or misaligned Q, K, V, G, O are reported (LA_ERR_NULL / LA_ERR_ALIGN) before any
 *    CUDA call, as for la_forward_bidir.
 *  - All calls, on any stream, share the one scratch array, which keeps whatever the last call
 *    left in it.  Nothing in it needs clearing (each call writes every byte it later reads),
 *    but calls whose GPU work overlaps in time race on it: serialise them. */
int la_forward_bidir_static(const la_problem* p, const void* Q, const void* K, const void* V,
                            const void* G, void* O, cudaStream_t stream);

/* Static description of a status code. */
const char* la_status_string(int status);

/* Synchronises `stream`, then reads and clears the current device's error word.
 * Returns LA_OK, LA_ERR_DEVICE if a kernel gave up on a bounded wait since the last
 * call, or LA_ERR_CUDA if the synchronisation itself failed. */
int la_device_error(cudaStream_t stream);

/* Number of kernels the last successful entry point on this host thread queued. */
int la_last_launch_count(void);

/* Host-only self-check of the library's work decomposition (no CUDA call): exact 32-bit
 * fast division, and for a set of problem shapes every tile owned by exactly one CTA, every
 * partial-state slot in range, and every unit's tiles covering its tokens.  Returns 0 on
 * success, a positive code naming the failed check otherwise. */
int la_selftest_host(void);

#ifdef __cplusplus
}
#endif

#endif /* LA_H_ */
