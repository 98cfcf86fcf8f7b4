/*
 * qknr.h -- fused per-head QK-RMSNorm + rotate-half RoPE for NVIDIA B200
 * (sm_100a): forward and backward, as a plain C ABI.
 *
 * What it computes. Chronicals (arXiv 2601.02609), abstract, contribution
 * (1), fuses the query/key normalisation with the rotary embedding
 * ("QK-RoPE") so Q and K cross HBM once. For every token and every head of
 * Q (weight gamma_q) and of K (weight gamma_k), with x the head's D values
 * and m the token's position:
 *
 *   r         = 1 / sqrt(mean_d(x_d^2) + eps)       saved as fp32
 *   n_d       = x_d * r * gamma_d
 *   w_i       = theta^(-2i/R),  i < R/2             (R = rotary_dim)
 *   y_i       = n_i cos(m w_i) - n_{i+R/2} sin(m w_i)
 *   y_{i+R/2} = n_{i+R/2} cos(m w_i) + n_i sin(m w_i)
 *   y_d       = n_d                                 for R <= d < D
 *
 * The per-(token, head) inverse RMS is the one statistic kept for the
 * backward ("QK-Normed MLA: QK normalization without full key caching",
 * abstract). Rotating only the first R < D dims is partial RoPE ("Fractional
 * Rotation, Full Potential? Investigating Performance and Convergence of
 * Partial RoPE", abstract); R = 0 leaves plain per-head RMSNorm (the NoPE
 * layers of "Rope to Nope and Back Again: A New Hybrid Attention Strategy",
 * abstract). Optional int32 position ids carry packed sequences whose
 * positions restart per document (Chronicals, abstract, contribution (4)).
 *
 * Layout. Every tensor is dense and row-major (the _strided forms below
 * also take Q and K, and dQ and dK, with a token stride):
 *   q, q_out, dq_out, dq   [B, S, Hq,  D]     k, k_out, dk_out, dk [B, S, Hkv, D]
 *   rstd_q [B, S, Hq] fp32, rstd_k [B, S, Hkv] fp32
 *   gamma_q, gamma_k [D] in the I/O dtype;  dgamma_q, dgamma_k [D] fp32
 *   pos_ids [B, S] int32, or NULL for position = s (restarting every batch row)
 * I/O dtype is fp32 or bf16 for all of q, k, gamma, outputs and gradients;
 * arithmetic is fp32 with fp64 rotary-angle reduction.
 *
 * Pointers and state. All pointers are device pointers (or managed memory)
 * owned by the caller; the library allocates no memory. It does keep a
 * little state: per-device caches of the SM count, the shared-memory limit,
 * kernel occupancy and kernel attributes (filled on first use, thread-safe),
 * and one sticky device flag per kernel family that a kernel sets when it
 * gives up a bounded internal wait (read and cleared by
 * qknr_pipeline_error). Neither affects results, so concurrent calls on
 * different streams are safe. Vector pointers
 * (q, k, gamma, outputs, gradients) must be 16-byte aligned; rstd, dgamma
 * and pos_ids 4-byte aligned. An output may alias its own input exactly
 * (q_out == q, dq == dq_out) for in-place use; any other overlap is rejected.
 * A tensor with zero heads (Hq == 0 or Hkv == 0) may pass NULL for its
 * pointers. B == 0 or S == 0 is an empty problem: nothing is launched except
 * the backward's zeroing of dgamma.
 *
 * Asynchrony and errors. A call validates every argument on the host first;
 * on any failure it returns a non-zero status and enqueues nothing. On
 * success it enqueues its work on `stream` and returns without waiting; a
 * fault during execution surfaces at the caller's next synchronisation, as
 * for any CUDA launch. A launch the runtime refuses returns QKNR_ERR_CUDA.
 *
 * Limits. 2 <= D <= 256 with D * elem_bytes a multiple of 16 (whole 16-byte
 * vectors; with an odd number of them per row the call runs the plain-load
 * kernels); rotary_dim even, 0 <= rotary_dim <= D, and
 * (rotary_dim / 2) * elem_bytes a multiple of 16; theta finite and > 0;
 * eps finite and >= 0. Other shapes return QKNR_ERR_UNSUPPORTED or
 * QKNR_ERR_INVALID_ARG.
 */
#ifndef QKNR_H
#define QKNR_H

#include <stdint.h>

#if defined(__GNUC__)
#define QKNR_API __attribute__((visibility("default")))
#else
#define QKNR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; NULL is the legacy default stream. */
struct CUstream_st;
typedef struct CUstream_st *qknr_stream_t;

typedef enum {
    QKNR_F32 = 0,  /* 4-byte IEEE float I/O */
    QKNR_BF16 = 1  /* 2-byte bfloat16 I/O, outputs rounded to nearest even */
} qknr_dtype;

typedef enum {
    QKNR_OK = 0,
    QKNR_ERR_INVALID_ARG = 1, /* bad size, NULL pointer, overlap, bad theta/eps */
    QKNR_ERR_ALIGNMENT = 2,   /* a pointer is not aligned as stated above */
    QKNR_ERR_UNSUPPORTED = 3, /* a valid shape this build does not handle */
    QKNR_ERR_CUDA = 4         /* the CUDA runtime refused the launch */
} qknr_status;

/*
 * Forward: q_out/k_out = rope(rmsnorm(q|k) * gamma), rstd_q/rstd_k = r.
 * Chronicals (arXiv 2601.02609), abstract, contribution (1).
 *
 *   q, k            inputs, [B,S,Hq,D] / [B,S,Hkv,D], dtype
 *   gamma_q/gamma_k per-dim weights [D], dtype
 *   pos_ids         [B,S] int32 positions, or NULL (position = s)
 *   q_out, k_out    outputs, same shapes as q, k (may equal q, k)
 *   rstd_q, rstd_k  fp32 [B,S,Hq] / [B,S,Hkv] inverse RMS, saved for bwd
 *   B, S, Hq, Hkv, D, rotary_dim, theta, eps   as defined above
 *   dtype           I/O element type
 *   stream          stream to enqueue on
 */
QKNR_API qknr_status qk_norm_rope_fwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             void *q_out, void *k_out,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Backward of qk_norm_rope_fwd. Given the forward's inputs, its saved
 * rstd and the upstream gradients dq_out/dk_out, writes
 *   dq, dk            gradients w.r.t. q and k (may equal dq_out, dk_out)
 *   dgamma_q/dgamma_k fp32 [D] gradients w.r.t. gamma, OVERWRITTEN (the
 *                     call zeroes them on `stream` first, by a small kernel
 *                     of its own); either may be NULL to skip it.
 * Per row, with g the inverse rotation of dy and xh = x * r:
 *   dgamma_d += g_d * xh_d;   h = g * gamma;
 *   dx = r * (h - xh * <h, xh> / D).
 * dgamma is summed with fp32 atomics, one pass per thread block, so its
 * last bits may differ run to run; dq and dk are bitwise reproducible.
 */
QKNR_API qknr_status qk_norm_rope_bwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             void *dq, void *dk,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Strided-input forms, for Q and K read straight out of a fused QKV
 * projection buffer with no copy pass in between (Chronicals, arXiv
 * 2601.02609, abstract, contribution (1): the fused kernels remove memory
 * traffic; reading the projection output in place is this library's reading
 * of that, the pages give no layout). Heads stay contiguous within a token
 * and D contiguous within a head; tokens t = b * S + s are evenly spaced:
 *
 *   row (t, h) of q  starts at  q + t * q_token_stride + h * D   (elements)
 *   row (t, h) of k  starts at  k + t * k_token_stride + h * D
 *
 * e.g. for qkv [B, S, (Hq + 2 Hkv) * D]: q = qkv, k = qkv + Hq * D and both
 * strides (Hq + 2 Hkv) * D. A stride must be >= H * D of its tensor and a
 * whole number of 16 bytes (else QKNR_ERR_INVALID_ARG / QKNR_ERR_ALIGNMENT);
 * H * D elements is the dense layout of qk_norm_rope_fwd / _bwd, which
 * these calls then match exactly.
 *
 * Forward: q_out, k_out, rstd_q, rstd_k are dense as in qk_norm_rope_fwd
 * (the layout attention kernels read). An output may alias its input only
 * when that input is dense.
 */
QKNR_API qknr_status qk_norm_rope_fwd_strided(const void *q, const void *k,
                             int64_t q_token_stride, int64_t k_token_stride,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             void *q_out, void *k_out,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Backward with strided q, k (as in qk_norm_rope_fwd_strided) and strided
 * gradients dq, dk (row (t, h) of dq at dq + t * dq_token_stride + h * D),
 * e.g. written straight into the Q and K slots of a dQKV buffer whose V slot
 * another kernel fills. dq_out, dk_out, rstd and dgamma are dense as in
 * qk_norm_rope_bwd. Strided outputs may share a buffer with each other and
 * with other tensors' slots as long as their bytes do not overlap; dq may
 * alias dq_out (dk, dk_out) only when both are dense.
 */
QKNR_API qknr_status qk_norm_rope_bwd_strided(const void *q, const void *k,
                             int64_t q_token_stride, int64_t k_token_stride,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             void *dq, void *dk,
                             int64_t dq_token_stride, int64_t dk_token_stride,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Mean-centred form (QK-LayerNorm, "Nyonic Technical Report", abstract:
 * rotary embeddings with QK-LayerNorm): per (token, head) row
 *   mu = mean_d x_d,  r = 1 / sqrt(mean_d (x_d - mu)^2 + eps)  (saved fp32)
 *   n_d = (x_d - mu) * r * gamma_d,  then the same rotate-half RoPE,
 * with the learned weight and no bias (the page names no bias). Backward,
 * with g the inverse rotation of dy and xh = (x - mu) r:
 *   dgamma_d += g_d xh_d;  h = g * gamma;
 *   dx = r * (h - mean(h) - xh * mean(h * xh)).
 * The mean is recomputed from x in the backward, so rstd is still the one
 * saved statistic. Arguments, layouts, aliasing and errors exactly as for
 * qk_norm_rope_fwd / qk_norm_rope_bwd.
 */
QKNR_API qknr_status qk_layernorm_rope_fwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             void *q_out, void *k_out,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

QKNR_API qknr_status qk_layernorm_rope_bwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             void *dq, void *dk,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Per-head QK-RMSNorm alone, for the layers that use no positional
 * embedding ("Rope to Nope and Back Again: A New Hybrid Attention Strategy",
 * abstract: NoPE and QK-Norm layers; "Fractional Rotation, Full Potential?",
 * abstract: NoPE stabilised by QK-Norm). The same op as qk_norm_rope_fwd /
 * _bwd with rotary_dim = 0 (no positions, no theta): q_out = q * r * gamma_q,
 * and the backward of it. Arguments, layouts and errors as there.
 */
QKNR_API qknr_status qk_norm_fwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             void *q_out, void *k_out,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv, int D, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

QKNR_API qknr_status qk_norm_bwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             void *dq, void *dk,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv, int D, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * The inverse-RMS statistic alone: rstd = 1 / sqrt(mean_d x_d^2 + eps) for
 * every (token, head) row of q and of k, fp32 [B,S,Hq] / [B,S,Hkv], with no
 * normalised rows written. This is the dynamic half of a split RMSNorm:
 * "QK-Normed MLA: QK normalization without full key caching", abstract,
 * absorbs the static key-side weight into the query projection and keeps
 * one inverse-RMS scalar per token and KV group, computed here from the
 * projected rows (one read of the rows, 4 bytes written per row). Equal bit
 * for bit to the rstd that qk_norm_fwd saves (and qk_norm_rope_fwd when
 * rotary_dim is 0 or D; with a partial span its fp32 sum is taken in another
 * order, within the same D * 2^-24 bound). Either tensor may have zero
 * heads; layouts, alignment and errors as for qk_norm_rope_fwd.
 */
QKNR_API qknr_status qk_rms_stats(const void *q, const void *k,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv, int D, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Rotate-half RoPE alone, no normalisation: q_out = R(m) q, k_out = R(m) k
 * over the first rotary_dim dims (the rest copied), or with inverse != 0
 * the transpose R(m)^T = R(-m), which strips RoPE from rotated rows, e.g.
 * cached keys before a position-free mapping (cross-model KV cache
 * transfer, abstract, on the papers listing the sources include). The
 * gradient of either direction is the other direction applied to the
 * upstream gradient, so there is no separate backward. Positions, layouts,
 * aliasing (q_out may be q) and errors as for qk_norm_rope_fwd; no gamma,
 * no eps, no rstd.
 */
QKNR_API qknr_status qk_rope_apply(const void *q, const void *k,
                             const int32_t *pos_ids,
                             void *q_out, void *k_out,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta, int inverse,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Layerwise QK-RMSNorm + RoPE under tensor parallelism. "SwiftQK: Fast and
 * Communication-Efficient Tensor Parallelism for Query-Key Normalization"
 * (abstract, on the papers listing the sources include): a layerwise
 * QK-norm normalises each token's whole hidden vector (all heads of q, and
 * separately all heads of k), so when the heads are split over ranks only
 * one scalar statistic per token and tensor has to cross GPUs. Each rank
 * holds Hq of the Hq_total query heads and Hkv of the Hkv_total key heads
 * (dense [B,S,Hq,D] / [B,S,Hkv,D] rows) and the matching slices of the
 * learned weights: gamma_q [Hq*D], gamma_k [Hkv*D], the rank's part of the
 * full-hidden gamma. Per token t (T = B*S):
 *
 *   1. qk_layerwise_stats: s_t = sum over the rank's heads and dims of x^2,
 *      fp32 [T] (sumsq_q from q, sumsq_k from k).
 *   2. the caller sums s_t over the ranks (an all-reduce of T fp32 values;
 *      with one rank, nothing), giving S_t.
 *   3. qk_layerwise_norm_rope_fwd: r_t = 1/sqrt(S_t/(H_total*D) + eps),
 *      saved fp32 [T] in rstd_q / rstd_k; out = R(m) (x r_t gamma) on every
 *      head row, the rotate-half rotation of qk_norm_rope_fwd.
 *
 * Backward: with g = R(m)^T dy, hh = g gamma and xh = x r_t,
 *   4. qk_layerwise_bwd_dots: p_t = sum over the rank of hh . xh, fp32 [T].
 *   5. the caller sums p_t over the ranks, giving P_t.
 *   6. qk_layerwise_norm_rope_bwd: dx = r_t (hh - xh P_t/(H_total*D)) and
 *      dgamma[h*D + d] = sum over tokens of g xh (the rank's slice; fp32,
 *      zeroed by the call, may be NULL).
 *
 * One rank holding every head (Hq_total = Hq, Hkv_total = Hkv) may pass
 * NULL for both sumsq pointers of step 3, or both dot pointers of step 6:
 * the call then takes the statistic itself in the same pass (steps 1-2 or
 * 4-5 skipped; the second read of each row comes from on-chip memory or
 * L2, mostly). NULL sums
 * with totals above the local counts are QKNR_ERR_INVALID_ARG.
 *
 * pos_ids as for qk_norm_rope_fwd (NULL: position s of each row). Either
 * tensor may have zero local heads (its pointers are then unused). Rows,
 * gamma, outputs: 16-byte aligned; fp32 vectors: 4-byte aligned. Shapes as
 * for qk_norm_rope_fwd; Hq_total >= Hq, Hkv_total >= Hkv (else
 * QKNR_ERR_INVALID_ARG). The backward keeps the rank's dgamma partial sums
 * in shared memory: (Hq + Hkv) * D * 4 bytes at most 200 KiB, else
 * QKNR_ERR_UNSUPPORTED. No output may overlap an input or another output
 * (QKNR_ERR_INVALID_ARG), except exactly in place: q_out = q, k_out = k,
 * dq = dq_out, dk = dk_out. T = 0 or no heads: nothing launched (the
 * backward still zeroes dgamma).
 */
QKNR_API qknr_status qk_layerwise_stats(const void *q, const void *k,
                             float *sumsq_q, float *sumsq_k,
                             int B, int S, int Hq, int Hkv, int D,
                             qknr_dtype dtype, qknr_stream_t stream);

QKNR_API qknr_status qk_layerwise_norm_rope_fwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *sumsq_q, const float *sumsq_k,
                             void *q_out, void *k_out,
                             float *rstd_q, float *rstd_k,
                             int B, int S, int Hq, int Hkv,
                             int Hq_total, int Hkv_total, int D,
                             int rotary_dim, float theta, float eps,
                             qknr_dtype dtype, qknr_stream_t stream);

QKNR_API qknr_status qk_layerwise_bwd_dots(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             float *dot_q, float *dot_k,
                             int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, float theta,
                             qknr_dtype dtype, qknr_stream_t stream);

QKNR_API qknr_status qk_layerwise_norm_rope_bwd(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             const float *dot_q, const float *dot_k,
                             void *dq, void *dk,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv,
                             int Hq_total, int Hkv_total, int D,
                             int rotary_dim, float theta,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * qk_layerwise_norm_rope_bwd that adds to dgamma_q / dgamma_k instead of
 * overwriting them (no zeroing): for a backward split into token chunks,
 * each chunk's call adds its tokens' share, and the caller zeroes dgamma
 * once before the first. Everything else as qk_layerwise_norm_rope_bwd.
 */
QKNR_API qknr_status qk_layerwise_norm_rope_bwd_acc(const void *q, const void *k,
                             const void *gamma_q, const void *gamma_k,
                             const int32_t *pos_ids,
                             const float *rstd_q, const float *rstd_k,
                             const void *dq_out, const void *dk_out,
                             const float *dot_q, const float *dot_k,
                             void *dq, void *dk,
                             float *dgamma_q, float *dgamma_k,
                             int B, int S, int Hq, int Hkv,
                             int Hq_total, int Hkv_total, int D,
                             int rotary_dim, float theta,
                             qknr_dtype dtype, qknr_stream_t stream);

/*
 * Launch geometry of the layerwise pipelined kernels for a shape, for
 * inspection and host-side checks; no CUDA call is made. mode 0: the dots
 * (qk_layerwise_bwd_dots), 1: the backward (qk_layerwise_norm_rope_bwd),
 * 2: the statistics and the forward (qk_layerwise_stats,
 * qk_layerwise_norm_rope_fwd: one warp per token, so [12] is 1 and [13]
 * the consumer warps, with no dQ_out / dK_out or partial-sum sections);
 * sms: the SM count to plan for. geom (22 int64, caller-owned) receives
 *   [0] 1 if the plan for `sms` SMs is the pipelined kernel, 0 if it is
 *       the plain-load kernel (then the rest is 0); this is the plan the
 *       library follows on a device with `sms` SMs unless the environment
 *       variable QKNR_SIMPLE_KERNELS=1 forces the plain-load kernels,
 *   [1] lanes per head row, [2] tokens per stage, [3] stages,
 *   [4] bytes per stage, [5..9] byte offsets within a stage of the K rows,
 *       dQ_out rows, dK_out rows, (cos, sin) table and per-token scalars,
 *   [10] offset of the per-token partial-sum table and [11] of the gamma
 *       table in the dynamic shared memory,
 *   [12] warps per token, [13] token groups, [14] head blocks,
 *   [15] tokens per CTA, [16] CTAs, [17] dynamic shared memory bytes,
 *   [18] threads per CTA, [19] tokens of each CTA's first tile (the
 *       token pipeline starts on half a tile; the head-block one on [2]),
 *   [20] 1 when the consumer warps fill their own tokens' (cos, sin)
 *       tables (few rows a token), 0 when the producer warp fills them,
 *   [21] offset of the stage's token positions (int32 each).
 * Shapes are checked as for qk_layerwise_norm_rope_bwd (with the totals
 * equal to the local head counts); a bad mode, sms or NULL geom is
 * QKNR_ERR_INVALID_ARG.
 */
QKNR_API qknr_status qk_layerwise_geometry(int mode, int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, qknr_dtype dtype, int sms,
                             int64_t *geom);

/*
 * Launch plan of the per-head entry points for a shape, for inspection and
 * host-side checks (profilers name the kernel by these template values); no
 * CUDA call is made. kind 0: every forward form (qk_norm_rope_fwd and
 * _strided, qk_norm_fwd, qk_rope_apply, qk_rms_stats); 1: the backward
 * (qk_norm_rope_bwd and _strided, qk_norm_bwd); 2 / 3: the mean-centred
 * forward / backward (qk_layernorm_rope_*). strided: bit 0 (1) when q (k)
 * has a token stride other than its dense one. sms: the SM count to plan
 * for; smem_optin: shared memory per block available by opt-in (0: 227 KB,
 * B200's). plan (15 int64, caller-owned) receives
 *   [0] 1 if the plan is the pipelined kernel, 0 if the plain-load kernel
 *       (then only [1], [2], [5] and [13] are set); the library follows it
 *       on a device with these limits unless QKNR_SIMPLE_KERNELS=1,
 *   [1] lanes per head row, [2] units (pairs of 16-byte vectors) per lane,
 *   [3] consumer warps, [4] producer warps, [5] 1 if mean-centred,
 *   [6] tensor-copy mask (bit 0 q, bit 1 k), [7] tokens per tile,
 *   [8] stages in the ring, [9] bytes per stage, [10] tokens per CTA,
 *   [11] CTAs, [12] dynamic shared memory bytes, [13] threads per CTA,
 *   [14] tokens of each CTA's first tile (a forward without tensor copies
 *       starts on half a tile; otherwise [7]).
 * The pipelined kernels are named qknr_fwd_pipe_kernel<T, [1], [2], [3],
 * [4], [5], [6] != 0> and qknr_bwd_pipe_kernel<T, [1], [3], [4], [5],
 * [6] != 0>. Shapes are checked as for the entry points; a bad kind,
 * strided, sms or NULL plan is QKNR_ERR_INVALID_ARG. B * S == 0 or no heads:
 * all zeros.
 */
QKNR_API qknr_status qk_norm_rope_plan(int kind, int B, int S, int Hq, int Hkv, int D,
                             int rotary_dim, qknr_dtype dtype, int strided, int sms,
                             int smem_optin, int64_t *plan);

/* Static English text for a status code; never NULL. */
QKNR_API const char *qknr_strerror(qknr_status status);

/* The CUDA runtime error of the last QKNR_ERR_CUDA on this thread (0 if none). */
QKNR_API int qknr_last_cuda_error(void);

/*
 * Diagnostic of the timeout path: launches on `stream` a one-block kernel in
 * which one thread waits, with the same bounded wait the pipelined kernels
 * of `family` use (0: the per-head kernels, 1: the layerwise kernels), on a
 * shared-memory barrier that nothing completes, for at most limit_cycles SM
 * clock cycles (1 <= limit_cycles <= 2^31; the clock is read every 256th
 * test of the barrier, each test bounded by its suspend hint, so the wait
 * lasts a few milliseconds at least). The wait gives up, sets bit 0 of the
 * flag qknr_pipeline_error reports, and the kernel returns; nothing else is
 * touched and the context stays usable. A bad family or limit is
 * QKNR_ERR_INVALID_ARG; a refused launch QKNR_ERR_CUDA.
 */
QKNR_API qknr_status qknr_wait_selftest(int family, int64_t limit_cycles, qknr_stream_t stream);

/*
 * Diagnostic flag of the current device's pipelined kernels: non-zero if
 * a kernel gave up an internal wait (bounded at 2 s; the results of that
 * launch are then incomplete). Synchronises with the device. With reset
 * != 0 the flag is cleared. Returns -1 if the flag cannot be read.
 */
QKNR_API int qknr_pipeline_error(int reset);

#ifdef __cplusplus
}
#endif

#endif /* QKNR_H */
