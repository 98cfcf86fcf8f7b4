// Layerwise QK-RMSNorm + rotate-half RoPE, shaped for tensor parallelism.
//
// "SwiftQK: Fast and Communication-Efficient Tensor Parallelism for
// Query-Key Normalization" (abstract): under tensor parallelism a layerwise
// QK-norm needs the statistic of each token's whole hidden vector (all heads),
// while each rank holds only a slice of the heads, so only scalar statistics
// have to cross GPUs. Per token t and tensor (Q or K), with the full hidden
// vector spread over ranks as head slices:
//
//   forward:  s_t = sum over this rank's heads and dims of x^2      (stats)
//             S_t = sum over ranks of s_t                            (caller)
//             r_t = 1 / sqrt(S_t / (H_total D) + eps)
//             n[h, d] = x[h, d] r_t gamma[h D + d], rotate each head row
//   backward: p_t = sum over this rank of (g gamma) . (x r_t)        (dots)
//             P_t = sum over ranks of p_t                            (caller)
//             dx = r_t (g gamma - x r_t P_t / (H_total D)),
//             dgamma[h D + d] += g x r_t, g = R^T dy
//
// The exchange itself (an all-reduce of one fp32 per token and tensor) is
// the caller's: NCCL through torch.distributed in the Python binding, token
// chunk by token chunk on a side stream so that each chunk's all-reduce
// overlaps the next chunk's statistics. A rank holding every head passes no
// totals and gets one pass each way.
//
// Three kernel families, all staged through shared memory by bulk copies
// except the last. The token-per-warp pipeline (qknr_lw_tok_kernel) takes
// the statistics and the forward: a warp owns whole tokens, so each
// per-token sum is one warp reduction. The head-block pipeline
// (qknr_lw_pipe_kernel) takes the dots and the backward: a warp owns fixed
// head blocks of a token group, so dgamma is summed in registers, and the
// group's warps meet per token for the sum. Plain-load kernels (one warp
// walks all of a token's local heads with 16-byte loads) take every shape
// neither pipeline fits.
#include "qknr.h"
#include "qknr_kernels.cuh"

#include <cstdint>
#include <cstdlib>

namespace qknr {

qknr_status cuda_fail(cudaError_t e);  // defined beside the per-head entry points
// zeroes two float ranges by one kernel launch (beside the per-head entry points)
qknr_status zero_f32(float *a, int64_t na, float *b, int64_t nb, cudaStream_t st);

namespace {

constexpr int kLwMaxDgammaBytes = 200 * 1024;
constexpr int kLwGeomLen = 22;  // entries qk_layerwise_geometry writes

struct LwArgs {
    const void *q, *k;        // this rank's heads: [T, Hq, D], [T, Hkv, D]
    const void *gq, *gk;      // gamma slices [Hq * D], [Hkv * D]
    const int32_t *pos;       // position ids [T] or NULL (s within the batch row)
    const void *dqo, *dko;    // upstream gradients (backward)
    void *qo, *ko;            // forward outputs, or dq, dk (backward)
    const float *sq, *sk;     // per-token totals over ranks (S_t or P_t)
    float *wq, *wk;           // per-token outputs: partial sums (stats, dots) or rstd (forward)
    const float *rq, *rk;     // saved rstd (backward)
    float *dgq, *dgk;         // dgamma slices (backward), zeroed by the caller
    int64_t T;
    int S, Hq, Hkv, D, R;
    float inv_q, inv_k;       // 1 / (H_total D) of each tensor
    float theta, eps;
    int tpw;                  // tokens per warp
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The warp's token range.
__device__ __forceinline__ void warp_tokens(const LwArgs &a, int64_t *t0, int64_t *t1) {
    const int64_t gw = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    *t0 = gw * a.tpw;
    *t1 = min(*t0 + (int64_t)a.tpw, a.T);
}

// The row (token t, head h of the local Q heads then K heads) a lane reads.
template <typename T>
__device__ __forceinline__ const char *row_of(const void *qb, const void *kb, const LwArgs &a,
                                              int64_t t, int h) {
    const int rowb = a.D * (int)sizeof(T);
    return h < a.Hq ? (const char *)qb + (t * a.Hq + h) * rowb
                    : (const char *)kb + (t * a.Hkv + (h - a.Hq)) * rowb;
}

// Per-token (cos, sin) table of the warp (lanes split the R/2 angles).
__device__ __forceinline__ void token_cs(float2 *cs, const double *s_omega, int half, int64_t pos,
                                         int lane) {
    __syncwarp();
    for (int i = lane; i < half; i += 32) cs[i] = rope_cos_sin(pos, s_omega[i]);
    __syncwarp();
}

// Sums of x^2 over token t's local Q heads (.x) and K heads (.y), the warp
// totals in every lane.
template <typename T, int LPR>
__device__ __forceinline__ float2 token_sumsq(const LwArgs &a, const Lane<LPR, Io<T>::V> &L,
                                              int64_t t) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR;
    const int H = a.Hq + a.Hkv;
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    float sq = 0.f, sk = 0.f;
    for (int p = 0; p < H; p += SLOTS) {
        const int h = p + L.slot;
        if (!(L.on && h < H)) continue;
        const char *row = row_of<T>(a.q, a.k, a, t, h);
        const Vec16 xa = ld16(row + offA), xb = L.onB ? ld16(row + offB) : zero16();
        float s = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < V / 2; ++k2) {
            const float2 va = IO::get2(xa, k2), vb = IO::get2(xb, k2);
            s = fmaf(va.x, va.x, s); s = fmaf(va.y, va.y, s);
            s = fmaf(vb.x, vb.x, s); s = fmaf(vb.y, vb.y, s);
        }
        if (h < a.Hq) sq += s;
        else sk += s;
    }
    return make_float2(warp_sum(sq), warp_sum(sk));
}

// Sums of (g gamma) . (x r) over token t's local Q heads (.x) and K heads
// (.y), g = R(m)^T dy; the warp totals in every lane.
template <typename T, int LPR>
__device__ __forceinline__ float2 token_dots(const LwArgs &a, const Lane<LPR, Io<T>::V> &L,
                                             const float2 *cs, int64_t t, float rq, float rk) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR;
    const int H = a.Hq + a.Hkv, rowb = a.D * (int)sizeof(T);
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    float pq = 0.f, pk = 0.f;
    for (int p = 0; p < H; p += SLOTS) {
        const int h = p + L.slot;
        if (!(L.on && h < H)) continue;
        const bool isq = h < a.Hq;
        const int hh = isq ? h : h - a.Hq;
        const int64_t ri = (isq ? t * a.Hq : t * a.Hkv) + hh;
        const char *row = (const char *)(isq ? a.q : a.k) + ri * rowb;
        const char *drow = (const char *)(isq ? a.dqo : a.dko) + ri * rowb;
        const char *grow = (const char *)(isq ? a.gq : a.gk) + hh * rowb;
        // a half unit (odd vector count) keeps its B vectors at zero
        const Vec16 xa = ld16(row + offA), xb = L.onB ? ld16(row + offB) : zero16();
        const Vec16 da = ld16(drow + offA), db = L.onB ? ld16(drow + offB) : zero16();
        const Vec16 ga = ld16(grow + offA), gb = L.onB ? ld16(grow + offB) : zero16();
        float dot = 0.f;
#pragma unroll
        for (int k2 = 0; k2 < V / 2; ++k2) {
            const float2 va = IO::get2(xa, k2), vb = IO::get2(xb, k2);
            const float2 ea = IO::get2(da, k2), eb = IO::get2(db, k2);
            const float2 wa = IO::get2(ga, k2), wb = IO::get2(gb, k2);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float2 c = lane_cs(cs, L.rot, L.eA + 2 * k2 + q);
                const float dA = q ? ea.y : ea.x, dB = q ? eb.y : eb.x;
                const float gA = fmaf(dA, c.x, dB * c.y), gB = fmaf(dB, c.x, -dA * c.y);
                dot = fmaf(gA * (q ? wa.y : wa.x), q ? va.y : va.x, dot);
                dot = fmaf(gB * (q ? wb.y : wb.x), q ? vb.y : vb.x, dot);
            }
        }
        if (isq) pq = fmaf(dot, rq, pq);
        else pk = fmaf(dot, rk, pk);
    }
    return make_float2(warp_sum(pq), warp_sum(pk));
}

// ---------------------------------------------------------------- stats
template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads) qknr_lw_stats_kernel(const LwArgs a) {
    const Lane<LPR, Io<T>::V> L(threadIdx.x & 31, a.D, a.R);
    int64_t t0, t1;
    warp_tokens(a, &t0, &t1);
    for (int64_t t = t0; t < t1; ++t) {
        const float2 s = token_sumsq<T, LPR>(a, L, t);
        if ((threadIdx.x & 31) == 0) {
            if (a.Hq) a.wq[t] = s.x;
            if (a.Hkv) a.wk[t] = s.y;
        }
    }
}

// -------------------------------------------------------------- forward
// With a.sq == NULL the rank holds every head: the statistic is taken in
// the same pass (the rows are read twice, the second time from cache).
template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads) qknr_lw_fwd_kernel(const LwArgs a) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR;
    __shared__ double s_omega[kMaxHalf];
    __shared__ float2 s_cs[kWarps][kMaxHalf];
    const int half = a.R >> 1;
    for (int i = threadIdx.x; i < half; i += kThreads)
        s_omega[i] = pow((double)a.theta, -2.0 * (double)i / (double)a.R);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Lane<LPR, V> L(lane, a.D, a.R);
    const int H = a.Hq + a.Hkv, rowb = a.D * (int)sizeof(T);
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    const bool local = a.sq == nullptr && a.sk == nullptr;
    // the sums of squares use the layout of qk_layerwise_stats (no rotary
    // span), so both paths add the same terms in the same order
    const Lane<LPR, V> Ls(lane, a.D, 0);
    float2 *cs = s_cs[warp];
    int64_t t0, t1;
    warp_tokens(a, &t0, &t1);
    PosIter pit(a.pos, a.S, t0);
    for (int64_t t = t0; t < t1; ++t) {
        token_cs(cs, s_omega, half, pit.next(t), lane);
        float2 tot;
        if (local) {
            tot = token_sumsq<T, LPR>(a, Ls, t);
        } else {
            tot.x = a.Hq ? a.sq[t] : 0.f;
            tot.y = a.Hkv ? a.sk[t] : 0.f;
        }
        const float rq = a.Hq ? rsqrtf(fmaf(tot.x, a.inv_q, a.eps)) : 0.f;
        const float rk = a.Hkv ? rsqrtf(fmaf(tot.y, a.inv_k, a.eps)) : 0.f;
        if (lane == 0) {
            if (a.Hq) a.wq[t] = rq;
            if (a.Hkv) a.wk[t] = rk;
        }
        for (int p = 0; p < H; p += SLOTS) {
            const int h = p + L.slot;
            if (!(L.on && h < H)) continue;
            const bool isq = h < a.Hq;
            const int hh = isq ? h : h - a.Hq;
            const int64_t ri = (isq ? t * a.Hq : t * a.Hkv) + hh;
            const char *row = (const char *)(isq ? a.q : a.k) + ri * rowb;
            const char *grow = (const char *)(isq ? a.gq : a.gk) + hh * rowb;
            const Vec16 xa = ld16(row + offA), xb = L.onB ? ld16(row + offB) : zero16();
            const Vec16 ga = ld16(grow + offA), gb = L.onB ? ld16(grow + offB) : zero16();
            const float r = isq ? rq : rk;
            Vec16 ya, yb;
#pragma unroll
            for (int k2 = 0; k2 < V / 2; ++k2) {
                const float2 va = IO::get2(xa, k2), vb = IO::get2(xb, k2);
                const float2 wa = IO::get2(ga, k2), wb = IO::get2(gb, k2);
                const int e = 2 * k2;
                const float2 c0 = lane_cs(cs, L.rot, L.eA + e), c1 = lane_cs(cs, L.rot, L.eA + e + 1);
                const float na0 = va.x * wa.x * r, na1 = va.y * wa.y * r;
                const float nb0 = vb.x * wb.x * r, nb1 = vb.y * wb.y * r;
                IO::put2(ya, k2, fmaf(na0, c0.x, -nb0 * c0.y), fmaf(na1, c1.x, -nb1 * c1.y));
                IO::put2(yb, k2, fmaf(nb0, c0.x, na0 * c0.y), fmaf(nb1, c1.x, na1 * c1.y));
            }
            char *out = (char *)(isq ? a.qo : a.ko) + ri * rowb;
            st16(out + offA, ya);
            if (L.onB) st16(out + offB, yb);
        }
    }
}

// ----------------------------------------------------------------- dots
template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads) qknr_lw_dots_kernel(const LwArgs a) {
    __shared__ double s_omega[kMaxHalf];
    __shared__ float2 s_cs[kWarps][kMaxHalf];
    const int half = a.R >> 1;
    for (int i = threadIdx.x; i < half; i += kThreads)
        s_omega[i] = pow((double)a.theta, -2.0 * (double)i / (double)a.R);
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Lane<LPR, Io<T>::V> L(lane, a.D, a.R);
    float2 *cs = s_cs[warp];
    int64_t t0, t1;
    warp_tokens(a, &t0, &t1);
    PosIter pit(a.pos, a.S, t0);
    for (int64_t t = t0; t < t1; ++t) {
        token_cs(cs, s_omega, half, pit.next(t), lane);
        const float rq = a.Hq ? a.rq[t] : 0.f, rk = a.Hkv ? a.rk[t] : 0.f;
        const float2 p = token_dots<T, LPR>(a, L, cs, t, rq, rk);
        if (lane == 0) {
            if (a.Hq) a.wq[t] = p.x;
            if (a.Hkv) a.wk[t] = p.y;
        }
    }
}

// ------------------------------------------------------------- backward
// dx and dgamma from the all-rank dot sums a.sq / a.sk, or, with both NULL
// (the rank holds every head), from the dots taken in the same pass.
template <typename T, int LPR>
__global__ void __launch_bounds__(kThreads) qknr_lw_bwd_kernel(const LwArgs a) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR;
    extern __shared__ float s_dg[];  // (Hq + Hkv) * D dgamma partial sums of the block
    __shared__ double s_omega[kMaxHalf];
    __shared__ float2 s_cs[kWarps][kMaxHalf];
    const int half = a.R >> 1;
    const int H = a.Hq + a.Hkv, rowb = a.D * (int)sizeof(T);
    for (int i = threadIdx.x; i < half; i += kThreads)
        s_omega[i] = pow((double)a.theta, -2.0 * (double)i / (double)a.R);
    for (int i = threadIdx.x; i < H * a.D; i += kThreads) s_dg[i] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Lane<LPR, V> L(lane, a.D, a.R);
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    const bool local = a.sq == nullptr && a.sk == nullptr;
    float2 *cs = s_cs[warp];
    int64_t t0, t1;
    warp_tokens(a, &t0, &t1);
    PosIter pit(a.pos, a.S, t0);
    for (int64_t t = t0; t < t1; ++t) {
        token_cs(cs, s_omega, half, pit.next(t), lane);
        const float rq = a.Hq ? a.rq[t] : 0.f, rk = a.Hkv ? a.rk[t] : 0.f;
        float2 tot;
        if (local) {
            tot = token_dots<T, LPR>(a, L, cs, t, rq, rk);
        } else {
            tot.x = a.Hq ? a.sq[t] : 0.f;
            tot.y = a.Hkv ? a.sk[t] : 0.f;
        }
        // dx = r (hh - (x r) P / (H_total D)): nq, nk are the factors of x
        const float nq = -rq * tot.x * a.inv_q, nk = -rk * tot.y * a.inv_k;
        for (int p = 0; p < H; p += SLOTS) {
            const int h = p + L.slot;
            if (!(L.on && h < H)) continue;
            const bool isq = h < a.Hq;
            const int hh = isq ? h : h - a.Hq;
            const int64_t ri = (isq ? t * a.Hq : t * a.Hkv) + hh;
            const char *row = (const char *)(isq ? a.q : a.k) + ri * rowb;
            const char *drow = (const char *)(isq ? a.dqo : a.dko) + ri * rowb;
            const char *grow = (const char *)(isq ? a.gq : a.gk) + hh * rowb;
            const Vec16 xa = ld16(row + offA), xb = L.onB ? ld16(row + offB) : zero16();
            const Vec16 da = ld16(drow + offA), db = L.onB ? ld16(drow + offB) : zero16();
            const Vec16 ga = ld16(grow + offA), gb = L.onB ? ld16(grow + offB) : zero16();
            const float r = isq ? rq : rk, nd = isq ? nq : nk;
            float *dg = s_dg + (isq ? 0 : a.Hq * a.D) + hh * a.D;
            Vec16 oa, ob;
#pragma unroll
            for (int k2 = 0; k2 < V / 2; ++k2) {
                const float2 va = IO::get2(xa, k2), vb = IO::get2(xb, k2);
                const float2 ea = IO::get2(da, k2), eb = IO::get2(db, k2);
                const float2 wa = IO::get2(ga, k2), wb = IO::get2(gb, k2);
                float outA[2], outB[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int e = 2 * k2 + q;
                    const float2 c = lane_cs(cs, L.rot, L.eA + e);
                    const float dA = q ? ea.y : ea.x, dB = q ? eb.y : eb.x;
                    const float xA = q ? va.y : va.x, xB = q ? vb.y : vb.x;
                    const float gA = fmaf(dA, c.x, dB * c.y), gB = fmaf(dB, c.x, -dA * c.y);
                    const float hA = gA * (q ? wa.y : wa.x), hB = gB * (q ? wb.y : wb.x);
                    outA[q] = r * fmaf(xA, nd, hA);
                    outB[q] = r * fmaf(xB, nd, hB);
                    atomicAdd(dg + L.eA + e, gA * xA * r);
                    if (L.onB) atomicAdd(dg + L.eB + e, gB * xB * r);
                }
                IO::put2(oa, k2, outA[0], outA[1]);
                IO::put2(ob, k2, outB[0], outB[1]);
            }
            char *out = (char *)(isq ? a.qo : a.ko) + ri * rowb;
            st16(out + offA, oa);
            if (L.onB) st16(out + offB, ob);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < H * a.D; i += kThreads) {
        const bool isq = i < a.Hq * a.D;
        float *g = isq ? a.dgq : a.dgk;
        if (g) atomicAdd(g + (isq ? i : i - a.Hq * a.D), s_dg[i]);
    }
}

// ------------------------------------------------------------------------
// Pipelined dots and backward (the statistics and the forward use the
// plain-load kernels above). One producer warp streams stages of TT whole
// tokens (their Q rows, K rows and upstream gradients: each one contiguous
// range) into a shared-memory ring with 1-D bulk copies and fills the
// stage's (cos, sin) table and per-token scalars; G * NTG consumer warps (at
// most kLwCWMax, chosen per shape so that every warp owns the same number of
// head blocks) share each stage. Consumer warp w owns head block set
// {wb + G nb} (a block is the SLOTS rows one warp covers at once) of token
// group tg (tokens tg, tg + NTG, ...), so the rows, gamma elements and
// dgamma sums a lane touches are the same for the whole kernel: dgamma is
// summed in registers, then per CTA in shared memory, and added to global
// memory once per element and CTA. Per-token sums over all heads are
// reduced across the G warps of a token through a small shared table and a
// per-stage barrier, in a fixed order, so the one-pass and the two-phase
// calls add the same terms in the same order.
constexpr int kLwCWMax = 15;                   // consumer warps at most (+1: 16 warps, 128 registers)
constexpr int kLwNBMax = 2;                    // head blocks one consumer warp may own
constexpr int kLwMaxStages = 4;
constexpr int kLwStageTarget = 96 * 1024;
constexpr int kLwRingBytes = 200 * 1024;
constexpr int kMaxTileTokensLw = 32;
constexpr int kLwSmemBytes = 220 * 1024;       // dynamic shared memory at most
constexpr int kLwTokStageTarget = 96 * 1024;   // statistics / forward stage
constexpr long long kLwWaitCycles = 4000000000ll;  // ~2 s per wait at 1.9 GHz

enum LwMode { kLwDots = 0, kLwBwd = 1 };

// Sticky error flag of the pipelined layerwise kernels (bit 0: a wait gave
// up, the launch's results are then incomplete; bit 1: shared memory not
// aligned for bulk copies, nothing computed).
__device__ unsigned int g_lw_error;

struct LwGeom {
    int TT, NS, stage_bytes;
    int off_k, off_dq, off_dk, off_cs;  // sections of a stage (Q rows at 0)
    int off_sc;                         // stage: per-token scalars float4 {rq, rk, sq, sk}
    int off_pos;                        // stage: token positions, int32
    int off_parts;                      // per-token partial sums [NS][TT][G] float2
    int off_gamma;                      // gamma_q then gamma_k rows, I/O dtype
    int G, NTG, HB;                     // warps per token, token groups, head blocks
    int64_t tpc;                        // tokens per CTA
    int cs_by_consumers;                // each warp fills its tokens' (cos, sin) table
};

__device__ __forceinline__ uint32_t lw_smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void lw_bar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void lw_bar_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void lw_bar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool lw_bar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
// Wait for the phase of parity `parity`, for at most `limit` cycles (by
// default kLwWaitCycles); false (with the error flag set) if it never
// completes.
__device__ __forceinline__ bool lw_wait(uint32_t bar, uint32_t parity,
                                        long long limit = kLwWaitCycles) {
    if (lw_bar_test(bar, parity)) return true;
    const long long c0 = clock64();
    uint32_t nap = 32;
#pragma unroll 1
    for (uint32_t n = 1;; ++n) {
        if (lw_bar_test(bar, parity)) return true;
        if (n > 2) {
            __nanosleep(nap);
            nap = nap < 256 ? nap * 2 : 256;
        }
        if ((n & 255u) == 0 && clock64() - c0 > limit) {
            atomicOr(&g_lw_error, 1u);
            return false;
        }
    }
}

// Diagnostic: lw_wait with a limit of `limit` cycles on a barrier nothing
// arrives on (see qknr_wait_selftest_kernel).
__global__ void qknr_lw_wait_selftest_kernel(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = lw_smem_u32(&bar);
    lw_bar_init(b, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    lw_wait(b, 0, limit);
}
// Bulk copy global -> shared (dst, src, bytes multiples of 16), counted in
// bytes on `bar`; the rows are read once, so they may leave L2 first.
__device__ __forceinline__ void lw_bulk(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                        uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t lw_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void lw_st_stream(void *p, const Vec16 &v) {
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
}

__device__ __forceinline__ float2 neg2f(float2 v) { return make_float2(-v.x, -v.y); }

// Token j's sums over all heads: its G per-warp partials added in warp order
// (the same order wherever a total is formed).
__device__ __forceinline__ float2 token_total(const float2 *parts, int j, int G) {
    float2 tot = parts[j * G];
    for (int w2 = 1; w2 < G; ++w2) {
        const float2 p = parts[j * G + w2];
        tot.x += p.x;
        tot.y += p.y;
    }
    return tot;
}

// Shared-memory loads at 32-bit shared addresses (the pipelined consumers
// keep every shared address in 32 bits). Volatile keeps them in order with
// the mbarrier waits and arrivals around them.
__device__ __forceinline__ Vec16 lw_lds16(uint32_t addr) {
    Vec16 r;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3])
                 : "r"(addr));
    return r;
}
__device__ __forceinline__ float4 lw_ldsf4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ float2 lw_ldsf2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}
// Row h of token j in a stage whose Q rows start at q0 and K rows at k0.
__device__ __forceinline__ uint32_t stage_row32(uint32_t q0, uint32_t k0, int j, int h, int Hq,
                                                int Hkv, int rowb) {
    return h < Hq ? q0 + (uint32_t)((j * Hq + h) * rowb) : k0 + (uint32_t)((j * Hkv + (h - Hq)) * rowb);
}
// A lane's (cos, sin) pairs for elements eA .. eA + V - 1 come from its
// token's table: float4 per pair, pair k of unit w at k U + w (U = hp / (V/2)
// rotating units). The byte offsets are fixed for the kernel; lanes past the
// rotary span load none and take (1, 1, 0, 0).
template <int V> struct LwCsOffsets {
    uint32_t o[V / 2];
    template <typename LaneT>
    __device__ __forceinline__ LwCsOffsets(const LaneT &L, int U) {
        const int w = L.eA / V;
#pragma unroll
        for (int k = 0; k < V / 2; ++k) o[k] = (uint32_t)(k * U + w) * 16u;
    }
};
template <int V, typename LaneT>
__device__ __forceinline__ void lane_cs4_32(float4 (&c)[V / 2], uint32_t tok,
                                            const LwCsOffsets<V> &co, const LaneT &L) {
    if (L.rot) {
#pragma unroll
        for (int k = 0; k < V / 2; ++k) c[k] = lw_ldsf4(tok + co.o[k]);
    } else {
#pragma unroll
        for (int k = 0; k < V / 2; ++k) c[k] = make_float4(1.f, 1.f, 0.f, 0.f);
    }
}

// The producer warp's share of a stage's (cos, sin) table: pair P of a token
// (angles 2P, 2P + 1) is one float4 (c_2P, c_2P+1, s_2P, s_2P+1) stored at
// (P mod W) U + P / W (W = V/2 pairs per lane, U = hp / W rotating units), so
// the lanes of a row read consecutive entries. The work split is fixed for
// the kernel: with hp <= 32 pairs lane (jo, P) takes pair P of tokens jo,
// jo + tpp, ... (tpp = 32 / hp tokens per pass); beyond that every lane loops
// over pairs lane + 32 k of every token.
template <int V> struct LwCsWork {
    int hp, tpp, jo, P, dst;
    uint64_t F0, F1;
    __device__ __forceinline__ LwCsWork(const uint64_t *s_step, int half, int lane) {
        hp = half >> 1;
        tpp = (hp > 0 && hp <= 32) ? 32 / hp : 0;
        jo = 0;
        P = -1;
        dst = 0;
        F0 = F1 = 0;
        if (tpp > 0 && lane < tpp * hp) {
            jo = lane / hp;
            P = lane - jo * hp;
            F0 = s_step[2 * P];
            F1 = s_step[2 * P + 1];
            const int pw = P / (V / 2);
            dst = (P - pw * (V / 2)) * (hp / (V / 2)) + pw;
        }
    }
    // table of na tokens whose positions are s_pos[0..na)
    __device__ __forceinline__ void fill(float4 *cs, const int32_t *s_pos, const uint64_t *s_step,
                                         int na, int lane) const {
        if (tpp > 0) {
            if (P >= 0)
                for (int j = jo; j < na; j += tpp) {
                    const int32_t m = s_pos[j];
                    const float2 c0 = rope_cos_sin_fixed(m, F0);
                    const float2 c1 = rope_cos_sin_fixed(m, F1);
                    cs[j * hp + dst] = make_float4(c0.x, c1.x, c0.y, c1.y);
                }
        } else {
            for (int q = lane; q < hp; q += 32) {
                const uint64_t G0 = s_step[2 * q], G1 = s_step[2 * q + 1];
                const int pw = q / (V / 2);
                const int d = (q - pw * (V / 2)) * (hp / (V / 2)) + pw;
                for (int j = 0; j < na; ++j) {
                    const int32_t m = s_pos[j];
                    const float2 c0 = rope_cos_sin_fixed(m, G0);
                    const float2 c1 = rope_cos_sin_fixed(m, G1);
                    cs[j * hp + d] = make_float4(c0.x, c1.x, c0.y, c1.y);
                }
            }
        }
    }
};

template <typename T, int LPR, int MODE, int NBM>
__global__ void __launch_bounds__((kLwCWMax + 1) * 32, 1)
    qknr_lw_pipe_kernel(const LwArgs a, const LwGeom g) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR, E = (int)sizeof(T);
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t s_step[kMaxHalf];      // fixed-point angle step per rotary pair
    __shared__ int32_t s_pos[kMaxTileTokensLw];  // producer: positions of the stage's tokens
    const int half = a.R >> 1;
    const int nthr = blockDim.x, ncw = g.G * g.NTG;  // consumer warps; the producer is warp ncw
    for (int i = threadIdx.x; i < half; i += nthr) s_step[i] = turn_step(i, a.R, a.theta);
    const uint32_t bar0 = lw_smem_u32(smem);  // full[NS], empty[NS], parts[NS]
    if (bar0 & 127u) {  // bulk copies need 16-byte aligned stages: compute nothing
        if (threadIdx.x == 0) atomicOr(&g_lw_error, 2u);
        return;
    }
    __shared__ int s_abort;  // a consumer warp gave up a wait: skip the dgamma phase
    __shared__ __align__(8) uint64_t s_tgbar[kLwCWMax];  // one per token group: its warps' partials are in
    unsigned char *ring = smem + 128;
    float2 *parts_all = reinterpret_cast<float2 *>(smem + g.off_parts);
    if (threadIdx.x == 0) s_abort = 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t_lo = (int64_t)blockIdx.x * g.tpc;
    const int64_t t_hi = min(a.T, t_lo + g.tpc);
    const int ntiles = t_hi > t_lo ? (int)((t_hi - t_lo + g.TT - 1) / g.TT) : 0;
    const int H = a.Hq + a.Hkv, rowb = a.D * E;
    unsigned char *s_gamma = smem + g.off_gamma;  // every CTA reads the weights once
    if (threadIdx.x == 0) {
        for (int s = 0; s < g.NS; ++s) {
            lw_bar_init(bar0 + 8 * s, 32);                   // the producer warp's lanes
            lw_bar_init(bar0 + 8 * (g.NS + s), ncw);       // one per consumer warp
        }
        for (int t = 0; t < g.NTG; ++t) lw_bar_init(lw_smem_u32(&s_tgbar[t]), g.G);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    grid_dep_wait();  // no global memory is touched above this line
    grid_dep_launch();
    {
        const int nq = a.Hq * rowb / 16, nk = a.Hkv * rowb / 16;
        for (int i = threadIdx.x; i < nq + nk; i += nthr) {
            const Vec16 v = i < nq ? ld16((const char *)a.gq + 16 * i)
                                   : ld16((const char *)a.gk + 16 * (i - nq));
            st16(s_gamma + 16 * i, v);
        }
    }
    __syncthreads();

    if (warp == ncw) {
        // ---------------------------------------------------------- producer
        const uint64_t pol = lw_evict_first();
        const bool totals = MODE == kLwBwd && !(a.sq == nullptr && a.sk == nullptr);
        const bool need_cs = half > 0;
        int s_cur = (int)(t_lo % a.S);  // row position of the tile's first token
        const LwCsWork<V> csw(s_step, half, lane);
        int issued = 0;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % g.NS;
            const uint32_t ph = (uint32_t)(i / g.NS) & 1u;
            const int64_t t0 = t_lo + (int64_t)i * g.TT;
            const int na = (int)min((int64_t)g.TT, t_hi - t0);
            // this stage's per-token values, loaded before the wait for the
            // slot so that their latency overlaps it: saved rstd, all-rank
            // totals (second phase of a sharded call), positions
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            int32_t pos = 0;
            if (lane < na) {
                const int64_t t = t0 + lane;
                v.x = a.Hq ? a.rq[t] : 0.f;
                v.y = a.Hkv ? a.rk[t] : 0.f;
                if (totals) {
                    v.z = a.Hq ? a.sq[t] : 0.f;
                    v.w = a.Hkv ? a.sk[t] : 0.f;
                }
                if (need_cs) {
                    if (a.pos) {
                        pos = a.pos[t];
                    } else {
                        int p = s_cur + lane;
                        while (p >= a.S) p -= a.S;
                        pos = p;
                    }
                }
            }
            s_cur += g.TT;
            while (s_cur >= a.S) s_cur -= a.S;
            if (i >= g.NS && !lw_wait(bar0 + 8 * (g.NS + s), ph ^ 1u)) break;
            unsigned char *st = ring + (size_t)s * g.stage_bytes;
            const uint32_t full = bar0 + 8 * s;
            if (lane == 0) {
                const uint32_t bq = (uint32_t)(na * a.Hq * rowb);
                const uint32_t bk = (uint32_t)(na * a.Hkv * rowb);
                lw_bar_expect(full, 2u * (bq + bk));
                if (bq) lw_bulk(lw_smem_u32(st), (const char *)a.q + t0 * a.Hq * rowb, bq, full, pol);
                if (bk)
                    lw_bulk(lw_smem_u32(st + g.off_k), (const char *)a.k + t0 * a.Hkv * rowb, bk,
                            full, pol);
                if (bq)
                    lw_bulk(lw_smem_u32(st + g.off_dq), (const char *)a.dqo + t0 * a.Hq * rowb, bq,
                            full, pol);
                if (bk)
                    lw_bulk(lw_smem_u32(st + g.off_dk), (const char *)a.dko + t0 * a.Hkv * rowb, bk,
                            full, pol);
            }
            if (lane < na) reinterpret_cast<float4 *>(st + g.off_sc)[lane] = v;
            if (need_cs && g.cs_by_consumers) {
                if (lane < na) reinterpret_cast<int32_t *>(st + g.off_pos)[lane] = pos;
            } else if (need_cs) {
                if (lane < na) s_pos[lane] = pos;
                __syncwarp();
                csw.fill(reinterpret_cast<float4 *>(st + g.off_cs), s_pos, s_step, na, lane);
                __syncwarp();
            }
            lw_bar_arrive(full);
            ++issued;
        }
        // leave only once every copy issued has landed
        for (int i = max(0, issued - g.NS); i < issued; ++i)
            if (!lw_wait(bar0 + 8 * (i % g.NS), (uint32_t)(i / g.NS) & 1u)) break;
        return;
    }

    // -------------------------------------------------------------- consumers
    // Token group tg (warps tg G .. tg G + G - 1) takes tokens tg, tg + NTG,
    // ... of every stage, UA at a time; warp wb of the group owns head blocks
    // wb, wb + G (at most NBM), so each lane keeps the same rows, elements
    // and dgamma sums for the whole kernel. Per round a warp un-rotates dy,
    // forms hh = g gamma and xh = x r, adds g xh to its dgamma sums and keeps
    // hh, xh in registers; when the per-token sums come from this pass, the
    // group's G warps post their partials and meet on the group's mbarrier,
    // every warp adds the G partials in warp order, and then finishes dx
    // from the registers (no second pass over the rows).
    const int tg = warp / g.G, wb = warp % g.G;
    const Lane<LPR, V> L(lane, a.D, a.R);
    const uint32_t offA = (uint32_t)(L.eA * E), offB = (uint32_t)(L.eB * E);
    const int hp = half >> 1;  // rotary pairs per token
    const LwCsOffsets<V> co(L, hp / (V / 2));
    const uint32_t ring32 = lw_smem_u32(ring), gam32 = lw_smem_u32(s_gamma);
    const bool local = MODE == kLwBwd && a.sq == nullptr && a.sk == nullptr;
    const bool need_parts = MODE == kLwDots || local;
    constexpr int UA = NBM == 1 ? 2 : 1;  // tokens per round
    const uint32_t tgbar = lw_smem_u32(&s_tgbar[tg]);
    uint32_t tg_phase = 0;
    float2 acc[NBM][V];  // dgamma sums: pairs of the A vector, then of the B vector
#pragma unroll
    for (int nb = 0; nb < NBM; ++nb)
#pragma unroll
        for (int k = 0; k < V; ++k) acc[nb][k] = make_float2(0.f, 0.f);
    bool aborted = false;

    for (int i = 0; i < ntiles && !aborted; ++i) {
        const int s = i % g.NS;
        const uint32_t ph = (uint32_t)(i / g.NS) & 1u;
        if (!lw_wait(bar0 + 8 * s, ph)) {
            aborted = true;
            break;
        }
        const int64_t t0 = t_lo + (int64_t)i * g.TT;
        const int na = (int)min((int64_t)g.TT, t_hi - t0);
        const uint32_t st = ring32 + (uint32_t)(s * g.stage_bytes);
        const uint32_t xq = st, xk = st + (uint32_t)g.off_k;
        const uint32_t dq0 = st + (uint32_t)g.off_dq, dk0 = st + (uint32_t)g.off_dk;
        const uint32_t cs_st = st + (uint32_t)g.off_cs, sc = st + (uint32_t)g.off_sc;
        float2 *parts = parts_all + (size_t)s * g.TT * g.G;

        for (int j0 = tg; j0 < na; j0 += UA * g.NTG) {
            float2 hh[UA][NBM][V], xh[UA][NBM][V];  // pairs of A, then of B
            float vq[UA], vk[UA];
#pragma unroll
            for (int u = 0; u < UA; ++u) {
                const int j = j0 + u * g.NTG;
                vq[u] = vk[u] = 0.f;
                const bool tok_ok = j < na;
                float4 c[V / 2];
                const int jt = tok_ok ? j : j0;
                if (NBM == 1 && half > 0 && g.cs_by_consumers && tok_ok) {
                    // every warp of the token's group fills the whole table
                    // before reading it (the same values, so the group's
                    // concurrent fills of one entry agree); planned only for
                    // one head block a warp, the register-lighter instance
                    const unsigned char *stg = ring + (size_t)s * g.stage_bytes;
                    const int32_t m = reinterpret_cast<const int32_t *>(stg + g.off_pos)[j];
                    float4 *tab = reinterpret_cast<float4 *>(ring + (size_t)s * g.stage_bytes +
                                                             g.off_cs) + j * hp;
                    for (int P = lane; P < hp; P += 32) {
                        const int pw = P / (V / 2);
                        const int dst = (P - pw * (V / 2)) * (hp / (V / 2)) + pw;
                        const float2 c0 = rope_cos_sin_fixed(m, s_step[2 * P]);
                        const float2 c1 = rope_cos_sin_fixed(m, s_step[2 * P + 1]);
                        tab[dst] = make_float4(c0.x, c1.x, c0.y, c1.y);
                    }
                    __syncwarp();
                }
                lane_cs4_32<V>(c, cs_st + (uint32_t)(jt * hp * 16), co, L);
                const float4 sv = lw_ldsf4(sc + (uint32_t)(jt * 16));
#pragma unroll
                for (int nb = 0; nb < NBM; ++nb) {
                    const int b = wb + nb * g.G;
                    const int h = b * SLOTS + L.slot;
                    const bool on = tok_ok && b < g.HB && L.on && h < H;
                    const bool isq = h < a.Hq;
                    const int hs = on ? h : 0;
                    const uint32_t row = stage_row32(xq, xk, on ? j : 0, hs, a.Hq, a.Hkv, rowb);
                    const uint32_t drow = stage_row32(dq0, dk0, on ? j : 0, hs, a.Hq, a.Hkv, rowb);
                    const uint32_t grow = gam32 + (uint32_t)(hs * rowb);
                    const Vec16 xa = lw_lds16(row + offA), xb = lw_lds16(row + offB);
                    const Vec16 da = lw_lds16(drow + offA), db = lw_lds16(drow + offB);
                    const Vec16 ga = lw_lds16(grow + offA), gb = lw_lds16(grow + offB);
                    const float r = on ? (isq ? sv.x : sv.y) : 0.f;  // off rows add nothing
                    const float2 r2 = make_float2(r, r);
                    float2 p2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int k2 = 0; k2 < V / 2; ++k2) {
                        const float2 c2 = make_float2(c[k2].x, c[k2].y);
                        const float2 s2 = make_float2(c[k2].z, c[k2].w);
                        const float2 ea = IO::get2(da, k2), eb = IO::get2(db, k2);
                        const float2 gA = __ffma2_rn(ea, c2, __fmul2_rn(eb, s2));
                        const float2 gB = __ffma2_rn(eb, c2, __fmul2_rn(ea, neg2f(s2)));
                        const float2 hA = __fmul2_rn(gA, IO::get2(ga, k2));
                        const float2 hB = __fmul2_rn(gB, IO::get2(gb, k2));
                        const float2 xA = __fmul2_rn(IO::get2(xa, k2), r2);
                        const float2 xB = __fmul2_rn(IO::get2(xb, k2), r2);
                        p2 = __ffma2_rn(hA, xA, p2);
                        p2 = __ffma2_rn(hB, xB, p2);
                        hh[u][nb][k2] = hA;
                        hh[u][nb][V / 2 + k2] = hB;
                        xh[u][nb][k2] = xA;
                        xh[u][nb][V / 2 + k2] = xB;
                        if (MODE == kLwBwd) {
                            acc[nb][k2] = __ffma2_rn(gA, xA, acc[nb][k2]);
                            acc[nb][V / 2 + k2] = __ffma2_rn(gB, xB, acc[nb][V / 2 + k2]);
                        }
                    }
                    const float pr = p2.x + p2.y;
                    vq[u] += isq ? pr : 0.f;
                    vk[u] += isq ? 0.f : pr;
                }
            }
            float2 tot[UA];
            if (need_parts) {
#pragma unroll
                for (int o = 16; o; o >>= 1)
#pragma unroll
                    for (int u = 0; u < UA; ++u) {
                        vq[u] += __shfl_xor_sync(0xffffffffu, vq[u], o);
                        vk[u] += __shfl_xor_sync(0xffffffffu, vk[u], o);
                    }
                if (lane == 0) {
#pragma unroll
                    for (int u = 0; u < UA; ++u) {
                        const int j = j0 + u * g.NTG;
                        if (j < na) parts[j * g.G + wb] = make_float2(vq[u], vk[u]);
                    }
                }
                // the group's G warps meet: every partial of these tokens is in
                __syncwarp();
                if (lane == 0) lw_bar_arrive(tgbar);
                if (!lw_wait(tgbar, tg_phase)) {
                    aborted = true;
                    break;
                }
                tg_phase ^= 1u;
#pragma unroll
                for (int u = 0; u < UA; ++u) {
                    const int j = j0 + u * g.NTG;
                    tot[u] = j < na ? token_total(parts, j, g.G) : make_float2(0.f, 0.f);
                }
                if (MODE == kLwDots) {
                    if (wb == 0 && lane == 0) {
#pragma unroll
                        for (int u = 0; u < UA; ++u) {
                            const int j = j0 + u * g.NTG;
                            if (j >= na) continue;
                            if (a.Hq) a.wq[t0 + j] = tot[u].x;
                            if (a.Hkv) a.wk[t0 + j] = tot[u].y;
                        }
                    }
                    continue;
                }
            } else {
#pragma unroll
                for (int u = 0; u < UA; ++u) {
                    const int j = j0 + u * g.NTG;
                    const float4 sv = lw_ldsf4(sc + (uint32_t)((j < na ? j : j0) * 16));
                    tot[u] = make_float2(sv.z, sv.w);
                }
            }
            if (MODE == kLwBwd) {
                // dx = r (hh - xh P / (H_total D)) from the registers
#pragma unroll
                for (int u = 0; u < UA; ++u) {
                    const int j = j0 + u * g.NTG;
                    if (j >= na) continue;
                    const int64_t t = t0 + j;
                    const float4 sv = lw_ldsf4(sc + (uint32_t)(j * 16));
                    const float nq = -tot[u].x * a.inv_q, nk = -tot[u].y * a.inv_k;
#pragma unroll
                    for (int nb = 0; nb < NBM; ++nb) {
                        const int b = wb + nb * g.G;
                        const int h = b * SLOTS + L.slot;
                        if (!(b < g.HB && L.on && h < H)) continue;
                        const bool isq = h < a.Hq;
                        const int hh_ = isq ? h : h - a.Hq;
                        const float r = isq ? sv.x : sv.y, nd = isq ? nq : nk;
                        const float2 r2 = make_float2(r, r), nd2 = make_float2(nd, nd);
                        Vec16 oa, ob;
#pragma unroll
                        for (int k2 = 0; k2 < V / 2; ++k2) {
                            const float2 oA = __fmul2_rn(r2, __ffma2_rn(xh[u][nb][k2], nd2, hh[u][nb][k2]));
                            const float2 oB = __fmul2_rn(
                                r2, __ffma2_rn(xh[u][nb][V / 2 + k2], nd2, hh[u][nb][V / 2 + k2]));
                            IO::put2(oa, k2, oA.x, oA.y);
                            IO::put2(ob, k2, oB.x, oB.y);
                        }
                        char *out = (char *)(isq ? a.qo : a.ko) +
                                    ((isq ? t * a.Hq : t * a.Hkv) + hh_) * rowb;
                        lw_st_stream(out + offA, oa);
                        lw_st_stream(out + offB, ob);
                    }
                }
            }
        }
        if (aborted) break;
        __syncwarp();
        if (lane == 0) lw_bar_arrive(bar0 + 8 * (g.NS + s));
    }
    if (aborted) s_abort = 1;

    if (MODE == kLwBwd) {
        // dgamma: the token groups of this CTA own the same elements, so sum
        // them in shared memory (the ring, free now) first, then one global
        // atomic add per element and CTA. After a consumer gave up a wait the
        // ring may still be receiving copies, so the phase is skipped (the
        // launch's results are incomplete then, and the error flag says so).
        float *s_red = reinterpret_cast<float *>(ring);
        const int nel = H * a.D, ct = ncw * 32;
        asm volatile("bar.sync 1, %0;" ::"r"(ct) : "memory");
        if (s_abort) return;
        for (int e = threadIdx.x; e < nel; e += ct) s_red[e] = 0.f;
        asm volatile("bar.sync 1, %0;" ::"r"(ct) : "memory");
        // the B vector of a rotary pair is e + R/2 elements on; the
        // geometry's element offsets say where each pair sum belongs
#pragma unroll
        for (int nb = 0; nb < NBM; ++nb) {
            const int b = wb + nb * g.G;
            if (b >= g.HB) break;
            const int h = b * SLOTS + L.slot;
            if (!(L.on && h < H)) continue;
            float *dg = s_red + h * a.D;
#pragma unroll
            for (int k2 = 0; k2 < V / 2; ++k2) {
                atomicAdd(dg + L.eA + 2 * k2, acc[nb][k2].x);
                atomicAdd(dg + L.eA + 2 * k2 + 1, acc[nb][k2].y);
                atomicAdd(dg + L.eB + 2 * k2, acc[nb][V / 2 + k2].x);
                atomicAdd(dg + L.eB + 2 * k2 + 1, acc[nb][V / 2 + k2].y);
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(ct) : "memory");
        const int nq = a.Hq * a.D;
        for (int e = threadIdx.x; e < nel; e += ct) {
            float *dg = e < nq ? a.dgq + e : a.dgk + (e - nq);
            if ((e < nq ? a.dgq : a.dgk) != nullptr) atomicAdd(dg, s_red[e]);
        }
    }
}

// ------------------------------------------------------------------------
// Pipelined statistics and forward. One producer warp streams stages of TT
// whole tokens (a CTA's first stage holds half as many; a stage's Q rows and
// K rows are two contiguous ranges) into the ring with bulk copies and writes the stage's per-token totals (second
// phase of a sharded call) and (cos, sin) table. Each consumer warp takes
// whole tokens, dealt round-robin and continuing across stages: it sums x^2
// over the token's rows in shared memory (one warp reduction per tensor, no
// cross-warp exchange), then normalises, rotates and stores every row of the
// token. Every row crosses HBM once. The statistics and the one-pass forward
// run the same summation, so the two-phase and one-pass results agree bit
// for bit.
enum LwTokMode { kTokStats = 0, kTokFwd = 1 };

struct LwTokGeom {
    int TT, NS, stage_bytes;
    int off_k, off_cs, off_sc;  // sections of a stage (Q rows at 0); scalars float2 {sq, sk}
    int off_pos;                // the stage's token positions, int32
    int off_gamma;              // gamma_q then gamma_k rows, I/O dtype
    int ncw;                    // consumer warps
    int64_t tpc;                // tokens per CTA
    int h0;                     // tokens of a CTA's first tile when shorter than TT (0: TT)
    int cs_by_consumers;        // each consumer warp fills its tokens' (cos, sin) table
};

// A CTA's tiles: the first holds h (a shorter first tile lets the consumers
// start before a whole stage has landed), every later one TT, the last what
// remains.
struct LwTiles {
    int64_t t_lo, t_hi;
    int TT, h, n;
    __device__ __forceinline__ LwTiles(int64_t lo, int64_t hi, int tt, int h0)
        : t_lo(lo), t_hi(hi), TT(tt) {
        const int64_t len = hi - lo;
        h = (h0 > 0 && len > tt) ? h0 : tt;
        n = len > 0 ? (len <= h ? 1 : 1 + (int)((len - h + tt - 1) / tt)) : 0;
    }
    __device__ __forceinline__ int64_t start(int i) const {
        return i == 0 ? t_lo : t_lo + h + (int64_t)(i - 1) * TT;
    }
    __device__ __forceinline__ int count(int i) const {
        return (int)min((int64_t)(i == 0 ? h : TT), t_hi - start(i));
    }
};

// Sums of x^2 over the rows of one token held in shared memory (Q rows at
// xq, K rows at xk), the warp totals in every lane.
template <typename T, int LPR>
__device__ __forceinline__ float2 tok_sumsq(uint32_t xq, uint32_t xk,
                                            const Lane<LPR, Io<T>::V> &L, int Hq, int H,
                                            int rowb, uint32_t offA, uint32_t offB) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR;
    float2 pq = make_float2(0.f, 0.f), pk = make_float2(0.f, 0.f);
    for (int p = 0; p < H; p += SLOTS) {
        const int h = p + L.slot;
        if (!(L.on && h < H)) continue;
        const bool isq = h < Hq;
        const uint32_t row = isq ? xq + (uint32_t)(h * rowb) : xk + (uint32_t)((h - Hq) * rowb);
        const Vec16 xa = lw_lds16(row + offA), xb = lw_lds16(row + offB);
        float2 s0 = make_float2(0.f, 0.f);
#pragma unroll
        for (int k2 = 0; k2 < V / 2; ++k2) {
            const float2 va = IO::get2(xa, k2), vb = IO::get2(xb, k2);
            s0 = __ffma2_rn(va, va, s0);
            s0 = __ffma2_rn(vb, vb, s0);
        }
        if (isq) pq = __fadd2_rn(pq, s0);
        else pk = __fadd2_rn(pk, s0);
    }
    float q = pq.x + pq.y, k = pk.x + pk.y;
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        q += __shfl_xor_sync(0xffffffffu, q, o);
        k += __shfl_xor_sync(0xffffffffu, k, o);
    }
    return make_float2(q, k);
}

template <typename T, int LPR, int MODE>
__global__ void __launch_bounds__((kLwCWMax + 1) * 32, 1)
    qknr_lw_tok_kernel(const LwArgs a, const LwTokGeom g) {
    using IO = Io<T>;
    constexpr int V = IO::V, SLOTS = 32 / LPR, E = (int)sizeof(T);
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ uint64_t s_step[kMaxHalf];        // fixed-point angle step per rotary pair
    __shared__ int32_t s_pos[kMaxTileTokensLw];  // producer: positions of the stage's tokens
    const int half = MODE == kTokFwd ? a.R >> 1 : 0;
    const int nthr = blockDim.x, ncw = g.ncw;  // the producer is warp ncw
    for (int i = threadIdx.x; i < half; i += nthr) s_step[i] = turn_step(i, a.R, a.theta);
    const uint32_t bar0 = lw_smem_u32(smem);  // full[NS], empty[NS]
    if (bar0 & 127u) {  // bulk copies need 16-byte aligned stages: compute nothing
        if (threadIdx.x == 0) atomicOr(&g_lw_error, 2u);
        return;
    }
    unsigned char *ring = smem + 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t_lo = (int64_t)blockIdx.x * g.tpc;
    const int64_t t_hi = min(a.T, t_lo + g.tpc);
    const LwTiles tiles(t_lo, t_hi, g.TT, g.h0);
    const int ntiles = tiles.n;
    const int H = a.Hq + a.Hkv, rowb = a.D * E;
    const unsigned char *s_gamma = smem + g.off_gamma;
    if (threadIdx.x == 0) {
        for (int s = 0; s < g.NS; ++s) {
            lw_bar_init(bar0 + 8 * s, 32);              // the producer warp's lanes
            lw_bar_init(bar0 + 8 * (g.NS + s), ncw);    // one per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    grid_dep_wait();  // no global memory is touched above this line
    grid_dep_launch();
    if (MODE == kTokFwd) {  // every CTA reads the weights once
        const int nq = a.Hq * rowb / 16, nk = a.Hkv * rowb / 16;
        for (int i = threadIdx.x; i < nq + nk; i += nthr) {
            const Vec16 v = i < nq ? ld16((const char *)a.gq + 16 * i)
                                   : ld16((const char *)a.gk + 16 * (i - nq));
            st16(smem + g.off_gamma + 16 * i, v);
        }
    }
    __syncthreads();
    const bool local = a.sq == nullptr && a.sk == nullptr;

    if (warp == ncw) {
        // ---------------------------------------------------------- producer
        const uint64_t pol = lw_evict_first();
        const bool totals = MODE == kTokFwd && !local;
        int s_cur = (int)(t_lo % a.S);  // row position of the tile's first token
        const LwCsWork<V> csw(s_step, half, lane);
        int issued = 0;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i % g.NS;
            const uint32_t ph = (uint32_t)(i / g.NS) & 1u;
            const int64_t t0 = tiles.start(i);
            const int na = tiles.count(i);
            // per-token values, loaded before the wait for the slot
            float2 v = make_float2(0.f, 0.f);
            int32_t pos = 0;
            if (lane < na) {
                const int64_t t = t0 + lane;
                if (totals) {
                    v.x = a.Hq ? a.sq[t] : 0.f;
                    v.y = a.Hkv ? a.sk[t] : 0.f;
                }
                if (half > 0) {
                    if (a.pos) {
                        pos = a.pos[t];
                    } else {
                        int p = s_cur + lane;
                        while (p >= a.S) p -= a.S;
                        pos = p;
                    }
                }
            }
            s_cur += na;
            while (s_cur >= a.S) s_cur -= a.S;
            if (i >= g.NS && !lw_wait(bar0 + 8 * (g.NS + s), ph ^ 1u)) break;
            unsigned char *st = ring + (size_t)s * g.stage_bytes;
            const uint32_t full = bar0 + 8 * s;
            if (lane == 0) {
                const uint32_t bq = (uint32_t)(na * a.Hq * rowb);
                const uint32_t bk = (uint32_t)(na * a.Hkv * rowb);
                lw_bar_expect(full, bq + bk);
                if (bq) lw_bulk(lw_smem_u32(st), (const char *)a.q + t0 * a.Hq * rowb, bq, full, pol);
                if (bk)
                    lw_bulk(lw_smem_u32(st + g.off_k), (const char *)a.k + t0 * a.Hkv * rowb, bk,
                            full, pol);
            }
            if (totals && lane < na) reinterpret_cast<float2 *>(st + g.off_sc)[lane] = v;
            if (half > 0 && g.cs_by_consumers) {
                if (lane < na) reinterpret_cast<int32_t *>(st + g.off_pos)[lane] = pos;
            } else if (half > 0) {
                if (lane < na) s_pos[lane] = pos;
                __syncwarp();
                csw.fill(reinterpret_cast<float4 *>(st + g.off_cs), s_pos, s_step, na, lane);
                __syncwarp();
            }
            lw_bar_arrive(full);
            ++issued;
        }
        // leave only once every copy issued has landed
        for (int i = max(0, issued - g.NS); i < issued; ++i)
            if (!lw_wait(bar0 + 8 * (i % g.NS), (uint32_t)(i / g.NS) & 1u)) break;
        return;
    }

    // ---------------------------------------------------------------- consumers
    const Lane<LPR, V> L(lane, a.D, a.R);
    const uint32_t offA = (uint32_t)(L.eA * E), offB = (uint32_t)(L.eB * E);
    // the sums use the lane layout without a rotary span (the statistics
    // call has none), so every call adds the same terms in the same order
    const Lane<LPR, V> Ls(lane, a.D, 0);
    const uint32_t offAs = (uint32_t)(Ls.eA * E), offBs = (uint32_t)(Ls.eB * E);
    const int hp = half >> 1;  // rotary pairs per token
    const LwCsOffsets<V> co(L, hp / (V / 2));
    const uint32_t ring32 = lw_smem_u32(ring), gam32 = lw_smem_u32(s_gamma);
    int pc = 0;                // tokens dealt before this stage, mod ncw
    for (int i = 0; i < ntiles; ++i) {
        const int s = i % g.NS;
        if (!lw_wait(bar0 + 8 * s, (uint32_t)(i / g.NS) & 1u)) break;
        const int64_t t0 = tiles.start(i);
        const int na = tiles.count(i);
        const uint32_t st = ring32 + (uint32_t)(s * g.stage_bytes);
        int j = warp - pc;
        if (j < 0) j += ncw;
        for (; j < na; j += ncw) {
            const int64_t t = t0 + j;
            const uint32_t xq = st + (uint32_t)(j * a.Hq * rowb);
            const uint32_t xk = st + (uint32_t)(g.off_k + j * a.Hkv * rowb);
            float2 tot;
            if (MODE == kTokStats || local) {
                tot = tok_sumsq<T, LPR>(xq, xk, Ls, a.Hq, H, rowb, offAs, offBs);
            } else {
                tot = lw_ldsf2(st + (uint32_t)(g.off_sc + 8 * j));
            }
            if (MODE == kTokStats) {
                if (lane == 0) {
                    if (a.Hq) a.wq[t] = tot.x;
                    if (a.Hkv) a.wk[t] = tot.y;
                }
                continue;
            }
            const float rq = a.Hq ? rsqrtf(fmaf(tot.x, a.inv_q, a.eps)) : 0.f;
            const float rk = a.Hkv ? rsqrtf(fmaf(tot.y, a.inv_k, a.eps)) : 0.f;
            if (lane == 0) {
                if (a.Hq) a.wq[t] = rq;
                if (a.Hkv) a.wk[t] = rk;
            }
            if (half > 0 && g.cs_by_consumers) {
                // this warp owns token j: its lanes fill the token's table
                // (pair P at the same entry as the producer's fill would)
                const int32_t m = reinterpret_cast<const int32_t *>(
                    ring + (size_t)s * g.stage_bytes + g.off_pos)[j];
                float4 *tab = reinterpret_cast<float4 *>(ring + (size_t)s * g.stage_bytes +
                                                         g.off_cs) + j * hp;
                for (int P = lane; P < hp; P += 32) {
                    const int pw = P / (V / 2);
                    const int dst = (P - pw * (V / 2)) * (hp / (V / 2)) + pw;
                    const float2 c0 = rope_cos_sin_fixed(m, s_step[2 * P]);
                    const float2 c1 = rope_cos_sin_fixed(m, s_step[2 * P + 1]);
                    tab[dst] = make_float4(c0.x, c1.x, c0.y, c1.y);
                }
                __syncwarp();
            }
            float4 c[V / 2];
            lane_cs4_32<V>(c, st + (uint32_t)(g.off_cs + j * hp * 16), co, L);
            for (int p = 0; p < H; p += SLOTS) {
                const int h = p + L.slot;
                if (!(L.on && h < H)) continue;
                const bool isq = h < a.Hq;
                const int hh = isq ? h : h - a.Hq;
                const uint32_t row = isq ? xq + (uint32_t)(h * rowb) : xk + (uint32_t)(hh * rowb);
                const uint32_t grow = gam32 + (uint32_t)(h * rowb);
                const Vec16 xa = lw_lds16(row + offA), xb = lw_lds16(row + offB);
                const Vec16 ga = lw_lds16(grow + offA), gb = lw_lds16(grow + offB);
                const float r = isq ? rq : rk;
                const float2 r2 = make_float2(r, r);
                Vec16 ya, yb;
#pragma unroll
                for (int k2 = 0; k2 < V / 2; ++k2) {
                    // r folded into cos and sin: y_A = u_A (r c) - u_B (r s),
                    // y_B = u_B (r c) + u_A (r s), u = x gamma
                    const float2 cr = __fmul2_rn(make_float2(c[k2].x, c[k2].y), r2);
                    const float2 sr = __fmul2_rn(make_float2(c[k2].z, c[k2].w), r2);
                    const float2 ua = __fmul2_rn(IO::get2(xa, k2), IO::get2(ga, k2));
                    const float2 ub = __fmul2_rn(IO::get2(xb, k2), IO::get2(gb, k2));
                    const float2 oa = __ffma2_rn(ua, cr, __fmul2_rn(ub, neg2f(sr)));
                    const float2 ob = __ffma2_rn(ub, cr, __fmul2_rn(ua, sr));
                    IO::put2(ya, k2, oa.x, oa.y);
                    IO::put2(yb, k2, ob.x, ob.y);
                }
                char *out = (char *)(isq ? a.qo : a.ko) + ((isq ? t * a.Hq : t * a.Hkv) + hh) * rowb;
                lw_st_stream(out + offA, ya);
                lw_st_stream(out + offB, yb);
            }
        }
        pc = (pc + na) % ncw;
        __syncwarp();
        if (lane == 0) lw_bar_arrive(bar0 + 8 * (g.NS + s));
    }
}

int lpr_of(int D, int esz) {
    const int units = (D / (16 / esz) + 1) / 2;  // the last one may be a half unit
    int l = 1;
    while (l < units) l <<= 1;
    return l;
}

int sm_count_of(int dev) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

// Enough warps for ~4 CTAs of 8 warps per SM, each warp a contiguous run.
void lw_geometry(int64_t T, int *grid, int *tpw) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int64_t warps_max = (int64_t)sm_count_of(dev) * 4 * kWarps;
    int64_t per = (T + warps_max - 1) / warps_max;
    if (per < 1) per = 1;
    *tpw = (int)per;
    const int64_t warps = (T + per - 1) / per;
    *grid = (int)((warps + kWarps - 1) / kWarps);
}

qknr_status cuda_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

enum class LwKernel { kStats, kFwd, kDots, kBwd };

bool simple_kernels_forced() {
    const char *e = std::getenv("QKNR_SIMPLE_KERNELS");
    return e && e[0] && e[0] != '0';
}

// Stage and ring sizes of the pipelined (dots, backward) kernels for this
// shape, or false if the shape does not fit them (the plain-load kernels run
// instead).
bool lw_plan(int mode, const LwArgs &a, int esz, int lpr, int sms, LwGeom *g, int *grid,
             int *smem, int *threads) {
    if ((a.D / (16 / esz)) & 1) return false;  // a half unit: the plain-load kernels take it
    const int slots = 32 / lpr, H = a.Hq + a.Hkv;
    const int HB = (H + slots - 1) / slots;
    // head blocks per warp, warps per token, token groups: every warp owns
    // NB blocks (the last one maybe fewer), at most kLwCWMax warps. Two
    // blocks a warp (one token a round instead of two) when that lets a
    // quarter more consumer warps run: more warps hide the shared-memory and
    // group-sync latencies (Llama-3-8B shape: 3 groups of 5 warps, not 1 of 10)
    int NB = (HB + kLwCWMax - 1) / kLwCWMax;
    if (NB > kLwNBMax) return false;
    if (NB == 1 && HB > 1) {
        const int G1 = HB, G2 = (HB + 1) / 2;
        if (4 * G2 * (kLwCWMax / G2) >= 5 * G1 * (kLwCWMax / G1)) NB = 2;
    }
    const int G = (HB + NB - 1) / NB;
    const int NTG = kLwCWMax / G;
    const int64_t rowb = (int64_t)a.D * esz;
    const int64_t xq = (int64_t)a.Hq * rowb, xk = (int64_t)a.Hkv * rowb;  // per token
    const int64_t csb = (int64_t)(a.R / 2) * 8;
    const int64_t per = 2 * (xq + xk) + csb + 16 + 4;  // rows, gradients, angles, scalars, position
    int64_t TT = kLwStageTarget / per;
    TT = TT > kMaxTileTokensLw ? kMaxTileTokensLw : TT;
    TT = (TT / NTG) * NTG;
    if (TT < NTG) TT = NTG;
    if (TT > kMaxTileTokensLw) return false;
    const int64_t stage = ((TT * per + 127) / 128) * 128;  // the position section is last
    const int64_t gbytes = ((xq + xk + 127) / 128) * 128;
    const int64_t budget = kLwSmemBytes - 128 - TT * G * 8 * kLwMaxStages - 128 - gbytes;
    int64_t NS = (budget < kLwRingBytes ? budget : kLwRingBytes) / stage;
    if (NS > kLwMaxStages) NS = kLwMaxStages;
    if (NS < 2) return false;
    if (NS * stage < (int64_t)H * a.D * 4) return false;  // the backward's dgamma sums
    g->TT = (int)TT;
    g->NS = (int)NS;
    g->stage_bytes = (int)stage;
    g->off_k = (int)(TT * xq);
    g->off_dq = (int)(TT * (xq + xk));
    g->off_dk = (int)(TT * (2 * xq + xk));
    g->off_cs = (int)(TT * 2 * (xq + xk));
    g->off_sc = g->off_cs + (int)(TT * csb);
    g->off_pos = g->off_sc + (int)(TT * 16);
    // few rows a token: the consumer warps fill their tokens' (cos, sin)
    // tables, as in the token pipeline (see lw_tok_plan)
    g->cs_by_consumers = (a.R > 0 && NB == 1 && xq + xk < 32 * (int64_t)a.R) ? 1 : 0;
    g->off_parts = 128 + (int)(NS * stage);
    g->off_gamma = g->off_parts + (int)(((NS * TT * G * 8 + 127) / 128) * 128);
    g->G = G;
    g->NTG = NTG;
    g->HB = HB;
    // one CTA per SM, the tokens split evenly (a CTA's last stage may be
    // partial), so no SM idles for want of whole stages
    const int64_t tiles = (a.T + TT - 1) / TT;
    int64_t nb = tiles < (int64_t)sms ? tiles : (int64_t)sms;
    g->tpc = (a.T + nb - 1) / nb;
    nb = (a.T + g->tpc - 1) / g->tpc;
    *grid = (int)nb;
    *smem = g->off_gamma + (int)gbytes;
    *threads = (G * NTG + 1) * 32;
    return true;
}

// Stage and ring sizes of the pipelined statistics and forward, or false if
// the shape does not fit them. One plan serves both kernels (the statistics
// leave the angle and weight sections unused), so a shape runs both phases of
// a sharded call in the same kernel family as the one-pass forward.
bool lw_tok_plan(const LwArgs &a, int esz, int sms, LwTokGeom *g, int *grid, int *smem,
                 int *threads) {
    if ((a.D / (16 / esz)) & 1) return false;  // a half unit: the plain-load kernels take it
    const int64_t rowb = (int64_t)a.D * esz;
    const int64_t xq = (int64_t)a.Hq * rowb, xk = (int64_t)a.Hkv * rowb;  // per token
    const int64_t csb = (int64_t)(a.R / 2) * 8;
    const int64_t per = xq + xk + csb + 8 + 4;  // rows, angles, totals, position
    int64_t TT = kLwTokStageTarget / per;
    TT = TT > kMaxTileTokensLw ? kMaxTileTokensLw : (TT < 1 ? 1 : TT);
    const int64_t off_cs = TT * (xq + xk);
    const int64_t off_sc = off_cs + TT * csb;
    const int64_t off_pos = off_sc + TT * 8;
    const int64_t stage = ((off_pos + TT * 4 + 127) / 128) * 128;
    const int64_t gbytes = ((xq + xk + 127) / 128) * 128;
    const int64_t budget = kLwSmemBytes - 128 - gbytes;
    int64_t NS = (budget < kLwRingBytes ? budget : kLwRingBytes) / stage;
    if (NS > kLwMaxStages) NS = kLwMaxStages;
    if (NS < 2 || off_cs > (1 << 20) - 1) return false;
    g->TT = (int)TT;
    g->NS = (int)NS;
    g->stage_bytes = (int)stage;
    g->off_k = (int)(TT * xq);
    g->off_cs = (int)off_cs;
    g->off_sc = (int)off_sc;
    g->off_pos = (int)off_pos;
    g->off_gamma = 128 + (int)(NS * stage);
    g->ncw = kLwCWMax;
    g->h0 = TT >= 2 ? (int)(TT / 2) : 0;  // half a first tile (see LwTiles)
    // The one producer warp fills every token's (cos, sin) table of the CTA,
    // two angles a lane for each four pairs of dims: when a token's rows are
    // few (a tensor-parallel rank's head slice), that outlasts the rows'
    // transfer, so the consumer warps fill the tables of their own tokens
    // instead (Llama-3-8B shape at 4 + 1 heads: the producer-filled forward
    // ran at 15% DRAM throughput, its consumers waiting on stages).
    g->cs_by_consumers = (a.R > 0 && xq + xk < 32 * (int64_t)a.R) ? 1 : 0;
    const int64_t tiles = (a.T + TT - 1) / TT;
    int64_t nb = tiles < (int64_t)sms ? tiles : (int64_t)sms;
    g->tpc = (a.T + nb - 1) / nb;
    nb = (a.T + g->tpc - 1) / g->tpc;
    *grid = (int)nb;
    *smem = g->off_gamma + (int)gbytes;
    *threads = (g->ncw + 1) * 32;
    return true;
}

template <typename T, int LPR, int MODE>
qknr_status lw_tok_launch(const LwArgs &a, const LwTokGeom &g, int grid, int smem, int threads,
                          cudaStream_t st) {
    auto kern = qknr_lw_tok_kernel<T, LPR, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_pdl(kern, grid, threads, smem, st, a, g);
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, int LPR, int MODE>
qknr_status lw_pipe_launch(const LwArgs &a, const LwGeom &g, int grid, int smem, int threads,
                           cudaStream_t st) {
    // head blocks a warp owns: one (two tokens a round) or two (one a round)
    auto kern = (g.HB + g.G - 1) / g.G <= 1 ? qknr_lw_pipe_kernel<T, LPR, MODE, 1>
                                            : qknr_lw_pipe_kernel<T, LPR, MODE, 2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    e = launch_pdl(kern, grid, threads, smem, st, a, g);
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, int LPR>
qknr_status lw_launch_t(LwKernel which, const LwArgs &a, cudaStream_t st) {
    // The statistics and the forward take the token-per-warp pipeline (no
    // cross-warp sums); the dots and the backward, whose dgamma sums need
    // fixed row ownership, take the head-block pipeline. Shapes neither fits
    // run the plain-load kernels.
    if (!simple_kernels_forced() && (which == LwKernel::kStats || which == LwKernel::kFwd)) {
        int dev = 0;
        cudaGetDevice(&dev);
        LwTokGeom g;
        int grid, smem, thr;
        if (lw_tok_plan(a, (int)sizeof(T), sm_count_of(dev), &g, &grid, &smem, &thr)) {
            return which == LwKernel::kStats
                       ? lw_tok_launch<T, LPR, kTokStats>(a, g, grid, smem, thr, st)
                       : lw_tok_launch<T, LPR, kTokFwd>(a, g, grid, smem, thr, st);
        }
    }
    if (!simple_kernels_forced() && (which == LwKernel::kDots || which == LwKernel::kBwd)) {
        int dev = 0;
        cudaGetDevice(&dev);
        const int mode = which == LwKernel::kDots ? kLwDots : kLwBwd;
        LwGeom g;
        int grid, smem, thr;
        if (lw_plan(mode, a, (int)sizeof(T), LPR, sm_count_of(dev), &g, &grid, &smem, &thr)) {
            return mode == kLwDots ? lw_pipe_launch<T, LPR, kLwDots>(a, g, grid, smem, thr, st)
                                   : lw_pipe_launch<T, LPR, kLwBwd>(a, g, grid, smem, thr, st);
        }
    }
    int grid, tpw;
    lw_geometry(a.T, &grid, &tpw);
    LwArgs b = a;
    b.tpw = tpw;
    switch (which) {
        case LwKernel::kStats: qknr_lw_stats_kernel<T, LPR><<<grid, kThreads, 0, st>>>(b); break;
        case LwKernel::kFwd: qknr_lw_fwd_kernel<T, LPR><<<grid, kThreads, 0, st>>>(b); break;
        case LwKernel::kDots: qknr_lw_dots_kernel<T, LPR><<<grid, kThreads, 0, st>>>(b); break;
        case LwKernel::kBwd: {
            const int smem = (a.Hq + a.Hkv) * a.D * 4;
            auto kern = qknr_lw_bwd_kernel<T, LPR>;
            if (smem > 48 * 1024 &&
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                    cudaSuccess)
                return QKNR_ERR_UNSUPPORTED;
            kern<<<grid, kThreads, smem, st>>>(b);
            break;
        }
    }
    return cuda_status();
}

template <typename T>
qknr_status lw_launch(LwKernel which, const LwArgs &a, cudaStream_t st) {
    switch (lpr_of(a.D, (int)sizeof(T))) {
        case 1: return lw_launch_t<T, 1>(which, a, st);
        case 2: return lw_launch_t<T, 2>(which, a, st);
        case 4: return lw_launch_t<T, 4>(which, a, st);
        case 8: return lw_launch_t<T, 8>(which, a, st);
        case 16: return lw_launch_t<T, 16>(which, a, st);
        case 32: return lw_launch_t<T, 32>(which, a, st);
    }
    return QKNR_ERR_UNSUPPORTED;
}

// Checks shared by the layerwise entry points (the shape rules of the
// per-head op; totals at least the local head counts).
qknr_status lw_check(int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total, int D, int R,
                     float theta, float eps, qknr_dtype dtype) {
    if (dtype != QKNR_F32 && dtype != QKNR_BF16) return QKNR_ERR_INVALID_ARG;
    if (B < 0 || S < 0 || Hq < 0 || Hkv < 0) return QKNR_ERR_INVALID_ARG;
    if (Hq_total < Hq || Hkv_total < Hkv) return QKNR_ERR_INVALID_ARG;
    if (D < 2 || (D & 1) || R < 0 || R > D || (R & 1)) return QKNR_ERR_INVALID_ARG;
    if (!(theta > 0.f) || !(theta < 3.0e38f)) return QKNR_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(eps < 3.0e38f)) return QKNR_ERR_INVALID_ARG;
    const int e = dtype == QKNR_F32 ? 4 : 2;
    if (D > kMaxD || (D * e) % 16 != 0 || ((R / 2) * e) % 16 != 0) return QKNR_ERR_UNSUPPORTED;
    return QKNR_OK;
}

bool al(const void *p, uintptr_t n) { return !p || ((uintptr_t)p % n) == 0; }

// A buffer an entry point reads or writes: [p, p + n).
struct Buf {
    const void *p;
    size_t n;
    const void *same;  // outputs only: the input this one may equal exactly (in place)
};

bool touch(const Buf &a, const Buf &b) {
    if (!a.p || !b.p || !a.n || !b.n) return false;
    const uintptr_t x = (uintptr_t)a.p, y = (uintptr_t)b.p;
    return x < y + b.n && y < x + a.n;
}

// No output overlaps another output or an input, except an output that is
// exactly its own input (same address, so each lane reads its elements
// before it writes them).
template <size_t NO, size_t NI>
bool disjoint(const Buf (&out)[NO], const Buf (&in)[NI]) {
    for (size_t i = 0; i < NO; ++i) {
        for (size_t j = i + 1; j < NO; ++j)
            if (touch(out[i], out[j])) return false;
        for (size_t j = 0; j < NI; ++j)
            if (touch(out[i], in[j]) && !(out[i].same && out[i].same == in[j].p &&
                                          out[i].p == in[j].p && out[i].n == in[j].n))
                return false;
    }
    return true;
}

qknr_status lw_run(LwKernel which, LwArgs a, qknr_dtype dtype, qknr_stream_t stream) {
    cudaStream_t st = (cudaStream_t)stream;
    return dtype == QKNR_F32 ? lw_launch<float>(which, a, st)
                             : lw_launch<__nv_bfloat16>(which, a, st);
}

}  // namespace
}  // namespace qknr

namespace qknr {

// Launches the layerwise family's wait self-test.
qknr_status lw_wait_selftest(long long limit, cudaStream_t st) {
    qknr_lw_wait_selftest_kernel<<<1, 32, 0, st>>>(limit);
    return cuda_status();
}

// The pipelined layerwise kernels' error flag (see g_lw_error); -1 if it
// cannot be read.
int lw_pipeline_error(int reset) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_lw_error, sizeof(v)) != cudaSuccess) return -1;
    if (reset && v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_lw_error, &zero, sizeof(zero)) != cudaSuccess) return -1;
    }
    return (int)v;
}

}  // namespace qknr

using namespace qknr;

extern "C" qknr_status qk_layerwise_geometry(int mode, int B, int S, int Hq, int Hkv, int D,
                                             int rotary_dim, qknr_dtype dtype, int sms,
                                             int64_t *geom) {
    if (!geom || mode < 0 || mode > 2 || sms < 1) return QKNR_ERR_INVALID_ARG;
    qknr_status s = lw_check(B, S, Hq, Hkv, Hq, Hkv, D, rotary_dim, 1.f, 0.f, dtype);
    if (s != QKNR_OK) return s;
    if (mode == 1 && (int64_t)(Hq + Hkv) * D * 4 > kLwMaxDgammaBytes) return QKNR_ERR_UNSUPPORTED;
    for (int i = 0; i < kLwGeomLen; ++i) geom[i] = 0;
    const int esz = dtype == QKNR_F32 ? 4 : 2;
    LwArgs a{};
    a.T = (int64_t)B * S; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    if (a.T == 0 || Hq + Hkv == 0) return QKNR_OK;
    const int lpr = lpr_of(D, esz);
    int grid, smem, thr;
    if (mode == 2) {
        LwTokGeom t;
        if (!lw_tok_plan(a, esz, sms, &t, &grid, &smem, &thr)) return QKNR_OK;
        const int64_t v[kLwGeomLen] = {1, lpr, t.TT, t.NS, t.stage_bytes, t.off_k, 0, 0,
                                       t.off_cs, t.off_sc, 0, t.off_gamma, 1, t.ncw,
                                       (Hq + Hkv + 32 / lpr - 1) / (32 / lpr), t.tpc, grid, smem,
                                       thr, t.h0 ? t.h0 : t.TT, t.cs_by_consumers, t.off_pos};
        for (int i = 0; i < kLwGeomLen; ++i) geom[i] = v[i];
        return QKNR_OK;
    }
    LwGeom g;
    if (!lw_plan(mode == 0 ? kLwDots : kLwBwd, a, esz, lpr, sms, &g, &grid, &smem, &thr))
        return QKNR_OK;
    const int64_t v[kLwGeomLen] = {1, lpr, g.TT, g.NS, g.stage_bytes, g.off_k, g.off_dq,
                                   g.off_dk, g.off_cs, g.off_sc, g.off_parts, g.off_gamma, g.G,
                                   g.NTG, g.HB, g.tpc, grid, smem, thr, g.TT, g.cs_by_consumers,
                                   g.off_pos};
    for (int i = 0; i < kLwGeomLen; ++i) geom[i] = v[i];
    return QKNR_OK;
}

extern "C" qknr_status qk_layerwise_stats(const void *q, const void *k, float *sumsq_q,
                                          float *sumsq_k, int B, int S, int Hq, int Hkv, int D,
                                          qknr_dtype dtype, qknr_stream_t stream) {
    qknr_status s = lw_check(B, S, Hq, Hkv, Hq, Hkv, D, 0, 1.f, 0.f, dtype);
    if (s != QKNR_OK) return s;
    const int64_t T = (int64_t)B * S;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    if ((Hq && (!q || !sumsq_q)) || (Hkv && (!k || !sumsq_k))) return QKNR_ERR_INVALID_ARG;
    if (!al(q, 16) || !al(k, 16) || !al(sumsq_q, 4) || !al(sumsq_k, 4)) return QKNR_ERR_ALIGNMENT;
    const size_t e = dtype == QKNR_F32 ? 4 : 2, nq = (size_t)T * Hq * D * e,
                 nk = (size_t)T * Hkv * D * e, nt = (size_t)T * 4;
    const Buf outs[] = {{sumsq_q, Hq ? nt : 0, nullptr}, {sumsq_k, Hkv ? nt : 0, nullptr}};
    const Buf ins[] = {{q, nq, nullptr}, {k, nk, nullptr}};
    if (!disjoint(outs, ins)) return QKNR_ERR_INVALID_ARG;
    LwArgs a{};
    a.q = q; a.k = k; a.wq = sumsq_q; a.wk = sumsq_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = 0;
    return lw_run(LwKernel::kStats, a, dtype, stream);
}

extern "C" qknr_status qk_layerwise_norm_rope_fwd(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k,
    const int32_t *pos_ids, const float *sumsq_q, const float *sumsq_k, void *q_out, void *k_out,
    float *rstd_q, float *rstd_k, int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total,
    int D, int rotary_dim, float theta, float eps, qknr_dtype dtype, qknr_stream_t stream) {
    qknr_status s = lw_check(B, S, Hq, Hkv, Hq_total, Hkv_total, D, rotary_dim, theta, eps, dtype);
    if (s != QKNR_OK) return s;
    const int64_t T = (int64_t)B * S;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    // no sums given: this rank holds every head and takes the statistic itself
    const bool local = !sumsq_q && !sumsq_k;
    if (local && (Hq_total != Hq || Hkv_total != Hkv)) return QKNR_ERR_INVALID_ARG;
    if (Hq && (!q || !gamma_q || (!local && !sumsq_q) || !q_out || !rstd_q))
        return QKNR_ERR_INVALID_ARG;
    if (Hkv && (!k || !gamma_k || (!local && !sumsq_k) || !k_out || !rstd_k))
        return QKNR_ERR_INVALID_ARG;
    if (!al(q, 16) || !al(k, 16) || !al(gamma_q, 16) || !al(gamma_k, 16) || !al(q_out, 16) ||
        !al(k_out, 16) || !al(sumsq_q, 4) || !al(sumsq_k, 4) || !al(rstd_q, 4) ||
        !al(rstd_k, 4) || !al(pos_ids, 4))
        return QKNR_ERR_ALIGNMENT;
    const size_t e = dtype == QKNR_F32 ? 4 : 2, nq = (size_t)T * Hq * D * e,
                 nk = (size_t)T * Hkv * D * e, nt = (size_t)T * 4;
    const size_t tq = Hq ? nt : 0, tk = Hkv ? nt : 0;
    const Buf outs[] = {{q_out, nq, q}, {k_out, nk, k}, {rstd_q, tq, nullptr},
                        {rstd_k, tk, nullptr}};
    const Buf ins[] = {{q, nq, nullptr}, {k, nk, nullptr}, {gamma_q, (size_t)Hq * D * e, nullptr},
                       {gamma_k, (size_t)Hkv * D * e, nullptr}, {pos_ids, nt, nullptr},
                       {sumsq_q, tq, nullptr}, {sumsq_k, tk, nullptr}};
    if (!disjoint(outs, ins)) return QKNR_ERR_INVALID_ARG;
    LwArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.qo = q_out; a.ko = k_out; a.sq = sumsq_q; a.sk = sumsq_k; a.wq = rstd_q; a.wk = rstd_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    a.inv_q = Hq_total ? 1.f / ((float)Hq_total * (float)D) : 0.f;
    a.inv_k = Hkv_total ? 1.f / ((float)Hkv_total * (float)D) : 0.f;
    a.theta = theta; a.eps = eps;
    return lw_run(LwKernel::kFwd, a, dtype, stream);
}

extern "C" qknr_status qk_layerwise_bwd_dots(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k,
    const int32_t *pos_ids, const float *rstd_q, const float *rstd_k, const void *dq_out,
    const void *dk_out, float *dot_q, float *dot_k, int B, int S, int Hq, int Hkv, int D,
    int rotary_dim, float theta, qknr_dtype dtype, qknr_stream_t stream) {
    qknr_status s = lw_check(B, S, Hq, Hkv, Hq, Hkv, D, rotary_dim, theta, 0.f, dtype);
    if (s != QKNR_OK) return s;
    const int64_t T = (int64_t)B * S;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    if (Hq && (!q || !gamma_q || !rstd_q || !dq_out || !dot_q)) return QKNR_ERR_INVALID_ARG;
    if (Hkv && (!k || !gamma_k || !rstd_k || !dk_out || !dot_k)) return QKNR_ERR_INVALID_ARG;
    if (!al(q, 16) || !al(k, 16) || !al(gamma_q, 16) || !al(gamma_k, 16) || !al(dq_out, 16) ||
        !al(dk_out, 16) || !al(rstd_q, 4) || !al(rstd_k, 4) || !al(dot_q, 4) || !al(dot_k, 4) ||
        !al(pos_ids, 4))
        return QKNR_ERR_ALIGNMENT;
    const size_t e = dtype == QKNR_F32 ? 4 : 2, nq = (size_t)T * Hq * D * e,
                 nk = (size_t)T * Hkv * D * e, nt = (size_t)T * 4;
    const size_t tq = Hq ? nt : 0, tk = Hkv ? nt : 0;
    const Buf outs[] = {{dot_q, tq, nullptr}, {dot_k, tk, nullptr}};
    const Buf ins[] = {{q, nq, nullptr}, {k, nk, nullptr}, {gamma_q, (size_t)Hq * D * e, nullptr},
                       {gamma_k, (size_t)Hkv * D * e, nullptr}, {pos_ids, nt, nullptr},
                       {rstd_q, tq, nullptr}, {rstd_k, tk, nullptr}, {dq_out, nq, nullptr},
                       {dk_out, nk, nullptr}};
    if (!disjoint(outs, ins)) return QKNR_ERR_INVALID_ARG;
    LwArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.rq = rstd_q; a.rk = rstd_k; a.dqo = dq_out; a.dko = dk_out; a.wq = dot_q; a.wk = dot_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim; a.theta = theta;
    return lw_run(LwKernel::kDots, a, dtype, stream);
}

namespace {
qknr_status lw_bwd_impl(const void *q, const void *k, const void *gamma_q, const void *gamma_k,
                        const int32_t *pos_ids, const float *rstd_q, const float *rstd_k,
                        const void *dq_out, const void *dk_out, const float *dot_q,
                        const float *dot_k, void *dq, void *dk, float *dgamma_q, float *dgamma_k,
                        int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total, int D,
                        int rotary_dim, float theta, qknr_dtype dtype, qknr_stream_t stream,
                        bool zero_dgamma) {
    qknr_status s = lw_check(B, S, Hq, Hkv, Hq_total, Hkv_total, D, rotary_dim, theta, 0.f, dtype);
    if (s != QKNR_OK) return s;
    // the block's dgamma partial sums live in shared memory
    if ((int64_t)(Hq + Hkv) * D * 4 > kLwMaxDgammaBytes) return QKNR_ERR_UNSUPPORTED;
    const int64_t T = (int64_t)B * S;
    if (!al(q, 16) || !al(k, 16) || !al(gamma_q, 16) || !al(gamma_k, 16) || !al(dq_out, 16) ||
        !al(dk_out, 16) || !al(dq, 16) || !al(dk, 16) || !al(rstd_q, 4) || !al(rstd_k, 4) ||
        !al(dot_q, 4) || !al(dot_k, 4) || !al(dgamma_q, 4) || !al(dgamma_k, 4) || !al(pos_ids, 4))
        return QKNR_ERR_ALIGNMENT;
    const bool work = T > 0 && Hq + Hkv > 0;
    // no dot sums given: this rank holds every head and takes them itself
    const bool local = !dot_q && !dot_k;
    if (local && (Hq_total != Hq || Hkv_total != Hkv)) return QKNR_ERR_INVALID_ARG;
    if (work && Hq && (!q || !gamma_q || !rstd_q || !dq_out || (!local && !dot_q) || !dq))
        return QKNR_ERR_INVALID_ARG;
    if (work && Hkv && (!k || !gamma_k || !rstd_k || !dk_out || (!local && !dot_k) || !dk))
        return QKNR_ERR_INVALID_ARG;
    {
        const size_t e = dtype == QKNR_F32 ? 4 : 2, nq = (size_t)T * Hq * D * e,
                     nk = (size_t)T * Hkv * D * e, nt = (size_t)T * 4;
        const size_t tq = Hq ? nt : 0, tk = Hkv ? nt : 0;
        const Buf outs[] = {{dq, nq, dq_out}, {dk, nk, dk_out},
                            {dgamma_q, (size_t)Hq * D * 4, nullptr},
                            {dgamma_k, (size_t)Hkv * D * 4, nullptr}};
        const Buf ins[] = {{q, nq, nullptr}, {k, nk, nullptr},
                           {gamma_q, (size_t)Hq * D * e, nullptr},
                           {gamma_k, (size_t)Hkv * D * e, nullptr}, {pos_ids, nt, nullptr},
                           {rstd_q, tq, nullptr}, {rstd_k, tk, nullptr}, {dq_out, nq, nullptr},
                           {dk_out, nk, nullptr}, {dot_q, tq, nullptr}, {dot_k, tk, nullptr}};
        if (!disjoint(outs, ins)) return QKNR_ERR_INVALID_ARG;
    }
    cudaStream_t st = (cudaStream_t)stream;
    if (zero_dgamma) {
        const qknr_status zs = zero_f32(dgamma_q, (int64_t)Hq * D, dgamma_k, (int64_t)Hkv * D, st);
        if (zs != QKNR_OK) return zs;
    }
    if (!work) return QKNR_OK;
    LwArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.rq = rstd_q; a.rk = rstd_k; a.dqo = dq_out; a.dko = dk_out; a.sq = dot_q; a.sk = dot_k;
    a.qo = dq; a.ko = dk; a.dgq = dgamma_q; a.dgk = dgamma_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim; a.theta = theta;
    a.inv_q = Hq_total ? 1.f / ((float)Hq_total * (float)D) : 0.f;
    a.inv_k = Hkv_total ? 1.f / ((float)Hkv_total * (float)D) : 0.f;
    return lw_run(LwKernel::kBwd, a, dtype, stream);
}
}  // namespace

extern "C" qknr_status qk_layerwise_norm_rope_bwd(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k,
    const int32_t *pos_ids, const float *rstd_q, const float *rstd_k, const void *dq_out,
    const void *dk_out, const float *dot_q, const float *dot_k, void *dq, void *dk,
    float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total,
    int D, int rotary_dim, float theta, qknr_dtype dtype, qknr_stream_t stream) {
    return lw_bwd_impl(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dot_q,
                       dot_k, dq, dk, dgamma_q, dgamma_k, B, S, Hq, Hkv, Hq_total, Hkv_total, D,
                       rotary_dim, theta, dtype, stream, true);
}

extern "C" qknr_status qk_layerwise_norm_rope_bwd_acc(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k,
    const int32_t *pos_ids, const float *rstd_q, const float *rstd_k, const void *dq_out,
    const void *dk_out, const float *dot_q, const float *dot_k, void *dq, void *dk,
    float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total,
    int D, int rotary_dim, float theta, qknr_dtype dtype, qknr_stream_t stream) {
    return lw_bwd_impl(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dot_q,
                       dot_k, dq, dk, dgamma_q, dgamma_k, B, S, Hq, Hkv, Hq_total, Hkv_total, D,
                       rotary_dim, theta, dtype, stream, false);
}
