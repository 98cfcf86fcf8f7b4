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
// the caller's: NCCL through torch.distributed in the Python binding.
// One warp walks all of a token's local heads, so each per-token sum is one
// warp reduction. gamma rows are read with the same 16-byte vectors as x rows
// (they are cached; every token reuses them).
#include "qknr.h"
#include "qknr_kernels.cuh"

#include <cstdint>

namespace qknr {

qknr_status cuda_fail(cudaError_t e);  // defined beside the per-head entry points

namespace {

constexpr int kLwMaxDgammaBytes = 200 * 1024;

struct LwArgs {
    const void *q, *k;        // this rank's heads: [T, Hq, D], [T, Hkv, D]
    const void *gq, *gk;      // gamma slices [Hq * D], [Hkv * D]
    const int32_t *pos;
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
        const Vec16 xa = ld16(row + offA), xb = ld16(row + offB);
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
        const Vec16 xa = ld16(row + offA), xb = ld16(row + offB);
        const Vec16 da = ld16(drow + offA), db = ld16(drow + offB);
        const Vec16 ga = ld16(grow + offA), gb = ld16(grow + offB);
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
            const Vec16 xa = ld16(row + offA), xb = ld16(row + offB);
            const Vec16 ga = ld16(grow + offA), gb = ld16(grow + offB);
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
            st16(out + offB, yb);
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
            const Vec16 xa = ld16(row + offA), xb = ld16(row + offB);
            const Vec16 da = ld16(drow + offA), db = ld16(drow + offB);
            const Vec16 ga = ld16(grow + offA), gb = ld16(grow + offB);
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
                    atomicAdd(dg + L.eB + e, gB * xB * r);
                }
                IO::put2(oa, k2, outA[0], outA[1]);
                IO::put2(ob, k2, outB[0], outB[1]);
            }
            char *out = (char *)(isq ? a.qo : a.ko) + ri * rowb;
            st16(out + offA, oa);
            st16(out + offB, ob);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < H * a.D; i += kThreads) {
        const bool isq = i < a.Hq * a.D;
        float *g = isq ? a.dgq : a.dgk;
        if (g) atomicAdd(g + (isq ? i : i - a.Hq * a.D), s_dg[i]);
    }
}

int lpr_of(int D, int esz) {
    const int dv2 = D / (2 * (16 / esz));
    int l = 1;
    while (l < dv2) l <<= 1;
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

template <typename T, int LPR>
qknr_status lw_launch_t(LwKernel which, const LwArgs &a, cudaStream_t st) {
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
    if (D > kMaxD || (D * e) % 32 != 0 || ((R / 2) * e) % 16 != 0) return QKNR_ERR_UNSUPPORTED;
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

using namespace qknr;

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

extern "C" qknr_status qk_layerwise_norm_rope_bwd(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k,
    const int32_t *pos_ids, const float *rstd_q, const float *rstd_k, const void *dq_out,
    const void *dk_out, const float *dot_q, const float *dot_k, void *dq, void *dk,
    float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv, int Hq_total, int Hkv_total,
    int D, int rotary_dim, float theta, qknr_dtype dtype, qknr_stream_t stream) {
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
    cudaError_t ce;
    if (dgamma_q && Hq &&
        (ce = cudaMemsetAsync(dgamma_q, 0, (size_t)Hq * D * 4, st)) != cudaSuccess)
        return cuda_fail(ce);
    if (dgamma_k && Hkv &&
        (ce = cudaMemsetAsync(dgamma_k, 0, (size_t)Hkv * D * 4, st)) != cudaSuccess)
        return cuda_fail(ce);
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
