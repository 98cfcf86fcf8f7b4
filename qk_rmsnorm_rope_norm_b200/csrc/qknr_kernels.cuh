// Device code of the fused per-head QK-RMSNorm + rotate-half RoPE, forward
// and backward, for sm_100a.
//
// The op is a streaming, HBM-bound map over (token, head) rows: each element
// is read once and written once, with ~10 fp32 operations per element, so
// there is no contraction and no tensor-core work. Chronicals (arXiv
// 2601.02609), abstract, contribution (1), fuses exactly this pair (norm and
// rotary on Q and K) to cut memory traffic; its Triton kernels target the
// A100 and are prior art only.
//
// Work mapping (one design for both directions):
//  * one warp owns one token at a time and walks all Hq + Hkv heads of it;
//    the token's R/2 rotary (cos, sin) pairs are computed once per warp into
//    a warp-private shared-memory table and reused by every head;
//  * LPR lanes share one head row; lane u of the group holds two 16-byte
//    vectors of the row, chosen so that every rotary pair (i, i + R/2) sits
//    in the same lane: for u < R/(2V) the vectors u and u + R/(2V) (V
//    elements per vector), otherwise the pass-through vectors u + R/(2V) and
//    u + D/(2V). Each load instruction of the group covers whole 32-byte
//    sectors; pass-through lanes rotate with (cos, sin) = (1, 0), which is
//    exact;
//  * the sum of squares (forward) and <h, xh> (backward) are reduced across
//    the LPR lanes with xor shuffles;
//  * gamma lives in shared memory as fp32 and (cos, sin) in the warp's
//    table, so registers hold little beyond the 16-byte vectors in flight;
//  * rotary angles are reduced modulo 2*pi in fp64 (Cody-Waite, two-part
//    2*pi) before an fp32 sincosf, so positions up to 2^31 keep an angle
//    error far below bf16 resolution.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
#include <utility>

namespace qknr {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxD = 256;
constexpr int kMaxHalf = kMaxD / 2;

// Resident CTAs per SM the register allocation is sized for.
#ifndef QKNR_FWD_MIN_CTAS
#define QKNR_FWD_MIN_CTAS 3
#endif
#ifndef QKNR_BWD_MIN_CTAS
#define QKNR_BWD_MIN_CTAS 2
#endif

// Programmatic dependent launch. The pipelined kernels (per-head and
// layerwise) and the dgamma zeroing kernel are launched with programmatic
// stream serialization allowed, so a kernel's CTAs may start while the
// previous kernel of the stream is still finishing: everything before
// grid_dep_wait() touches only the CTA's own shared memory (and, on the
// misaligned-shared-memory error path, the library's own error flag), and no
// input or output is read or written before it returns (the previous kernel
// has then completed and its writes are visible). grid_dep_launch() lets the
// next kernel of the stream start its own prologue once every CTA of this one
// has passed that point. Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// QKNR_PDL=0 in the environment launches those kernels plainly.
inline bool pdl_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("QKNR_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

// Launch with programmatic stream serialization (unless disabled). Only for
// kernels that call grid_dep_wait() before their first global access.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), int grid, int threads, int smem, cudaStream_t st,
                       A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// Forward variants (FwdArgs::mode bits).
constexpr int kModeRopeOnly = 1;  // rotation alone: r = 1, gamma = 1, no rstd written
constexpr int kModeInverse = 2;   // rotate by -m (the transpose): strips RoPE
constexpr int kModeStatsOnly = 4; // write rstd only, no normalised rows
constexpr int kModeLayerNorm = 8; // mean-centred (QK-LayerNorm): host-side choice of kernel

struct FwdArgs {
    const void *q, *k, *gq, *gk;
    const int32_t *pos;
    void *qo, *ko;
    float *rq, *rk;
    int64_t qts, kts;  // bytes from one token's rows of q (k) to the next token's
    int64_t T;  // tokens = B * S
    int S, Hq, Hkv, D, R;
    float theta, eps;
    int tpw;    // consecutive tokens per warp
    int mode;   // kMode* bits, 0 for the fused op
};

struct BwdArgs {
    const void *q, *k, *gq, *gk;
    const int32_t *pos;
    const float *rq, *rk;
    const void *dqo, *dko;
    void *dq, *dk;
    float *dgq, *dgk;
    int64_t qts, kts;    // token strides (bytes) of q and k
    int64_t dqts, dkts;  // token strides (bytes) of dq and dk
    int64_t T;
    int S, Hq, Hkv, D, R;
    float theta, eps;
    int tpw;
};

// ----------------------------------------------------------------- I/O types
// A 16-byte vector as four 32-bit words; element pairs (2k, 2k+1) are read
// and written together.
struct alignas(16) Vec16 {
    uint32_t w[4];
};

template <typename T> struct Io;

template <> struct Io<float> {
    static constexpr int V = 4;  // elements per 16-byte vector
    __device__ __forceinline__ static float2 get2(const Vec16 &r, int k) {
        return make_float2(__uint_as_float(r.w[2 * k]), __uint_as_float(r.w[2 * k + 1]));
    }
    __device__ __forceinline__ static void put2(Vec16 &r, int k, float a, float b) {
        r.w[2 * k] = __float_as_uint(a);
        r.w[2 * k + 1] = __float_as_uint(b);
    }
    __device__ __forceinline__ static float to_f32(const void *p, int i) {
        return reinterpret_cast<const float *>(p)[i];
    }
};

template <> struct Io<__nv_bfloat16> {
    static constexpr int V = 8;
    __device__ __forceinline__ static float2 get2(const Vec16 &r, int k) {
        return make_float2(__uint_as_float(r.w[k] << 16), __uint_as_float(r.w[k] & 0xffff0000u));
    }
    __device__ __forceinline__ static void put2(Vec16 &r, int k, float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // round to nearest even
        r.w[k] = *reinterpret_cast<uint32_t *>(&h);
    }
    __device__ __forceinline__ static float to_f32(const void *p, int i) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    }
};

__device__ __forceinline__ Vec16 ld16(const void *p) {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    Vec16 r;
    r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    return r;
}
__device__ __forceinline__ void st16(void *p, const Vec16 &v) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]);
}
__device__ __forceinline__ Vec16 zero16() {
    Vec16 r;
    r.w[0] = r.w[1] = r.w[2] = r.w[3] = 0u;
    return r;
}

// ------------------------------------------------------------- rotary angle
// cos/sin of pos * omega. The product is formed in fp64 (exact integer pos,
// 53-bit omega) and reduced to [-pi, pi] with a two-part 2*pi (Cody-Waite);
// only the reduced angle is rounded to fp32 for sincosf.
__device__ __forceinline__ float2 rope_cos_sin(int64_t pos, double omega) {
    const double kInv2Pi = 0.15915494309189533577;
    const double k2PiHi = 6.283185307179586232;      // nearest double to 2*pi
    const double k2PiLo = 2.4492935982947064e-16;    // 2*pi - k2PiHi
    const double phi = (double)pos * omega;
    const double n = rint(phi * kInv2Pi);
    double r = fma(-n, k2PiHi, phi);
    r = fma(-n, k2PiLo, r);
    float s, c;
    sincosf((float)r, &s, &c);
    return make_float2(c, s);
}

// Rotary angle in fixed point. F = round(2^64 * frac(omega / 2pi)) is the
// angle step per position in units of 2^-64 turns, so pos * F mod 2^64 is
// the angle mod one turn (integer wrap-around does the reduction; negative
// positions work in two's complement). Its top 32 bits, as a signed turn
// fraction in [-1/2, 1/2), feed the hardware sin/cos (absolute error
// ~2^-21 on [-pi, pi]). The error of F (~1e-16 relative) times |pos| < 2^31
// keeps the angle within ~2.4e-7 rad at the largest positions.
__device__ __forceinline__ uint64_t turn_step(int i, int R, float theta) {
    const double w = pow((double)theta, -2.0 * (double)i / (double)R);
    return __double2ull_rn(w * 0.15915494309189533577 * 18446744073709551616.0);
}
__device__ __forceinline__ float2 rope_cos_sin_fixed(int32_t pos, uint64_t F) {
    const uint32_t p = (uint32_t)pos, flo = (uint32_t)F, fhi = (uint32_t)(F >> 32);
    const uint32_t hi = __umulhi(p, flo) + p * fhi - (pos < 0 ? flo : 0u);
    const float turns = (float)(int32_t)hi * 2.3283064365386963e-10f;  // 2^-32
    float s, c;
    __sincosf(turns * 6.2831853071795865f, &s, &c);
    return make_float2(c, s);
}

// Per-CTA tables: inverse frequencies omega_i = theta^(-2i/R) in fp64, and
// gamma_q / gamma_k widened to fp32.
template <typename T>
__device__ __forceinline__ void fill_tables(double *s_omega, float (*s_g)[kMaxD],
                                            int D, int R, float theta,
                                            const void *gq, const void *gk) {
    const int half = R >> 1;
    for (int i = threadIdx.x; i < half; i += blockDim.x)
        s_omega[i] = pow((double)theta, -2.0 * (double)i / (double)R);
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        s_g[0][i] = gq ? Io<T>::to_f32(gq, i) : 1.f;  // no gamma: rotation alone
        s_g[1][i] = gk ? Io<T>::to_f32(gk, i) : 1.f;
    }
}

// Geometry of unit w of a head row of D elements (R rotary, V elements per
// 16-byte vector): the element offsets of its two vectors. The R / V rotary
// vectors form R / 2V units (w, w + R / 2V), so every rotary pair (i, i + R/2)
// sits in one unit; the P pass-through vectors form ceil(P / 2) units
// (j, j + ceil(P / 2)) after them. With P odd the last pass-through unit has
// no second vector (onB false; eB then repeats eA and must not be used).
// Units past the row (the unit count not a power of two) are off and point
// at element 0.
template <int V> struct UnitGeom {
    bool on, rot, onB;
    int eA, eB;
    __device__ __forceinline__ UnitGeom(int w, int D, int R) {
        const int Rv2 = R / (2 * V), P = D / V - 2 * Rv2, hp = (P + 1) >> 1;
        const int j = w - Rv2;
        on = w < Rv2 + hp;
        rot = w < Rv2;
        onB = rot || (on && j + hp < P);
        eA = on ? (rot ? w : 2 * Rv2 + j) * V : 0;
        eB = onB ? (rot ? w + Rv2 : 2 * Rv2 + j + hp) * V : eA;
    }
};

// Lane geometry: LPR lanes per row, lane u of the group owns unit u.
template <int LPR, int V> struct Lane {
    int u, slot;
    bool on, rot, onB;
    int eA, eB;  // element offsets of the lane's two vectors
    __device__ __forceinline__ Lane(int lane, int D, int R) {
        u = lane & (LPR - 1);
        slot = lane / LPR;
        const UnitGeom<V> G(u, D, R);
        on = G.on;
        rot = G.rot;
        onB = G.onB;
        eA = G.eA;
        eB = G.eB;
    }
};

template <int LPR>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// (cos, sin) for element eA + j of a lane; (1, 0) on pass-through lanes.
__device__ __forceinline__ float2 lane_cs(const float2 *cs, bool rot, int e) {
    const float2 v = cs[rot ? e : 0];
    return rot ? v : make_float2(1.f, 0.f);
}

// Position of the warp's next token: the given id, else s within the row.
struct PosIter {
    const int32_t *ids;
    int S, s;
    __device__ __forceinline__ PosIter(const int32_t *p, int S_, int64_t t0)
        : ids(p), S(S_), s((int)(t0 % S_)) {}
    __device__ __forceinline__ int64_t next(int64_t t) {
        const int64_t m = ids ? (int64_t)ids[t] : (int64_t)s;
        if (++s == S) s = 0;
        return m;
    }
};

// =================================================================== forward
// A warp covers 32 / LPR rows of one token per pass; P passes are loaded
// together so each lane keeps 2 * P 16-byte loads in flight.
// LN: the mean-centred variant (QK-LayerNorm): x - mean(x) in place of x.
template <typename T, int LPR, bool LN>
__global__ void __launch_bounds__(kThreads, QKNR_FWD_MIN_CTAS)
qknr_fwd_kernel(const FwdArgs a) {
    using IO = Io<T>;
    constexpr int V = IO::V;
    constexpr int SLOTS = 32 / LPR;
    constexpr int P = 2;
    __shared__ double s_omega[kMaxHalf];
    __shared__ float s_g[2][kMaxD];
    __shared__ float2 s_cs[kWarps][kMaxHalf];

    fill_tables<T>(s_omega, s_g, a.D, a.R, a.theta, a.Hq ? a.gq : nullptr,
                   a.Hkv ? a.gk : nullptr);
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Lane<LPR, V> L(lane, a.D, a.R);
    const int H = a.Hq + a.Hkv, half = a.R >> 1;
    const int npass = (H + SLOTS - 1) / SLOTS;
    const int rowb = a.D * (int)sizeof(T);
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    const float inv_d = 1.0f / (float)a.D;
    float2 *cs = s_cs[warp];

    const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;
    const int64_t t_begin = gw * a.tpw;
    const int64_t t_end = min(t_begin + (int64_t)a.tpw, a.T);
    PosIter pit(a.pos, a.S, t_begin);

    for (int64_t t = t_begin; t < t_end; ++t) {
        const int64_t pos = pit.next(t);
        const char *qrow = (const char *)a.q + t * a.qts;
        const char *krow = (const char *)a.k + t * a.kts;
        Vec16 xa[P], xb[P];
        auto load_chunk = [&](int p0) {
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                const int h = (p0 + pp) * SLOTS + L.slot;
                xa[pp] = xb[pp] = zero16();
                if (L.on && h < H) {
                    const char *row = h < a.Hq ? qrow + h * rowb : krow + (h - a.Hq) * rowb;
                    xa[pp] = ld16(row + offA);
                    if (L.onB) xb[pp] = ld16(row + offB);  // a half unit keeps B = 0
                }
            }
        };
        load_chunk(0);
        for (int i = lane; i < half; i += 32) {
            float2 v = rope_cos_sin(pos, s_omega[i]);
            if (a.mode & kModeInverse) v.y = -v.y;
            cs[i] = v;
        }
        __syncwarp();

        for (int p0 = 0; p0 < npass; p0 += P) {
            if (p0) load_chunk(p0);
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                float mu = 0.f;
                if (LN) {
                    float sx = 0.f;
#pragma unroll
                    for (int k2 = 0; k2 < V / 2; ++k2) {
                        const float2 va = IO::get2(xa[pp], k2), vb = IO::get2(xb[pp], k2);
                        sx += (va.x + va.y) + (vb.x + vb.y);
                    }
                    mu = group_sum<LPR>(sx) * inv_d;
                }
                float ss = 0.f;
#pragma unroll
                for (int k2 = 0; k2 < V / 2; ++k2) {
                    float2 va = IO::get2(xa[pp], k2), vb = IO::get2(xb[pp], k2);
                    if (LN && L.on) {
                        va.x -= mu; va.y -= mu;
                        if (L.onB) {
                            vb.x -= mu; vb.y -= mu;
                        }
                    }
                    ss = fmaf(va.x, va.x, ss); ss = fmaf(va.y, va.y, ss);
                    ss = fmaf(vb.x, vb.x, ss); ss = fmaf(vb.y, vb.y, ss);
                }
                ss = group_sum<LPR>(ss);
                const float r = (a.mode & kModeRopeOnly) ? 1.f : __frsqrt_rn(fmaf(ss, inv_d, a.eps));
                const int h = (p0 + pp) * SLOTS + L.slot;
                if (L.on && h < H) {
                    const bool isq = h < a.Hq;
                    const float *g = s_g[isq ? 0 : 1];
                    Vec16 ya, yb;
#pragma unroll
                    for (int k2 = 0; k2 < V / 2; ++k2) {
                        float2 va = IO::get2(xa[pp], k2), vb = IO::get2(xb[pp], k2);
                        if (LN) {
                            va.x -= mu; va.y -= mu; vb.x -= mu; vb.y -= mu;
                        }
                        const int e = 2 * k2;
                        const float2 c0 = lane_cs(cs, L.rot, L.eA + e);
                        const float2 c1 = lane_cs(cs, L.rot, L.eA + e + 1);
                        // n = (x * gamma) * r, the order the pipelined kernel uses
                        const float na0 = va.x * g[L.eA + e] * r, na1 = va.y * g[L.eA + e + 1] * r;
                        const float nb0 = vb.x * g[L.eB + e] * r, nb1 = vb.y * g[L.eB + e + 1] * r;
                        IO::put2(ya, k2, fmaf(na0, c0.x, -nb0 * c0.y), fmaf(na1, c1.x, -nb1 * c1.y));
                        IO::put2(yb, k2, fmaf(nb0, c0.x, na0 * c0.y), fmaf(nb1, c1.x, na1 * c1.y));
                    }
                    const int hh = isq ? h : h - a.Hq;
                    const int64_t rowi = isq ? t * a.Hq + hh : t * a.Hkv + hh;
                    char *out = (char *)(isq ? a.qo : a.ko) + rowi * rowb;
                    if (!(a.mode & kModeStatsOnly)) {
                        st16(out + offA, ya);
                        if (L.onB) st16(out + offB, yb);
                    }
                    if (L.u == 0 && !(a.mode & kModeRopeOnly)) (isq ? a.rq : a.rk)[rowi] = r;
                }
            }
        }
        __syncwarp();  // every lane has read the (cos, sin) table
    }
}

// ================================================================== backward
// Per row: g = R^T dy; xh = x r; h = g gamma; dgamma += g xh;
// dx = r (h - xh <h, xh> / D). The row is walked twice from the packed
// registers (once for <h, xh> and the dgamma terms, once for dx) so that no
// fp32 copy of the row is kept.
// LN: the mean-centred variant: xh = (x - mean) r and
// dx = r (h - mean(h) - xh <h, xh> / D).
template <typename T, int LPR, bool LN>
__global__ void __launch_bounds__(kThreads, QKNR_BWD_MIN_CTAS)
qknr_bwd_kernel(const BwdArgs a) {
    using IO = Io<T>;
    constexpr int V = IO::V;
    constexpr int SLOTS = 32 / LPR;
    constexpr int P = 2;
    __shared__ double s_omega[kMaxHalf];
    __shared__ float s_g[2][kMaxD];
    __shared__ float2 s_cs[kWarps][kMaxHalf];
    __shared__ float s_dg[2][kMaxD];
    __shared__ float4 s_acc[2][kWarps][V / 2][32];

    fill_tables<T>(s_omega, s_g, a.D, a.R, a.theta, a.Hq ? a.gq : nullptr,
                   a.Hkv ? a.gk : nullptr);
    for (int i = threadIdx.x; i < 2 * kMaxD; i += kThreads) (&s_dg[0][0])[i] = 0.f;
    for (int i = threadIdx.x; i < 2 * kWarps * (V / 2) * 32; i += kThreads)
        (&s_acc[0][0][0][0])[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Lane<LPR, V> L(lane, a.D, a.R);
    const int H = a.Hq + a.Hkv, half = a.R >> 1;
    const int npass = (H + SLOTS - 1) / SLOTS;
    const int rowb = a.D * (int)sizeof(T);
    const int offA = L.eA * (int)sizeof(T), offB = L.eB * (int)sizeof(T);
    const float inv_d = 1.0f / (float)a.D;
    float2 *cs = s_cs[warp];

    // dgamma partial sums live in shared memory, private to each lane: for
    // tensor z (0 = Q, 1 = K), float4 k of lane l of warp w is
    // s_acc[z][w][k][l] (k < V/4: elements eA..; else eB..), a layout in
    // which a warp's 16-byte accesses hit distinct banks.
    float4 (*acc_q)[32] = s_acc[0][warp];
    float4 (*acc_k)[32] = s_acc[1][warp];

    const int64_t gw = (int64_t)blockIdx.x * kWarps + warp;
    const int64_t t_begin = gw * a.tpw;
    const int64_t t_end = min(t_begin + (int64_t)a.tpw, a.T);
    PosIter pit(a.pos, a.S, t_begin);

    for (int64_t t = t_begin; t < t_end; ++t) {
        const int64_t pos = pit.next(t);
        Vec16 xa[P], xb[P], da[P], db[P];
        float rr[P];
        auto load_chunk = [&](int p0) {
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                const int h = (p0 + pp) * SLOTS + L.slot;
                xa[pp] = xb[pp] = da[pp] = db[pp] = zero16();
                rr[pp] = 0.f;
                if (L.on && h < H) {
                    const bool isq = h < a.Hq;
                    const int64_t rowi = isq ? t * a.Hq + h : t * a.Hkv + (h - a.Hq);
                    const int hh = isq ? h : h - a.Hq;
                    const char *xrow = (const char *)(isq ? a.q : a.k) + t * (isq ? a.qts : a.kts) + hh * rowb;
                    const char *drow = (const char *)(isq ? a.dqo : a.dko) + rowi * rowb;
                    xa[pp] = ld16(xrow + offA);
                    da[pp] = ld16(drow + offA);
                    if (L.onB) {  // a half unit keeps B = 0 (no gradient, no dgamma term)
                        xb[pp] = ld16(xrow + offB);
                        db[pp] = ld16(drow + offB);
                    }
                    rr[pp] = (isq ? a.rq : a.rk)[rowi];
                }
            }
        };
        load_chunk(0);
        for (int i = lane; i < half; i += 32) cs[i] = rope_cos_sin(pos, s_omega[i]);
        __syncwarp();

        for (int p0 = 0; p0 < npass; p0 += P) {
            if (p0) load_chunk(p0);
#pragma unroll
            for (int pp = 0; pp < P; ++pp) {
                const int h = (p0 + pp) * SLOTS + L.slot;
                const bool isq = h < a.Hq;
                const float *g = s_g[isq ? 0 : 1];
                const float r = rr[pp];
                float mu = 0.f;
                if (LN) {
                    float sx = 0.f;
#pragma unroll
                    for (int k2 = 0; k2 < V / 2; ++k2) {
                        const float2 xa2 = IO::get2(xa[pp], k2), xb2 = IO::get2(xb[pp], k2);
                        sx += (xa2.x + xa2.y) + (xb2.x + xb2.y);
                    }
                    mu = group_sum<LPR>(sx) * inv_d;
                }
                // walk 1: <h, xh> and the dgamma terms g * xh, four elements
                // of each half at a time (and, mean-centred, sum of h)
                float dot = 0.f, sh = 0.f;
                float4 (*acc)[32] = isq ? acc_q : acc_k;
#pragma unroll
                for (int qd = 0; qd < V / 4; ++qd) {
                    float tA[4], tB[4];
#pragma unroll
                    for (int k2 = 2 * qd; k2 < 2 * qd + 2; ++k2) {
                        const float2 xa2 = IO::get2(xa[pp], k2), xb2 = IO::get2(xb[pp], k2);
                        const float2 da2 = IO::get2(da[pp], k2), db2 = IO::get2(db[pp], k2);
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int e = 2 * k2 + q;
                            const float2 c = lane_cs(cs, L.rot, L.eA + e);
                            const float dA = q ? da2.y : da2.x, dB = q ? db2.y : db2.x;
                            const float xA = ((q ? xa2.y : xa2.x) - mu) * r;
                            const float xB = L.onB ? ((q ? xb2.y : xb2.x) - mu) * r : 0.f;
                            const float gA = fmaf(dA, c.x, dB * c.y);
                            const float gB = fmaf(dB, c.x, -dA * c.y);
                            tA[e & 3] = gA * xA;
                            tB[e & 3] = gB * xB;
                            dot = fmaf(gA * g[L.eA + e], xA, dot);
                            dot = fmaf(gB * g[L.eB + e], xB, dot);
                            if (LN) sh += gA * g[L.eA + e] + gB * g[L.eB + e];
                        }
                    }
                    float4 &sa = acc[qd][lane];
                    float4 &sb = acc[V / 4 + qd][lane];
                    float4 va = sa, vb = sb;
                    va.x += tA[0]; va.y += tA[1]; va.z += tA[2]; va.w += tA[3];
                    vb.x += tB[0]; vb.y += tB[1]; vb.z += tB[2]; vb.w += tB[3];
                    sa = va;
                    sb = vb;
                }
                dot = group_sum<LPR>(dot) * inv_d;
                const float mh = LN ? group_sum<LPR>(sh) * inv_d : 0.f;
                if (L.on && h < H) {
                    // walk 2: dx = r (h - xh * dot)
                    Vec16 oa, ob;
#pragma unroll
                    for (int k2 = 0; k2 < V / 2; ++k2) {
                        const float2 xa2 = IO::get2(xa[pp], k2), xb2 = IO::get2(xb[pp], k2);
                        const float2 da2 = IO::get2(da[pp], k2), db2 = IO::get2(db[pp], k2);
                        float outA[2], outB[2];
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const int e = 2 * k2 + q;
                            const float2 c = lane_cs(cs, L.rot, L.eA + e);
                            const float dA = q ? da2.y : da2.x, dB = q ? db2.y : db2.x;
                            const float xA = ((q ? xa2.y : xa2.x) - mu) * r;
                            const float xB = L.onB ? ((q ? xb2.y : xb2.x) - mu) * r : 0.f;
                            const float hA = fmaf(dA, c.x, dB * c.y) * g[L.eA + e];
                            const float hB = fmaf(dB, c.x, -dA * c.y) * g[L.eB + e];
                            outA[q] = r * fmaf(-xA, dot, LN ? hA - mh : hA);
                            outB[q] = r * fmaf(-xB, dot, LN ? hB - mh : hB);
                        }
                        IO::put2(oa, k2, outA[0], outA[1]);
                        IO::put2(ob, k2, outB[0], outB[1]);
                    }
                    const int hh = isq ? h : h - a.Hq;
                    char *out = (char *)(isq ? a.dq : a.dk) + t * (isq ? a.dqts : a.dkts) + hh * rowb;
                    st16(out + offA, oa);
                    if (L.onB) st16(out + offB, ob);
                }
            }
        }
        __syncwarp();  // every lane has read the (cos, sin) table
    }

    // dgamma: each lane's private sums, then the lanes of the same unit across
    // the warp's row slots (shuffles), then the CTA's warps (shared atomics),
    // then one global atomic pass per CTA.
    __syncwarp();
#pragma unroll
    for (int z = 0; z < 2; ++z) {
        float v[2 * V];
#pragma unroll
        for (int k = 0; k < V / 2; ++k) {
            const float4 f = s_acc[z][warp][k][lane];
            v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
        }
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
            for (int j = 0; j < 2 * V; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], o);
        }
        if (L.slot == 0 && L.on) {
#pragma unroll
            for (int e = 0; e < V; ++e) {
                atomicAdd(&s_dg[z][L.eA + e], v[e]);
                if (L.onB) atomicAdd(&s_dg[z][L.eB + e], v[V + e]);
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < a.D; i += kThreads) {
        if (a.dgq && a.Hq) atomicAdd(a.dgq + i, s_dg[0][i]);
        if (a.dgk && a.Hkv) atomicAdd(a.dgk + i, s_dg[1][i]);
    }
}

}  // namespace qknr
