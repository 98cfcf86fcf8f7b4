// Pipelined sm_100a kernels of the fused QK-RMSNorm + rotate-half RoPE.
//
// Same arithmetic as qknr_kernels.cuh; what changes is how bytes reach the
// SMs. A persistent CTA owns a contiguous run of tokens and streams it in
// tiles of TT tokens through a ring of NS shared-memory stages:
//
//  * warp NCW is the producer: one lane arms the stage's "full" mbarrier
//    with the expected byte count and issues bulk asynchronous copies
//    (cp.async.bulk, the TMA engine, no tensor map: every block of a tile is
//    one contiguous run of global memory) for the tile's Q rows and K rows
//    (and, backward, the upstream gradients and saved inverse RMS); its 32
//    lanes meanwhile compute the tile's rotary (cos, sin) table into the
//    stage, then all arrive on "full";
//  * warps 0..NCW-1 are consumers: they wait on "full", walk the tile's rows
//    (row passes dealt round-robin across the consumer warps, continuing
//    across tiles), write results straight to global memory with 16-byte
//    stores, and arrive on the stage's "empty" mbarrier so the producer can
//    refill it.
//
// Memory parallelism therefore comes from the copy engine (NS stages of
// ~16-32 KB in flight per CTA) rather than from registers, and the consumer
// registers hold gamma, the row and the dgamma partial sums in fp32, with
// packed FP32x2 arithmetic (FFMA2/FMUL2) on element pairs.
//
// Every mbarrier wait is bounded (about 2-4 s of SM clock cycles); on expiry
// the thread records an error in g_qknr_pipe_error and leaves its loop, and
// the producers wait (again bounded) for the copies they issued before the
// CTA exits.
#pragma once

#include "qknr_kernels.cuh"

namespace qknr {

constexpr int kMaxStages = 8;
constexpr int kMaxTileTokens = 32;
constexpr long long kWaitLimitCycles = 4000000000ll;  // ~2 s per wait at 1.9 GHz

// Sticky error flag of the pipelined kernels (bit 0: a wait timed out).
__device__ unsigned int g_qknr_pipe_error;

struct PipeGeom {
    int TT;            // tokens per tile (stage)
    int NS;            // stages in the ring
    int stage_bytes;   // bytes per stage (multiple of 128)
    int off_k;         // stage offsets: K rows of x
    int off_dq, off_dk;  // backward: upstream gradients of Q and K rows
    int off_cs;        // (cos, sin) table, TT * R/2 float2
    int off_rq, off_rk;  // backward: saved inverse RMS of Q and K rows
    uint32_t mq, mk;   // jj / Hq == umulhi(jj, mq) (mq == 0: Hq == 1); same for Hkv
    int64_t tpc;       // tokens per CTA (a multiple of TT)
};

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// One bounded-time test of the phase; a waiting thread may be suspended by
// the hardware (up to the hint) instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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
// Wait until the phase of parity `parity` has completed, for at most
// kWaitLimitCycles SM clock cycles (about 2-4 s; the cycle counter is cheap
// to read, unlike the global timer); false on expiry, with the error flag
// set. After a few tries a waiting warp may sleep between tests (backing off
// from 32 ns to `max_sleep` ns) so waiters leave the issue slots to the warps
// doing work.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t max_sleep = 256) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long c0 = clock64();
    uint32_t nap = 32;
#pragma unroll 1
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if (n > 2 && max_sleep) {
            __nanosleep(nap);
            nap = nap < max_sleep ? nap * 2 : max_sleep;
        }
        if ((n & 255u) == 0 && clock64() - c0 > kWaitLimitCycles) {
            atomicOr(&g_qknr_pipe_error, 1u);
            return false;
        }
    }
}
// Named barrier over the consumer warps only (id 1; id 0 is __syncthreads).
__device__ __forceinline__ void consumers_sync(int nthreads) {
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// Bulk copy global -> this CTA's shared memory, completion counted in bytes
// on `bar`. dst, src and bytes are multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}
// 16-byte store to global memory, streaming (written once, not re-read).
__device__ __forceinline__ void stg16(void *p, const Vec16 &v) {
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
}
__device__ __forceinline__ Vec16 lds16(const unsigned char *p) {
    const uint4 v = *reinterpret_cast<const uint4 *>(p);
    Vec16 r;
    r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
    return r;
}

// Everything a CTA knows about its run of tokens.
struct Run {
    int64_t t_lo, t_hi;
    int ntiles;
    __device__ __forceinline__ Run(int64_t T, const PipeGeom &g) {
        t_lo = (int64_t)blockIdx.x * g.tpc;
        t_hi = min(T, t_lo + g.tpc);
        ntiles = t_hi > t_lo ? (int)((t_hi - t_lo + g.TT - 1) / g.TT) : 0;
    }
};

// Producer: positions of a tile's tokens, one per lane (TT <= 32): the given
// id, else s within the batch row, from the row position s0 of the tile's
// first token.
__device__ __forceinline__ int32_t tile_pos(const int32_t *ids, int S, int64_t t0, int s0, int na,
                                            int lane) {
    if (lane >= na) return 0;
    if (ids) return ids[t0 + lane];
    const int s = s0 + lane;
    return s >= S ? s - S * (s / S) : s;
}

// (cos, sin) tables. Angles come in pairs (2P, 2P+1) stored as one float4
// (c_2P, c_2P+1, s_2P, s_2P+1), so a lane gets ready-made float2 operands.
// Unit u reads the V/2 pairs P = (V/2) u + k; within its block the pairs
// are rotated by (u * V/2) / 8 so that the eight lanes of a shared-memory
// phase hit eight distinct 16-byte bank groups.
template <int V>
__device__ __forceinline__ int cs_slot(int P) {
    constexpr int W = V / 2;
    const int u = P / W, k = P % W;
    return W * u + (k + ((u * W) >> 3)) % W;
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

// Producers: fill the stage's (cos, sin) table for na tokens. The NW = 32 *
// NPW producer lanes each own one angle index i and one token group; with
// R/2 <= NW there are G = NW / (R/2) groups and worker (grp, i) takes tokens
// grp, grp + G, ...; with R/2 > NW each worker loops over i in steps of NW
// and over all tokens. Lane t of every producer warp holds the position of
// token t in `pos`; a shuffle hands it out, and every loop has a trip count
// uniform across the warp so the shuffles are well defined.
template <int V, int NPW>
__device__ __forceinline__ void tile_angles(float *__restrict__ cs,
                                            const uint64_t *__restrict__ s_step, int half,
                                            int na, int32_t pos, int pw, int lane) {
    constexpr int NW = 32 * NPW;
    const int w = pw * 32 + lane;
    if (half <= NW) {
        const int G = NW / half;
        const int grp = w / half, i = w - grp * half;
        const bool on = grp < G;
        const uint64_t F = on ? s_step[i] : 0ull;
        float *q = cs + 4 * cs_slot<V>(i >> 1) + (i & 1);
#pragma unroll 4
        for (int tb = 0; tb < na; tb += G) {
            const int tl = tb + grp;
            const int32_t m = __shfl_sync(0xffffffffu, pos, tl & 31);
            const float2 v = rope_cos_sin_fixed(m, F);
            if (on && tl < na) {
                q[tl * half * 2] = v.x;
                q[tl * half * 2 + 2] = v.y;
            }
        }
    } else {
        for (int ib = 0; ib < half; ib += NW) {
            const int i = ib + w;
            const bool on = i < half;
            const uint64_t F = on ? s_step[i] : 0ull;
            float *q = cs + 4 * cs_slot<V>(on ? (i >> 1) : 0) + (i & 1);
#pragma unroll 4
            for (int tl = 0; tl < na; ++tl) {
                const int32_t m = __shfl_sync(0xffffffffu, pos, tl);
                const float2 v = rope_cos_sin_fixed(m, F);
                if (on) {
                    q[tl * half * 2] = v.x;
                    q[tl * half * 2 + 2] = v.y;
                }
            }
        }
    }
}

// Named barrier over the producer warps only (id 2).
__device__ __forceinline__ void producers_sync(int nthreads) {
    asm volatile("bar.sync 2, %0;" ::"r"(nthreads) : "memory");
}

// Consumer: the V/2 (cos, sin) float4 of unit u for one token; (1, 1, 0, 0)
// on pass-through units.
template <int V>
__device__ __forceinline__ void unit_table(const float4 *tok, bool rot, int u, float4 *cs) {
    constexpr int W = V / 2;
    if (rot) {
        const float4 *t = tok + W * u;
        const int sh = (u * W) >> 3;
#pragma unroll
        for (int k = 0; k < W; ++k) cs[k] = t[(k + sh) % W];
    } else {
#pragma unroll
        for (int k = 0; k < W; ++k) cs[k] = make_float4(1.f, 1.f, 0.f, 0.f);
    }
}

__device__ __forceinline__ float2 neg2(float2 v) { return make_float2(-v.x, -v.y); }
__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }

// Where row j of a tile lives: Q rows first (na * Hq), then K rows.
struct TileRow {
    bool isq;
    int jj;  // row index within its tensor's block of the tile
    int tl;  // token within the tile
    __device__ __forceinline__ TileRow(int j, int rows_q, const PipeGeom &g) {
        isq = j < rows_q;
        jj = isq ? j : j - rows_q;
        const uint32_t m = isq ? g.mq : g.mk;
        tl = m ? (int)__umulhi((uint32_t)jj, m) : jj;
    }
};

// U units per lane: lane (slot, u) owns units u + q * LPR, q < U. Unit w
// holds the two 16-byte vectors of a head row described in
// qknr_kernels.cuh (rotary partners in one unit); units past D / 2V are
// off (they read element 0 and are masked out).
template <int LPR, int V, int U> struct Units {
    int u, slot;
    bool on[U], rot[U];
    int eA[U], eB[U];
    float mask[U];
    __device__ __forceinline__ Units(int lane, int D, int R) {
        u = lane & (LPR - 1);
        slot = lane / LPR;
#pragma unroll
        for (int q = 0; q < U; ++q) {
            const UnitGeom<V> G(u + q * LPR, D, R);
            on[q] = G.on;
            rot[q] = G.rot;
            eA[q] = G.eA;
            eB[q] = G.eB;
            mask[q] = G.on ? 1.f : 0.f;
        }
    }
};

// Per-CTA table of gamma in unit order: s_gl[z][k][w] holds elements
// 4k..4k+3 of unit w's A vector (k < V/4) or of its B vector, as fp32, so
// a warp reads it without bank conflicts.
template <typename T, int V>
__device__ __forceinline__ void fill_unit_gamma(float4 (*s_gl)[V / 2][32], const void *gq,
                                                const void *gk, int D, int R, int tid, int nthreads) {
    constexpr int W = V / 2;
    for (int idx = tid; idx < 2 * W * 32; idx += nthreads) {
        const int z = idx / (W * 32), k = (idx / 32) % W, w = idx % 32;
        const UnitGeom<V> L(w, D, R);
        const void *gp = z ? gk : gq;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (L.on && gp) {
            const int e = (k < W / 2 ? L.eA + 4 * k : L.eB + 4 * (k - W / 2));
            v = make_float4(Io<T>::to_f32(gp, e), Io<T>::to_f32(gp, e + 1),
                            Io<T>::to_f32(gp, e + 2), Io<T>::to_f32(gp, e + 3));
        }
        s_gl[z][k][w] = v;
    }
}

// Barrier set-up, before the CTA-wide __syncthreads.
template <int NCW, int NPW>
__device__ __forceinline__ void init_barriers(uint32_t full0, uint32_t empty0, const PipeGeom &g) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < g.NS; ++s) {
            mbar_init(full0 + 8 * s, 32 * NPW);
            mbar_init(empty0 + 8 * s, NCW);
        }
        fence_mbar_init();
    }
}

// ================================================================== forward
// Per row: y_A = r (u_A c - u_B s), y_B = r (u_B c + u_A s), u = x * gamma.
template <typename T, int LPR, int U, int NCW, int NPW>
__global__ void __launch_bounds__((NCW + NPW) * 32, 1)
qknr_fwd_pipe_kernel(const FwdArgs a, const PipeGeom g) {
    using IO = Io<T>;
    constexpr int V = IO::V, W = V / 2;
    constexpr int SLOTS = 32 / LPR;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
    __shared__ uint64_t s_step[kMaxHalf];
    __shared__ __align__(16) float4 s_gl[2][W][32];
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(&bars[0]), empty0 = smem_u32(&bars[kMaxStages]);
    init_barriers<NCW, NPW>(full0, empty0, g);
    if (threadIdx.x == 0) s_abort = 0;
    __syncthreads();

    const Run run(a.T, g);
    const int rowb = a.D * (int)sizeof(T);
    const int half = a.R >> 1;

    if (warp < NPW) {
        // ----------------------------------------------------- producers
        // (the lowest warp ids, which the warp schedulers favour, so the
        // tables are ready before the consumers need them)
        const int pw = warp;
        const uint64_t pol = evict_first_policy();
        // copies of tile `it` into its stage, counted on the stage's barrier
        auto issue = [&](int it) {
            const int s = it % g.NS;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const uint32_t bq = (uint32_t)(na * a.Hq * rowb), bk = (uint32_t)(na * a.Hkv * rowb);
            const uint32_t bar = full0 + 8 * s;
            mbar_expect_tx(bar, bq + bk);
            if (bq) bulk_g2s(smem_u32(st), (const char *)a.q + t0 * a.Hq * rowb, bq, bar, pol);
            if (bk) bulk_g2s(smem_u32(st + g.off_k), (const char *)a.k + t0 * a.Hkv * rowb, bk, bar, pol);
        };
        // the first ring of copies goes out before any table is built
        const int first = min(g.NS, run.ntiles);
        if (pw == 0 && lane == 0)
            for (int it = 0; it < first; ++it) issue(it);
        for (int i = pw * 32 + lane; i < half; i += 32 * NPW) s_step[i] = turn_step(i, a.R, a.theta);
        producers_sync(32 * NPW);
        int issued = first;
        int s_row = run.ntiles ? (int)(run.t_lo % a.S) : 0;  // row position of the tile's first token
        int32_t pos_next = tile_pos(a.pos, a.S, run.t_lo, s_row,
                                    (int)min((int64_t)g.TT, run.t_hi - run.t_lo), lane);
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            const int32_t pos = pos_next;
            s_row += g.TT;
            while (s_row >= a.S) s_row -= a.S;
            if (it + 1 < run.ntiles) {
                const int64_t t1 = t0 + g.TT;
                pos_next = tile_pos(a.pos, a.S, t1, s_row, (int)min((int64_t)g.TT, run.t_hi - t1), lane);
            }
            if (it >= first) {
                // warp 0 waits for the stage and refills it; the others block
                // on a hardware barrier until it has (no spinning)
                bool ok = true;
                if (pw == 0) {
                    ok = mbar_wait(empty0 + 8 * s, ((it / g.NS) & 1) ^ 1, 512);
                    if (ok && lane == 0) issue(it);
                    if (!ok) s_abort = 1;
                }
                producers_sync(32 * NPW);
                if (s_abort) break;
                issued = it + 1;
            }
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            tile_angles<V, NPW>(reinterpret_cast<float *>(st + g.off_cs), s_step, half, na, pos, pw, lane);
            __syncwarp();
            mbar_arrive(full0 + 8 * s);
        }
        // the copies of the last stages must land before the CTA may exit
        for (int it = max(0, issued - g.NS); it < issued; ++it)
            mbar_wait(full0 + 8 * (it % g.NS), (it / g.NS) & 1);
    } else {
        // ------------------------------------------------------ consumers
        fill_unit_gamma<T, V>(s_gl, a.Hq ? a.gq : nullptr, a.Hkv ? a.gk : nullptr, a.D, a.R,
                              threadIdx.x - NPW * 32, NCW * 32);
        consumers_sync(NCW * 32);
        const Units<LPR, V, U> L(lane, a.D, a.R);
        int offA[U], offB[U];
#pragma unroll
        for (int q = 0; q < U; ++q) {
            offA[q] = L.eA[q] * (int)sizeof(T);
            offB[q] = L.eB[q] * (int)sizeof(T);
        }
        const float inv_d = 1.0f / (float)a.D;
        int pc = 0;  // passes dealt before this tile, mod NCW
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            if (!mbar_wait(full0 + 8 * s, (it / g.NS) & 1, 0)) break;
            const unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            const int rows_q = na * a.Hq, rows = na * (a.Hq + a.Hkv);
            char *out_q = (char *)a.qo + t0 * a.Hq * rowb;   // the tile's first rows
            char *out_k = (char *)a.ko + t0 * a.Hkv * rowb;
            float *r_q = a.rq + t0 * a.Hq;
            float *r_k = a.rk + t0 * a.Hkv;
            const float4 *cs_tile = reinterpret_cast<const float4 *>(st + g.off_cs);
            const int npass = (rows + SLOTS - 1) / SLOTS;
            int p = (warp - NPW) - pc;
            if (p < 0) p += NCW;
            for (; p < npass; p += NCW) {
                const int j = p * SLOTS + L.slot;
                const bool valid = j < rows;
                const TileRow tr(valid ? j : 0, rows_q, g);
                const unsigned char *src = st + (tr.isq ? 0 : g.off_k) + tr.jj * rowb;
                Vec16 xa[U], xb[U];
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    xa[q] = lds16(src + offA[q]);
                    xb[q] = lds16(src + offB[q]);
                }
                float ss = 0.f;
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const float2 va = IO::get2(xa[q], k), vb = IO::get2(xb[q], k);
                        s0 = __ffma2_rn(va, va, s0);
                        s1 = __ffma2_rn(vb, vb, s1);
                    }
                    ss = fmaf(L.mask[q], (s0.x + s1.x) + (s0.y + s1.y), ss);
                }
                ss = group_sum<LPR>(ss);
                const float r = rsqrtf(fmaf(ss, inv_d, a.eps));
                const float2 r2 = make_float2(r, r);
                const float4 *tok = cs_tile + tr.tl * (half >> 1);
                char *out = (tr.isq ? out_q : out_k) + tr.jj * rowb;
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    float4 cs[W], gv[W];
                    unit_table<V>(tok, L.rot[q], L.u + q * LPR, cs);
#pragma unroll
                    for (int k = 0; k < W; ++k) gv[k] = s_gl[tr.isq ? 0 : 1][k][L.u + q * LPR];
                    Vec16 ya, yb;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                        const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                        const float2 c = lo2(cs[k]), sn = hi2(cs[k]);
                        const float2 ua = __fmul2_rn(IO::get2(xa[q], k), ga);
                        const float2 ub = __fmul2_rn(IO::get2(xb[q], k), gb);
                        const float2 pa = __ffma2_rn(ua, c, __fmul2_rn(ub, neg2(sn)));
                        const float2 pb = __ffma2_rn(ub, c, __fmul2_rn(ua, sn));
                        const float2 oa = __fmul2_rn(pa, r2), ob = __fmul2_rn(pb, r2);
                        IO::put2(ya, k, oa.x, oa.y);
                        IO::put2(yb, k, ob.x, ob.y);
                    }
                    if (valid && L.on[q]) {
                        stg16(out + offA[q], ya);
                        stg16(out + offB[q], yb);
                    }
                }
                if (valid && L.u == 0) __stcs((tr.isq ? r_q : r_k) + tr.jj, r);
            }
            pc = (pc + npass) % NCW;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
        }
    }
}

// ================================================================= backward
// Per row: g = R^T dy; xh = x r; h = g gamma; dgamma += g xh;
// dx = r (h - xh <h, xh> / D). One unit per lane: the dgamma partial sums
// of both tensors stay in registers for the whole run.
template <typename T, int LPR, int NCW, int NPW>
__global__ void __launch_bounds__((NCW + NPW) * 32, 1)
qknr_bwd_pipe_kernel(const BwdArgs a, const PipeGeom g) {
    using IO = Io<T>;
    constexpr int V = IO::V, W = V / 2;
    constexpr int SLOTS = 32 / LPR;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
    __shared__ uint64_t s_step[kMaxHalf];
    __shared__ __align__(16) float4 s_gl[2][W][32];
    __shared__ volatile int s_abort;
    __shared__ float s_dg[2][kMaxD];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(&bars[0]), empty0 = smem_u32(&bars[kMaxStages]);
    init_barriers<NCW, NPW>(full0, empty0, g);
    if (threadIdx.x == 0) s_abort = 0;
    for (int i = threadIdx.x; i < 2 * kMaxD; i += blockDim.x) (&s_dg[0][0])[i] = 0.f;
    __syncthreads();

    const Run run(a.T, g);
    const int rowb = a.D * (int)sizeof(T);
    const int half = a.R >> 1;

    if (warp < NPW) {
        // ----------------------------------------------------- producers
        // (the lowest warp ids, which the warp schedulers favour, so the
        // tables are ready before the consumers need them)
        const int pw = warp;
        const uint64_t pol = evict_first_policy();
        auto issue = [&](int it) {
            const int s = it % g.NS;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const uint32_t bq = (uint32_t)(na * a.Hq * rowb), bk = (uint32_t)(na * a.Hkv * rowb);
            // inverse RMS: the 16-byte multiple of each block (the
            // producers fill in a tail of up to three floats)
            const uint32_t brq = (uint32_t)(na * a.Hq * 4) & ~15u;
            const uint32_t brk = (uint32_t)(na * a.Hkv * 4) & ~15u;
            const uint32_t bar = full0 + 8 * s;
            mbar_expect_tx(bar, 2 * (bq + bk) + brq + brk);
            if (bq) {
                bulk_g2s(smem_u32(st), (const char *)a.q + t0 * a.Hq * rowb, bq, bar, pol);
                bulk_g2s(smem_u32(st + g.off_dq), (const char *)a.dqo + t0 * a.Hq * rowb, bq, bar, pol);
            }
            if (bk) {
                bulk_g2s(smem_u32(st + g.off_k), (const char *)a.k + t0 * a.Hkv * rowb, bk, bar, pol);
                bulk_g2s(smem_u32(st + g.off_dk), (const char *)a.dko + t0 * a.Hkv * rowb, bk, bar, pol);
            }
            if (brq) bulk_g2s(smem_u32(st + g.off_rq), a.rq + t0 * a.Hq, brq, bar, pol);
            if (brk) bulk_g2s(smem_u32(st + g.off_rk), a.rk + t0 * a.Hkv, brk, bar, pol);
        };
        const int first = min(g.NS, run.ntiles);
        if (pw == 0 && lane == 0)
            for (int it = 0; it < first; ++it) issue(it);
        for (int i = pw * 32 + lane; i < half; i += 32 * NPW) s_step[i] = turn_step(i, a.R, a.theta);
        producers_sync(32 * NPW);
        int issued = first;
        int s_row = run.ntiles ? (int)(run.t_lo % a.S) : 0;  // row position of the tile's first token
        int32_t pos_next = tile_pos(a.pos, a.S, run.t_lo, s_row,
                                    (int)min((int64_t)g.TT, run.t_hi - run.t_lo), lane);
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            const int32_t pos = pos_next;
            s_row += g.TT;
            while (s_row >= a.S) s_row -= a.S;
            if (it + 1 < run.ntiles) {
                const int64_t t1 = t0 + g.TT;
                pos_next = tile_pos(a.pos, a.S, t1, s_row, (int)min((int64_t)g.TT, run.t_hi - t1), lane);
            }
            if (it >= first) {
                // warp 0 waits for the stage and refills it; the others block
                // on a hardware barrier until it has (no spinning)
                bool ok = true;
                if (pw == 0) {
                    ok = mbar_wait(empty0 + 8 * s, ((it / g.NS) & 1) ^ 1, 512);
                    if (ok && lane == 0) issue(it);
                    if (!ok) s_abort = 1;
                }
                producers_sync(32 * NPW);
                if (s_abort) break;
                issued = it + 1;
            }
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            if (pw == 0) {
                // inverse-RMS floats past the 16-byte multiple (at most three
                // per tensor, only in a tensor's last, partial tile)
                const int nq = na * a.Hq, nk = na * a.Hkv;
                const int cq = (nq * 4 & ~15) / 4, ck = (nk * 4 & ~15) / 4;
                if (lane < nq - cq)
                    reinterpret_cast<float *>(st + g.off_rq)[cq + lane] = a.rq[t0 * a.Hq + cq + lane];
                if (lane >= 4 && lane - 4 < nk - ck)
                    reinterpret_cast<float *>(st + g.off_rk)[ck + lane - 4] = a.rk[t0 * a.Hkv + ck + lane - 4];
            }
            tile_angles<V, NPW>(reinterpret_cast<float *>(st + g.off_cs), s_step, half, na, pos, pw, lane);
            __syncwarp();
            mbar_arrive(full0 + 8 * s);
        }
        for (int it = max(0, issued - g.NS); it < issued; ++it)
            mbar_wait(full0 + 8 * (it % g.NS), (it / g.NS) & 1);
    } else {
        // ------------------------------------------------------ consumers
        fill_unit_gamma<T, V>(s_gl, a.Hq ? a.gq : nullptr, a.Hkv ? a.gk : nullptr, a.D, a.R,
                              threadIdx.x - NPW * 32, NCW * 32);
        consumers_sync(NCW * 32);
        const Units<LPR, V, 1> L(lane, a.D, a.R);
        const int offA = L.eA[0] * (int)sizeof(T), offB = L.eB[0] * (int)sizeof(T);
        const int uu = L.u;
        const float inv_d = 1.0f / (float)a.D;
        // dgamma partial sums: [k] = elements (eA + 2k, eA + 2k + 1), same for B
        float2 aqa[W], aqb[W], aka[W], akb[W];
#pragma unroll
        for (int k = 0; k < W; ++k) aqa[k] = aqb[k] = aka[k] = akb[k] = make_float2(0.f, 0.f);
        int pc = 0;
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            if (!mbar_wait(full0 + 8 * s, (it / g.NS) & 1, 0)) break;
            const unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const int64_t t0 = run.t_lo + (int64_t)it * g.TT;
            const int na = (int)min((int64_t)g.TT, run.t_hi - t0);
            const int rows_q = na * a.Hq, rows = na * (a.Hq + a.Hkv);
            char *out_q = (char *)a.dq + t0 * a.Hq * rowb;
            char *out_k = (char *)a.dk + t0 * a.Hkv * rowb;
            const float4 *cs_tile = reinterpret_cast<const float4 *>(st + g.off_cs);
            const int npass = (rows + SLOTS - 1) / SLOTS;
            int p = (warp - NPW) - pc;
            if (p < 0) p += NCW;
            for (; p < npass; p += NCW) {
                const int j = p * SLOTS + L.slot;
                const bool valid = j < rows && L.on[0];
                const TileRow tr(j < rows ? j : 0, rows_q, g);
                const unsigned char *xs = st + (tr.isq ? 0 : g.off_k) + tr.jj * rowb;
                const unsigned char *ds = st + (tr.isq ? g.off_dq : g.off_dk) + tr.jj * rowb;
                const Vec16 xa = lds16(xs + offA), xb = lds16(xs + offB);
                const Vec16 da = lds16(ds + offA), db = lds16(ds + offB);
                float r = reinterpret_cast<const float *>(st + (tr.isq ? g.off_rq : g.off_rk))[tr.jj];
                r = valid ? r : 0.f;  // rows past the tile and off lanes add nothing
                float4 cs[W], gv[W];
                unit_table<V>(cs_tile + tr.tl * (half >> 1), L.rot[0], uu, cs);
#pragma unroll
                for (int k = 0; k < W; ++k) gv[k] = s_gl[tr.isq ? 0 : 1][k][uu];
                const float2 r2 = make_float2(r, r);
                float2 ha[W], hb[W], xha[W], xhb[W];
                float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                    const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                    const float2 c = lo2(cs[k]), sn = hi2(cs[k]);
                    const float2 dA = IO::get2(da, k), dB = IO::get2(db, k);
                    xha[k] = __fmul2_rn(IO::get2(xa, k), r2);
                    xhb[k] = __fmul2_rn(IO::get2(xb, k), r2);
                    const float2 gA = __ffma2_rn(dA, c, __fmul2_rn(dB, sn));
                    const float2 gB = __ffma2_rn(dB, c, __fmul2_rn(dA, neg2(sn)));
                    if (tr.isq) {
                        aqa[k] = __ffma2_rn(gA, xha[k], aqa[k]);
                        aqb[k] = __ffma2_rn(gB, xhb[k], aqb[k]);
                    } else {
                        aka[k] = __ffma2_rn(gA, xha[k], aka[k]);
                        akb[k] = __ffma2_rn(gB, xhb[k], akb[k]);
                    }
                    ha[k] = __fmul2_rn(gA, ga);
                    hb[k] = __fmul2_rn(gB, gb);
                    d0 = __ffma2_rn(ha[k], xha[k], d0);
                    d1 = __ffma2_rn(hb[k], xhb[k], d1);
                }
                const float dot = group_sum<LPR>((d0.x + d1.x) + (d0.y + d1.y)) * inv_d;
                if (valid) {
                    const float2 nd = make_float2(-dot, -dot);
                    Vec16 oa, ob;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const float2 va = __fmul2_rn(__ffma2_rn(xha[k], nd, ha[k]), r2);
                        const float2 vb = __fmul2_rn(__ffma2_rn(xhb[k], nd, hb[k]), r2);
                        IO::put2(oa, k, va.x, va.y);
                        IO::put2(ob, k, vb.x, vb.y);
                    }
                    char *out = (tr.isq ? out_q : out_k) + tr.jj * rowb;
                    stg16(out + offA, oa);
                    stg16(out + offB, ob);
                }
            }
            pc = (pc + npass) % NCW;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
        }
        // dgamma: lanes of one unit across the warp's row slots, then the
        // CTA's consumer warps (shared atomics)
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
            for (int k = 0; k < W; ++k) {
                aqa[k].x += __shfl_xor_sync(0xffffffffu, aqa[k].x, o);
                aqa[k].y += __shfl_xor_sync(0xffffffffu, aqa[k].y, o);
                aqb[k].x += __shfl_xor_sync(0xffffffffu, aqb[k].x, o);
                aqb[k].y += __shfl_xor_sync(0xffffffffu, aqb[k].y, o);
                aka[k].x += __shfl_xor_sync(0xffffffffu, aka[k].x, o);
                aka[k].y += __shfl_xor_sync(0xffffffffu, aka[k].y, o);
                akb[k].x += __shfl_xor_sync(0xffffffffu, akb[k].x, o);
                akb[k].y += __shfl_xor_sync(0xffffffffu, akb[k].y, o);
            }
        }
        if (L.slot == 0 && L.on[0]) {
            const int eA = L.eA[0], eB = L.eB[0];
#pragma unroll
            for (int k = 0; k < W; ++k) {
                atomicAdd(&s_dg[0][eA + 2 * k], aqa[k].x);
                atomicAdd(&s_dg[0][eA + 2 * k + 1], aqa[k].y);
                atomicAdd(&s_dg[0][eB + 2 * k], aqb[k].x);
                atomicAdd(&s_dg[0][eB + 2 * k + 1], aqb[k].y);
                atomicAdd(&s_dg[1][eA + 2 * k], aka[k].x);
                atomicAdd(&s_dg[1][eA + 2 * k + 1], aka[k].y);
                atomicAdd(&s_dg[1][eB + 2 * k], akb[k].x);
                atomicAdd(&s_dg[1][eB + 2 * k + 1], akb[k].y);
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < a.D; i += blockDim.x) {
        if (a.dgq && a.Hq) atomicAdd(a.dgq + i, s_dg[0][i]);
        if (a.dgk && a.Hkv) atomicAdd(a.dgk + i, s_dg[1][i]);
    }
}

}  // namespace qknr
