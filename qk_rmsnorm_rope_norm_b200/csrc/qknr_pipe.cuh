// Pipelined sm_100a kernels of the fused QK-RMSNorm + rotate-half RoPE.
//
// Same arithmetic as qknr_kernels.cuh; what changes is how bytes reach the
// SMs. A persistent CTA owns a contiguous run of tokens and streams it in
// tiles through a ring of NS shared-memory stages (the forward's first tile
// holds half the tokens of the others, see Run):
//
//  * warps 0..NPW-1 are the producers: lane 0 of warp 0 arms the stage's
//    "full" mbarrier with the expected byte count and issues asynchronous
//    bulk copies for the tile's Q rows and K rows (and, backward, the
//    upstream gradients and saved inverse RMS): cp.async.bulk, the TMA
//    engine, one contiguous run of global memory a block, or a 3-D tensor
//    copy when Q / K are strided slices of a fused QKV buffer. All NPW * 32
//    producer lanes meanwhile compute the tile's rotary (cos, sin) table
//    into the stage, then arrive on "full";
//  * the NCW warps after them are consumers: they wait on "full", walk the
//    tile's rows (row passes dealt round-robin across the consumer warps,
//    continuing across tiles), write results straight to global memory
//    with 16-byte stores, and arrive on the stage's "empty" mbarrier so the
//    producers can refill it.
//
// Memory parallelism therefore comes from the copy engine (two or three
// stages of ~80 KB in flight per CTA) rather than from registers, and the
// consumer registers hold the row and the dgamma partial sums in fp32
// (gamma and the angle table are read from shared memory), with packed
// FP32x2 arithmetic (FFMA2/FMUL2) on element pairs.
//
// Every mbarrier wait is bounded (about 2-4 s of SM clock cycles); on expiry
// the thread records an error in g_qknr_pipe_error and leaves its loop, and
// the producers wait (again bounded) for the copies they issued before the
// CTA exits.
#pragma once

#include <cuda.h>  // CUtensorMap (the type only)

#include "qknr_kernels.cuh"

namespace qknr {

constexpr int kMaxStages = 8;
constexpr int kMaxTileTokens = 32;
constexpr long long kWaitLimitCycles = 4000000000ll;  // ~2 s per wait at 1.9 GHz

// Sticky error flag of the pipelined kernels (bit 0: a wait timed out;
// bit 1: shared memory unfit for tensor copies, nothing computed).
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
    int64_t tpc;       // tokens per CTA
    int tmap;          // bit 0 (1): Q (K) rows arrive by 3-D tensor copy (strided input)
    int h0;            // tokens of a CTA's first tile when shorter than TT (0: TT)
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
// `limit` SM clock cycles (by default kWaitLimitCycles, about 2-4 s; the
// cycle counter is cheap to read, unlike the global timer); false on expiry,
// with the error flag set. After a few tries a waiting warp may sleep between
// tests (backing off from 32 ns to `max_sleep` ns) so waiters leave the issue
// slots to the warps doing work. The clock is read every 256th test, and
// every test is itself bounded (its suspend hint), so the wait ends.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t max_sleep = 256,
                                          long long limit = kWaitLimitCycles) {
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
        if ((n & 255u) == 0 && clock64() - c0 > limit) {
            atomicOr(&g_qknr_pipe_error, 1u);
            return false;
        }
    }
}

// Diagnostic: one thread waits, with mbar_wait and a limit of `limit`
// cycles, on a barrier nothing arrives on, so the wait gives up and sets the
// error flag; the kernel then returns. It checks the timeout path without a
// fault or a hang.
__global__ void qknr_wait_selftest_kernel(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    mbar_wait(b, 0, 256, limit);
}
// Zeroes the dgamma accumulators ahead of a backward launch. Launched with
// programmatic stream serialization like the pipelined kernels, it overlaps
// the previous kernel's tail, and the backward that follows overlaps its own
// prologue with this one; two memset nodes in its place would end both
// overlaps (about 6 us of launch gaps a backward call on B200).
__global__ void __launch_bounds__(256) qknr_zero_kernel(float *a, int64_t na, float *b,
                                                        int64_t nb) {
    grid_dep_wait();  // the previous kernel of the stream may still use a or b
    grid_dep_launch();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < na + nb; i += stride) {
        if (i < na) a[i] = 0.f;
        else b[i - na] = 0.f;
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
// Tensor copy global -> this CTA's shared memory of the box at (c0, c1, c2)
// of a 3-D tensor map {D, heads, tokens} (a strided Q or K: one token's rows
// contiguous, tokens a fixed stride apart). The whole box is always counted
// on `bar`; elements past the tensor's end read as zero.
__device__ __forceinline__ void tensor_g2s(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                           int c2, uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
        : "memory");
}
// Tensor maps of strided Q and K, a kernel parameter only of the TM
// instantiations (the dense ones take an empty one).
struct TensorMaps {
    CUtensorMap q, k;
};
struct NoTensorMaps {};
template <bool TM> struct MapsArg {
    using type = NoTensorMaps;
};
template <> struct MapsArg<true> {
    using type = TensorMaps;
};
template <bool TM>
__device__ __forceinline__ const CUtensorMap *map_of(const typename MapsArg<TM>::type &m, int z) {
    if constexpr (TM) return z ? &m.k : &m.q;
    else return nullptr;
}

// First token of the tensor-copy box of a tile [t0, t0 + na) in a run ending
// at t_hi: the tile itself when it is whole, else the box that ends with the
// run (so a partial last tile re-reads the end of the previous tile instead
// of the next run's tokens), or token 0 when the run is shorter than a box.
__device__ __forceinline__ int64_t box_start(int64_t t0, int64_t t_hi, int TT) {
    return t0 + TT <= t_hi ? t0 : max((int64_t)0, t_hi - TT);
}

// 16-byte store to global memory, streaming (written once, not re-read).
__device__ __forceinline__ void stg16(void *p, const Vec16 &v) {
    __stcs(reinterpret_cast<uint4 *>(p), make_uint4(v.w[0], v.w[1], v.w[2], v.w[3]));
}
// 16-byte shared-memory loads at 32-bit shared addresses (the consumers keep
// every address in 32 bits). Volatile keeps them in order with the mbarrier
// waits and arrivals around them.
__device__ __forceinline__ Vec16 lds16(uint32_t addr) {
    Vec16 r;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3])
                 : "r"(addr));
    return r;
}
__device__ __forceinline__ float4 ldsf4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

// Everything a CTA knows about its run of tokens: tile 0 holds h0 tokens
// (a shorter first tile lets the consumers start on a partly filled ring
// instead of waiting for a whole stage), every later tile TT, the last one
// what remains.
struct Run {
    int64_t t_lo, t_hi;
    int ntiles, h0, TT;
    __device__ __forceinline__ Run(int64_t T, const PipeGeom &g) {
        t_lo = (int64_t)blockIdx.x * g.tpc;
        t_hi = min(T, t_lo + g.tpc);
        TT = g.TT;
        const int64_t L = t_hi - t_lo;
        h0 = (g.h0 > 0 && L > g.TT) ? g.h0 : g.TT;
        ntiles = L > 0 ? (L <= h0 ? 1 : 1 + (int)((L - h0 + g.TT - 1) / g.TT)) : 0;
    }
    __device__ __forceinline__ int64_t start(int it) const {
        return it == 0 ? t_lo : t_lo + h0 + (int64_t)(it - 1) * TT;
    }
    __device__ __forceinline__ int count(int it) const {
        return (int)min((int64_t)(it == 0 ? h0 : TT), t_hi - start(it));
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
    if (half <= 0) return;  // no rotary span (NoPE): no table
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

// Consumer: shared-memory byte offsets of a register pair's (cos, sin) and
// gamma operands, fixed for the kernel. The table of a token holds R/2V
// units of V/2 float4 (c_2P, c_2P+1, s_2P, s_2P+1); unit w's float4 k sits at
// W w + (k + ((w W) >> 3)) mod W (the rotation that spreads a shared-memory
// phase over eight bank groups; W = V/2); a pass-through unit reads none and
// takes (cos, sin) = (1, 0). Gamma's first vector of the pair is
// rows kb, kb + 1, ... of the fp32 table at column w (^ X in the B half), its
// second vector rows W/2 - kb, ...: a float4 row is 32 float4 (512 bytes).
template <int V, int X> struct PairOffsets {
    static constexpr int W = V / 2;
    uint32_t cs[W];   // from the token's table (rotary units)
    uint32_t g1, g2;  // gamma, first and second vector, float4 j at + j * 512
    __device__ __forceinline__ void set(int w, int kb) {
        const int sh = (w * W) >> 3;
#pragma unroll
        for (int k = 0; k < W; ++k) cs[k] = (uint32_t)(W * w + ((k + sh) & (W - 1))) * 16u;
        const int k1 = kb, k2 = W / 2 - kb;
        g1 = (uint32_t)(k1 * 32 + (w ^ (k1 >= W / 2 ? X : 0))) * 16u;
        g2 = (uint32_t)(k2 * 32 + (w ^ (k2 >= W / 2 ? X : 0))) * 16u;
    }
};

__device__ __forceinline__ float2 neg2(float2 v) { return make_float2(-v.x, -v.y); }
__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }

// Where row j of a tile lives: Q rows first (na * Hq), then K rows.
struct TileRow {
    bool isq;
    int jj;  // row index within its tensor's block of the tile
    int tl;  // token within the tile
    __device__ __forceinline__ TileRow(bool q, int j, const PipeGeom &g) {
        isq = q;
        jj = j;
        const uint32_t m = isq ? g.mq : g.mk;
        tl = m ? (int)__umulhi((uint32_t)jj, m) : jj;
    }
};

// Row passes of a tile: the Q rows, then the K rows from a fresh pass, so
// every pass is all Q or all K (the tensor is uniform across the warp).
struct TilePasses {
    int pq, npass, rows_q, rows_k;
    __device__ __forceinline__ TilePasses(int na, int Hq, int Hkv, int slots) {
        rows_q = na * Hq;
        rows_k = na * Hkv;
        pq = (rows_q + slots - 1) / slots;
        npass = pq + (rows_k + slots - 1) / slots;
    }
};

// Register pairs of a lane. Lane (slot, u) owns units u + q * LPR (q < U),
// each unit being the two 16-byte vectors of a head row described in
// qknr_kernels.cuh (rotary partners in one unit). Pair p holds unit
// u + q LPR with c = (p + slot) mod 2U, q = c mod U, and its two vectors in
// swapped order when c >= U. Load instruction k (first vectors for k < U,
// second vectors after) then reads combination (k + slot) mod 2U, so the
// rows of a shared-memory phase (rows are 128 or 256 bytes apart and would
// otherwise all hit the same banks) read distinct bank groups. A swapped
// pair computes the same rotation with the sine negated. Units past D / 2V
// are off (they read element 0 and are masked out).
template <int LPR, int V, int U> struct Pairs {
    int u, slot;
    bool on[U], rot[U];
    int w[U];               // unit index
    int first[U], second[U];  // element offsets of the pair's two vectors
    int kb[U];              // gamma-table half of the first vector (0: A, V/4: B)
    float sgn[U];           // +1, or -1 when the halves are swapped
    float mask[U];
    __device__ __forceinline__ Pairs(int lane, int D, int R) {
        u = lane & (LPR - 1);
        slot = lane / LPR;
#pragma unroll
        for (int p = 0; p < U; ++p) {
            const int c = (p + slot) % (2 * U);
            const bool sw = c >= U;
            const int q = sw ? c - U : c;
            w[p] = u + q * LPR;
            const UnitGeom<V> G(w[p], D, R);
            on[p] = G.on;
            rot[p] = G.rot;
            first[p] = sw ? G.eB : G.eA;
            second[p] = sw ? G.eA : G.eB;
            kb[p] = sw ? V / 4 : 0;
            sgn[p] = sw ? -1.f : 1.f;
            mask[p] = G.on ? 1.f : 0.f;
        }
    }
};

// Column swizzle of the gamma table: with at most 4 units per row group the
// B half is stored at column w ^ 4, which keeps a phase's reads on distinct
// banks under the pair rotation above.
template <int LPR, int U> struct GammaSwz {
    static constexpr int X = (LPR * U <= 4) ? 4 : 0;
};

// Per-CTA table of gamma in unit order: s_gl[z][k][w ^ (k >= V/4 ? X : 0)]
// holds elements 4k..4k+3 of unit w's A vector (k < V/4) or 4(k - V/4)..
// of its B vector, as fp32, so a warp reads it without bank conflicts.
template <typename T, int V, int X>
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
        } else if (L.on) {
            v = make_float4(1.f, 1.f, 1.f, 1.f);  // no gamma: rotation alone
        }
        s_gl[z][k][w ^ (k >= W / 2 ? X : 0)] = v;
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
// Per row: y_A = r (u_A c - u_B s), y_B = r (u_B c + u_A s), u = x * gamma,
// evaluated as u_A (r c) - u_B (r s) and u_B (r c) + u_A (r s).
// LN: the mean-centred variant (QK-LayerNorm, x - mean(x) in place of x).
// The mode word of FwdArgs selects the rotation alone, the inverse rotation
// or the statistic alone (0: the fused op). TM: Q / K rows arrive by 3-D
// tensor copy (strided inputs); the dense instantiations hold no
// tensor-copy code.
template <typename T, int LPR, int U, int NCW, int NPW, bool LN, bool TM>
__global__ void __launch_bounds__((NCW + NPW) * 32, 1)
qknr_fwd_pipe_kernel(const FwdArgs a, const PipeGeom g,
                     const __grid_constant__ typename MapsArg<TM>::type maps) {
    using IO = Io<T>;
    const int mode = a.mode;
    constexpr int V = IO::V, W = V / 2;
    constexpr int SLOTS = 32 / LPR;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
    __shared__ uint64_t s_step[kMaxHalf];
    __shared__ __align__(16) float4 s_gl[2][W][32];
    __shared__ volatile int s_abort;

    // tensor copies land on 128-byte boundaries (the stage offsets are
    // multiples of 128); should the dynamic base not be, report and stop
    const int tmap = TM ? g.tmap : 0;
    if (tmap && (smem_u32(smem) & 127u)) {
        if (threadIdx.x == 0) atomicOr(&g_qknr_pipe_error, 2u);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(&bars[0]), empty0 = smem_u32(&bars[kMaxStages]);
    init_barriers<NCW, NPW>(full0, empty0, g);
    if (threadIdx.x == 0) s_abort = 0;
    const int half = a.R >> 1;
    // the angle steps depend on the arguments only: taken before the wait
    for (int i = threadIdx.x; i < half; i += blockDim.x) s_step[i] = turn_step(i, a.R, a.theta);
    grid_dep_wait();
    grid_dep_launch();
    __syncthreads();

    const Run run(a.T, g);
    const int rowb = a.D * (int)sizeof(T);

    if (warp < NPW) {
        // ----------------------------------------------------- producers
        // (the lowest warp ids, which the warp schedulers favour, so the
        // tables are ready before the consumers need them)
        const int pw = warp;
        const uint64_t pol = evict_first_policy();
        // copies of tile `it` into its stage, counted on the stage's barrier
        auto issue = [&](int it) {
            const int s = it % g.NS;
            const int64_t t0 = run.start(it);
            const int na = run.count(it);
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const uint32_t bq = (uint32_t)(na * a.Hq * rowb), bk = (uint32_t)(na * a.Hkv * rowb);
            // a tensor copy moves its whole box of TT tokens
            const uint32_t xq = (tmap & 1) && bq ? (uint32_t)(g.TT * a.Hq * rowb) : bq;
            const uint32_t xk = (tmap & 2) && bk ? (uint32_t)(g.TT * a.Hkv * rowb) : bk;
            const int bs = (int)box_start(t0, run.t_hi, g.TT);
            const uint32_t bar = full0 + 8 * s;
            mbar_expect_tx(bar, xq + xk);
            if (bq) {
                if (tmap & 1) tensor_g2s(smem_u32(st), map_of<TM>(maps, 0), 0, 0, bs, bar, pol);
                else bulk_g2s(smem_u32(st), (const char *)a.q + t0 * a.qts, bq, bar, pol);
            }
            if (bk) {
                if (tmap & 2) tensor_g2s(smem_u32(st + g.off_k), map_of<TM>(maps, 1), 0, 0, bs, bar, pol);
                else bulk_g2s(smem_u32(st + g.off_k), (const char *)a.k + t0 * a.kts, bk, bar, pol);
            }
        };
        // the first ring of copies goes out before any table is built
        const int first = min(g.NS, run.ntiles);
        if (pw == 0 && lane == 0)
            for (int it = 0; it < first; ++it) issue(it);
        int issued = first;
        int s_row = run.ntiles ? (int)(run.t_lo % a.S) : 0;  // row position of the tile's first token
        int32_t pos_next = tile_pos(a.pos, a.S, run.t_lo, s_row, run.ntiles ? run.count(0) : 0, lane);
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            const int64_t t0 = run.start(it);
            const int na = run.count(it);
            const int32_t pos = pos_next;
            s_row += na;
            while (s_row >= a.S) s_row -= a.S;
            if (it + 1 < run.ntiles) {
                const int64_t t1 = t0 + na;
                pos_next = tile_pos(a.pos, a.S, t1, s_row, run.count(it + 1), lane);
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
        constexpr int X = GammaSwz<LPR, U>::X;
        fill_unit_gamma<T, V, X>(s_gl, a.Hq ? a.gq : nullptr, a.Hkv ? a.gk : nullptr, a.D, a.R,
                                 threadIdx.x - NPW * 32, NCW * 32);
        consumers_sync(NCW * 32);
        const Pairs<LPR, V, U> L(lane, a.D, a.R);
        uint32_t off1[U], off2[U];
        float sgn[U];  // sine sign of each pair (negated again for the inverse rotation)
        PairOffsets<V, X> po[U];
#pragma unroll
        for (int q = 0; q < U; ++q) {
            off1[q] = (uint32_t)(L.first[q] * (int)sizeof(T));
            off2[q] = (uint32_t)(L.second[q] * (int)sizeof(T));
            sgn[q] = (mode & kModeInverse) ? -L.sgn[q] : L.sgn[q];
            po[q].set(L.w[q], L.kb[q]);
        }
        const uint32_t smem0 = smem_u32(smem);
        const uint32_t gq0 = smem_u32(&s_gl[0][0][0]), gk0 = smem_u32(&s_gl[1][0][0]);
        const float inv_d = 1.0f / (float)a.D;
        int pc = 0;  // passes dealt before this tile, mod NCW
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            if (!mbar_wait(full0 + 8 * s, (it / g.NS) & 1, 0)) break;
            const uint32_t st = smem0 + (uint32_t)(s * g.stage_bytes);
            const int64_t t0 = run.start(it);
            const int na = run.count(it);

            // tokens of a tensor-copy box before the tile (partial last tile)
            const int skip = (int)(t0 - box_start(t0, run.t_hi, g.TT));
            const int xq0 = (tmap & 1) ? skip * a.Hq * rowb : 0;
            const int xk0 = (tmap & 2) ? skip * a.Hkv * rowb : 0;
            char *out_q = (char *)a.qo + t0 * a.Hq * rowb;   // the tile's first rows
            char *out_k = (char *)a.ko + t0 * a.Hkv * rowb;
            float *r_q = a.rq + t0 * a.Hq;
            float *r_k = a.rk + t0 * a.Hkv;
            const uint32_t cs_tile = st + (uint32_t)g.off_cs;
            const TilePasses tp(na, a.Hq, a.Hkv, SLOTS);
            const int npass = tp.npass;
            int p = (warp - NPW) - pc;
            if (p < 0) p += NCW;
            for (; p < npass; p += NCW) {
                const bool isq = p < tp.pq;  // uniform across the warp
                const int j = (isq ? p : p - tp.pq) * SLOTS + L.slot;
                const bool valid = j < (isq ? tp.rows_q : tp.rows_k);
                const TileRow tr(isq, valid ? j : 0, g);
                const uint32_t src = st + (uint32_t)((tr.isq ? xq0 : g.off_k + xk0) + tr.jj * rowb);
                Vec16 xa[U], xb[U];
#pragma unroll
                for (int q = 0; q < U; ++q) xa[q] = lds16(src + off1[q]);
#pragma unroll
                for (int q = 0; q < U; ++q) xb[q] = lds16(src + off2[q]);
                float r = 1.f;  // rotation alone: no normalisation
                float2 nm2 = make_float2(0.f, 0.f);  // -mean (mean-centred variant)
                if (LN) {
                    float sx = 0.f;
#pragma unroll
                    for (int q = 0; q < U; ++q) {
                        float2 s0 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < W; ++k)
                            s0 = __fadd2_rn(s0, __fadd2_rn(IO::get2(xa[q], k), IO::get2(xb[q], k)));
                        sx = fmaf(L.mask[q], s0.x + s0.y, sx);
                    }
                    const float mu = group_sum<LPR>(sx) * inv_d;
                    nm2 = make_float2(-mu, -mu);
                }
                if (!(mode & kModeRopeOnly)) {
                    float ss = 0.f;
#pragma unroll
                    for (int q = 0; q < U; ++q) {
                        float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < W; ++k) {
                            float2 va = IO::get2(xa[q], k), vb = IO::get2(xb[q], k);
                            if (LN) {
                                va = __fadd2_rn(va, nm2);
                                vb = __fadd2_rn(vb, nm2);
                            }
                            s0 = __ffma2_rn(va, va, s0);
                            s1 = __ffma2_rn(vb, vb, s1);
                        }
                        ss = fmaf(L.mask[q], (s0.x + s1.x) + (s0.y + s1.y), ss);
                    }
                    ss = group_sum<LPR>(ss);
                    r = rsqrtf(fmaf(ss, inv_d, a.eps));
                }
                const float2 r2 = make_float2(r, r);
                const uint32_t tok = cs_tile + (uint32_t)(tr.tl * (half >> 1) * 16);
                const uint32_t gtab = tr.isq ? gq0 : gk0;
                char *out = (tr.isq ? out_q : out_k) + tr.jj * rowb;
#pragma unroll
                for (int q = 0; q < U && !(mode & kModeStatsOnly); ++q) {
                    float4 cs[W], gv[W];
                    if (L.rot[q]) {
#pragma unroll
                        for (int k = 0; k < W; ++k) cs[k] = ldsf4(tok + po[q].cs[k]);
                    } else {  // pass-through unit: (cos, sin) = (1, 0), no load
#pragma unroll
                        for (int k = 0; k < W; ++k) cs[k] = make_float4(1.f, 1.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int k = 0; k < W / 2; ++k) {
                        gv[k] = ldsf4(gtab + po[q].g1 + 512u * k);
                        gv[W / 2 + k] = ldsf4(gtab + po[q].g2 + 512u * k);
                    }
                    // r (and the pair's sine sign) folded into cos and sin
                    const float rs = r * sgn[q];
                    const float2 rs2 = make_float2(rs, rs);
                    Vec16 ya, yb;
#pragma unroll
                    for (int k = 0; k < W; ++k) {
                        const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                        const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                        const float2 c = __fmul2_rn(lo2(cs[k]), r2), sn = __fmul2_rn(hi2(cs[k]), rs2);
                        float2 xa2 = IO::get2(xa[q], k), xb2 = IO::get2(xb[q], k);
                        if (LN) {
                            xa2 = __fadd2_rn(xa2, nm2);
                            xb2 = __fadd2_rn(xb2, nm2);
                        }
                        const float2 ua = __fmul2_rn(xa2, ga);
                        const float2 ub = __fmul2_rn(xb2, gb);
                        const float2 oa = __ffma2_rn(ua, c, __fmul2_rn(ub, neg2(sn)));
                        const float2 ob = __ffma2_rn(ub, c, __fmul2_rn(ua, sn));
                        IO::put2(ya, k, oa.x, oa.y);
                        IO::put2(yb, k, ob.x, ob.y);
                    }
                    if (valid && L.on[q]) {
                        stg16(out + off1[q], ya);
                        stg16(out + off2[q], yb);
                    }
                }
                if (valid && L.u == 0 && !(mode & kModeRopeOnly)) __stcs((tr.isq ? r_q : r_k) + tr.jj, r);
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
// LN: the mean-centred variant: x_hat = (x - mean) r and
// dx = r (h - mean(h) - x_hat <h, x_hat> / D). TM as for the forward.
template <typename T, int LPR, int NCW, int NPW, bool LN, bool TM>
__global__ void __launch_bounds__((NCW + NPW) * 32, 1)
qknr_bwd_pipe_kernel(const BwdArgs a, const PipeGeom g,
                     const __grid_constant__ typename MapsArg<TM>::type maps) {
    using IO = Io<T>;
    constexpr int V = IO::V, W = V / 2;
    constexpr int SLOTS = 32 / LPR;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
    __shared__ uint64_t s_step[kMaxHalf];
    __shared__ __align__(16) float4 s_gl[2][W][32];
    __shared__ volatile int s_abort;
    __shared__ float s_dg[2][kMaxD];

    // tensor copies land on 128-byte boundaries (the stage offsets are
    // multiples of 128); should the dynamic base not be, report and stop
    const int tmap = TM ? g.tmap : 0;
    if (tmap && (smem_u32(smem) & 127u)) {
        if (threadIdx.x == 0) atomicOr(&g_qknr_pipe_error, 2u);
        return;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(&bars[0]), empty0 = smem_u32(&bars[kMaxStages]);
    init_barriers<NCW, NPW>(full0, empty0, g);
    if (threadIdx.x == 0) s_abort = 0;
    for (int i = threadIdx.x; i < 2 * kMaxD; i += blockDim.x) (&s_dg[0][0])[i] = 0.f;
    const int half = a.R >> 1;
    // the angle steps depend on the arguments only: taken before the wait
    for (int i = threadIdx.x; i < half; i += blockDim.x) s_step[i] = turn_step(i, a.R, a.theta);
    grid_dep_wait();
    grid_dep_launch();
    __syncthreads();

    const Run run(a.T, g);
    const int rowb = a.D * (int)sizeof(T);

    if (warp < NPW) {
        // ----------------------------------------------------- producers
        // (the lowest warp ids, which the warp schedulers favour, so the
        // tables are ready before the consumers need them)
        const int pw = warp;
        const uint64_t pol = evict_first_policy();
        auto issue = [&](int it) {
            const int s = it % g.NS;
            const int64_t t0 = run.start(it);
            const int na = run.count(it);
            unsigned char *st = smem + (size_t)s * g.stage_bytes;
            const uint32_t bq = (uint32_t)(na * a.Hq * rowb), bk = (uint32_t)(na * a.Hkv * rowb);
            // inverse RMS: the 16-byte multiple of each block (the
            // producers fill in a tail of up to three floats)
            const uint32_t brq = (uint32_t)(na * a.Hq * 4) & ~15u;
            const uint32_t brk = (uint32_t)(na * a.Hkv * 4) & ~15u;
            // a tensor copy moves its whole box of TT tokens
            const uint32_t xq = (tmap & 1) && bq ? (uint32_t)(g.TT * a.Hq * rowb) : bq;
            const uint32_t xk = (tmap & 2) && bk ? (uint32_t)(g.TT * a.Hkv * rowb) : bk;
            const int bs = (int)box_start(t0, run.t_hi, g.TT);
            const uint32_t bar = full0 + 8 * s;
            mbar_expect_tx(bar, xq + xk + bq + bk + brq + brk);
            if (bq) {
                if (tmap & 1) tensor_g2s(smem_u32(st), map_of<TM>(maps, 0), 0, 0, bs, bar, pol);
                else bulk_g2s(smem_u32(st), (const char *)a.q + t0 * a.qts, bq, bar, pol);
                bulk_g2s(smem_u32(st + g.off_dq), (const char *)a.dqo + t0 * a.Hq * rowb, bq, bar, pol);
            }
            if (bk) {
                if (tmap & 2) tensor_g2s(smem_u32(st + g.off_k), map_of<TM>(maps, 1), 0, 0, bs, bar, pol);
                else bulk_g2s(smem_u32(st + g.off_k), (const char *)a.k + t0 * a.kts, bk, bar, pol);
                bulk_g2s(smem_u32(st + g.off_dk), (const char *)a.dko + t0 * a.Hkv * rowb, bk, bar, pol);
            }
            if (brq) bulk_g2s(smem_u32(st + g.off_rq), a.rq + t0 * a.Hq, brq, bar, pol);
            if (brk) bulk_g2s(smem_u32(st + g.off_rk), a.rk + t0 * a.Hkv, brk, bar, pol);
        };
        const int first = min(g.NS, run.ntiles);
        if (pw == 0 && lane == 0)
            for (int it = 0; it < first; ++it) issue(it);
        int issued = first;
        int s_row = run.ntiles ? (int)(run.t_lo % a.S) : 0;  // row position of the tile's first token
        int32_t pos_next = tile_pos(a.pos, a.S, run.t_lo, s_row, run.ntiles ? run.count(0) : 0, lane);
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            const int64_t t0 = run.start(it);
            const int na = run.count(it);
            const int32_t pos = pos_next;
            s_row += na;
            while (s_row >= a.S) s_row -= a.S;
            if (it + 1 < run.ntiles) {
                const int64_t t1 = t0 + na;
                pos_next = tile_pos(a.pos, a.S, t1, s_row, run.count(it + 1), lane);
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
        constexpr int X = GammaSwz<LPR, 1>::X;
        fill_unit_gamma<T, V, X>(s_gl, a.Hq ? a.gq : nullptr, a.Hkv ? a.gk : nullptr, a.D, a.R,
                                 threadIdx.x - NPW * 32, NCW * 32);
        consumers_sync(NCW * 32);
        const Pairs<LPR, V, 1> L(lane, a.D, a.R);
        const uint32_t off1 = (uint32_t)(L.first[0] * (int)sizeof(T));
        const uint32_t off2 = (uint32_t)(L.second[0] * (int)sizeof(T));
        const float2 sg = make_float2(L.sgn[0], L.sgn[0]);
        PairOffsets<V, X> po;
        po.set(L.w[0], L.kb[0]);
        const uint32_t smem0 = smem_u32(smem);
        const uint32_t gq0 = smem_u32(&s_gl[0][0][0]), gk0 = smem_u32(&s_gl[1][0][0]);
        const float inv_d = 1.0f / (float)a.D;
        // dgamma partial sums: [k] = elements (first + 2k, first + 2k + 1),
        // same for the second vector
        float2 aqa[W], aqb[W], aka[W], akb[W];
#pragma unroll
        for (int k = 0; k < W; ++k) aqa[k] = aqb[k] = aka[k] = akb[k] = make_float2(0.f, 0.f);
        int pc = 0;
        for (int it = 0; it < run.ntiles; ++it) {
            const int s = it % g.NS;
            if (!mbar_wait(full0 + 8 * s, (it / g.NS) & 1, 0)) break;
            const uint32_t st = smem0 + (uint32_t)(s * g.stage_bytes);
            const int64_t t0 = run.start(it);
            const int na = run.count(it);

            // tokens of a tensor-copy box before the tile (partial last tile)
            const int skip = (int)(t0 - box_start(t0, run.t_hi, g.TT));
            const int xq0 = (tmap & 1) ? skip * a.Hq * rowb : 0;
            const int xk0 = (tmap & 2) ? skip * a.Hkv * rowb : 0;
            char *out_q = (char *)a.dq + t0 * a.dqts;
            char *out_k = (char *)a.dk + t0 * a.dkts;
            const uint32_t cs_tile = st + (uint32_t)g.off_cs;
            const TilePasses tp(na, a.Hq, a.Hkv, SLOTS);
            const int npass = tp.npass;
            int p = (warp - NPW) - pc;
            if (p < 0) p += NCW;
            for (; p < npass; p += NCW) {
                const bool isq = p < tp.pq;  // uniform across the warp
                const int j = (isq ? p : p - tp.pq) * SLOTS + L.slot;
                const bool in = j < (isq ? tp.rows_q : tp.rows_k);
                const bool valid = in && L.on[0];
                const TileRow tr(isq, in ? j : 0, g);
                const uint32_t xs = st + (uint32_t)((tr.isq ? xq0 : g.off_k + xk0) + tr.jj * rowb);
                const uint32_t ds = st + (uint32_t)((tr.isq ? g.off_dq : g.off_dk) + tr.jj * rowb);
                const Vec16 xa = lds16(xs + off1), da = lds16(ds + off1);
                const Vec16 xb = lds16(xs + off2), db = lds16(ds + off2);
                float r;
                asm volatile("ld.shared.f32 %0, [%1];"
                             : "=f"(r)
                             : "r"(st + (uint32_t)((tr.isq ? g.off_rq : g.off_rk) + 4 * tr.jj)));
                r = valid ? r : 0.f;  // rows past the tile and off lanes add nothing
                float4 cs[W], gv[W];
                if (L.rot[0]) {
                    const uint32_t cb = cs_tile + (uint32_t)(tr.tl * (half >> 1) * 16);
#pragma unroll
                    for (int k = 0; k < W; ++k) cs[k] = ldsf4(cb + po.cs[k]);
                } else {  // pass-through unit: (cos, sin) = (1, 0), no load
#pragma unroll
                    for (int k = 0; k < W; ++k) cs[k] = make_float4(1.f, 1.f, 0.f, 0.f);
                }
                const uint32_t gtab = tr.isq ? gq0 : gk0;
#pragma unroll
                for (int k = 0; k < W / 2; ++k) {
                    gv[k] = ldsf4(gtab + po.g1 + 512u * k);
                    gv[W / 2 + k] = ldsf4(gtab + po.g2 + 512u * k);
                }
                const float2 r2 = make_float2(r, r);
                if constexpr (LN) {
                // one pass forms g (dy un-rotated) and the row sums of x,
                // h = g gamma and h x; with mu = mean(x), xh = (x - mu) r:
                //   <h, xh> / D = r (sum(h x) / D - mu mean(h))
                //   dx = r (h - mean(h) - xh <h, xh> / D) = r h + A x + B
                // so dx and the dgamma terms g xh come from x and g alone
                float2 xA[W], xB[W], gAv[W], gBv[W];
                float2 sx = make_float2(0.f, 0.f), sh = make_float2(0.f, 0.f);
                float2 shx = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                    const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                    const float2 c = lo2(cs[k]), sn = __fmul2_rn(hi2(cs[k]), sg);
                    const float2 dA = IO::get2(da, k), dB = IO::get2(db, k);
                    xA[k] = IO::get2(xa, k);
                    xB[k] = IO::get2(xb, k);
                    gAv[k] = __ffma2_rn(dA, c, __fmul2_rn(dB, sn));
                    gBv[k] = __ffma2_rn(dB, c, __fmul2_rn(dA, neg2(sn)));
                    const float2 hA = __fmul2_rn(gAv[k], ga), hB = __fmul2_rn(gBv[k], gb);
                    sx = __fadd2_rn(sx, __fadd2_rn(xA[k], xB[k]));
                    sh = __fadd2_rn(sh, __fadd2_rn(hA, hB));
                    shx = __ffma2_rn(hA, xA[k], __ffma2_rn(hB, xB[k], shx));
                }
                const float mu = group_sum<LPR>(L.on[0] ? sx.x + sx.y : 0.f) * inv_d;
                const float mh = group_sum<LPR>(sh.x + sh.y) * inv_d;
                const float dd = r * (group_sum<LPR>(shx.x + shx.y) * inv_d - mu * mh);
                const float A = -r * r * dd, Bc = r * (r * dd * mu - mh);
                const float2 A2 = make_float2(A, A), B2 = make_float2(Bc, Bc);
                const float2 nmr2 = make_float2(-mu * r, -mu * r);
                Vec16 oa, ob;
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                    const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                    const float2 xhA = __ffma2_rn(xA[k], r2, nmr2), xhB = __ffma2_rn(xB[k], r2, nmr2);
                    if (tr.isq) {
                        aqa[k] = __ffma2_rn(gAv[k], xhA, aqa[k]);
                        aqb[k] = __ffma2_rn(gBv[k], xhB, aqb[k]);
                    } else {
                        aka[k] = __ffma2_rn(gAv[k], xhA, aka[k]);
                        akb[k] = __ffma2_rn(gBv[k], xhB, akb[k]);
                    }
                    const float2 va = __ffma2_rn(xA[k], A2, __ffma2_rn(__fmul2_rn(gAv[k], ga), r2, B2));
                    const float2 vb = __ffma2_rn(xB[k], A2, __ffma2_rn(__fmul2_rn(gBv[k], gb), r2, B2));
                    IO::put2(oa, k, va.x, va.y);
                    IO::put2(ob, k, vb.x, vb.y);
                }
                if (valid) {
                    // row (tl, h) of dq / dk, whose tokens may be strided
                    const int hz = tr.isq ? a.Hq : a.Hkv;
                    char *out = (tr.isq ? out_q : out_k) + (int64_t)tr.tl * (tr.isq ? a.dqts : a.dkts) +
                                (tr.jj - tr.tl * hz) * rowb;
                    stg16(out + off1, oa);
                    stg16(out + off2, ob);
                }
                } else {
                float2 ha[W], hb[W], xha[W], xhb[W];
                float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < W; ++k) {
                    const float2 ga = (k & 1) ? hi2(gv[k >> 1]) : lo2(gv[k >> 1]);
                    const float2 gb = (k & 1) ? hi2(gv[W / 2 + (k >> 1)]) : lo2(gv[W / 2 + (k >> 1)]);
                    const float2 c = lo2(cs[k]), sn = __fmul2_rn(hi2(cs[k]), sg);
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
                    // row (tl, h) of dq / dk, whose tokens may be strided
                    const int hz = tr.isq ? a.Hq : a.Hkv;
                    char *out = (tr.isq ? out_q : out_k) + (int64_t)tr.tl * (tr.isq ? a.dqts : a.dkts) +
                                (tr.jj - tr.tl * hz) * rowb;
                    stg16(out + off1, oa);
                    stg16(out + off2, ob);
                }
                }
            }
            pc = (pc + npass) % NCW;
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
        }
        // dgamma: back to (A, B) order on swapped lanes, then lanes of one
        // unit across the warp's row slots, then the CTA's consumer warps
        // (shared atomics)
        const bool sw = L.sgn[0] < 0.f;
#pragma unroll
        for (int k = 0; k < W; ++k) {
            const float2 q1 = aqa[k], q2 = aqb[k], k1 = aka[k], k2 = akb[k];
            aqa[k] = sw ? q2 : q1;
            aqb[k] = sw ? q1 : q2;
            aka[k] = sw ? k2 : k1;
            akb[k] = sw ? k1 : k2;
        }
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
            const int eA = sw ? L.second[0] : L.first[0], eB = sw ? L.first[0] : L.second[0];
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
