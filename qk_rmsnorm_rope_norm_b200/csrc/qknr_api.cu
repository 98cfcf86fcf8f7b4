// C ABI of the fused QK-RMSNorm + RoPE library: host-side validation,
// launch geometry and dispatch to the sm_100a kernels in qknr_kernels.cuh.
// Declarations and the full contract are in include/qknr.h.
#include "qknr.h"
#include "qknr_pipe.cuh"

#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <utility>

namespace qknr {

thread_local int g_last_cuda_error = 0;

// Records the CUDA error behind a QKNR_ERR_CUDA (every entry point of the
// library, in either source file, reports through here).
qknr_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return QKNR_ERR_CUDA;
}

namespace {

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

// The bytes a buffer covers: [p, p + n), and when ts > 0 only the first
// `row` bytes of every ts-byte token step (a strided Q or K in a fused QKV
// buffer, where the other slots belong to other tensors).
struct Span {
    const char *p;
    size_t n;
    size_t row = 0;
    size_t ts = 0;
};

// Span covering T tokens of `row` bytes, `ts` bytes apart (ts == row: dense).
Span strided(const void *p, int64_t T, size_t row, size_t ts) {
    if (!p || T <= 0 || row == 0) return Span{(const char *)p, 0};
    Span s{(const char *)p, (size_t)(T - 1) * ts + row};
    if (ts != row) {
        s.row = row;
        s.ts = ts;
    }
    return s;
}

bool overlaps(Span a, Span b) {
    if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
    if (!(a.p < b.p + b.n && b.p < a.p + a.n)) return false;
    if (a.ts && a.ts == b.ts) {
        // two combs of the same pitch: disjoint when b's row sits in a's gap
        const int64_t d = (int64_t)(b.p - a.p), ts = (int64_t)a.ts;
        const int64_t r = ((d % ts) + ts) % ts;
        return !((int64_t)a.row <= r && r + (int64_t)b.row <= ts);
    }
    return true;
}

// Shape checks shared by both directions.
qknr_status check_shape(int B, int S, int Hq, int Hkv, int D, int R,
                        float theta, float eps, qknr_dtype dtype) {
    if (dtype != QKNR_F32 && dtype != QKNR_BF16) return QKNR_ERR_INVALID_ARG;
    if (B < 0 || S < 0 || Hq < 0 || Hkv < 0) return QKNR_ERR_INVALID_ARG;
    if (D < 2 || (D & 1)) return QKNR_ERR_INVALID_ARG;
    if (R < 0 || R > D || (R & 1)) return QKNR_ERR_INVALID_ARG;
    if (!(theta > 0.f) || !std::isfinite(theta)) return QKNR_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return QKNR_ERR_INVALID_ARG;
    const int e = dtype == QKNR_F32 ? 4 : 2;
    if (D > kMaxD) return QKNR_ERR_UNSUPPORTED;
    if ((D * e) % 16 != 0) return QKNR_ERR_UNSUPPORTED;
    if (((R / 2) * e) % 16 != 0) return QKNR_ERR_UNSUPPORTED;
    return QKNR_OK;
}

// Outputs are all[first_out..n_all). Output i may coincide exactly with the
// one input all[may_equal[i - first_out]] (in-place use); any other overlap
// between an output and another buffer is an error.
qknr_status check_overlaps(const Span *all, int n_all, int first_out, const int *may_equal) {
    for (int i = first_out; i < n_all; ++i) {
        for (int j = 0; j < n_all; ++j) {
            if (j == i || !overlaps(all[i], all[j])) continue;
            if (j == may_equal[i - first_out] && all[j].p == all[i].p && all[j].n == all[i].n &&
                all[j].ts == all[i].ts)
                continue;
            return QKNR_ERR_INVALID_ARG;
        }
    }
    return QKNR_OK;
}

// Units (pairs of 16-byte vectors) of a row: an odd count of vectors leaves
// the last pass-through unit with one vector.
int units_per_row(int D, int e) { return (D / (16 / e) + 1) / 2; }

int next_pow2(int x) {
    int l = 1;
    while (l < x) l <<= 1;
    return l;
}

int lanes_per_row(int D, int e) { return next_pow2(units_per_row(D, e)); }

// Occupancy (resident CTAs per SM) of one kernel on one device. `cache` is
// owned by the kernel's launcher (one array per template instantiation).
int resident_ctas(const void *kernel, int dev, std::atomic<int> *cache) {
    if (dev >= 0 && dev < 64) {
        int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) != cudaSuccess || n < 1)
        n = 1;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

int sm_count(int dev) {
    static std::atomic<int> cache[64];
    if (dev >= 0 && dev < 64) {
        int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        n = 1;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Tokens per warp so that one wave of resident warps covers all tokens.
void geometry(const void *kernel, std::atomic<int> *cache, int64_t T, int *grid, int *tpw) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int64_t cap = (int64_t)sm_count(dev) * resident_ctas(kernel, dev, cache) * kWarps;
    int64_t t = (T + cap - 1) / cap;
    if (t < 1) t = 1;
    const int64_t warps = (T + t - 1) / t;
    *tpw = (int)t;
    *grid = (int)((warps + kWarps - 1) / kWarps);
}

// ------------------------------------------------------------ pipelined
#ifndef QKNR_FWD_PIPE_WARPS
#define QKNR_FWD_PIPE_WARPS 16
#endif
#ifndef QKNR_BWD_PIPE_WARPS
#define QKNR_BWD_PIPE_WARPS 12
#endif
#ifndef QKNR_PRODUCER_WARPS
#define QKNR_PRODUCER_WARPS 4
#endif
// Consumer warps per CTA. Measured on B200: 16 for the forward on rows of
// more than 128 bytes per lane group (LPR * U > 4: Llama-3-8B and partial
// RoPE shapes 3-5% faster than with 12); 12 (512 threads, so 128 registers a
// thread) for the forward on short rows (Qwen2.5-0.5B shape 7% faster), for
// every backward (14 or 16 fit in 96 registers without spills but run 2-5%
// slower) and for the mean-centred kernels (which spill at 96 registers).
// Four producer warps: with two, the forward's angle tables take longer to
// fill (Qwen2.5-0.5B-shaped forward 7% slower).
constexpr int kFwdPipeWarps = QKNR_FWD_PIPE_WARPS;
constexpr int kFwdPipeWarpsShortRow = 12;
constexpr int kBwdPipeWarps = QKNR_BWD_PIPE_WARPS;
constexpr int kBwdPipeWarpsLN = 12;
constexpr int kFwdPipeWarpsLN = 12;
constexpr int kProducerWarps = QKNR_PRODUCER_WARPS;  // copy issue + rotary tables
constexpr int fwd_pipe_warps(int lpr, int u, bool ln) {
    return ln ? kFwdPipeWarpsLN : (lpr * u <= 4 ? kFwdPipeWarpsShortRow : kFwdPipeWarps);
}
constexpr int bwd_pipe_warps(bool ln) { return ln ? kBwdPipeWarpsLN : kBwdPipeWarps; }
#ifndef QKNR_STAGE_TARGET_BYTES
#define QKNR_STAGE_TARGET_BYTES 81920
#endif
// Rows per stage, in bytes. Measured on B200: stages of ~80 KB (two or three
// in the ring) beat eight stages of ~24 KB by 1.2-1.9x, because each bulk
// copy and each full/empty hand-off has a fixed cost.
constexpr int kStageTargetBytes = QKNR_STAGE_TARGET_BYTES;
constexpr int kStaticSmemReserve = 8192; // barriers, angle steps, gamma, dgamma tables
constexpr int kDefaultSmemOptin = 232448;  // B200: 227 KB of shared memory per block, opt-in
constexpr int kPlanLen = 15;             // entries qk_norm_rope_plan writes

int align128(int x) { return (x + 127) & ~127; }

int max_dyn_smem(int dev) {
    static std::atomic<int> cache[64];
    if (dev >= 0 && dev < 64) {
        int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        n = 48 * 1024;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// The launch plan of one call: which kernel runs and with what geometry.
// The dispatch below and the qk_norm_rope_plan query both come from here.
struct Plan {
    bool pipe;        // the pipelined kernel (else the plain-load one)
    int lpr, u;       // lanes per head row, units per lane
    int ncw, npw;     // consumer and producer warps
    bool ln;          // mean-centred instantiation
    PipeGeom g;
    int grid, smem, threads;
};

// Tile and ring sizes for one problem; false when the pipelined kernels do
// not apply (an odd number of 16-byte vectors per row, a token too large for
// two stages, or unaligned rstd buffers). `sms` CTAs at most, `optin` bytes
// of shared memory per block.
bool plan_pipe(bool bwd, bool ln, int64_t T, int Hq, int Hkv, int D, int R, int esz, int sms,
               int optin, const void *rq, const void *rk, Plan *p) {
    const int rowb = D * esz, H = Hq + Hkv, half = R / 2;
    const int units = units_per_row(D, esz);
    *p = Plan{};
    p->lpr = next_pow2(units);
    p->u = 1;
    p->threads = kThreads;
    if ((D / (16 / esz)) & 1) return false;  // a half unit: the plain-load kernels take it
    if (bwd && ((rq && ((uintptr_t)rq & 15)) || (rk && ((uintptr_t)rk & 15)))) return false;
    // backward tiles must start rstd blocks on 16-byte boundaries
    int m = 1;
    if (bwd) {
        while ((m * Hq) % 4 || (m * Hkv) % 4) m <<= 1;  // m in {1, 2, 4}
    }
    const int per_tok = (bwd ? 2 : 1) * H * rowb;
    int TT = kStageTargetBytes / (per_tok > 0 ? per_tok : 1);
    TT = TT < 1 ? 1 : (TT > kMaxTileTokens ? kMaxTileTokens : TT);
    TT = ((TT + m - 1) / m) * m;
    if (TT > kMaxTileTokens) TT = kMaxTileTokens;  // a multiple of 4 already
    if (T < TT) TT = (int)(((T + m - 1) / m) * m);
    PipeGeom q{};
    q.TT = TT;
    int off = align128(TT * Hq * rowb);
    q.off_k = off;
    off = align128(off + TT * Hkv * rowb);
    if (bwd) {
        q.off_dq = off;
        off = align128(off + TT * Hq * rowb);
        q.off_dk = off;
        off = align128(off + TT * Hkv * rowb);
    }
    q.off_cs = off;
    off = align128(off + TT * half * 8);
    if (bwd) {
        q.off_rq = off;
        off = align128(off + TT * Hq * 4);
        q.off_rk = off;
        off = align128(off + TT * Hkv * 4);
    }
    q.stage_bytes = off > 0 ? off : 128;
    const int budget = optin - kStaticSmemReserve;
    int NS = budget / q.stage_bytes;
    if (NS > kMaxStages) NS = kMaxStages;
    if (NS < 2) return false;
    q.NS = NS;
    // one CTA per SM; each owns a contiguous run of tokens (a multiple of m)
    int64_t tpc = (T + sms - 1) / sms;
    tpc = ((tpc + m - 1) / m) * m;
    if (tpc < 1) tpc = 1;
    q.tpc = tpc;
    // forward: a first tile of half the tokens. The copies of a CTA's first
    // ring all go out at once and share the DRAM queue with every other
    // CTA's, so a whole first stage lands late; consumers that start on a
    // half tile overlap that wait (Qwen2.5-0.5B-shaped forward 15.4 ->
    // 14.3 us on B200, the large shapes 1-2% faster). The backward gains
    // nothing from it and keeps whole tiles.
    if (!bwd && TT >= 2) q.h0 = TT / 2;
    q.mq = Hq > 1 ? (uint32_t)(0x100000000ull / (uint64_t)Hq + 1) : 0u;
    q.mk = Hkv > 1 ? (uint32_t)(0x100000000ull / (uint64_t)Hkv + 1) : 0u;
    // the kernel instantiation: two units per lane once a forward row has
    // three or more (halving the per-row overhead per element)
    if (!bwd && units >= 3) {
        p->u = 2;
        p->lpr = next_pow2((units + 1) / 2);
    }
    p->ncw = bwd ? bwd_pipe_warps(ln) : fwd_pipe_warps(p->lpr, p->u, ln);
    p->npw = kProducerWarps;
    p->ln = ln;
    p->pipe = true;
    p->g = q;
    p->grid = (int)((T + tpc - 1) / tpc);
    p->smem = NS * q.stage_bytes;
    p->threads = (p->ncw + p->npw) * 32;
    return true;
}

bool allow_dyn_smem(const void *kernel, int dev, std::atomic<int> *cache, int bytes) {
    if (dev < 0 || dev >= 64) return false;
    if (cache[dev].load(std::memory_order_relaxed) >= bytes) return true;
    const int want = max_dyn_smem(dev) - kStaticSmemReserve;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, want) !=
        cudaSuccess)
        return false;
    cache[dev].store(want, std::memory_order_relaxed);
    return want >= bytes;
}

bool pipe_disabled() {
    const char *e = std::getenv("QKNR_SIMPLE_KERNELS");
    return e && e[0] == '1';
}

}  // namespace

// na floats at a and nb at b set to zero on the stream (either may be null
// with a count of 0), by one programmatic-dependent launch.
qknr_status zero_f32(float *a, int64_t na, float *b, int64_t nb, cudaStream_t st) {
    if (!a) na = 0;
    if (!b) nb = 0;
    if (na + nb == 0) return QKNR_OK;
    const int64_t blocks = (na + nb + 2047) / 2048;
    const cudaError_t e =
        launch_pdl(qknr_zero_kernel, (int)(blocks < 16 ? blocks : 16), 256, 0, st, a, na, b, nb);
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

namespace {

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::atomic<void *> fn{nullptr};
    static std::atomic<int> tried{0};
    void *f = fn.load(std::memory_order_acquire);
    if (f || tried.load(std::memory_order_acquire)) return (PFN_cuTensorMapEncodeTiled_v12000)f;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        f = nullptr;
    fn.store(f, std::memory_order_release);
    tried.store(1, std::memory_order_release);
    return (PFN_cuTensorMapEncodeTiled_v12000)f;
}

// 3-D tensor map {D, H, T} over rows whose tokens are ts bytes apart (heads
// contiguous within a token), box {D, H, TT}: one tile's block in one copy.
bool encode_rows(CUtensorMap *m, const void *base, int esz, int D, int H, int64_t T, int64_t ts,
                 int TT) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || H > 256 || D > 256 || T >= ((int64_t)1 << 31)) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * esz, (cuuint64_t)ts};
    const cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)H, (cuuint32_t)TT};
    const cuuint32_t unit[3] = {1, 1, 1};
    return enc(m, esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void *>(base), dims, strides, box, unit, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps for strided Q / K inputs (bit 0 / 1 of the returned mask);
// -1 when a strided input cannot be described by one (the caller then uses
// the plain-load kernels).
int input_maps(const void *q, const void *k, int64_t qts, int64_t kts, int Hq, int Hkv, int D,
               int esz, int64_t T, int TT, CUtensorMap *mq, CUtensorMap *mk) {
    const int64_t rowb = (int64_t)D * esz;
    int mask = 0;
    *mq = CUtensorMap{};
    *mk = CUtensorMap{};
    if (Hq > 0 && qts != Hq * rowb) {
        if (!encode_rows(mq, q, esz, D, Hq, T, qts, TT)) return -1;
        mask |= 1;
    }
    if (Hkv > 0 && kts != Hkv * rowb) {
        if (!encode_rows(mk, k, esz, D, Hkv, T, kts, TT)) return -1;
        mask |= 2;
    }
    return mask;
}

template <typename T, int LPR, int U, bool LN, bool TM>
qknr_status launch_fwd_pipe_tm(const FwdArgs &a, const PipeGeom &g, const CUtensorMap &mq,
                               const CUtensorMap &mk, int grid, int smem, int dev, cudaStream_t st,
                               bool *launched) {
    static std::atomic<int> smem_ok[64];
    constexpr int NCW = fwd_pipe_warps(LPR, U, LN);
    auto kern = qknr_fwd_pipe_kernel<T, LPR, U, NCW, kProducerWarps, LN, TM>;
    *launched = false;
    if (!allow_dyn_smem((const void *)kern, dev, smem_ok, smem)) return QKNR_OK;
    *launched = true;
    typename MapsArg<TM>::type maps{};
    if constexpr (TM) maps = TensorMaps{mq, mk};
    cudaError_t e = launch_pdl(kern, grid, (NCW + kProducerWarps) * 32, smem, st, a, g, maps);
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, int LPR, bool LN, bool TM>
qknr_status launch_bwd_pipe_tm(const BwdArgs &a, const PipeGeom &g, const CUtensorMap &mq,
                               const CUtensorMap &mk, int grid, int smem, int dev, cudaStream_t st,
                               bool *launched) {
    static std::atomic<int> smem_ok[64];
    constexpr int NCW = bwd_pipe_warps(LN);
    auto kern = qknr_bwd_pipe_kernel<T, LPR, NCW, kProducerWarps, LN, TM>;
    *launched = false;
    if (!allow_dyn_smem((const void *)kern, dev, smem_ok, smem)) return QKNR_OK;
    *launched = true;
    typename MapsArg<TM>::type maps{};
    if constexpr (TM) maps = TensorMaps{mq, mk};
    cudaError_t e = launch_pdl(kern, grid, (NCW + kProducerWarps) * 32, smem, st, a, g, maps);
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

// The tensor-copy instantiation only for the forms that take strided inputs
// (the fused RMSNorm op); every other form is dense.
template <typename T, int LPR, int U, bool LN>
qknr_status launch_fwd_pipe(const FwdArgs &a, const PipeGeom &g, const CUtensorMap &mq,
                            const CUtensorMap &mk, int grid, int smem, int dev, cudaStream_t st,
                            bool *launched) {
    if constexpr (!LN) {
        if (g.tmap)
            return launch_fwd_pipe_tm<T, LPR, U, LN, true>(a, g, mq, mk, grid, smem, dev, st,
                                                           launched);
    }
    return launch_fwd_pipe_tm<T, LPR, U, LN, false>(a, g, mq, mk, grid, smem, dev, st, launched);
}

template <typename T, int LPR, bool LN>
qknr_status launch_bwd_pipe(const BwdArgs &a, const PipeGeom &g, const CUtensorMap &mq,
                            const CUtensorMap &mk, int grid, int smem, int dev, cudaStream_t st,
                            bool *launched) {
    if constexpr (!LN) {
        if (g.tmap)
            return launch_bwd_pipe_tm<T, LPR, LN, true>(a, g, mq, mk, grid, smem, dev, st, launched);
    }
    return launch_bwd_pipe_tm<T, LPR, LN, false>(a, g, mq, mk, grid, smem, dev, st, launched);
}

// Pipelined forward when the plan takes it.
template <typename T, bool LN>
bool try_fwd_pipe(const FwdArgs &a, cudaStream_t st, qknr_status *status) {
    int dev = 0;
    cudaGetDevice(&dev);
    Plan p;
    if (pipe_disabled() ||
        !plan_pipe(false, LN, a.T, a.Hq, a.Hkv, a.D, a.R, (int)sizeof(T), sm_count(dev),
                   max_dyn_smem(dev), nullptr, nullptr, &p))
        return false;
    PipeGeom g = p.g;
    CUtensorMap mq, mk;
    g.tmap = input_maps(a.q, a.k, a.qts, a.kts, a.Hq, a.Hkv, a.D, (int)sizeof(T), a.T, g.TT, &mq, &mk);
    if (g.tmap < 0) return false;
    if (g.tmap) g.h0 = 0;  // a tensor copy moves whole boxes of TT tokens
    const int grid = p.grid, smem = p.smem;
    bool launched = false;
    qknr_status s = QKNR_OK;
    if (p.u == 2) {
        switch (p.lpr) {
            case 2: s = launch_fwd_pipe<T, 2, 2, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
            case 4: s = launch_fwd_pipe<T, 4, 2, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
            case 8: s = launch_fwd_pipe<T, 8, 2, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
            case 16: s = launch_fwd_pipe<T, 16, 2, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        }
    } else {
        switch (p.lpr) {
            case 1: s = launch_fwd_pipe<T, 1, 1, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
            case 2: s = launch_fwd_pipe<T, 2, 1, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        }
    }
    *status = s;
    return launched;
}

template <typename T, bool LN>
bool try_bwd_pipe(const BwdArgs &a, cudaStream_t st, qknr_status *status) {
    int dev = 0;
    cudaGetDevice(&dev);
    Plan p;
    if (pipe_disabled() ||
        !plan_pipe(true, LN, a.T, a.Hq, a.Hkv, a.D, a.R, (int)sizeof(T), sm_count(dev),
                   max_dyn_smem(dev), a.rq, a.rk, &p))
        return false;
    PipeGeom g = p.g;
    CUtensorMap mq, mk;
    g.tmap = input_maps(a.q, a.k, a.qts, a.kts, a.Hq, a.Hkv, a.D, (int)sizeof(T), a.T, g.TT, &mq, &mk);
    if (g.tmap < 0) return false;
    if (g.tmap) g.h0 = 0;  // a tensor copy moves whole boxes of TT tokens
    const int grid = p.grid, smem = p.smem;
    bool launched = false;
    qknr_status s = QKNR_OK;
    switch (p.lpr) {
        case 1: s = launch_bwd_pipe<T, 1, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        case 2: s = launch_bwd_pipe<T, 2, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        case 4: s = launch_bwd_pipe<T, 4, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        case 8: s = launch_bwd_pipe<T, 8, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        case 16: s = launch_bwd_pipe<T, 16, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
        case 32: s = launch_bwd_pipe<T, 32, LN>(a, g, mq, mk, grid, smem, dev, st, &launched); break;
    }
    *status = s;
    return launched;
}

template <typename T, int LPR, bool LN>
qknr_status launch_fwd(FwdArgs a, cudaStream_t st) {
    static std::atomic<int> occ[64];
    auto kern = qknr_fwd_kernel<T, LPR, LN>;
    int grid, tpw;
    geometry((const void *)kern, occ, a.T, &grid, &tpw);
    a.tpw = tpw;
    kern<<<grid, kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, int LPR, bool LN>
qknr_status launch_bwd(BwdArgs a, cudaStream_t st) {
    static std::atomic<int> occ[64];
    auto kern = qknr_bwd_kernel<T, LPR, LN>;
    int grid, tpw;
    geometry((const void *)kern, occ, a.T, &grid, &tpw);
    a.tpw = tpw;
    kern<<<grid, kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, bool LN>
qknr_status dispatch_fwd(const FwdArgs &a, int lpr, cudaStream_t st) {
    qknr_status ps;
    if (try_fwd_pipe<T, LN>(a, st, &ps)) return ps;
    switch (lpr) {
        case 1: return launch_fwd<T, 1, LN>(a, st);
        case 2: return launch_fwd<T, 2, LN>(a, st);
        case 4: return launch_fwd<T, 4, LN>(a, st);
        case 8: return launch_fwd<T, 8, LN>(a, st);
        case 16: return launch_fwd<T, 16, LN>(a, st);
        case 32: return launch_fwd<T, 32, LN>(a, st);
    }
    return QKNR_ERR_UNSUPPORTED;
}

template <typename T, bool LN>
qknr_status dispatch_bwd(const BwdArgs &a, int lpr, cudaStream_t st) {
    qknr_status ps;
    if (try_bwd_pipe<T, LN>(a, st, &ps)) return ps;
    switch (lpr) {
        case 1: return launch_bwd<T, 1, LN>(a, st);
        case 2: return launch_bwd<T, 2, LN>(a, st);
        case 4: return launch_bwd<T, 4, LN>(a, st);
        case 8: return launch_bwd<T, 8, LN>(a, st);
        case 16: return launch_bwd<T, 16, LN>(a, st);
        case 32: return launch_bwd<T, 32, LN>(a, st);
    }
    return QKNR_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace qknr

using namespace qknr;

namespace qknr {
namespace {

// Token strides (elements) of a strided input or output: at least the rows
// of one token, and a whole number of 16-byte steps.
qknr_status check_stride(int64_t ts, int H, int D, size_t e) {
    if (H == 0) return QKNR_OK;
    if (ts < (int64_t)H * D) return QKNR_ERR_INVALID_ARG;
    if ((ts * (int64_t)e) % 16 != 0) return QKNR_ERR_ALIGNMENT;
    return QKNR_OK;
}

qknr_status fwd_impl(const void *q, const void *k, int64_t q_ts, int64_t k_ts,
                     const void *gamma_q, const void *gamma_k, const int32_t *pos_ids, void *q_out,
                     void *k_out, float *rstd_q, float *rstd_k, int B, int S, int Hq, int Hkv,
                     int D, int rotary_dim, float theta, float eps, qknr_dtype dtype,
                     qknr_stream_t stream, int mode = 0) {
    qknr_status st = check_shape(B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype);
    if (st != QKNR_OK) return st;
    const int64_t T = (int64_t)B * S;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    const size_t e = dtype == QKNR_F32 ? 4 : 2;
    if (mode & kModeRopeOnly) {  // rotation alone: no gamma, no rstd
        gamma_q = gamma_k = nullptr;
        rstd_q = rstd_k = nullptr;
        if ((Hq > 0 && (!q || !q_out)) || (Hkv > 0 && (!k || !k_out))) return QKNR_ERR_INVALID_ARG;
    } else if (mode & kModeStatsOnly) {  // rstd alone: no gamma, no rows written
        gamma_q = gamma_k = nullptr;
        q_out = k_out = nullptr;
        if ((Hq > 0 && (!q || !rstd_q)) || (Hkv > 0 && (!k || !rstd_k))) return QKNR_ERR_INVALID_ARG;
    } else {
        if (Hq > 0 && (!q || !q_out || !rstd_q || !gamma_q)) return QKNR_ERR_INVALID_ARG;
        if (Hkv > 0 && (!k || !k_out || !rstd_k || !gamma_k)) return QKNR_ERR_INVALID_ARG;
    }
    if ((st = check_stride(q_ts, Hq, D, e)) != QKNR_OK) return st;
    if ((st = check_stride(k_ts, Hkv, D, e)) != QKNR_OK) return st;
    const void *vec[] = {q, k, gamma_q, gamma_k, q_out, k_out};
    for (const void *p : vec)
        if (p && !aligned(p, 16)) return QKNR_ERR_ALIGNMENT;
    if ((rstd_q && !aligned(rstd_q, 4)) || (rstd_k && !aligned(rstd_k, 4)) ||
        (pos_ids && !aligned(pos_ids, 4)))
        return QKNR_ERR_ALIGNMENT;

    const size_t rq = (size_t)Hq * D * e, rk = (size_t)Hkv * D * e;  // bytes per token
    const size_t nq = (size_t)T * Hq, nk = (size_t)T * Hkv;
    Span all[] = {
        strided(q, Hq ? T : 0, rq, (size_t)q_ts * e), strided(k, Hkv ? T : 0, rk, (size_t)k_ts * e),
        {(const char *)gamma_q, Hq ? D * e : 0}, {(const char *)gamma_k, Hkv ? D * e : 0},
        {(const char *)pos_ids, pos_ids ? (size_t)T * 4 : 0},
        {(const char *)q_out, nq * D * e},      {(const char *)k_out, nk * D * e},
        {(const char *)rstd_q, rstd_q ? nq * 4 : 0}, {(const char *)rstd_k, rstd_k ? nk * 4 : 0},
    };
    const int may_equal[] = {0, 1, -1, -1};  // q_out may be a dense q, k_out a dense k
    if (check_overlaps(all, 9, 5, may_equal) != QKNR_OK) return QKNR_ERR_INVALID_ARG;

    FwdArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.qo = q_out; a.ko = k_out; a.rq = rstd_q; a.rk = rstd_k;
    a.qts = q_ts * (int64_t)e; a.kts = k_ts * (int64_t)e;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    a.theta = theta; a.eps = eps; a.mode = mode;
    const int lpr = lanes_per_row(D, (int)e);
    cudaStream_t cs = (cudaStream_t)stream;
    if (mode & kModeLayerNorm)
        return dtype == QKNR_F32 ? dispatch_fwd<float, true>(a, lpr, cs)
                                 : dispatch_fwd<__nv_bfloat16, true>(a, lpr, cs);
    return dtype == QKNR_F32 ? dispatch_fwd<float, false>(a, lpr, cs)
                             : dispatch_fwd<__nv_bfloat16, false>(a, lpr, cs);
}

qknr_status bwd_impl(const void *q, const void *k, int64_t q_ts, int64_t k_ts,
                     const void *gamma_q, const void *gamma_k, const int32_t *pos_ids,
                     const float *rstd_q, const float *rstd_k, const void *dq_out,
                     const void *dk_out, void *dq, void *dk, int64_t dq_ts, int64_t dk_ts,
                     float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv, int D,
                     int rotary_dim, float theta, float eps, qknr_dtype dtype,
                     qknr_stream_t stream, int mode = 0) {
    qknr_status st = check_shape(B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype);
    if (st != QKNR_OK) return st;
    const int64_t T = (int64_t)B * S;
    const size_t e = dtype == QKNR_F32 ? 4 : 2;
    const bool work = T > 0 && Hq + Hkv > 0;
    if (work && Hq > 0 && (!q || !gamma_q || !rstd_q || !dq_out || !dq)) return QKNR_ERR_INVALID_ARG;
    if (work && Hkv > 0 && (!k || !gamma_k || !rstd_k || !dk_out || !dk)) return QKNR_ERR_INVALID_ARG;
    if ((st = check_stride(q_ts, Hq, D, e)) != QKNR_OK) return st;
    if ((st = check_stride(k_ts, Hkv, D, e)) != QKNR_OK) return st;
    if ((st = check_stride(dq_ts, Hq, D, e)) != QKNR_OK) return st;
    if ((st = check_stride(dk_ts, Hkv, D, e)) != QKNR_OK) return st;
    const void *vec[] = {q, k, gamma_q, gamma_k, dq_out, dk_out, dq, dk};
    for (const void *p : vec)
        if (p && !aligned(p, 16)) return QKNR_ERR_ALIGNMENT;
    if ((rstd_q && !aligned(rstd_q, 4)) || (rstd_k && !aligned(rstd_k, 4)) ||
        (pos_ids && !aligned(pos_ids, 4)) || (dgamma_q && !aligned(dgamma_q, 4)) ||
        (dgamma_k && !aligned(dgamma_k, 4)))
        return QKNR_ERR_ALIGNMENT;

    const int64_t Tq = work && Hq ? T : 0, Tk = work && Hkv ? T : 0;
    const size_t rq = (size_t)Hq * D * e, rk = (size_t)Hkv * D * e;  // bytes per token
    const size_t nq = (size_t)Tq * Hq, nk = (size_t)Tk * Hkv;
    Span all[] = {
        strided(q, Tq, rq, (size_t)q_ts * e),    strided(k, Tk, rk, (size_t)k_ts * e),
        {(const char *)gamma_q, Hq ? D * e : 0},  {(const char *)gamma_k, Hkv ? D * e : 0},
        {(const char *)pos_ids, pos_ids && work ? (size_t)T * 4 : 0},
        {(const char *)rstd_q, nq * 4},          {(const char *)rstd_k, nk * 4},
        {(const char *)dq_out, nq * D * e},      {(const char *)dk_out, nk * D * e},
        strided(dq, Tq, rq, (size_t)dq_ts * e),  strided(dk, Tk, rk, (size_t)dk_ts * e),
        {(const char *)dgamma_q, dgamma_q ? (size_t)D * 4 : 0},
        {(const char *)dgamma_k, dgamma_k ? (size_t)D * 4 : 0},
    };
    const int may_equal[] = {7, 8, -1, -1};  // a dense dq may be dq_out, a dense dk dk_out
    if (check_overlaps(all, 13, 9, may_equal) != QKNR_OK) return QKNR_ERR_INVALID_ARG;

    cudaStream_t cs = (cudaStream_t)stream;
    // dgamma is accumulated by atomics, so it starts from zero; one small
    // kernel clears both (chained to the backward launch that follows)
    if ((st = zero_f32(dgamma_q, D, dgamma_k, D, cs)) != QKNR_OK) return st;
    if (!work) return QKNR_OK;

    BwdArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.rq = rstd_q; a.rk = rstd_k; a.dqo = dq_out; a.dko = dk_out;
    a.dq = dq; a.dk = dk; a.dgq = dgamma_q; a.dgk = dgamma_k;
    a.qts = q_ts * (int64_t)e; a.kts = k_ts * (int64_t)e;
    a.dqts = dq_ts * (int64_t)e; a.dkts = dk_ts * (int64_t)e;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    a.theta = theta; a.eps = eps;
    const int lpr = lanes_per_row(D, (int)e);
    if (mode & kModeLayerNorm)
        return dtype == QKNR_F32 ? dispatch_bwd<float, true>(a, lpr, cs)
                                 : dispatch_bwd<__nv_bfloat16, true>(a, lpr, cs);
    return dtype == QKNR_F32 ? dispatch_bwd<float, false>(a, lpr, cs)
                             : dispatch_bwd<__nv_bfloat16, false>(a, lpr, cs);
}

}  // namespace
}  // namespace qknr

extern "C" qknr_status qk_norm_rope_fwd(const void *q, const void *k,
                                        const void *gamma_q, const void *gamma_k,
                                        const int32_t *pos_ids, void *q_out, void *k_out,
                                        float *rstd_q, float *rstd_k, int B, int S, int Hq,
                                        int Hkv, int D, int rotary_dim, float theta, float eps,
                                        qknr_dtype dtype, qknr_stream_t stream) {
    return fwd_impl(q, k, (int64_t)Hq * D, (int64_t)Hkv * D, gamma_q, gamma_k, pos_ids, q_out,
                    k_out, rstd_q, rstd_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype, stream);
}

extern "C" qknr_status qk_norm_rope_fwd_strided(const void *q, const void *k, int64_t q_token_stride,
                                                int64_t k_token_stride, const void *gamma_q,
                                                const void *gamma_k, const int32_t *pos_ids,
                                                void *q_out, void *k_out, float *rstd_q,
                                                float *rstd_k, int B, int S, int Hq, int Hkv, int D,
                                                int rotary_dim, float theta, float eps,
                                                qknr_dtype dtype, qknr_stream_t stream) {
    return fwd_impl(q, k, q_token_stride, k_token_stride, gamma_q, gamma_k, pos_ids, q_out, k_out,
                    rstd_q, rstd_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype, stream);
}

extern "C" qknr_status qk_norm_rope_bwd(const void *q, const void *k,
                                        const void *gamma_q, const void *gamma_k,
                                        const int32_t *pos_ids, const float *rstd_q,
                                        const float *rstd_k, const void *dq_out,
                                        const void *dk_out, void *dq, void *dk,
                                        float *dgamma_q, float *dgamma_k, int B, int S, int Hq,
                                        int Hkv, int D, int rotary_dim, float theta, float eps,
                                        qknr_dtype dtype, qknr_stream_t stream) {
    const int64_t qts = (int64_t)Hq * D, kts = (int64_t)Hkv * D;
    return bwd_impl(q, k, qts, kts, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dq,
                    dk, qts, kts, dgamma_q, dgamma_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps,
                    dtype, stream);
}

extern "C" qknr_status qk_norm_rope_bwd_strided(
    const void *q, const void *k, int64_t q_token_stride, int64_t k_token_stride,
    const void *gamma_q, const void *gamma_k, const int32_t *pos_ids, const float *rstd_q,
    const float *rstd_k, const void *dq_out, const void *dk_out, void *dq, void *dk,
    int64_t dq_token_stride, int64_t dk_token_stride, float *dgamma_q, float *dgamma_k, int B,
    int S, int Hq, int Hkv, int D, int rotary_dim, float theta, float eps, qknr_dtype dtype,
    qknr_stream_t stream) {
    return bwd_impl(q, k, q_token_stride, k_token_stride, gamma_q, gamma_k, pos_ids, rstd_q,
                    rstd_k, dq_out, dk_out, dq, dk, dq_token_stride, dk_token_stride, dgamma_q,
                    dgamma_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype, stream);
}

extern "C" qknr_status qk_layernorm_rope_fwd(const void *q, const void *k, const void *gamma_q,
                                             const void *gamma_k, const int32_t *pos_ids,
                                             void *q_out, void *k_out, float *rstd_q,
                                             float *rstd_k, int B, int S, int Hq, int Hkv, int D,
                                             int rotary_dim, float theta, float eps,
                                             qknr_dtype dtype, qknr_stream_t stream) {
    return fwd_impl(q, k, (int64_t)Hq * D, (int64_t)Hkv * D, gamma_q, gamma_k, pos_ids, q_out,
                    k_out, rstd_q, rstd_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype, stream,
                    kModeLayerNorm);
}

extern "C" qknr_status qk_layernorm_rope_bwd(
    const void *q, const void *k, const void *gamma_q, const void *gamma_k, const int32_t *pos_ids,
    const float *rstd_q, const float *rstd_k, const void *dq_out, const void *dk_out, void *dq,
    void *dk, float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv, int D,
    int rotary_dim, float theta, float eps, qknr_dtype dtype, qknr_stream_t stream) {
    const int64_t qts = (int64_t)Hq * D, kts = (int64_t)Hkv * D;
    return bwd_impl(q, k, qts, kts, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dq,
                    dk, qts, kts, dgamma_q, dgamma_k, B, S, Hq, Hkv, D, rotary_dim, theta, eps,
                    dtype, stream, kModeLayerNorm);
}

extern "C" qknr_status qk_norm_fwd(const void *q, const void *k, const void *gamma_q,
                                   const void *gamma_k, void *q_out, void *k_out, float *rstd_q,
                                   float *rstd_k, int B, int S, int Hq, int Hkv, int D, float eps,
                                   qknr_dtype dtype, qknr_stream_t stream) {
    return fwd_impl(q, k, (int64_t)Hq * D, (int64_t)Hkv * D, gamma_q, gamma_k, nullptr, q_out,
                    k_out, rstd_q, rstd_k, B, S, Hq, Hkv, D, 0, 1.0f, eps, dtype, stream);
}

extern "C" qknr_status qk_norm_bwd(const void *q, const void *k, const void *gamma_q,
                                   const void *gamma_k, const float *rstd_q, const float *rstd_k,
                                   const void *dq_out, const void *dk_out, void *dq, void *dk,
                                   float *dgamma_q, float *dgamma_k, int B, int S, int Hq, int Hkv,
                                   int D, float eps, qknr_dtype dtype, qknr_stream_t stream) {
    const int64_t qts = (int64_t)Hq * D, kts = (int64_t)Hkv * D;
    return bwd_impl(q, k, qts, kts, gamma_q, gamma_k, nullptr, rstd_q, rstd_k, dq_out, dk_out, dq,
                    dk, qts, kts, dgamma_q, dgamma_k, B, S, Hq, Hkv, D, 0, 1.0f, eps, dtype,
                    stream);
}

extern "C" qknr_status qk_rms_stats(const void *q, const void *k, float *rstd_q, float *rstd_k,
                                    int B, int S, int Hq, int Hkv, int D, float eps,
                                    qknr_dtype dtype, qknr_stream_t stream) {
    return fwd_impl(q, k, (int64_t)Hq * D, (int64_t)Hkv * D, nullptr, nullptr, nullptr, nullptr,
                    nullptr, rstd_q, rstd_k, B, S, Hq, Hkv, D, 0, 1.0f, eps, dtype, stream,
                    kModeStatsOnly);
}

extern "C" qknr_status qk_rope_apply(const void *q, const void *k, const int32_t *pos_ids,
                                     void *q_out, void *k_out, int B, int S, int Hq, int Hkv,
                                     int D, int rotary_dim, float theta, int inverse,
                                     qknr_dtype dtype, qknr_stream_t stream) {
    const int mode = kModeRopeOnly | (inverse ? kModeInverse : 0);
    return fwd_impl(q, k, (int64_t)Hq * D, (int64_t)Hkv * D, nullptr, nullptr, pos_ids, q_out,
                    k_out, nullptr, nullptr, B, S, Hq, Hkv, D, rotary_dim, theta, 0.0f, dtype,
                    stream, mode);
}

extern "C" qknr_status qk_norm_rope_plan(int kind, int B, int S, int Hq, int Hkv, int D,
                                         int rotary_dim, qknr_dtype dtype, int strided, int sms,
                                         int smem_optin, int64_t *plan) {
    if (!plan || kind < 0 || kind > 3 || strided < 0 || strided > 3 || sms < 1 ||
        smem_optin < 0)
        return QKNR_ERR_INVALID_ARG;
    const qknr_status st = check_shape(B, S, Hq, Hkv, D, rotary_dim, 1.f, 0.f, dtype);
    if (st != QKNR_OK) return st;
    for (int i = 0; i < kPlanLen; ++i) plan[i] = 0;
    const int64_t T = (int64_t)B * S;
    const int esz = dtype == QKNR_F32 ? 4 : 2;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    Plan p;
    const bool bwd = kind & 1, ln = (kind & 2) != 0;
    if (!plan_pipe(bwd, ln, T, Hq, Hkv, D, rotary_dim, esz, sms,
                   smem_optin ? smem_optin : kDefaultSmemOptin, nullptr, nullptr, &p)) {
        plan[1] = lanes_per_row(D, esz);
        plan[2] = 1;
        plan[5] = ln;
        plan[13] = kThreads;
        return QKNR_OK;
    }
    // tensor copies serve strided inputs of the RMSNorm forms only
    const int tm = ln ? 0 : ((strided & 1) && Hq ? 1 : 0) | ((strided & 2) && Hkv ? 2 : 0);
    const int64_t h0 = tm || p.g.h0 == 0 ? p.g.TT : p.g.h0;
    const int64_t v[kPlanLen] = {1, p.lpr, p.u, p.ncw, p.npw, p.ln, tm, p.g.TT, p.g.NS,
                                 p.g.stage_bytes, p.g.tpc, p.grid, p.smem, p.threads, h0};
    for (int i = 0; i < kPlanLen; ++i) plan[i] = v[i];
    return QKNR_OK;
}

extern "C" const char *qknr_strerror(qknr_status s) {
    switch (s) {
        case QKNR_OK: return "success";
        case QKNR_ERR_INVALID_ARG: return "invalid argument (size, NULL pointer, overlap, theta or eps)";
        case QKNR_ERR_ALIGNMENT: return "pointer not aligned (16 bytes for vectors, 4 for fp32/int32 arrays)";
        case QKNR_ERR_UNSUPPORTED: return "unsupported shape (D <= 256, D*elem a multiple of 16, (R/2)*elem a multiple of 16)";
        case QKNR_ERR_CUDA: return "the CUDA runtime refused the launch (see qknr_last_cuda_error)";
    }
    return "unknown status";
}

extern "C" int qknr_last_cuda_error(void) { return g_last_cuda_error; }

namespace qknr {
int lw_pipeline_error(int reset);  // the layerwise kernels' flag, same bits
qknr_status lw_wait_selftest(long long limit, cudaStream_t st);
}

extern "C" qknr_status qknr_wait_selftest(int family, int64_t limit_cycles, qknr_stream_t stream) {
    if ((family != 0 && family != 1) || limit_cycles < 1 || limit_cycles > ((int64_t)1 << 31))
        return QKNR_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    if (family == 1) return qknr::lw_wait_selftest((long long)limit_cycles, st);
    qknr::qknr_wait_selftest_kernel<<<1, 32, 0, st>>>((long long)limit_cycles);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

extern "C" int qknr_pipeline_error(int reset) {
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, qknr::g_qknr_pipe_error, sizeof(v)) != cudaSuccess) return -1;
    if (reset && v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(qknr::g_qknr_pipe_error, &zero, sizeof(zero)) != cudaSuccess)
            return -1;
    }
    const int lw = qknr::lw_pipeline_error(reset);
    if (lw < 0) return -1;
    return (int)(v | (unsigned int)lw);
}
