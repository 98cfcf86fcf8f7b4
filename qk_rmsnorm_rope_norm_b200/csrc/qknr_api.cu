// C ABI of the fused QK-RMSNorm + RoPE library: host-side validation,
// launch geometry and dispatch to the sm_100a kernels in qknr_kernels.cuh.
// Declarations and the full contract are in include/qknr.h.
#include "qknr.h"
#include "qknr_kernels.cuh"

#include <atomic>
#include <cmath>
#include <cstdint>

namespace qknr {
namespace {

thread_local int g_last_cuda_error = 0;

qknr_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return QKNR_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

struct Span {
    const char *p;
    size_t n;
};

bool overlaps(Span a, Span b) {
    if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
    return a.p < b.p + b.n && b.p < a.p + a.n;
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
    if ((D * e) % 32 != 0) return QKNR_ERR_UNSUPPORTED;
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
            if (j == may_equal[i - first_out] && all[j].p == all[i].p && all[j].n == all[i].n)
                continue;
            return QKNR_ERR_INVALID_ARG;
        }
    }
    return QKNR_OK;
}

int lanes_per_row(int D, int e) {
    const int V = 16 / e;
    const int units = D / (2 * V);
    int l = 1;
    while (l < units) l <<= 1;
    return l;
}

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

template <typename T, int LPR>
qknr_status launch_fwd(FwdArgs a, cudaStream_t st) {
    static std::atomic<int> occ[64];
    auto kern = qknr_fwd_kernel<T, LPR>;
    int grid, tpw;
    geometry((const void *)kern, occ, a.T, &grid, &tpw);
    a.tpw = tpw;
    kern<<<grid, kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T, int LPR>
qknr_status launch_bwd(BwdArgs a, cudaStream_t st) {
    static std::atomic<int> occ[64];
    auto kern = qknr_bwd_kernel<T, LPR>;
    int grid, tpw;
    geometry((const void *)kern, occ, a.T, &grid, &tpw);
    a.tpw = tpw;
    kern<<<grid, kThreads, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKNR_OK : cuda_fail(e);
}

template <typename T>
qknr_status dispatch_fwd(const FwdArgs &a, int lpr, cudaStream_t st) {
    switch (lpr) {
        case 1: return launch_fwd<T, 1>(a, st);
        case 2: return launch_fwd<T, 2>(a, st);
        case 4: return launch_fwd<T, 4>(a, st);
        case 8: return launch_fwd<T, 8>(a, st);
        case 16: return launch_fwd<T, 16>(a, st);
        case 32: return launch_fwd<T, 32>(a, st);
    }
    return QKNR_ERR_UNSUPPORTED;
}

template <typename T>
qknr_status dispatch_bwd(const BwdArgs &a, int lpr, cudaStream_t st) {
    switch (lpr) {
        case 1: return launch_bwd<T, 1>(a, st);
        case 2: return launch_bwd<T, 2>(a, st);
        case 4: return launch_bwd<T, 4>(a, st);
        case 8: return launch_bwd<T, 8>(a, st);
        case 16: return launch_bwd<T, 16>(a, st);
        case 32: return launch_bwd<T, 32>(a, st);
    }
    return QKNR_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace qknr

using namespace qknr;

extern "C" qknr_status qk_norm_rope_fwd(const void *q, const void *k,
                                        const void *gamma_q, const void *gamma_k,
                                        const int32_t *pos_ids, void *q_out, void *k_out,
                                        float *rstd_q, float *rstd_k, int B, int S, int Hq,
                                        int Hkv, int D, int rotary_dim, float theta, float eps,
                                        qknr_dtype dtype, qknr_stream_t stream) {
    qknr_status st = check_shape(B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype);
    if (st != QKNR_OK) return st;
    const int64_t T = (int64_t)B * S;
    if (T == 0 || Hq + Hkv == 0) return QKNR_OK;
    const size_t e = dtype == QKNR_F32 ? 4 : 2;
    if (Hq > 0 && (!q || !q_out || !rstd_q || !gamma_q)) return QKNR_ERR_INVALID_ARG;
    if (Hkv > 0 && (!k || !k_out || !rstd_k || !gamma_k)) return QKNR_ERR_INVALID_ARG;
    const void *vec[] = {q, k, gamma_q, gamma_k, q_out, k_out};
    for (const void *p : vec)
        if (p && !aligned(p, 16)) return QKNR_ERR_ALIGNMENT;
    if ((rstd_q && !aligned(rstd_q, 4)) || (rstd_k && !aligned(rstd_k, 4)) ||
        (pos_ids && !aligned(pos_ids, 4)))
        return QKNR_ERR_ALIGNMENT;

    const size_t nq = (size_t)T * Hq, nk = (size_t)T * Hkv;
    Span all[] = {
        {(const char *)q, nq * D * e},          {(const char *)k, nk * D * e},
        {(const char *)gamma_q, Hq ? D * e : 0}, {(const char *)gamma_k, Hkv ? D * e : 0},
        {(const char *)pos_ids, pos_ids ? (size_t)T * 4 : 0},
        {(const char *)q_out, nq * D * e},      {(const char *)k_out, nk * D * e},
        {(const char *)rstd_q, nq * 4},         {(const char *)rstd_k, nk * 4},
    };
    const int may_equal[] = {0, 1, -1, -1};  // q_out may be q, k_out may be k
    if (check_overlaps(all, 9, 5, may_equal) != QKNR_OK) return QKNR_ERR_INVALID_ARG;

    FwdArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.qo = q_out; a.ko = k_out; a.rq = rstd_q; a.rk = rstd_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    a.theta = theta; a.eps = eps;
    const int lpr = lanes_per_row(D, (int)e);
    cudaStream_t cs = (cudaStream_t)stream;
    return dtype == QKNR_F32 ? dispatch_fwd<float>(a, lpr, cs)
                             : dispatch_fwd<__nv_bfloat16>(a, lpr, cs);
}

extern "C" qknr_status qk_norm_rope_bwd(const void *q, const void *k,
                                        const void *gamma_q, const void *gamma_k,
                                        const int32_t *pos_ids, const float *rstd_q,
                                        const float *rstd_k, const void *dq_out,
                                        const void *dk_out, void *dq, void *dk,
                                        float *dgamma_q, float *dgamma_k, int B, int S, int Hq,
                                        int Hkv, int D, int rotary_dim, float theta, float eps,
                                        qknr_dtype dtype, qknr_stream_t stream) {
    qknr_status st = check_shape(B, S, Hq, Hkv, D, rotary_dim, theta, eps, dtype);
    if (st != QKNR_OK) return st;
    const int64_t T = (int64_t)B * S;
    const size_t e = dtype == QKNR_F32 ? 4 : 2;
    const bool work = T > 0 && Hq + Hkv > 0;
    if (work && Hq > 0 && (!q || !gamma_q || !rstd_q || !dq_out || !dq)) return QKNR_ERR_INVALID_ARG;
    if (work && Hkv > 0 && (!k || !gamma_k || !rstd_k || !dk_out || !dk)) return QKNR_ERR_INVALID_ARG;
    const void *vec[] = {q, k, gamma_q, gamma_k, dq_out, dk_out, dq, dk};
    for (const void *p : vec)
        if (p && !aligned(p, 16)) return QKNR_ERR_ALIGNMENT;
    if ((rstd_q && !aligned(rstd_q, 4)) || (rstd_k && !aligned(rstd_k, 4)) ||
        (pos_ids && !aligned(pos_ids, 4)) || (dgamma_q && !aligned(dgamma_q, 4)) ||
        (dgamma_k && !aligned(dgamma_k, 4)))
        return QKNR_ERR_ALIGNMENT;

    const size_t nq = work ? (size_t)T * Hq : 0, nk = work ? (size_t)T * Hkv : 0;
    Span all[] = {
        {(const char *)q, nq * D * e},           {(const char *)k, nk * D * e},
        {(const char *)gamma_q, Hq ? D * e : 0},  {(const char *)gamma_k, Hkv ? D * e : 0},
        {(const char *)pos_ids, pos_ids && work ? (size_t)T * 4 : 0},
        {(const char *)rstd_q, nq * 4},          {(const char *)rstd_k, nk * 4},
        {(const char *)dq_out, nq * D * e},      {(const char *)dk_out, nk * D * e},
        {(const char *)dq, nq * D * e},          {(const char *)dk, nk * D * e},
        {(const char *)dgamma_q, dgamma_q ? D * 4 : 0},
        {(const char *)dgamma_k, dgamma_k ? D * 4 : 0},
    };
    const int may_equal[] = {7, 8, -1, -1};  // dq may be dq_out, dk may be dk_out
    if (check_overlaps(all, 13, 9, may_equal) != QKNR_OK) return QKNR_ERR_INVALID_ARG;

    cudaStream_t cs = (cudaStream_t)stream;
    if (dgamma_q) {
        cudaError_t ce = cudaMemsetAsync(dgamma_q, 0, (size_t)D * 4, cs);
        if (ce != cudaSuccess) return cuda_fail(ce);
    }
    if (dgamma_k) {
        cudaError_t ce = cudaMemsetAsync(dgamma_k, 0, (size_t)D * 4, cs);
        if (ce != cudaSuccess) return cuda_fail(ce);
    }
    if (!work) return QKNR_OK;

    BwdArgs a{};
    a.q = q; a.k = k; a.gq = gamma_q; a.gk = gamma_k; a.pos = pos_ids;
    a.rq = rstd_q; a.rk = rstd_k; a.dqo = dq_out; a.dko = dk_out;
    a.dq = dq; a.dk = dk; a.dgq = dgamma_q; a.dgk = dgamma_k;
    a.T = T; a.S = S; a.Hq = Hq; a.Hkv = Hkv; a.D = D; a.R = rotary_dim;
    a.theta = theta; a.eps = eps;
    const int lpr = lanes_per_row(D, (int)e);
    return dtype == QKNR_F32 ? dispatch_bwd<float>(a, lpr, cs)
                             : dispatch_bwd<__nv_bfloat16>(a, lpr, cs);
}

extern "C" const char *qknr_strerror(qknr_status s) {
    switch (s) {
        case QKNR_OK: return "success";
        case QKNR_ERR_INVALID_ARG: return "invalid argument (size, NULL pointer, overlap, theta or eps)";
        case QKNR_ERR_ALIGNMENT: return "pointer not aligned (16 bytes for vectors, 4 for fp32/int32 arrays)";
        case QKNR_ERR_UNSUPPORTED: return "unsupported shape (D <= 256, D*elem a multiple of 32, (R/2)*elem a multiple of 16)";
        case QKNR_ERR_CUDA: return "the CUDA runtime refused the launch (see qknr_last_cuda_error)";
    }
    return "unknown status";
}

extern "C" int qknr_last_cuda_error(void) { return g_last_cuda_error; }
