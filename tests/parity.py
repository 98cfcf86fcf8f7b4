"""GPU-vs-oracle comparison helpers for the parity tests.

Tolerances (written here, used by every parity test):

* fp32 I/O: max-abs 1e-5 on q_out, k_out, dq, dk.
* bf16 I/O: max-abs 2e-2 on every element whose oracle value has |ref| < 8
  (below 8 half a bf16 ulp is at most 1/64, so a correctly rounded result
  meets 2e-2 with room for the fp32 arithmetic); on every element,
  |ref| >= 8 included, the GPU value must be within one bf16 ulp of the
  exact value (faithful rounding: the fp32 result rounded once to nearest
  even), with an absolute floor of 1e-5 for values near zero. From |ref| = 8
  up half an ulp alone is 1/32 > 2e-2, so faithful rounding is the
  meaningful bound there; the count of such elements is reported.
* rstd (fp32 in both cases): relative D * 2^-24, the worst-case error of an
  fp32 sum of D squares (the root halves it).
* dgamma: normwise relative error max|gpu - ref| / max|ref| <= 1e-3 (bf16),
  1e-5 (fp32): dgamma sums up to millions of zero-mean terms, so single
  components can sit near zero and an elementwise relative test would be
  ill-conditioned.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle
import workloads

ABS_TOL = {"f32": 1e-5, "bf16": 2e-2}
DGAMMA_REL = {"f32": 1e-5, "bf16": 1e-3}
ORDER_ONE = 8.0
ULP_FLOOR = 1e-5


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at magnitude |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def gpu_run(inp: workloads.Inputs, device="cuda", fwd_only=False, norm="rms"):
    """Run the CUDA fwd (+ bwd) through the C ABI on ``inp``; CPU results.
    ``norm="layer"``: the mean-centred (QK-LayerNorm) entry points."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    w = inp.w
    dev = torch.device(device)
    q, k = inp.q.to(dev), inp.k.to(dev)
    gq, gk = inp.gamma_q.to(dev), inp.gamma_k.to(dev)
    pos = None if inp.pos is None else inp.pos.to(dev)
    qo, ko, rq, rk = qknr.qk_norm_rope_fwd(q, k, gq, gk, pos, rotary_dim=w.rotary_dim,
                                           theta=w.theta, eps=w.eps, norm=norm)
    out = {"q_out": qo, "k_out": ko, "rstd_q": rq, "rstd_k": rk}
    if not fwd_only:
        dqo, dko = inp.dq_out.to(dev), inp.dk_out.to(dev)
        dq, dk, dgq, dgk = qknr.qk_norm_rope_bwd(q, k, gq, gk, pos, rq, rk, dqo, dko,
                                                 rotary_dim=w.rotary_dim, theta=w.theta,
                                                 eps=w.eps, norm=norm)
        out.update(dq=dq, dk=dk, dgamma_q=dgq, dgamma_k=dgk)
    torch.cuda.synchronize()
    return {n: t.cpu() for n, t in out.items()}


class Stats:
    def __init__(self, dtype: str, D: int):
        self.dtype = dtype
        self.D = D
        self.max_abs = {}        # over |ref| < ORDER_ONE (all elements for fp32)
        self.max_ulp = {}        # bf16: max err / ulp(max(|ref|, |gpu|))
        self.n_big = {}          # count of |ref| >= ORDER_ONE
        self.rstd_rel = 0.0

    def elem(self, name, got, ref):
        got = np.asarray(got, np.float64)
        ref = np.asarray(ref, np.float64)
        err = np.abs(got - ref)
        if self.dtype == "f32":
            m = float(err.max()) if err.size else 0.0
        else:
            small = np.abs(ref) < ORDER_ONE
            m = float(err[small].max()) if small.any() else 0.0
            ulp = np.maximum(bf16_ulp(np.maximum(np.abs(ref), np.abs(got))), ULP_FLOOR)
            u = float((err / ulp).max()) if err.size else 0.0
            self.max_ulp[name] = max(self.max_ulp.get(name, 0.0), u)
            self.n_big[name] = self.n_big.get(name, 0) + int((~small).sum())
        self.max_abs[name] = max(self.max_abs.get(name, 0.0), m)

    def rstd(self, got, ref):
        got = np.asarray(got, np.float64)
        ref = np.asarray(ref, np.float64)
        if ref.size:
            self.rstd_rel = max(self.rstd_rel, float((np.abs(got - ref) / ref).max()))

    def check(self, dgamma=None):
        tol = ABS_TOL[self.dtype]
        for n, m in self.max_abs.items():
            assert m <= tol, f"{n}: max-abs err {m:.3e} > {tol:g}"
        for n, u in self.max_ulp.items():
            assert u <= 1.0, f"{n}: {u:.3f} bf16 ulps from the exact value"
        rtol = self.D * 2.0 ** -24
        assert self.rstd_rel <= rtol, f"rstd rel err {self.rstd_rel:.3e} > {rtol:.3e}"
        if dgamma:
            for n, (got, ref) in dgamma.items():
                got = np.asarray(got, np.float64)
                ref = np.asarray(ref, np.float64)
                if not np.abs(ref).max() > 0:      # tensor with no rows
                    assert np.all(got == 0), f"{n}: expected zeros"
                    continue
                rel = float(np.abs(got - ref).max() / np.abs(ref).max())
                assert rel <= DGAMMA_REL[self.dtype], f"{n}: normwise rel err {rel:.3e}"
                assert np.abs(got).max() > 0, f"{n} is zero"

    def merge(self, other: "Stats"):
        """Fold in the statistics of another chunk of the same tensors."""
        for n, m in other.max_abs.items():
            self.max_abs[n] = max(self.max_abs.get(n, 0.0), m)
        for n, u in other.max_ulp.items():
            self.max_ulp[n] = max(self.max_ulp.get(n, 0.0), u)
        for n, c in other.n_big.items():
            self.n_big[n] = self.n_big.get(n, 0) + c
        self.rstd_rel = max(self.rstd_rel, other.rstd_rel)

    def summary(self):
        return dict(max_abs=self.max_abs, max_ulp=self.max_ulp, n_big=self.n_big,
                    rstd_rel=self.rstd_rel)


def _workers() -> int:
    try:
        n = len(os.sched_getaffinity(0))
    except Exception:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def ordered_map(fn, items, workers=None):
    """fn over items on a pool of host threads (the oracle is C called through
    ctypes, which releases the GIL), results in item order, at most 2x
    ``workers`` chunks in flight so memory stays bounded."""
    items = list(items)
    workers = workers or _workers()
    if workers == 1 or len(items) <= 1:
        for it in items:
            yield fn(it)
        return
    with ThreadPoolExecutor(workers) as ex:
        pending = []
        i = 0
        while i < len(items) or pending:
            while i < len(items) and len(pending) < 2 * workers:
                pending.append(ex.submit(fn, items[i]))
                i += 1
            yield pending.pop(0).result()


def compare_with_oracle(inp: workloads.Inputs, got: dict, chunk_tokens: int = 1024,
                        bwd: bool = True, norm: str = "rms") -> Stats:
    """Every element of the GPU results against the oracle, token chunk by
    token chunk (the oracle runs in fp64 on the CPU, chunks on parallel host
    threads; dgamma partials are added in chunk order). ``norm="layer"``
    compares with the oracle's mean-centred form."""
    w = inp.w
    T = w.B * w.S
    orc = oracle.get()
    m_all = oracle.positions(None if inp.pos is None else inp.pos.numpy(), w.B, w.S)
    q = inp.q.reshape(T, w.Hq, w.D)
    k = inp.k.reshape(T, w.Hkv, w.D)

    def view(name, H, last=w.D):
        return got[name].reshape(T, H, last)

    def one(t0):
        t1 = min(T, t0 + chunk_tokens)
        st = Stats(w.dtype, w.D)
        m = m_all[t0:t1]
        fwd = orc.ln_fwd if norm == "layer" else orc.fwd
        qo, ko, rq, rk = fwd(q[t0:t1], k[t0:t1], inp.gamma_q, inp.gamma_k, m,
                             w.rotary_dim, w.theta, w.eps)
        st.elem("q_out", oracle.as_f64(view("q_out", w.Hq)[t0:t1]), qo)
        st.elem("k_out", oracle.as_f64(view("k_out", w.Hkv)[t0:t1]), ko)
        st.rstd(oracle.as_f64(view("rstd_q", w.Hq, 1)[t0:t1]).reshape(-1), rq.reshape(-1))
        st.rstd(oracle.as_f64(view("rstd_k", w.Hkv, 1)[t0:t1]).reshape(-1), rk.reshape(-1))
        cq = ck = None
        if bwd:
            dqo = inp.dq_out.reshape(T, w.Hq, w.D)[t0:t1]
            dko = inp.dk_out.reshape(T, w.Hkv, w.D)[t0:t1]
            if norm == "layer":
                dq, dk, cq, ck = orc.ln_bwd(q[t0:t1], k[t0:t1], inp.gamma_q, inp.gamma_k, m,
                                            dqo, dko, w.rotary_dim, w.theta, w.eps)
            else:
                dq, dk, cq, ck = orc.bwd(q[t0:t1], k[t0:t1], inp.gamma_q, inp.gamma_k, m,
                                         dqo, dko, w.rotary_dim, w.theta, w.eps)
            st.elem("dq", oracle.as_f64(view("dq", w.Hq)[t0:t1]), dq)
            st.elem("dk", oracle.as_f64(view("dk", w.Hkv)[t0:t1]), dk)
        return st, cq, ck

    total = Stats(w.dtype, w.D)
    dgq = np.zeros(w.D)
    dgk = np.zeros(w.D)
    for st, cq, ck in ordered_map(one, range(0, T, chunk_tokens)):
        total.merge(st)
        if cq is not None:
            dgq, dgk = dgq + cq, dgk + ck
    total.dgamma = {"dgamma_q": (got["dgamma_q"].numpy(), dgq),
                    "dgamma_k": (got["dgamma_k"].numpy(), dgk)} if bwd else None
    return total


def check(inp, got, **kw) -> Stats:
    st = compare_with_oracle(inp, got, **kw)
    if st.n_big:
        print("elements with |ref| >= %g (held to one bf16 ulp):" % ORDER_ONE, st.n_big)
    st.check(st.dgamma)
    return st
