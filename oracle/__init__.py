"""CPU oracle for the fused QK-RMSNorm + RoPE path (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The CUDA library and its Python
binding never do; the two implementations share no code.

The arithmetic lives in ``qknr_oracle.c`` (plain fp64 C, one row at a time);
this module only converts arrays to fp64, resolves each token's position and
calls it through ctypes. See the C file's header for the definition and the
passages it follows.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def _p(a: np.ndarray, ptr=_D):
    return a.ctypes.data_as(ptr)


def positions(pos_ids, B: int, S: int) -> np.ndarray:
    """Each token's position: the given int32 id, else s within its batch row."""
    if pos_ids is None:
        return np.tile(np.arange(S, dtype=np.int64), B)
    p = np.asarray(pos_ids).reshape(B * S)
    return p.astype(np.int64)


def as_f64(a) -> np.ndarray:
    """Exact upcast of a torch tensor / numpy array (fp32 or bf16) to fp64."""
    if hasattr(a, "detach"):
        import torch
        a = a.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


class Oracle:
    """Handle on one compiled oracle shared object."""

    def __init__(self, lib_path: Optional[str] = None):
        if lib_path is None:
            if _build.needs_build():
                _build.build()
            lib_path = _build.LIB
        self.path = lib_path
        self.lib = lib = ctypes.CDLL(lib_path)
        c_int, c_dbl, c_i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.oracle_inv_freq.restype = c_dbl
        lib.oracle_inv_freq.argtypes = [c_int, c_int, c_dbl]
        lib.oracle_rstd.restype = c_dbl
        lib.oracle_rstd.argtypes = [_D, c_int, c_dbl]
        lib.oracle_fwd.restype = None
        lib.oracle_fwd.argtypes = [_D, _D, _D, _D, _I64, c_i64, c_int, c_int,
                                   c_int, c_int, c_dbl, c_dbl, _D, _D, _D, _D]
        lib.oracle_bwd.restype = None
        lib.oracle_bwd.argtypes = [_D, _D, _D, _D, _I64, _D, _D, c_i64, c_int,
                                   c_int, c_int, c_int, c_dbl, c_dbl,
                                   _D, _D, _D, _D]
        lib.oracle_fwd_rows.restype = None
        lib.oracle_fwd_rows.argtypes = [_D, _D, _I64, c_i64, c_int, c_int,
                                        c_dbl, c_dbl, _D, _D]
        lib.oracle_bwd_rows.restype = None
        lib.oracle_bwd_rows.argtypes = [_D, _D, _D, _I64, c_i64, c_int, c_int,
                                        c_dbl, c_dbl, _D, _D]
        lib.oracle_ln_fwd_rows.restype = None
        lib.oracle_ln_fwd_rows.argtypes = [_D, _D, _I64, c_i64, c_int, c_int,
                                           c_dbl, c_dbl, _D, _D]
        lib.oracle_ln_bwd_rows.restype = None
        lib.oracle_ln_bwd_rows.argtypes = [_D, _D, _D, _I64, c_i64, c_int,
                                           c_int, c_dbl, c_dbl, _D, _D]
        lib.oracle_lw_fwd.restype = None
        lib.oracle_lw_fwd.argtypes = [_D, _D, _I64, c_i64, c_int, c_int, c_int,
                                      c_dbl, c_dbl, _D, _D]
        lib.oracle_lw_bwd.restype = None
        lib.oracle_lw_bwd.argtypes = [_D, _D, _D, _I64, c_i64, c_int, c_int,
                                      c_int, c_dbl, c_dbl, _D, _D]
        lib.oracle_rope_rows.restype = None
        lib.oracle_rope_rows.argtypes = [_D, _I64, c_i64, c_int, c_int, c_dbl,
                                         c_int, _D]

    # ---------------------------------------------------------------- scalars
    def inv_freq(self, i: int, R: int, theta: float) -> float:
        return self.lib.oracle_inv_freq(i, R, theta)

    # ---------------------------------------------------------------- tensors
    def fwd(self, q, k, gamma_q, gamma_k, m, R: int, theta: float, eps: float):
        """Forward over tokens. q [..., Hq, D], k [..., Hkv, D] (leading dims
        flatten to tokens in C order), m: per-token positions (len T).

        Returns fp64 (q_out, k_out, rstd_q, rstd_k) shaped like the inputs.
        """
        q, k = as_f64(q), as_f64(k)
        gq, gk = as_f64(gamma_q), as_f64(gamma_k)
        Hq, D = q.shape[-2], q.shape[-1]
        Hkv = k.shape[-2]
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(-1))
        T = m.size
        q_out = np.empty_like(q)
        k_out = np.empty_like(k)
        rq = np.empty(q.shape[:-1], dtype=np.float64)
        rk = np.empty(k.shape[:-1], dtype=np.float64)
        self.lib.oracle_fwd(_p(q), _p(k), _p(gq), _p(gk), _p(m, _I64), T, Hq,
                            Hkv, D, R, float(theta), float(eps), _p(q_out),
                            _p(k_out), _p(rq), _p(rk))
        return q_out, k_out, rq, rk

    def bwd(self, q, k, gamma_q, gamma_k, m, dq_out, dk_out, R: int,
            theta: float, eps: float, dgamma_q=None, dgamma_k=None):
        """Backward over tokens. Returns fp64 (dq, dk, dgamma_q, dgamma_k).

        When ``dgamma_q`` / ``dgamma_k`` (fp64 [D]) are given they are
        accumulated into and returned (for evaluating a long run of tokens in
        consecutive pieces); otherwise fresh zeroed arrays are used.
        """
        q, k = as_f64(q), as_f64(k)
        dqo, dko = as_f64(dq_out), as_f64(dk_out)
        gq, gk = as_f64(gamma_q), as_f64(gamma_k)
        Hq, D = q.shape[-2], q.shape[-1]
        Hkv = k.shape[-2]
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(-1))
        T = m.size
        dq = np.empty_like(q)
        dk = np.empty_like(k)
        dgq = np.zeros(D) if dgamma_q is None else dgamma_q
        dgk = np.zeros(D) if dgamma_k is None else dgamma_k
        self.lib.oracle_bwd(_p(q), _p(k), _p(gq), _p(gk), _p(m, _I64),
                            _p(dqo), _p(dko), T, Hq, Hkv, D, R, float(theta),
                            float(eps), _p(dq), _p(dk), _p(dgq), _p(dgk))
        return dq, dk, dgq, dgk

    def fwd_rows(self, x, gamma, m, R: int, theta: float, eps: float):
        """Independent rows x [n, D], each at its own position m [n]."""
        x, g = as_f64(x), as_f64(gamma)
        n, D = x.shape
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(n))
        y = np.empty_like(x)
        r = np.empty(n)
        self.lib.oracle_fwd_rows(_p(x), _p(g), _p(m, _I64), n, D, R,
                                 float(theta), float(eps), _p(y), _p(r))
        return y, r

    def bwd_rows(self, x, gamma, dy, m, R: int, theta: float, eps: float):
        """Independent rows; returns (dx [n,D], per-row dgamma terms [n,D])."""
        x, g, dy = as_f64(x), as_f64(gamma), as_f64(dy)
        n, D = x.shape
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(n))
        dx = np.empty_like(x)
        dgr = np.empty_like(x)
        self.lib.oracle_bwd_rows(_p(x), _p(g), _p(dy), _p(m, _I64), n, D, R,
                                 float(theta), float(eps), _p(dx), _p(dgr))
        return dx, dgr


    def ln_fwd_rows(self, x, gamma, m, R: int, theta: float, eps: float):
        """Mean-centred (QK-LayerNorm) forward of independent rows."""
        x, g = as_f64(x), as_f64(gamma)
        n, D = x.shape
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(n))
        y = np.empty_like(x)
        r = np.empty(n)
        self.lib.oracle_ln_fwd_rows(_p(x), _p(g), _p(m, _I64), n, D, R,
                                    float(theta), float(eps), _p(y), _p(r))
        return y, r

    def ln_bwd_rows(self, x, gamma, dy, m, R: int, theta: float, eps: float):
        """Mean-centred backward of independent rows; (dx, per-row dgamma terms)."""
        x, g, dy = as_f64(x), as_f64(gamma), as_f64(dy)
        n, D = x.shape
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(n))
        dx = np.empty_like(x)
        dgr = np.empty_like(x)
        self.lib.oracle_ln_bwd_rows(_p(x), _p(g), _p(dy), _p(m, _I64), n, D, R,
                                    float(theta), float(eps), _p(dx), _p(dgr))
        return dx, dgr

    def ln_fwd(self, q, k, gamma_q, gamma_k, m, R: int, theta: float, eps: float):
        """Mean-centred forward over tokens, shaped like ``fwd``."""
        m = np.asarray(m, dtype=np.int64).reshape(-1)
        out = []
        for x, g in ((as_f64(q), gamma_q), (as_f64(k), gamma_k)):
            H, D = x.shape[-2], x.shape[-1]
            y, r = self.ln_fwd_rows(x.reshape(-1, D), g, np.repeat(m, H), R, theta, eps)
            out += [y.reshape(x.shape), r.reshape(x.shape[:-1])]
        return out[0], out[2], out[1], out[3]

    def ln_bwd(self, q, k, gamma_q, gamma_k, m, dq_out, dk_out, R: int, theta: float,
               eps: float):
        """Mean-centred backward over tokens, shaped like ``bwd``."""
        m = np.asarray(m, dtype=np.int64).reshape(-1)
        out = []
        for x, g, dy in ((as_f64(q), gamma_q, dq_out), (as_f64(k), gamma_k, dk_out)):
            H, D = x.shape[-2], x.shape[-1]
            dx, t = self.ln_bwd_rows(x.reshape(-1, D), g, as_f64(dy).reshape(-1, D),
                                     np.repeat(m, H), R, theta, eps)
            out += [dx.reshape(x.shape), t.sum(axis=0)]
        return out[0], out[2], out[1], out[3]

    def lw_fwd(self, x, gamma, m, R: int, theta: float, eps: float):
        """Layerwise forward of one tensor x [..., H, D] (leading dims are
        tokens), gamma [H*D]: one statistic per token over all its heads.
        Returns (y like x, rstd [tokens])."""
        x, g = as_f64(x), as_f64(gamma).reshape(-1)
        H, D = x.shape[-2], x.shape[-1]
        T = x.size // (H * D)
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(T))
        y = np.empty_like(x)
        r = np.empty(T)
        self.lib.oracle_lw_fwd(_p(x), _p(g), _p(m, _I64), T, H, D, R, float(theta),
                               float(eps), _p(y), _p(r))
        return y, r

    def lw_bwd(self, x, gamma, dy, m, R: int, theta: float, eps: float):
        """Layerwise backward of one tensor; returns (dx like x, dgamma [H*D])."""
        x, g, dy = as_f64(x), as_f64(gamma).reshape(-1), as_f64(dy)
        H, D = x.shape[-2], x.shape[-1]
        T = x.size // (H * D)
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(T))
        dx = np.empty_like(x)
        dg = np.zeros(H * D)
        self.lib.oracle_lw_bwd(_p(x), _p(g), _p(dy), _p(m, _I64), T, H, D, R,
                               float(theta), float(eps), _p(dx), _p(dg))
        return dx, dg

    def rope_rows(self, x, m, R: int, theta: float, inverse: bool = False):
        """Rotation alone of rows x [n, D] at positions m [n]: R(m) x, or
        R(m)^T x with ``inverse``."""
        x = as_f64(x)
        n, D = x.shape
        m = np.ascontiguousarray(np.asarray(m, dtype=np.int64).reshape(n))
        y = np.empty_like(x)
        self.lib.oracle_rope_rows(_p(x), _p(m, _I64), n, D, R, float(theta),
                                  1 if inverse else 0, _p(y))
        return y

    def rope(self, q, k, m, R: int, theta: float, inverse: bool = False):
        """Rotation alone over tokens: q [..., Hq, D], k [..., Hkv, D],
        m per-token positions (len T). Returns fp64 (q_out, k_out)."""
        m = np.asarray(m, dtype=np.int64).reshape(-1)
        out = []
        for x in (as_f64(q), as_f64(k)):
            H, D = x.shape[-2], x.shape[-1]
            rows = x.reshape(-1, D)
            y = self.rope_rows(rows, np.repeat(m, H), R, theta, inverse)
            out.append(y.reshape(x.shape))
        return out[0], out[1]


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from this directory's C source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def reference_outputs(inp, t0: int = 0, t1: Optional[int] = None):
    """Oracle fwd + bwd for workload inputs (``workloads.Inputs``) over the
    flattened token range [t0, t1). Returns a dict of fp64 arrays."""
    w = inp.w
    orc = get()
    T = w.B * w.S
    t1 = T if t1 is None else t1
    m = positions(None if inp.pos is None else inp.pos.numpy(), w.B, w.S)[t0:t1]
    q = inp.q.reshape(T, w.Hq, w.D)[t0:t1]
    k = inp.k.reshape(T, w.Hkv, w.D)[t0:t1]
    qo, ko, rq, rk = orc.fwd(q, k, inp.gamma_q, inp.gamma_k, m, w.rotary_dim,
                             w.theta, w.eps)
    out = {"q_out": qo, "k_out": ko, "rstd_q": rq, "rstd_k": rk}
    if inp.dq_out is not None:
        dqo = inp.dq_out.reshape(T, w.Hq, w.D)[t0:t1]
        dko = inp.dk_out.reshape(T, w.Hkv, w.D)[t0:t1]
        dq, dk, dgq, dgk = orc.bwd(q, k, inp.gamma_q, inp.gamma_k, m, dqo, dko,
                                   w.rotary_dim, w.theta, w.eps)
        out.update(dq=dq, dk=dk, dgamma_q=dgq, dgamma_k=dgk)
    return out
