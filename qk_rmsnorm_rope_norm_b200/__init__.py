"""Fused per-head QK-RMSNorm + rotate-half RoPE for NVIDIA B200 (sm_100a).

Thin ctypes binding of ``libqknr.so`` (the C ABI declared in
``include/qknr.h``). This module only marshals arguments: it checks tensor
metadata, allocates outputs the caller did not pass, and hands raw device
pointers and the current CUDA stream to the library. Every step of the
computation runs in the library's CUDA kernels; there is no fallback, and
every entry point raises if the library is missing or a tensor is not on a
CUDA device.

Names follow the C ABI: ``qk_norm_rope_fwd`` / ``qk_norm_rope_bwd`` (which
also take Q / K slices of a fused QKV buffer, dispatching to the
``_strided`` entry points). The autograd wrappers ``QKNormRoPE`` and
``QKNormRoPEFromQKV`` chain them for training code. The layerwise form for
tensor parallelism (``qk_layerwise_*``) is chained by
``QKLayerwiseNormRoPE``, which sums the per-token partial statistics over a
``torch.distributed`` group between its kernel calls.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["qk_norm_rope_fwd", "qk_norm_rope_bwd", "qknr_strerror", "QKNormRoPE",
           "QKNormRoPEFromQKV", "qk_norm_rope_qkv", "split_qkv",
           "qk_norm_fwd", "qk_norm_bwd", "qk_rope_apply", "QKRoPE", "qk_rms_stats",
           "prepare_fwd", "prepare_bwd", "PreparedCall",
           "qk_norm_rope", "QKNRError", "library_path", "load_library", "pipeline_error",
           "qk_layerwise_stats", "qk_layerwise_norm_rope_fwd", "qk_layerwise_bwd_dots",
           "qk_layerwise_norm_rope_bwd", "QKLayerwiseNormRoPE", "qk_layerwise_norm_rope",
           "all_reduce_stats", "layerwise_geometry", "launch_plan", "kernel_name",
           "wait_selftest", "token_chunks", "chunk_count", "run_chunked", "layerwise_chunked_fwd",
           "layerwise_chunked_bwd", "MIN_CHUNK_TOKENS", "MIN_CHUNK_BYTES"]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqknr.so")

QKNR_OK, QKNR_ERR_INVALID_ARG, QKNR_ERR_ALIGNMENT, QKNR_ERR_UNSUPPORTED, QKNR_ERR_CUDA = range(5)
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}

_lib = None


class QKNRError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = qknr_strerror(status)
        if status == QKNR_ERR_CUDA:
            msg += f" (cudaError {load_library().qknr_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load ``libqknr.so`` (build it with ``python -m qk_rmsnorm_rope_norm_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m qk_rmsnorm_rope_norm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.qk_norm_rope_fwd.restype = i32
    lib.qk_norm_rope_fwd.argtypes = [vp] * 9 + [i32] * 6 + [f32, f32, i32, vp]
    lib.qk_norm_rope_bwd.restype = i32
    lib.qk_norm_rope_bwd.argtypes = [vp] * 13 + [i32] * 6 + [f32, f32, i32, vp]
    i64 = ctypes.c_int64
    lib.qk_norm_rope_fwd_strided.restype = i32
    lib.qk_norm_rope_fwd_strided.argtypes = [vp, vp, i64, i64] + [vp] * 7 + [i32] * 6 + \
        [f32, f32, i32, vp]
    for n in ("qk_layernorm_rope_fwd", "qk_layernorm_rope_bwd"):
        fn, ref = getattr(lib, n), getattr(lib, n.replace("layernorm", "norm"))
        fn.restype, fn.argtypes = ref.restype, ref.argtypes
    lib.qk_norm_fwd.restype = i32
    lib.qk_norm_fwd.argtypes = [vp] * 8 + [i32] * 5 + [f32, i32, vp]
    lib.qk_norm_bwd.restype = i32
    lib.qk_norm_bwd.argtypes = [vp] * 12 + [i32] * 5 + [f32, i32, vp]
    lib.qk_rms_stats.restype = i32
    lib.qk_rms_stats.argtypes = [vp] * 4 + [i32] * 5 + [f32, i32, vp]
    lib.qk_rope_apply.restype = i32
    lib.qk_rope_apply.argtypes = [vp] * 5 + [i32] * 6 + [f32, i32, i32, vp]
    lib.qk_norm_rope_bwd_strided.restype = i32
    lib.qk_norm_rope_bwd_strided.argtypes = [vp, vp, i64, i64] + [vp] * 9 + [i64, i64] + \
        [vp] * 2 + [i32] * 6 + [f32, f32, i32, vp]
    lib.qk_layerwise_stats.restype = i32
    lib.qk_layerwise_stats.argtypes = [vp] * 4 + [i32] * 5 + [i32, vp]
    lib.qk_layerwise_norm_rope_fwd.restype = i32
    lib.qk_layerwise_norm_rope_fwd.argtypes = [vp] * 11 + [i32] * 8 + [f32, f32, i32, vp]
    lib.qk_layerwise_bwd_dots.restype = i32
    lib.qk_layerwise_bwd_dots.argtypes = [vp] * 11 + [i32] * 6 + [f32, i32, vp]
    lib.qk_layerwise_norm_rope_bwd.restype = i32
    lib.qk_layerwise_norm_rope_bwd.argtypes = [vp] * 15 + [i32] * 8 + [f32, i32, vp]
    lib.qk_layerwise_norm_rope_bwd_acc.restype = i32
    lib.qk_layerwise_norm_rope_bwd_acc.argtypes = lib.qk_layerwise_norm_rope_bwd.argtypes
    lib.qk_layerwise_geometry.restype = i32
    lib.qk_layerwise_geometry.argtypes = [i32] * 9 + [vp]
    lib.qk_norm_rope_plan.restype = i32
    lib.qk_norm_rope_plan.argtypes = [i32] * 11 + [vp]
    lib.qknr_strerror.restype = ctypes.c_char_p
    lib.qknr_strerror.argtypes = [i32]
    lib.qknr_last_cuda_error.restype = i32
    lib.qknr_last_cuda_error.argtypes = []
    lib.qknr_pipeline_error.restype = i32
    lib.qknr_pipeline_error.argtypes = [i32]
    lib.qknr_wait_selftest.restype = i32
    lib.qknr_wait_selftest.argtypes = [i32, i64, vp]
    _lib = lib
    return lib


def qknr_strerror(status: int) -> str:
    return load_library().qknr_strerror(int(status)).decode()


def pipeline_error(reset: bool = False) -> int:
    """Non-zero if a pipelined kernel on the current device gave up a bounded
    internal wait since the flag was last cleared (synchronises)."""
    return int(load_library().qknr_pipeline_error(1 if reset else 0))


def wait_selftest(family: int = 0, limit_cycles: int = 100_000, stream=None) -> None:
    """Run the bounded-wait self-test of a kernel family (0: per-head, 1:
    layerwise): a wait on a barrier nothing completes gives up and sets the
    flag that ``pipeline_error`` reports."""
    st = load_library().qknr_wait_selftest(int(family), int(limit_cycles), _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qknr_wait_selftest")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(name: str, t: torch.Tensor):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _token_stride(name: str, t: torch.Tensor) -> int:
    """Elements between consecutive tokens of a [B, S, H, D] CUDA tensor whose
    heads and dims are dense and whose tokens (t = b * S + s) are evenly
    spaced: a dense tensor, or a Q / K slice of a fused QKV buffer."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() != 4:
        raise ValueError(f"{name} must be [B, S, H, D]")
    B, S, H, D = t.shape
    if t.is_contiguous():
        return H * D
    st = t.stride()
    ts = st[1] if S > 1 else (st[0] if B > 1 else H * D)
    ok = (D <= 1 or st[3] == 1) and (H <= 1 or st[2] == D) and ts >= H * D
    ok = ok and (B <= 1 or S <= 1 or st[0] == S * st[1]) and (S > 1 or B <= 1 or st[0] == ts)
    if not ok:
        raise ValueError(f"{name} must be dense within each token, with tokens evenly spaced "
                         f"(strides {tuple(st)})")
    return int(ts)


def _shape(q: torch.Tensor, k: torch.Tensor):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, S, H, D]")
    B, S, Hq, D = q.shape
    if k.shape[0] != B or k.shape[1] != S or k.shape[3] != D:
        raise ValueError(f"k shape {tuple(k.shape)} does not match q {tuple(q.shape)}")
    return B, S, Hq, k.shape[2], D


def qk_norm_rope_fwd(q, k, gamma_q, gamma_k, pos_ids=None, *, rotary_dim: int,
                     theta: float, eps: float, q_out=None, k_out=None,
                     rstd_q=None, rstd_k=None, stream=None, norm: str = "rms"):
    """Forward. Returns ``(q_out, k_out, rstd_q, rstd_k)``.

    q [B,S,Hq,D], k [B,S,Hkv,D] (fp32 or bf16, contiguous, CUDA); gamma_q,
    gamma_k [D] same dtype; pos_ids optional int32 [B,S]. Outputs not given
    are allocated; ``q_out=q`` / ``k_out=k`` runs in place. ``norm="layer"``
    selects the mean-centred form (C ``qk_layernorm_rope_fwd``; dense q, k).
    """
    lib = load_library()
    qts, kts = _token_stride("q", q), _token_stride("k", k)
    for n, t in (("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    if q.dtype not in _DTYPES or k.dtype != q.dtype or gamma_q.dtype != q.dtype \
            or gamma_k.dtype != q.dtype:
        raise ValueError("q, k, gamma_q, gamma_k must share one dtype (float32 or bfloat16)")
    if pos_ids is not None:
        _need_cuda("pos_ids", pos_ids)
        if pos_ids.dtype != torch.int32 or tuple(pos_ids.shape) != (B, S):
            raise ValueError("pos_ids must be int32 [B, S]")
    q_out = torch.empty(q.shape, dtype=q.dtype, device=q.device) if q_out is None else q_out
    k_out = torch.empty(k.shape, dtype=k.dtype, device=k.device) if k_out is None else k_out
    if rstd_q is None:
        rstd_q = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device)
    if rstd_k is None:
        rstd_k = torch.empty((B, S, Hkv), dtype=torch.float32, device=q.device)
    for n, t in (("q_out", q_out), ("k_out", k_out), ("rstd_q", rstd_q), ("rstd_k", rstd_k)):
        _need_cuda(n, t)
    if q_out.shape != q.shape or k_out.shape != k.shape or q_out.dtype != q.dtype \
            or k_out.dtype != q.dtype:
        raise ValueError("q_out / k_out must match q / k in shape and dtype")
    if rstd_q.dtype != torch.float32 or rstd_k.dtype != torch.float32 or \
            tuple(rstd_q.shape) != (B, S, Hq) or tuple(rstd_k.shape) != (B, S, Hkv):
        raise ValueError("rstd_q / rstd_k must be float32 [B,S,Hq] / [B,S,Hkv]")
    fn, name, args = _fwd_args(lib, q, k, qts, kts, gamma_q, gamma_k, pos_ids, q_out, k_out,
                               rstd_q, rstd_k, rotary_dim, theta, eps, stream, norm)
    st = fn(*args)
    if st != QKNR_OK:
        raise QKNRError(st, name)
    return q_out, k_out, rstd_q, rstd_k


def _fwd_args(lib, q, k, qts, kts, gamma_q, gamma_k, pos_ids, q_out, k_out, rstd_q, rstd_k,
              rotary_dim, theta, eps, stream, norm="rms"):
    """(C function, its name, argument tuple): the dense entry point when q and
    k are dense, else the strided one."""
    B, S, Hq, Hkv, D = _shape(q, k)
    tail = (_ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(q_out), _ptr(k_out),
            _ptr(rstd_q), _ptr(rstd_k), B, S, Hq, Hkv, D, int(rotary_dim), float(theta),
            float(eps), _DTYPES[q.dtype], _stream(stream))
    if norm not in ("rms", "layer"):
        raise ValueError("norm must be 'rms' or 'layer'")
    if norm == "layer":
        if qts != Hq * D or kts != Hkv * D:
            raise ValueError("the mean-centred form takes dense q and k")
        return lib.qk_layernorm_rope_fwd, "qk_layernorm_rope_fwd", (_ptr(q), _ptr(k)) + tail
    if qts == Hq * D and kts == Hkv * D:
        return lib.qk_norm_rope_fwd, "qk_norm_rope_fwd", (_ptr(q), _ptr(k)) + tail
    return lib.qk_norm_rope_fwd_strided, "qk_norm_rope_fwd_strided", \
        (_ptr(q), _ptr(k), qts, kts) + tail


def qk_norm_rope_bwd(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, *,
                     rotary_dim: int, theta: float, eps: float, dq=None, dk=None,
                     dgamma_q=None, dgamma_k=None, need_dgamma: bool = True, stream=None,
                     norm: str = "rms"):
    """Backward. Returns ``(dq, dk, dgamma_q, dgamma_k)`` (dgamma fp32 [D]).

    ``dq=dq_out`` / ``dk=dk_out`` runs in place. With ``need_dgamma=False``
    and no dgamma buffers given, the gamma gradients are skipped (None).
    """
    lib = load_library()
    qts, kts = _token_stride("q", q), _token_stride("k", k)
    for n, t in (("gamma_q", gamma_q), ("gamma_k", gamma_k),
                 ("rstd_q", rstd_q), ("rstd_k", rstd_k), ("dq_out", dq_out), ("dk_out", dk_out)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype for t in (k, gamma_q, gamma_k, dq_out, dk_out)):
        raise ValueError("q, k, gamma, dq_out, dk_out must share one dtype")
    if dq_out.shape != q.shape or dk_out.shape != k.shape:
        raise ValueError("dq_out / dk_out must match q / k")
    if rstd_q.dtype != torch.float32 or rstd_k.dtype != torch.float32 or \
            tuple(rstd_q.shape) != (B, S, Hq) or tuple(rstd_k.shape) != (B, S, Hkv):
        raise ValueError("rstd_q / rstd_k must be float32 [B,S,Hq] / [B,S,Hkv]")
    if pos_ids is not None:
        _need_cuda("pos_ids", pos_ids)
        if pos_ids.dtype != torch.int32 or tuple(pos_ids.shape) != (B, S):
            raise ValueError("pos_ids must be int32 [B, S]")
    dq = torch.empty(q.shape, dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=k.dtype, device=k.device) if dk is None else dk
    if need_dgamma:
        if dgamma_q is None:
            dgamma_q = torch.empty(D, dtype=torch.float32, device=q.device)
        if dgamma_k is None:
            dgamma_k = torch.empty(D, dtype=torch.float32, device=q.device)
    dqts, dkts = _token_stride("dq", dq), _token_stride("dk", dk)
    if dq.shape != q.shape or dk.shape != k.shape or dq.dtype != q.dtype or dk.dtype != q.dtype:
        raise ValueError("dq / dk must match q / k in shape and dtype")
    for n, t in (("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k)):
        if t is not None:
            _need_cuda(n, t)
            if t.dtype != torch.float32 or t.numel() != D:
                raise ValueError(f"{n} must be float32 [D]")
    fn, name, args = _bwd_args(lib, q, k, qts, kts, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k,
                               dq_out, dk_out, dq, dk, dqts, dkts, dgamma_q, dgamma_k,
                               rotary_dim, theta, eps, stream, norm)
    st = fn(*args)
    if st != QKNR_OK:
        raise QKNRError(st, name)
    return dq, dk, dgamma_q, dgamma_k


def _bwd_args(lib, q, k, qts, kts, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out,
              dq, dk, dqts, dkts, dgamma_q, dgamma_k, rotary_dim, theta, eps, stream, norm="rms"):
    B, S, Hq, Hkv, D = _shape(q, k)
    tail = (B, S, Hq, Hkv, D, int(rotary_dim), float(theta), float(eps), _DTYPES[q.dtype],
            _stream(stream))
    dense = qts == Hq * D and kts == Hkv * D and dqts == Hq * D and dkts == Hkv * D
    if norm not in ("rms", "layer"):
        raise ValueError("norm must be 'rms' or 'layer'")
    if norm == "layer" and not dense:
        raise ValueError("the mean-centred form takes dense q, k, dq and dk")
    if dense:
        fn = lib.qk_layernorm_rope_bwd if norm == "layer" else lib.qk_norm_rope_bwd
        return fn, fn.__name__, (
            _ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(rstd_q),
            _ptr(rstd_k), _ptr(dq_out), _ptr(dk_out), _ptr(dq), _ptr(dk), _ptr(dgamma_q),
            _ptr(dgamma_k)) + tail
    return lib.qk_norm_rope_bwd_strided, "qk_norm_rope_bwd_strided", (
        _ptr(q), _ptr(k), qts, kts, _ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(rstd_q),
        _ptr(rstd_k), _ptr(dq_out), _ptr(dk_out), _ptr(dq), _ptr(dk), dqts, dkts,
        _ptr(dgamma_q), _ptr(dgamma_k)) + tail


class QKNormRoPE(torch.autograd.Function):
    """Autograd wrapper: forward saves q, k, gamma and rstd; backward calls
    ``qk_norm_rope_bwd``. gamma gradients are returned in gamma's dtype."""

    @staticmethod
    def forward(ctx, q, k, gamma_q, gamma_k, pos_ids, rotary_dim, theta, eps, norm="rms"):
        q_out, k_out, rq, rk = qk_norm_rope_fwd(q, k, gamma_q, gamma_k, pos_ids,
                                                rotary_dim=rotary_dim, theta=theta, eps=eps,
                                                norm=norm)
        ctx.save_for_backward(q, k, gamma_q, gamma_k, rq, rk)
        ctx.pos_ids = pos_ids
        ctx.cfg = (rotary_dim, theta, eps, norm)
        ctx.mark_non_differentiable(rq, rk)
        return q_out, k_out

    @staticmethod
    def backward(ctx, dq_out, dk_out):
        q, k, gq, gk, rq, rk = ctx.saved_tensors
        R, theta, eps, norm = ctx.cfg
        dq, dk, dgq, dgk = qk_norm_rope_bwd(
            q, k, gq, gk, ctx.pos_ids, rq, rk, dq_out.contiguous(), dk_out.contiguous(),
            rotary_dim=R, theta=theta, eps=eps,
            need_dgamma=ctx.needs_input_grad[2] or ctx.needs_input_grad[3], norm=norm)
        dgq = None if dgq is None else dgq.to(gq.dtype)
        dgk = None if dgk is None else dgk.to(gk.dtype)
        return dq, dk, dgq, dgk, None, None, None, None, None


def qk_norm_rope(q, k, gamma_q, gamma_k, pos_ids=None, *, rotary_dim: int, theta: float,
                 eps: float, norm: str = "rms"):
    """Differentiable fused op; returns ``(q_out, k_out)``. ``norm="layer"``
    is the mean-centred (QK-LayerNorm) form."""
    return QKNormRoPE.apply(q, k, gamma_q, gamma_k, pos_ids, rotary_dim, theta, eps, norm)


def qk_norm_fwd(q, k, gamma_q, gamma_k, *, eps: float, q_out=None, k_out=None,
                rstd_q=None, rstd_k=None, stream=None):
    """Per-head QK-RMSNorm alone (the NoPE layers' op, C ``qk_norm_fwd``).
    Returns ``(q_out, k_out, rstd_q, rstd_k)``; tensors as for
    ``qk_norm_rope_fwd`` (dense)."""
    lib = load_library()
    for n, t in (("q", q), ("k", k), ("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k, gamma_q, gamma_k)
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    rstd_q = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device) if rstd_q is None else rstd_q
    rstd_k = torch.empty((B, S, Hkv), dtype=torch.float32, device=q.device) if rstd_k is None else rstd_k
    _check_outputs(q, k, q_out, k_out, rstd_q, rstd_k)
    st = lib.qk_norm_fwd(_ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(q_out), _ptr(k_out),
                         _ptr(rstd_q), _ptr(rstd_k), B, S, Hq, Hkv, D, float(eps),
                         _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_norm_fwd")
    return q_out, k_out, rstd_q, rstd_k


def qk_norm_bwd(q, k, gamma_q, gamma_k, rstd_q, rstd_k, dq_out, dk_out, *, eps: float,
                dq=None, dk=None, dgamma_q=None, dgamma_k=None, stream=None):
    """Backward of ``qk_norm_fwd`` (C ``qk_norm_bwd``); returns
    ``(dq, dk, dgamma_q, dgamma_k)``, dgamma fp32 [D]."""
    lib = load_library()
    for n, t in (("q", q), ("k", k), ("gamma_q", gamma_q), ("gamma_k", gamma_k),
                 ("rstd_q", rstd_q), ("rstd_k", rstd_k), ("dq_out", dq_out), ("dk_out", dk_out)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k, gamma_q, gamma_k, dq_out, dk_out)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dgamma_q = torch.empty(D, dtype=torch.float32, device=q.device) if dgamma_q is None else dgamma_q
    dgamma_k = torch.empty(D, dtype=torch.float32, device=q.device) if dgamma_k is None else dgamma_k
    for n, t in (("dq", dq), ("dk", dk), ("dgamma_q", dgamma_q), ("dgamma_k", dgamma_k)):
        _need_cuda(n, t)
    st = lib.qk_norm_bwd(_ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(rstd_q),
                         _ptr(rstd_k), _ptr(dq_out), _ptr(dk_out), _ptr(dq), _ptr(dk),
                         _ptr(dgamma_q), _ptr(dgamma_k), B, S, Hq, Hkv, D, float(eps),
                         _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_norm_bwd")
    return dq, dk, dgamma_q, dgamma_k


def qk_rope_apply(q, k, pos_ids=None, *, rotary_dim: int, theta: float, inverse: bool = False,
                  q_out=None, k_out=None, stream=None):
    """Rotate-half RoPE alone (C ``qk_rope_apply``): R(m) q, R(m) k, or with
    ``inverse`` the transpose R(-m), which strips RoPE from rotated rows.
    Returns ``(q_out, k_out)``; ``q_out=q`` runs in place."""
    lib = load_library()
    for n, t in (("q", q), ("k", k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k)
    if pos_ids is not None:
        _need_cuda("pos_ids", pos_ids)
        if pos_ids.dtype != torch.int32 or tuple(pos_ids.shape) != (B, S):
            raise ValueError("pos_ids must be int32 [B, S]")
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    for n, t in (("q_out", q_out), ("k_out", k_out)):
        _need_cuda(n, t)
    if q_out.shape != q.shape or k_out.shape != k.shape or q_out.dtype != q.dtype \
            or k_out.dtype != q.dtype:
        raise ValueError("q_out / k_out must match q / k in shape and dtype")
    st = lib.qk_rope_apply(_ptr(q), _ptr(k), _ptr(pos_ids), _ptr(q_out), _ptr(k_out), B, S, Hq,
                           Hkv, D, int(rotary_dim), float(theta), 1 if inverse else 0,
                           _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_rope_apply")
    return q_out, k_out


def qk_rms_stats(q, k, *, eps: float, rstd_q=None, rstd_k=None, stream=None):
    """Inverse-RMS statistic alone (C ``qk_rms_stats``): fp32 ``(rstd_q,
    rstd_k)`` [B,S,Hq] / [B,S,Hkv], no normalised rows written."""
    lib = load_library()
    for n, t in (("q", q), ("k", k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k)
    rstd_q = torch.empty((B, S, Hq), dtype=torch.float32, device=q.device) if rstd_q is None else rstd_q
    rstd_k = torch.empty((B, S, Hkv), dtype=torch.float32, device=q.device) if rstd_k is None else rstd_k
    for n, t in (("rstd_q", rstd_q), ("rstd_k", rstd_k)):
        _need_cuda(n, t)
    if rstd_q.dtype != torch.float32 or rstd_k.dtype != torch.float32 or \
            tuple(rstd_q.shape) != (B, S, Hq) or tuple(rstd_k.shape) != (B, S, Hkv):
        raise ValueError("rstd_q / rstd_k must be float32 [B,S,Hq] / [B,S,Hkv]")
    st = lib.qk_rms_stats(_ptr(q), _ptr(k), _ptr(rstd_q), _ptr(rstd_k), B, S, Hq, Hkv, D,
                          float(eps), _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_rms_stats")
    return rstd_q, rstd_k


class QKRoPE(torch.autograd.Function):
    """Autograd wrapper of ``qk_rope_apply``: the gradient of a rotation is
    the opposite rotation of the upstream gradient."""

    @staticmethod
    def forward(ctx, q, k, pos_ids, rotary_dim, theta, inverse):
        ctx.cfg = (pos_ids, rotary_dim, theta, inverse)
        return qk_rope_apply(q, k, pos_ids, rotary_dim=rotary_dim, theta=theta, inverse=inverse)

    @staticmethod
    def backward(ctx, dq_out, dk_out):
        pos_ids, R, theta, inverse = ctx.cfg
        dq, dk = qk_rope_apply(dq_out.contiguous(), dk_out.contiguous(), pos_ids, rotary_dim=R,
                               theta=theta, inverse=not inverse)
        return dq, dk, None, None, None, None


def _same_dtype(*ts):
    if ts[0].dtype not in _DTYPES or any(t.dtype != ts[0].dtype for t in ts):
        raise ValueError("tensors must share one dtype (float32 or bfloat16)")


def _check_outputs(q, k, q_out, k_out, rstd_q, rstd_k):
    B, S, Hq, Hkv, D = _shape(q, k)
    for n, t in (("q_out", q_out), ("k_out", k_out), ("rstd_q", rstd_q), ("rstd_k", rstd_k)):
        _need_cuda(n, t)
    if q_out.shape != q.shape or k_out.shape != k.shape or q_out.dtype != q.dtype \
            or k_out.dtype != q.dtype:
        raise ValueError("q_out / k_out must match q / k in shape and dtype")
    if rstd_q.dtype != torch.float32 or rstd_k.dtype != torch.float32 or \
            tuple(rstd_q.shape) != (B, S, Hq) or tuple(rstd_k.shape) != (B, S, Hkv):
        raise ValueError("rstd_q / rstd_k must be float32 [B,S,Hq] / [B,S,Hkv]")


def split_qkv(qkv: torch.Tensor, Hq: int, Hkv: int):
    """Views ``(q, k, v)`` of a fused projection output qkv [B, S, (Hq + 2 Hkv) D]:
    q [B,S,Hq,D], k and v [B,S,Hkv,D], tokens (Hq + 2 Hkv) D elements apart."""
    if qkv.dim() != 3 or qkv.shape[2] % (Hq + 2 * Hkv):
        raise ValueError("qkv must be [B, S, (Hq + 2 Hkv) * D]")
    B, S, W = qkv.shape
    D = W // (Hq + 2 * Hkv)
    q = qkv[..., :Hq * D].unflatten(-1, (Hq, D))
    k = qkv[..., Hq * D:(Hq + Hkv) * D].unflatten(-1, (Hkv, D))
    v = qkv[..., (Hq + Hkv) * D:].unflatten(-1, (Hkv, D))
    return q, k, v


class QKNormRoPEFromQKV(torch.autograd.Function):
    """Fused op on a QKV projection output: q and k are read in place from
    qkv, and the backward writes dq and dk straight into the Q and K slots of
    one dqkv buffer (dv fills the V slot), so no split or concat is copied."""

    @staticmethod
    def forward(ctx, qkv, gamma_q, gamma_k, pos_ids, Hq, Hkv, rotary_dim, theta, eps):
        q, k, v = split_qkv(qkv, Hq, Hkv)
        q_out, k_out, rq, rk = qk_norm_rope_fwd(q, k, gamma_q, gamma_k, pos_ids,
                                                rotary_dim=rotary_dim, theta=theta, eps=eps)
        ctx.save_for_backward(qkv, gamma_q, gamma_k, rq, rk)
        ctx.pos_ids = pos_ids
        ctx.cfg = (Hq, Hkv, rotary_dim, theta, eps)
        ctx.mark_non_differentiable(rq, rk)
        return q_out, k_out, v

    @staticmethod
    def backward(ctx, dq_out, dk_out, dv):
        qkv, gq, gk, rq, rk = ctx.saved_tensors
        Hq, Hkv, R, theta, eps = ctx.cfg
        q, k, _ = split_qkv(qkv, Hq, Hkv)
        dqkv = torch.empty_like(qkv)
        dq, dk, dvs = split_qkv(dqkv, Hq, Hkv)
        if dv is None:
            dvs.zero_()
        else:
            dvs.copy_(dv)
        _, _, dgq, dgk = qk_norm_rope_bwd(
            q, k, gq, gk, ctx.pos_ids, rq, rk, dq_out.contiguous(), dk_out.contiguous(),
            rotary_dim=R, theta=theta, eps=eps, dq=dq, dk=dk,
            need_dgamma=ctx.needs_input_grad[1] or ctx.needs_input_grad[2])
        dgq = None if dgq is None else dgq.to(gq.dtype)
        dgk = None if dgk is None else dgk.to(gk.dtype)
        return dqkv, dgq, dgk, None, None, None, None, None, None


def qk_norm_rope_qkv(qkv, gamma_q, gamma_k, pos_ids=None, *, Hq: int, Hkv: int,
                     rotary_dim: int, theta: float, eps: float):
    """Differentiable fused op on qkv [B, S, (Hq + 2 Hkv) D]; returns
    ``(q_out, k_out, v)`` with q_out, k_out dense [B,S,H,D] and v a view."""
    return QKNormRoPEFromQKV.apply(qkv, gamma_q, gamma_k, pos_ids, Hq, Hkv, rotary_dim, theta,
                                   eps)


class PreparedCall:
    """A C ABI call with every argument marshalled once.

    ``prepare_fwd`` / ``prepare_bwd`` check the tensors exactly like
    ``qk_norm_rope_fwd`` / ``qk_norm_rope_bwd`` and keep the ctypes argument
    tuple, so each later ``call()`` is a single foreign call (for tight loops
    such as benchmarks). The tensors must stay alive and unchanged in shape.
    """

    def __init__(self, fn, args, name, keep):
        self._fn, self._args, self._name, self._keep = fn, args, name, keep

    def __call__(self):
        st = self._fn(*self._args)
        if st != QKNR_OK:
            raise QKNRError(st, self._name)


def prepare_fwd(q, k, gamma_q, gamma_k, pos_ids, q_out, k_out, rstd_q, rstd_k, *,
                rotary_dim, theta, eps, stream=None, norm="rms") -> PreparedCall:
    lib = load_library()
    # one checked call validates the tensors (and runs the op once)
    qk_norm_rope_fwd(q, k, gamma_q, gamma_k, pos_ids, rotary_dim=rotary_dim, theta=theta,
                     eps=eps, q_out=q_out, k_out=k_out, rstd_q=rstd_q, rstd_k=rstd_k,
                     stream=stream, norm=norm)
    fn, name, args = _fwd_args(lib, q, k, _token_stride("q", q), _token_stride("k", k), gamma_q,
                               gamma_k, pos_ids, q_out, k_out, rstd_q, rstd_k, rotary_dim,
                               theta, eps, stream, norm)
    keep = (q, k, gamma_q, gamma_k, pos_ids, q_out, k_out, rstd_q, rstd_k)
    return PreparedCall(fn, args, name, keep)


def prepare_bwd(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dq, dk,
                dgamma_q, dgamma_k, *, rotary_dim, theta, eps, stream=None,
                norm="rms") -> PreparedCall:
    lib = load_library()
    qk_norm_rope_bwd(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out,
                     rotary_dim=rotary_dim, theta=theta, eps=eps, dq=dq, dk=dk,
                     dgamma_q=dgamma_q, dgamma_k=dgamma_k, stream=stream, norm=norm)
    fn, name, args = _bwd_args(lib, q, k, _token_stride("q", q), _token_stride("k", k), gamma_q,
                               gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dq, dk,
                               _token_stride("dq", dq), _token_stride("dk", dk), dgamma_q,
                               dgamma_k, rotary_dim, theta, eps, stream, norm)
    keep = (q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, dq, dk,
            dgamma_q, dgamma_k)
    return PreparedCall(fn, args, name, keep)


# --------------------------------------------------------------------------
# Layerwise QK-norm under tensor parallelism ("SwiftQK: Fast and
# Communication-Efficient Tensor Parallelism for Query-Key Normalization",
# abstract): each rank holds a slice of the heads; the statistic of the full
# hidden vector is one fp32 per token and tensor, summed over the ranks.


def _token_vec(name, t, T, device):
    if t is None:
        return torch.empty(T, dtype=torch.float32, device=device)
    _need_cuda(name, t)
    if t.dtype != torch.float32 or t.numel() != T:
        raise ValueError(f"{name} must be float32 with B*S = {T} elements")
    return t


def _lw_inputs(q, k, gamma_q, gamma_k, pos_ids):
    for n, t in (("q", q), ("k", k), ("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k, gamma_q, gamma_k)
    if gamma_q.numel() != Hq * D or gamma_k.numel() != Hkv * D:
        raise ValueError(f"gamma_q / gamma_k must hold Hq*D = {Hq * D} / Hkv*D = {Hkv * D} "
                         "elements (this rank's slice of the full-hidden weight)")
    if pos_ids is not None:
        _need_cuda("pos_ids", pos_ids)
        if pos_ids.dtype != torch.int32 or tuple(pos_ids.shape) != (B, S):
            raise ValueError("pos_ids must be int32 [B, S]")
    return B, S, Hq, Hkv, D


def _totals(Hq, Hkv, Hq_total, Hkv_total, group):
    world = 1
    if group is not None:
        import torch.distributed as dist
        world = dist.get_world_size(group)
    return (Hq * world if Hq_total is None else int(Hq_total),
            Hkv * world if Hkv_total is None else int(Hkv_total))


def _sharded(q, k, Hq_total, Hkv_total, group) -> bool:
    """True when some heads live on other ranks (the statistics must be
    exchanged); False when this rank holds every head (one pass each way)."""
    if group is not None:
        import torch.distributed as dist
        if dist.get_world_size(group) > 1:
            return True
    return Hq_total != q.shape[2] or Hkv_total != k.shape[2]


def all_reduce_stats(tensors, group=None):
    """Sum per-token partial statistics over the ranks of ``group`` (NCCL on
    GPUs, any torch.distributed backend); no-op without a group or with one
    rank. Both tensors go in one call when they can be viewed as one buffer."""
    if group is None:
        return tensors
    import torch.distributed as dist
    if dist.get_world_size(group) == 1:
        return tensors
    flat = torch.cat([t.reshape(-1) for t in tensors])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    out, off = [], 0
    for t in tensors:
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t))
        out.append(t)
        off += n
    return out


def qk_layerwise_stats(q, k, *, sumsq_q=None, sumsq_k=None, stream=None):
    """Per-token partial sums of squares over this rank's heads (C
    ``qk_layerwise_stats``): fp32 ``(sumsq_q, sumsq_k)``, [B*S] each."""
    lib = load_library()
    for n, t in (("q", q), ("k", k)):
        _need_cuda(n, t)
    B, S, Hq, Hkv, D = _shape(q, k)
    _same_dtype(q, k)
    sumsq_q = _token_vec("sumsq_q", sumsq_q, B * S, q.device)
    sumsq_k = _token_vec("sumsq_k", sumsq_k, B * S, q.device)
    st = lib.qk_layerwise_stats(_ptr(q), _ptr(k), _ptr(sumsq_q), _ptr(sumsq_k), B, S, Hq, Hkv,
                                D, _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_layerwise_stats")
    return sumsq_q, sumsq_k


def qk_layerwise_norm_rope_fwd(q, k, gamma_q, gamma_k, pos_ids, sumsq_q, sumsq_k, *,
                               rotary_dim: int, theta: float, eps: float, Hq_total: int,
                               Hkv_total: int, q_out=None, k_out=None, rstd_q=None,
                               rstd_k=None, stream=None):
    """Normalise with the all-rank sums of squares and rotate (C
    ``qk_layerwise_norm_rope_fwd``). Returns ``(q_out, k_out, rstd_q, rstd_k)``,
    rstd fp32 [B*S]. ``sumsq_q = sumsq_k = None``: this rank holds every
    head, and the statistic is taken in the same pass."""
    lib = load_library()
    B, S, Hq, Hkv, D = _lw_inputs(q, k, gamma_q, gamma_k, pos_ids)
    T = B * S
    if sumsq_q is not None or sumsq_k is not None:
        sumsq_q = _token_vec("sumsq_q", sumsq_q, T, q.device)
        sumsq_k = _token_vec("sumsq_k", sumsq_k, T, q.device)
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    for n, t in (("q_out", q_out), ("k_out", k_out)):
        _need_cuda(n, t)
    if q_out.shape != q.shape or k_out.shape != k.shape or q_out.dtype != q.dtype \
            or k_out.dtype != q.dtype:
        raise ValueError("q_out / k_out must match q / k in shape and dtype")
    rstd_q = _token_vec("rstd_q", rstd_q, T, q.device)
    rstd_k = _token_vec("rstd_k", rstd_k, T, q.device)
    st = lib.qk_layerwise_norm_rope_fwd(
        _ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(sumsq_q),
        _ptr(sumsq_k), _ptr(q_out), _ptr(k_out), _ptr(rstd_q), _ptr(rstd_k), B, S, Hq, Hkv,
        int(Hq_total), int(Hkv_total), D, int(rotary_dim), float(theta), float(eps),
        _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_layerwise_norm_rope_fwd")
    return q_out, k_out, rstd_q, rstd_k


def qk_layerwise_bwd_dots(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, *,
                          rotary_dim: int, theta: float, dot_q=None, dot_k=None, stream=None):
    """Per-token partial sums of (g gamma) . (x rstd) over this rank's heads,
    g the un-rotated upstream gradient (C ``qk_layerwise_bwd_dots``)."""
    lib = load_library()
    B, S, Hq, Hkv, D = _lw_inputs(q, k, gamma_q, gamma_k, pos_ids)
    T = B * S
    for n, t, ref in (("dq_out", dq_out, q), ("dk_out", dk_out, k)):
        _need_cuda(n, t)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{n} must match its input in shape and dtype")
    rstd_q = _token_vec("rstd_q", rstd_q, T, q.device)
    rstd_k = _token_vec("rstd_k", rstd_k, T, q.device)
    dot_q = _token_vec("dot_q", dot_q, T, q.device)
    dot_k = _token_vec("dot_k", dot_k, T, q.device)
    st = lib.qk_layerwise_bwd_dots(
        _ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(rstd_q),
        _ptr(rstd_k), _ptr(dq_out), _ptr(dk_out), _ptr(dot_q), _ptr(dot_k), B, S, Hq, Hkv, D,
        int(rotary_dim), float(theta), _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_layerwise_bwd_dots")
    return dot_q, dot_k


def qk_layerwise_norm_rope_bwd(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out,
                               dot_q, dot_k, *, rotary_dim: int, theta: float, Hq_total: int,
                               Hkv_total: int, dq=None, dk=None, dgamma_q=None, dgamma_k=None,
                               need_dgamma: bool = True, accumulate: bool = False, stream=None):
    """dq, dk and this rank's dgamma slices from the all-rank dot sums (C
    ``qk_layerwise_norm_rope_bwd``). Returns ``(dq, dk, dgamma_q, dgamma_k)``;
    dgamma fp32 [Hq*D] / [Hkv*D], or None without ``need_dgamma``.
    ``dot_q = dot_k = None``: this rank holds every head, and the dots are
    taken in the same pass. ``accumulate``: add to the given dgamma instead
    of overwriting it (C ``qk_layerwise_norm_rope_bwd_acc``)."""
    lib = load_library()
    B, S, Hq, Hkv, D = _lw_inputs(q, k, gamma_q, gamma_k, pos_ids)
    T = B * S
    for n, t, ref in (("dq_out", dq_out, q), ("dk_out", dk_out, k)):
        _need_cuda(n, t)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{n} must match its input in shape and dtype")
    for n, t in (("rstd_q", rstd_q), ("rstd_k", rstd_k), ("dot_q", dot_q), ("dot_k", dot_k)):
        if t is not None:  # (None dot sums: the one-pass backward)
            _token_vec(n, t, T, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    for n, t, ref in (("dq", dq, q), ("dk", dk, k)):
        _need_cuda(n, t)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{n} must match its input in shape and dtype")
    if accumulate and need_dgamma and (dgamma_q is None or dgamma_k is None):
        raise ValueError("accumulate needs the dgamma buffers to add to")
    if need_dgamma:
        dgamma_q = torch.empty(Hq * D, dtype=torch.float32, device=q.device) \
            if dgamma_q is None else dgamma_q
        dgamma_k = torch.empty(Hkv * D, dtype=torch.float32, device=q.device) \
            if dgamma_k is None else dgamma_k
        for n, t, m in (("dgamma_q", dgamma_q, Hq * D), ("dgamma_k", dgamma_k, Hkv * D)):
            _need_cuda(n, t)
            if t.dtype != torch.float32 or t.numel() != m:
                raise ValueError(f"{n} must be float32 with {m} elements")
    fn = lib.qk_layerwise_norm_rope_bwd_acc if accumulate else lib.qk_layerwise_norm_rope_bwd
    st = fn(
        _ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k), _ptr(pos_ids), _ptr(rstd_q),
        _ptr(rstd_k), _ptr(dq_out), _ptr(dk_out), _ptr(dot_q), _ptr(dot_k), _ptr(dq), _ptr(dk),
        _ptr(dgamma_q if need_dgamma else None), _ptr(dgamma_k if need_dgamma else None),
        B, S, Hq, Hkv, int(Hq_total), int(Hkv_total), D, int(rotary_dim), float(theta),
        _DTYPES[q.dtype], _stream(stream))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_layerwise_norm_rope_bwd")
    return dq, dk, (dgamma_q if need_dgamma else None), (dgamma_k if need_dgamma else None)


def token_chunks(T: int, n: int):
    """[t0, t1) ranges of ``n`` near-equal runs covering tokens 0..T-1."""
    n = max(1, min(int(n), T)) if T > 0 else 1
    return [(T * i // n, T * (i + 1) // n) for i in range(n)]


def run_chunked(n: int, partial, exchange, finish, lag: int = 1):
    """The exchange schedule of a sharded layerwise call, over ``n`` token
    chunks: ``partial(i)`` enqueues chunk i's per-token partial sums,
    ``exchange(i)`` starts their sum over the ranks (on a side stream, or as
    an asynchronous collective), and ``finish(i)`` waits for that sum and
    enqueues the element-wise pass of chunk i. Chunk i is finished only after
    chunk i + ``lag``'s partial sums are enqueued, so the exchange of chunk i
    runs while the next chunk's statistics are taken ("SwiftQK", abstract:
    the exchange of scalar statistics overlapped with element-wise work)."""
    for i in range(n):
        partial(i)
        exchange(i)
        if i >= lag:
            finish(i - lag)
    for j in range(max(0, n - lag), n):
        finish(j)


_COMM_STREAMS = {}


def _comm_stream(device) -> torch.cuda.Stream:
    idx = torch.device(device).index
    if idx is None:
        idx = torch.cuda.current_device()
    st = _COMM_STREAMS.get(idx)
    if st is None:
        st = _COMM_STREAMS[idx] = torch.cuda.Stream(device=idx)
    return st


def _flat_tokens(t: torch.Tensor) -> torch.Tensor:
    B, S = t.shape[0], t.shape[1]
    return t.reshape((B * S,) + tuple(t.shape[2:]))


_POSITIONS = {}


def _chunk_positions(pos_ids, B: int, S: int, device) -> torch.Tensor:
    """Every token's position as int32 [B*S]: the given ids, else s within
    the batch row (written once per shape and device, then reused)."""
    if pos_ids is not None:
        return pos_ids.reshape(B * S)
    key = (B, S, str(torch.device(device)))
    p = _POSITIONS.get(key)
    if p is None:
        p = (torch.arange(B * S, device=device, dtype=torch.int64) % S).to(torch.int32)
        if not torch.cuda.is_current_stream_capturing():
            _POSITIONS[key] = p
    return p


def _all_reduce_exchange(group):
    import torch.distributed as dist

    def ex(buf, span):
        dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return ex


MIN_CHUNK_TOKENS = 4096  # a chunk's kernels should outlast their launch and event overhead
# Rows (this rank's Q and K) a chunk should hold. Chunk i's exchange is
# hidden only behind chunk i + 1's statistics pass, so a chunk whose
# statistics take less than one small all-reduce (a few to ~15 us across
# NVSwitch) adds exposed exchanges instead of hiding one; 96 MiB of rows is
# ~15 us of HBM time for the statistics pass on B200.
MIN_CHUNK_BYTES = 96 << 20


def chunk_count(T: int, row_bytes: int, chunks: int, min_chunk: int = MIN_CHUNK_TOKENS,
                min_chunk_bytes: int = MIN_CHUNK_BYTES) -> int:
    """Token chunks of a sharded layerwise call: at most ``chunks``, each of
    at least ``min_chunk`` tokens and (when > 0) ``min_chunk_bytes`` of the
    rank's rows (``row_bytes`` over all T tokens); at least one."""
    if T <= 0:
        return 1
    n = min(int(chunks), T // max(1, int(min_chunk)))
    if min_chunk_bytes > 0:
        n = min(n, int(row_bytes) // int(min_chunk_bytes))
    return max(1, n)


class _Chunks:
    """Token chunks of one sharded layerwise call and the direct library
    arguments of each chunk (the tensors are checked once, by the caller)."""

    def __init__(self, q, k, chunks, pos_ids, min_chunk, min_chunk_bytes):
        B, S, Hq, Hkv, D = _shape(q, k)
        self.T = T = B * S
        n = chunk_count(T, T * (Hq + Hkv) * D * q.element_size(), chunks, min_chunk,
                        min_chunk_bytes)
        self.spans = token_chunks(T, n)
        self.dev = q.device
        self.Hq, self.Hkv, self.D = Hq, Hkv, D
        self.esz = q.element_size()
        self.dt = _DTYPES[q.dtype]
        self.pos = _chunk_positions(pos_ids, B, S, q.device)
        self.comp, self.comm = torch.cuda.current_stream(q.device), _comm_stream(q.device)
        self.st = _stream(self.comp)
        self.bufs = [torch.empty((2, t1 - t0), dtype=torch.float32, device=q.device)
                     for t0, t1 in self.spans]
        self.done = [None] * len(self.spans)

    def rows(self, t: torch.Tensor, i: int, H: int):
        """Pointer to token spans[i][0] of a [B, S, H, D] tensor (None without heads)."""
        if t is None or H == 0:
            return None
        return ctypes.c_void_p(t.data_ptr() + self.spans[i][0] * H * self.D * self.esz)

    def vec(self, t: torch.Tensor, i: int):
        """Pointer to token spans[i][0] of a per-token fp32 or int32 vector."""
        return None if t is None else ctypes.c_void_p(t.data_ptr() + 4 * self.spans[i][0])

    def sums(self, i: int):
        b = self.bufs[i]
        n = b.shape[1]
        return ctypes.c_void_p(b.data_ptr()), ctypes.c_void_p(b.data_ptr() + 4 * n)

    def n(self, i: int) -> int:
        return self.spans[i][1] - self.spans[i][0]

    def exchange(self, i: int, fn):
        ev = torch.cuda.Event()
        ev.record(self.comp)
        with torch.cuda.stream(self.comm):
            self.comm.wait_event(ev)
            fn(self.bufs[i], self.spans[i])
            self.done[i] = torch.cuda.Event()
            self.done[i].record(self.comm)

    def wait(self, i: int):
        self.comp.wait_event(self.done[i])


def _ok(st: int, where: str):
    if st != QKNR_OK:
        raise QKNRError(st, where)


def layerwise_chunked_fwd(q, k, gamma_q, gamma_k, pos_ids, *, rotary_dim: int, theta: float,
                          eps: float, Hq_total: int, Hkv_total: int, exchange, chunks: int = 4,
                          min_chunk: int = MIN_CHUNK_TOKENS,
                          min_chunk_bytes: int = MIN_CHUNK_BYTES):
    """Forward of a rank holding a slice of the heads, in token chunks:
    stats of chunk i -> ``exchange(buf, (t0, t1))`` of its [2, n] partial
    sums (q row, k row) of tokens [t0, t1), on a side stream (the default
    exchange is an all-reduce over the group) -> normalise and rotate chunk
    i, with chunk i's exchange overlapping chunk i + 1's statistics
    (``run_chunked``). The tokens are cut into ``chunks`` runs of at least
    ``min_chunk`` tokens and ``min_chunk_bytes`` bytes of this rank's rows
    (fewer runs for short calls or narrow slices; one run is the plain
    stats -> exchange -> normalise sequence). Returns ``(q_out, k_out,
    rstd_q, rstd_k)``, rstd fp32 [B*S]."""
    lib = load_library()
    B, S, Hq, Hkv, D = _lw_inputs(q, k, gamma_q, gamma_k, pos_ids)
    T = B * S
    q_out, k_out = torch.empty_like(q), torch.empty_like(k)
    rstd_q = torch.empty(T, dtype=torch.float32, device=q.device)
    rstd_k = torch.empty(T, dtype=torch.float32, device=q.device)
    if T == 0:
        return q_out, k_out, rstd_q, rstd_k
    c = _Chunks(q, k, chunks, pos_ids, min_chunk, min_chunk_bytes)
    gq, gk = _ptr(gamma_q), _ptr(gamma_k)

    def partial(i):
        sq, sk = c.sums(i)
        _ok(lib.qk_layerwise_stats(c.rows(q, i, Hq), c.rows(k, i, Hkv), sq, sk, 1, c.n(i), Hq,
                                   Hkv, D, c.dt, c.st), "qk_layerwise_stats")

    def finish(i):
        c.wait(i)
        sq, sk = c.sums(i)
        _ok(lib.qk_layerwise_norm_rope_fwd(
            c.rows(q, i, Hq), c.rows(k, i, Hkv), gq, gk, c.vec(c.pos, i), sq, sk,
            c.rows(q_out, i, Hq), c.rows(k_out, i, Hkv), c.vec(rstd_q, i), c.vec(rstd_k, i), 1,
            c.n(i), Hq, Hkv, int(Hq_total), int(Hkv_total), D, int(rotary_dim), float(theta),
            float(eps), c.dt, c.st), "qk_layerwise_norm_rope_fwd")

    run_chunked(len(c.spans), partial, lambda i: c.exchange(i, exchange), finish)
    return q_out, k_out, rstd_q, rstd_k


def layerwise_chunked_bwd(q, k, gamma_q, gamma_k, pos_ids, rstd_q, rstd_k, dq_out, dk_out, *,
                          rotary_dim: int, theta: float, Hq_total: int, Hkv_total: int,
                          exchange, chunks: int = 4, need_dgamma: bool = True,
                          min_chunk: int = MIN_CHUNK_TOKENS,
                          min_chunk_bytes: int = MIN_CHUNK_BYTES):
    """Backward of a rank holding a slice of the heads, in token chunks:
    dots of chunk i -> ``exchange(buf, (t0, t1))`` -> dx and the chunk's
    dgamma share (added into one dgamma per tensor, zeroed once), overlapped
    as in ``layerwise_chunked_fwd``. Returns ``(dq, dk, dgamma_q,
    dgamma_k)``."""
    lib = load_library()
    B, S, Hq, Hkv, D = _lw_inputs(q, k, gamma_q, gamma_k, pos_ids)
    T = B * S
    for n, t, ref in (("dq_out", dq_out, q), ("dk_out", dk_out, k)):
        _need_cuda(n, t)
        if t.shape != ref.shape or t.dtype != ref.dtype:
            raise ValueError(f"{n} must match its input in shape and dtype")
    rq = _token_vec("rstd_q", rstd_q.reshape(-1) if rstd_q is not None else None, T, q.device)
    rk = _token_vec("rstd_k", rstd_k.reshape(-1) if rstd_k is not None else None, T, q.device)
    dq, dk = torch.empty_like(q), torch.empty_like(k)
    dgq = dgk = None
    if need_dgamma:
        dgq = torch.zeros(Hq * D, dtype=torch.float32, device=q.device)
        dgk = torch.zeros(Hkv * D, dtype=torch.float32, device=q.device)
    if T == 0:
        return dq, dk, dgq, dgk
    c = _Chunks(q, k, chunks, pos_ids, min_chunk, min_chunk_bytes)
    gq, gk = _ptr(gamma_q), _ptr(gamma_k)
    fn = lib.qk_layerwise_norm_rope_bwd_acc if need_dgamma else lib.qk_layerwise_norm_rope_bwd

    def partial(i):
        pq, pk = c.sums(i)
        _ok(lib.qk_layerwise_bwd_dots(
            c.rows(q, i, Hq), c.rows(k, i, Hkv), gq, gk, c.vec(c.pos, i), c.vec(rq, i),
            c.vec(rk, i), c.rows(dq_out, i, Hq), c.rows(dk_out, i, Hkv), pq, pk, 1, c.n(i), Hq,
            Hkv, D, int(rotary_dim), float(theta), c.dt, c.st), "qk_layerwise_bwd_dots")

    def finish(i):
        c.wait(i)
        pq, pk = c.sums(i)
        _ok(fn(c.rows(q, i, Hq), c.rows(k, i, Hkv), gq, gk, c.vec(c.pos, i), c.vec(rq, i),
               c.vec(rk, i), c.rows(dq_out, i, Hq), c.rows(dk_out, i, Hkv), pq, pk,
               c.rows(dq, i, Hq), c.rows(dk, i, Hkv), _ptr(dgq), _ptr(dgk), 1, c.n(i), Hq, Hkv,
               int(Hq_total), int(Hkv_total), D, int(rotary_dim), float(theta), c.dt, c.st),
            "qk_layerwise_norm_rope_bwd")

    run_chunked(len(c.spans), partial, lambda i: c.exchange(i, exchange), finish)
    return dq, dk, dgq, dgk


DEFAULT_EXCHANGE_CHUNKS = 4


class QKLayerwiseNormRoPE(torch.autograd.Function):
    """Autograd wrapper of the layerwise path: stats -> sum over ``group``
    -> normalise and rotate; backward: dots -> sum over ``group`` -> dx and
    dgamma. The gradients of gamma are this rank's slices (they are not
    reduced over the group: each rank owns its slice)."""

    @staticmethod
    def forward(ctx, q, k, gamma_q, gamma_k, pos_ids, rotary_dim, theta, eps, Hq_total,
                Hkv_total, group, chunks):
        if _sharded(q, k, Hq_total, Hkv_total, group):
            # stats -> sum over the ranks -> normalise, chunk by chunk, each
            # chunk's exchange overlapping the next chunk's statistics
            qo, ko, rq, rk = layerwise_chunked_fwd(
                q, k, gamma_q, gamma_k, pos_ids, rotary_dim=rotary_dim, theta=theta, eps=eps,
                Hq_total=Hq_total, Hkv_total=Hkv_total, exchange=_all_reduce_exchange(group),
                chunks=chunks)
        else:
            qo, ko, rq, rk = qk_layerwise_norm_rope_fwd(
                q, k, gamma_q, gamma_k, pos_ids, None, None, rotary_dim=rotary_dim, theta=theta,
                eps=eps, Hq_total=Hq_total, Hkv_total=Hkv_total)
        ctx.save_for_backward(q, k, gamma_q, gamma_k, rq, rk)
        ctx.cfg = (pos_ids, rotary_dim, theta, Hq_total, Hkv_total, group, chunks)
        return qo, ko

    @staticmethod
    def backward(ctx, dq_out, dk_out):
        q, k, gq, gk, rq, rk = ctx.saved_tensors
        pos_ids, R, theta, Hqt, Hkvt, group, chunks = ctx.cfg
        dq_out, dk_out = dq_out.contiguous(), dk_out.contiguous()
        need = ctx.needs_input_grad[2] or ctx.needs_input_grad[3]
        if _sharded(q, k, Hqt, Hkvt, group):
            dq, dk, dgq, dgk = layerwise_chunked_bwd(
                q, k, gq, gk, pos_ids, rq, rk, dq_out, dk_out, rotary_dim=R, theta=theta,
                Hq_total=Hqt, Hkv_total=Hkvt, exchange=_all_reduce_exchange(group),
                chunks=chunks, need_dgamma=need)
        else:
            dq, dk, dgq, dgk = qk_layerwise_norm_rope_bwd(
                q, k, gq, gk, pos_ids, rq, rk, dq_out, dk_out, None, None, rotary_dim=R,
                theta=theta, Hq_total=Hqt, Hkv_total=Hkvt, need_dgamma=need)
        if need:
            dgq, dgk = dgq.view_as(gq).to(gq.dtype), dgk.view_as(gk).to(gk.dtype)
        return dq, dk, dgq, dgk, None, None, None, None, None, None, None, None


def qk_layerwise_norm_rope(q, k, gamma_q, gamma_k, pos_ids=None, *, rotary_dim: int,
                           theta: float, eps: float, Hq_total: Optional[int] = None,
                           Hkv_total: Optional[int] = None, group=None,
                           chunks: int = DEFAULT_EXCHANGE_CHUNKS):
    """Layerwise QK-RMSNorm + RoPE with autograd. q, k hold this rank's
    heads; gamma_q / gamma_k this rank's [Hq*D] / [Hkv*D] slices of the
    full-hidden weights. The head totals default to the local counts times
    the group size (an even split). A sharded call exchanges the per-token
    sums in ``chunks`` token chunks, each chunk's all-reduce overlapping the
    next chunk's statistics."""
    B, S, Hq, Hkv, D = _shape(q, k)
    Hqt, Hkvt = _totals(Hq, Hkv, Hq_total, Hkv_total, group)
    return QKLayerwiseNormRoPE.apply(q.contiguous(), k.contiguous(), gamma_q.contiguous(),
                                     gamma_k.contiguous(), pos_ids, rotary_dim, theta, eps, Hqt,
                                     Hkvt, group, int(chunks))


_GEOM_KEYS = ("pipelined", "lpr", "TT", "NS", "stage_bytes", "off_k", "off_dq", "off_dk",
              "off_cs", "off_sc", "off_parts", "off_gamma", "G", "NTG", "HB", "tpc", "grid",
              "smem", "threads", "first_tile", "cs_by_consumers", "off_pos")


def layerwise_geometry(mode: str, B: int, S: int, Hq: int, Hkv: int, D: int, rotary_dim: int,
                       dtype=torch.bfloat16, sms: int = 148) -> dict:
    """Launch geometry of the pipelined layerwise ``"dots"`` or ``"bwd"``
    kernel, or of the ``"tok"`` kernel (statistics and forward), for a shape
    (C ``qk_layerwise_geometry``; host only, no GPU)."""
    lib = load_library()
    out = (ctypes.c_int64 * len(_GEOM_KEYS))()
    st = lib.qk_layerwise_geometry({"dots": 0, "bwd": 1, "tok": 2}[mode], B, S, Hq, Hkv, D,
                                   rotary_dim,
                                   _DTYPES[dtype], sms, ctypes.cast(out, ctypes.c_void_p))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_layerwise_geometry")
    return dict(zip(_GEOM_KEYS, (int(v) for v in out)))


_PLAN_KEYS = ("pipelined", "lpr", "units", "consumer_warps", "producer_warps", "ln", "tmap",
              "TT", "NS", "stage_bytes", "tpc", "grid", "smem", "threads", "first_tile")
_PLAN_KINDS = {"fwd": 0, "bwd": 1, "ln_fwd": 2, "ln_bwd": 3}


def launch_plan(kind: str, B: int, S: int, Hq: int, Hkv: int, D: int, rotary_dim: int,
                dtype=torch.bfloat16, strided: int = 0, sms: int = 148,
                smem_optin: int = 0) -> dict:
    """Launch plan of the per-head entry points (C ``qk_norm_rope_plan``; host
    only, no GPU): ``kind`` is "fwd", "bwd", "ln_fwd" or "ln_bwd"."""
    lib = load_library()
    out = (ctypes.c_int64 * len(_PLAN_KEYS))()
    st = lib.qk_norm_rope_plan(_PLAN_KINDS[kind], B, S, Hq, Hkv, D, rotary_dim, _DTYPES[dtype],
                               strided, sms, smem_optin, ctypes.cast(out, ctypes.c_void_p))
    if st != QKNR_OK:
        raise QKNRError(st, "qk_norm_rope_plan")
    return dict(zip(_PLAN_KEYS, (int(v) for v in out)))


def kernel_name(kind: str, B: int, S: int, Hq: int, Hkv: int, D: int, rotary_dim: int,
                dtype=torch.bfloat16, strided: int = 0, sms: int = 148,
                smem_optin: int = 0) -> str:
    """The kernel a call of this shape launches, named as profilers print it
    (template arguments included), from the library's own launch plan."""
    p = launch_plan(kind, B, S, Hq, Hkv, D, rotary_dim, dtype, strided, sms, smem_optin)
    t = "__nv_bfloat16" if dtype == torch.bfloat16 else "float"
    bwd = kind.endswith("bwd")
    if not p["pipelined"]:
        return f"qknr_{'bwd' if bwd else 'fwd'}_kernel<{t}, {p['lpr']}, {p['ln']}>"
    tm = int(p["tmap"] != 0)
    if bwd:
        return (f"qknr_bwd_pipe_kernel<{t}, {p['lpr']}, {p['consumer_warps']}, "
                f"{p['producer_warps']}, {p['ln']}, {tm}>")
    return (f"qknr_fwd_pipe_kernel<{t}, {p['lpr']}, {p['units']}, {p['consumer_warps']}, "
            f"{p['producer_warps']}, {p['ln']}, {tm}>")
