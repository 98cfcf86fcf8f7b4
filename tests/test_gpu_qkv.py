"""Q and K read in place from a fused QKV projection buffer, and dQ / dK
written in place into a dQKV buffer (the ``_strided`` entry points).

The strided calls run the same kernels and arithmetic as the dense ones; only
the addressing differs (one 3-D tensor copy per tile block instead of a flat
bulk copy, and strided dQ / dK stores). So their outputs must equal the dense
calls' bit for bit (dgamma, summed with atomics, to its normwise tolerance),
and they are also checked against the oracle directly. The V slot and any
padding between tokens must come back untouched.
"""
import os

import numpy as np
import pytest
import torch

import parity
import workloads
import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

pytestmark = pytest.mark.gpu

SENTINEL = -3.0


@pytest.fixture(scope="module")
def cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    qbuild.build()
    qknr.load_library()
    return torch.device("cuda")


def _cfg(w):
    return dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)


def pack_qkv(inp, cuda, pad=0, seed=11):
    """qkv [B, S, (Hq + 2 Hkv) D + pad] holding inp's q and k and a seeded v;
    returns (qkv, q view, k view, v view)."""
    w = inp.w
    B, S, Hq, Hkv, D = w.B, w.S, w.Hq, w.Hkv, w.D
    W = (Hq + 2 * Hkv) * D
    full = torch.full((B, S, W + pad), SENTINEL, dtype=inp.q.dtype, device=cuda)
    qkv = full[..., :W] if pad else full
    q, k, v = qknr.split_qkv(qkv, Hq, Hkv)
    q.copy_(inp.q.to(cuda))
    k.copy_(inp.k.to(cuda))
    g = torch.Generator().manual_seed(seed)
    v.copy_(torch.randn(v.shape, generator=g).to(v.dtype))
    return full, q, k, v


def run_strided(inp, cuda, pad=0):
    """fwd + bwd through the strided entry points; CPU results plus the two
    buffers (to check the untouched slots)."""
    w = inp.w
    full, q, k, v = pack_qkv(inp, cuda, pad)
    gq, gk = inp.gamma_q.to(cuda), inp.gamma_k.to(cuda)
    pos = None if inp.pos is None else inp.pos.to(cuda)
    qo, ko, rq, rk = qknr.qk_norm_rope_fwd(q, k, gq, gk, pos, **_cfg(w))
    dfull = torch.full_like(full, SENTINEL)
    W = (w.Hq + 2 * w.Hkv) * w.D
    dq, dk, dv = qknr.split_qkv(dfull[..., :W] if pad else dfull, w.Hq, w.Hkv)
    _, _, dgq, dgk = qknr.qk_norm_rope_bwd(q, k, gq, gk, pos, rq, rk, inp.dq_out.to(cuda),
                                           inp.dk_out.to(cuda), dq=dq, dk=dk, **_cfg(w))
    torch.cuda.synchronize()
    got = {"q_out": qo, "k_out": ko, "rstd_q": rq, "rstd_k": rk, "dq": dq.contiguous(),
           "dk": dk.contiguous(), "dgamma_q": dgq, "dgamma_k": dgk}
    got = {n: t.cpu() for n, t in got.items()}
    # the V slot and the padding of dqkv are never written; qkv is unchanged
    assert bool((dv == SENTINEL).all())
    if pad:
        assert bool((dfull[..., W:] == SENTINEL).all())
        assert bool((full[..., W:] == SENTINEL).all())
    assert torch.equal(q.cpu(), inp.q) and torch.equal(k.cpu(), inp.k)
    return got


def assert_same_as_dense(inp, got, dense):
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(got[n], dense[n]), n
    rel = parity.DGAMMA_REL[inp.w.dtype]
    for n in ("dgamma_q", "dgamma_k"):
        ref = dense[n].double()
        scale = float(ref.abs().max()) or 1.0
        assert float((got[n].double() - ref).abs().max()) / scale <= rel, n


CASES = [
    # name, overrides, pad (elements between tokens past the V slot)
    ("qwen2.5-0.5b", dict(B=2, S=333), 0),
    ("qwen2.5-0.5b", dict(B=1, S=700), 8),
    ("llama3-8b-qknorm", dict(B=1, S=301), 0),
    ("partial-rope-64k", dict(B=1, S=517), 24),
    ("tiny", dict(), 0),
    ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=24, rotary_dim=16), 4),
]


@pytest.mark.parametrize("name,over,pad", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in o.items())}-pad{p}"
                              for n, o, p in CASES])
def test_qkv_matches_dense_bitwise(cuda, name, over, pad):
    inp = workloads.make_inputs(name, **over)
    dense = parity.gpu_run(inp)
    got = run_strided(inp, cuda, pad)
    assert_same_as_dense(inp, got, dense)


def test_qkv_against_oracle(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=3, S=129)
    parity.check(inp, run_strided(inp, cuda, pad=8))


def test_qkv_packed_positions(cuda):
    inp = workloads.make_inputs("bfd-packed")
    parity.check(inp, run_strided(inp, cuda))


@pytest.mark.parametrize("B,S", [(1, 1), (1, 3), (2, 5), (5, 1), (3, 41)])
def test_qkv_short_runs(cuda, B, S):
    # runs shorter than a tile: the tensor-copy box reads past the last token
    # (zero fill) or into the previous run
    inp = workloads.make_inputs("llama3-8b-qknorm", seed=9, B=B, S=S, Hq=6, Hkv=2)
    assert_same_as_dense(inp, run_strided(inp, cuda, pad=8), parity.gpu_run(inp))


@pytest.mark.parametrize("Hq,Hkv", [(4, 0), (0, 4), (1, 1), (33, 1)])
def test_qkv_head_counts(cuda, Hq, Hkv):
    inp = workloads.make_inputs("llama3-8b-qknorm", seed=4, B=2, S=37, Hq=Hq, Hkv=Hkv)
    assert_same_as_dense(inp, run_strided(inp, cuda), parity.gpu_run(inp))


def test_qkv_simple_kernels(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=2, S=129)
    os.environ["QKNR_SIMPLE_KERNELS"] = "1"
    try:
        got = run_strided(inp, cuda, pad=8)
        dense = parity.gpu_run(inp)
    finally:
        del os.environ["QKNR_SIMPLE_KERNELS"]
    assert_same_as_dense(inp, got, dense)
    parity.check(inp, got)


def test_qkv_autograd(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=2, S=65)
    w = inp.w
    full, q, k, v = pack_qkv(inp, cuda)
    qkv = full.detach().requires_grad_(True)
    gq = inp.gamma_q.to(cuda).requires_grad_(True)
    gk = inp.gamma_k.to(cuda).requires_grad_(True)
    qo, ko, vo = qknr.qk_norm_rope_qkv(qkv, gq, gk, Hq=w.Hq, Hkv=w.Hkv, **_cfg(w))
    dv = torch.randn_like(vo)
    dqo, dko = inp.dq_out.to(cuda), inp.dk_out.to(cuda)
    torch.autograd.backward([qo, ko, vo], [dqo, dko, dv])
    # the dense op on copies
    q2 = q.detach().contiguous().requires_grad_(True)
    k2 = k.detach().contiguous().requires_grad_(True)
    gq2 = inp.gamma_q.to(cuda).requires_grad_(True)
    gk2 = inp.gamma_k.to(cuda).requires_grad_(True)
    qo2, ko2 = qknr.qk_norm_rope(q2, k2, gq2, gk2, **_cfg(w))
    torch.autograd.backward([qo2, ko2], [dqo, dko])
    assert torch.equal(qo, qo2) and torch.equal(ko, ko2) and torch.equal(vo, v)
    dq, dk, dvv = qknr.split_qkv(qkv.grad, w.Hq, w.Hkv)
    assert torch.equal(dq, q2.grad) and torch.equal(dk, k2.grad) and torch.equal(dvv, dv)
    for a, b in ((gq.grad, gq2.grad), (gk.grad, gk2.grad)):
        scale = float(b.double().abs().max()) or 1.0
        assert float((a.double() - b.double()).abs().max()) / scale <= 1e-2


def test_strided_error_codes(cuda):
    lib = qknr.load_library()
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=16)
    w = inp.w
    full, q, k, v = pack_qkv(inp, cuda)
    ts = (w.Hq + 2 * w.Hkv) * w.D
    gq, gk = inp.gamma_q.to(cuda), inp.gamma_k.to(cuda)
    qo = torch.empty(q.shape, dtype=q.dtype, device=cuda)
    ko = torch.empty(k.shape, dtype=k.dtype, device=cuda)
    rq = torch.empty(w.B, w.S, w.Hq, device=cuda)
    rk = torch.empty(w.B, w.S, w.Hkv, device=cuda)
    P = qknr._ptr
    st = qknr._stream(None)

    def fwd(qts, kts, qout=qo):
        return lib.qk_norm_rope_fwd_strided(P(q), P(k), qts, kts, P(gq), P(gk), None, P(qout),
                                            P(ko), P(rq), P(rk), w.B, w.S, w.Hq, w.Hkv, w.D,
                                            w.rotary_dim, w.theta, w.eps, 1, st)

    assert fwd(w.Hq * w.D - 8, ts) == qknr.QKNR_ERR_INVALID_ARG      # rows would overlap
    assert fwd(ts + 4, ts) == qknr.QKNR_ERR_ALIGNMENT                 # 8-byte step
    assert fwd(ts, ts, qout=full) == qknr.QKNR_ERR_INVALID_ARG        # q_out on top of qkv
    assert fwd(ts, ts) == qknr.QKNR_OK
    dfull = torch.empty_like(full)
    dq, dk, _ = qknr.split_qkv(dfull, w.Hq, w.Hkv)
    dqo, dko = inp.dq_out.to(cuda), inp.dk_out.to(cuda)

    def bwd(dq_ptr, dk_ptr, dqts, dkts):
        return lib.qk_norm_rope_bwd_strided(P(q), P(k), ts, ts, P(gq), P(gk), None, P(rq),
                                            P(rk), P(dqo), P(dko), dq_ptr, dk_ptr, dqts, dkts,
                                            None, None, w.B, w.S, w.Hq, w.Hkv, w.D,
                                            w.rotary_dim, w.theta, w.eps, 1, st)

    # dq, dk interleaved in one buffer without touching: accepted
    assert bwd(P(dq), P(dk), ts, ts) == qknr.QKNR_OK
    # dk shifted into dq's rows: rejected
    shifted = ctypes_ptr(dq, 64)
    assert bwd(P(dq), shifted, ts, ts) == qknr.QKNR_ERR_INVALID_ARG
    # dq written over the qkv input: rejected
    assert bwd(P(q), P(dk), ts, ts) == qknr.QKNR_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert qknr.pipeline_error() == 0


def ctypes_ptr(t, byte_offset):
    import ctypes
    return ctypes.c_void_p(t.data_ptr() + byte_offset)
