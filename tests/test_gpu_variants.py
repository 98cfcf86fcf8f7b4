"""The NoPE, rotation-only and statistics-only entry points (qk_norm_fwd /
qk_norm_bwd, qk_rope_apply, qk_rms_stats) through the C ABI.

qk_norm_* must equal qk_norm_rope_* at rotary_dim = 0 bit for bit (the same
kernels), and match the oracle. qk_rope_apply, forward and inverse, is checked
element by element against the oracle's rotation alone (``rope_rows``),
including extreme and negative positions and partial rotary spans; position 0
and the dims past rotary_dim must come back bitwise unchanged. qk_rms_stats
must equal the rstd the fused forward saves at rotary_dim = 0, bit for bit. Both kernel
families (pipelined and plain-load) are covered.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import parity
import workloads
import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    qbuild.build()
    qknr.load_library()
    return torch.device("cuda")


@pytest.fixture(params=["pipelined", "plain"])
def kernels(request):
    if request.param == "plain":
        os.environ["QKNR_SIMPLE_KERNELS"] = "1"
    yield request.param
    os.environ.pop("QKNR_SIMPLE_KERNELS", None)


def positions_of(inp):
    w = inp.w
    return oracle.positions(None if inp.pos is None else inp.pos.numpy(), w.B, w.S)


def check_elems(dtype, name, got, ref):
    """Elementwise bound of parity.py: fp32 max-abs 1e-5; bf16 max-abs 2e-2
    where |ref| < 8 and within one bf16 ulp everywhere."""
    st = parity.Stats(dtype, got.shape[-1])
    st.elem(name, got.double().numpy().reshape(-1), np.asarray(ref).reshape(-1))
    tol = parity.ABS_TOL[dtype]
    assert st.max_abs[name] <= tol, f"{name}: max-abs {st.max_abs[name]:.3e} > {tol}"
    if dtype == "bf16":
        assert st.max_ulp[name] <= 1.0, f"{name}: {st.max_ulp[name]:.3f} bf16 ulp"


def rope_on_gpu(inp, cuda, inverse, x=None):
    w = inp.w
    q = (inp.q if x is None else x[0]).to(cuda)
    k = (inp.k if x is None else x[1]).to(cuda)
    pos = None if inp.pos is None else inp.pos.to(cuda)
    qo, ko = qknr.qk_rope_apply(q, k, pos, rotary_dim=w.rotary_dim, theta=w.theta,
                                inverse=inverse)
    torch.cuda.synchronize()
    return qo.cpu(), ko.cpu()


ROPE_CASES = [
    ("qwen2.5-0.5b", dict(B=2, S=333)),
    ("llama3-8b-qknorm", dict(B=1, S=257)),
    ("partial-rope-64k", dict(B=1, S=777)),
    ("bfd-packed", dict()),
    ("tiny", dict()),
    ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=24, rotary_dim=16)),
    ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=20, rotary_dim=16)),
    ("llama3-8b-qknorm", dict(B=1, S=77, Hq=4, Hkv=2, D=72, rotary_dim=64)),
]


@pytest.mark.parametrize("inverse", [False, True], ids=["fwd", "inverse"])
@pytest.mark.parametrize("name,over", ROPE_CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in o.items())}"
                              for n, o in ROPE_CASES])
def test_rope_apply_vs_oracle(cuda, kernels, name, over, inverse):
    inp = workloads.make_inputs(name, **over)
    w = inp.w
    qo, ko = rope_on_gpu(inp, cuda, inverse)
    rq, rk = oracle.get().rope(inp.q, inp.k, positions_of(inp), w.rotary_dim, w.theta, inverse)
    check_elems(w.dtype, "q_out", qo, rq)
    check_elems(w.dtype, "k_out", ko, rk)
    # dims past the rotary span are copied
    R = w.rotary_dim
    assert torch.equal(qo[..., R:], inp.q[..., R:]) and torch.equal(ko[..., R:], inp.k[..., R:])


def test_rope_extreme_positions(cuda, kernels):
    for dtype, D, R in (("bf16", 128, 64), ("f32", 64, 64), ("bf16", 80, 16)):
        inp = workloads.make_inputs("tiny", seed=3, B=2, S=40, Hq=3, Hkv=2, D=D,
                                    rotary_dim=R, dtype=dtype, theta=1e4)
        rng = np.random.default_rng(3)
        pos = rng.integers(-2 ** 31, 2 ** 31 - 1, size=(2, 40))
        pos.reshape(-1)[:6] = [0, 1, -1, 2 ** 31 - 1, -(2 ** 31), 65535]
        inp.pos = torch.from_numpy(pos.astype(np.int32))
        for inverse in (False, True):
            qo, ko = rope_on_gpu(inp, cuda, inverse)
            rq, rk = oracle.get().rope(inp.q, inp.k, pos.reshape(-1), R, inp.w.theta, inverse)
            check_elems(dtype, "q_out", qo, rq)
            check_elems(dtype, "k_out", ko, rk)


def test_rope_position_zero_is_identity(cuda, kernels):
    inp = workloads.make_inputs("bfd-packed")
    starts = (inp.pos == 0) & inp.valid
    for inverse in (False, True):
        qo, ko = rope_on_gpu(inp, cuda, inverse)
        assert torch.equal(qo[starts], inp.q[starts]) and torch.equal(ko[starts], inp.k[starts])


def test_rope_inverse_undoes_forward(cuda):
    # fp32 I/O: the round trip returns the input to fp32 rounding
    inp = workloads.make_inputs("tiny", seed=8, B=2, S=64, Hq=4, Hkv=2, D=64, rotary_dim=64,
                                dtype="f32", theta=1e6)
    y = rope_on_gpu(inp, cuda, False)
    back = rope_on_gpu(inp, cuda, True, x=y)
    for a, b in zip(back, (inp.q, inp.k)):
        assert float((a - b).abs().max()) <= 1e-5


def test_rope_in_place(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=100)
    w = inp.w
    ref = rope_on_gpu(inp, cuda, False)
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    qknr.qk_rope_apply(q, k, rotary_dim=w.rotary_dim, theta=w.theta, q_out=q, k_out=k)
    torch.cuda.synchronize()
    assert torch.equal(q.cpu(), ref[0]) and torch.equal(k.cpu(), ref[1])


def test_rope_autograd_is_inverse_rotation(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=50)
    w = inp.w
    q = inp.q.to(cuda).requires_grad_(True)
    k = inp.k.to(cuda).requires_grad_(True)
    qo, ko = qknr.QKRoPE.apply(q, k, None, w.rotary_dim, w.theta, False)
    torch.autograd.backward([qo, ko], [inp.dq_out.to(cuda), inp.dk_out.to(cuda)])
    rq, rk = oracle.get().rope(inp.dq_out, inp.dk_out, positions_of(inp), w.rotary_dim,
                               w.theta, True)
    check_elems(w.dtype, "dq", q.grad.cpu(), rq)
    check_elems(w.dtype, "dk", k.grad.cpu(), rk)


@pytest.mark.parametrize("name,over", [("qwen2.5-0.5b", dict(B=2, S=129)),
                                       ("llama3-8b-qknorm", dict(B=1, S=200)),
                                       ("tiny", dict())])
def test_qk_norm_is_rotary_dim_zero(cuda, kernels, name, over):
    inp = workloads.make_inputs(name, rotary_dim=0, **over)
    w = inp.w
    dense = parity.gpu_run(inp)  # qk_norm_rope_* with rotary_dim = 0
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    gq, gk = inp.gamma_q.to(cuda), inp.gamma_k.to(cuda)
    qo, ko, rq, rk = qknr.qk_norm_fwd(q, k, gq, gk, eps=w.eps)
    dq, dk, dgq, dgk = qknr.qk_norm_bwd(q, k, gq, gk, rq, rk, inp.dq_out.to(cuda),
                                        inp.dk_out.to(cuda), eps=w.eps)
    torch.cuda.synchronize()
    got = {"q_out": qo, "k_out": ko, "rstd_q": rq, "rstd_k": rk, "dq": dq, "dk": dk,
           "dgamma_q": dgq, "dgamma_k": dgk}
    got = {n: t.cpu() for n, t in got.items()}
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(got[n], dense[n]), n
    parity.check(inp, got)


@pytest.mark.parametrize("name,over", [("qwen2.5-0.5b", dict(B=2, S=333)),
                                       ("llama3-8b-qknorm", dict(B=1, S=300)),
                                       ("tiny", dict()),
                                       ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=24, rotary_dim=16))])
def test_rms_stats_equal_saved_rstd(cuda, kernels, name, over):
    """qk_rms_stats equals, bit for bit, the rstd the fused forward saves with
    no rotary span (same lane layout, so the same fp32 summation order), and
    the oracle's inverse RMS to the fp32 bound."""
    inp = workloads.make_inputs(name, **dict(over, rotary_dim=0))
    w = inp.w
    dense = parity.gpu_run(inp, fwd_only=True)
    rq, rk = qknr.qk_rms_stats(inp.q.to(cuda), inp.k.to(cuda), eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(rq.cpu(), dense["rstd_q"]) and torch.equal(rk.cpu(), dense["rstd_k"])
    rows = inp.q.double().numpy().reshape(-1, w.D)
    _, ref_q = oracle.get().fwd_rows(rows, np.ones(w.D), np.zeros(len(rows), np.int64), 0,
                                     w.theta, w.eps)
    rel = np.abs(rq.cpu().double().numpy().reshape(-1) - ref_q) / ref_q
    assert float(rel.max()) <= w.D * 2.0 ** -24


def test_no_pipeline_timeouts(cuda):
    assert qknr.pipeline_error() == 0
