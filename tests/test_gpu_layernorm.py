"""The mean-centred form (QK-LayerNorm + RoPE, qk_layernorm_rope_fwd / _bwd)
through the C ABI, element by element against the oracle's mean-centred
functions, on the workload shapes and a sweep, in both kernel families; plus
the autograd wrapper and the bitwise determinism of outputs, rstd and dX.
Tolerances are those of parity.py.
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


def check_ln(inp):
    got = parity.gpu_run(inp, norm="layer")
    st = parity.compare_with_oracle(inp, got, norm="layer")
    st.check(st.dgamma)
    return got


CASES = [
    ("qwen2.5-0.5b", dict(B=2, S=333)),
    ("llama3-8b-qknorm", dict(B=1, S=301)),
    ("partial-rope-64k", dict(B=1, S=517)),
    ("bfd-packed", dict()),
    ("tiny", dict()),
]


@pytest.mark.parametrize("name,over", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in o.items())}" for n, o in CASES])
def test_layernorm_vs_oracle(cuda, kernels, name, over):
    check_ln(workloads.make_inputs(name, **over))


SHAPES = [("bf16", 16, 16), ("bf16", 64, 32), ("bf16", 80, 80), ("bf16", 128, 0),
          ("bf16", 256, 64), ("f32", 8, 8), ("f32", 24, 16), ("f32", 128, 128),
          ("bf16", 72, 64), ("bf16", 40, 16), ("f32", 12, 8), ("f32", 20, 0)]


@pytest.mark.parametrize("dtype,D,R", SHAPES, ids=[f"{a}-D{b}-R{c}" for a, b, c in SHAPES])
def test_layernorm_shape_sweep(cuda, kernels, dtype, D, R):
    inp = workloads.make_inputs("tiny", seed=12, B=3, S=37, Hq=5, Hkv=3, D=D, rotary_dim=R,
                                dtype=dtype, theta=1e4, qk_scale=2.0)
    # shift every row by a per-row constant: the mean-centred form must remove it
    g = torch.Generator().manual_seed(5)
    for t in (inp.q, inp.k):
        shift = (torch.randn(t.shape[:-1] + (1,), generator=g) * 4).to(t.dtype)
        t.copy_((t.double() + shift.double()).to(t.dtype))
    check_ln(inp)


def test_layernorm_full_bench_shape(cuda):
    check_ln(workloads.make_inputs(workloads.BENCH_WORKLOAD))


def test_layernorm_deterministic(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=2, S=500)
    a = parity.gpu_run(inp, norm="layer")
    b = parity.gpu_run(inp, norm="layer")
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(a[n], b[n]), n


def test_layernorm_differs_from_rmsnorm(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=64)
    a = parity.gpu_run(inp, norm="layer")
    b = parity.gpu_run(inp)
    assert not torch.equal(a["q_out"], b["q_out"])


def test_layernorm_autograd(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=80)
    w = inp.w
    q = inp.q.to(cuda).requires_grad_(True)
    k = inp.k.to(cuda).requires_grad_(True)
    gq = inp.gamma_q.to(cuda).requires_grad_(True)
    gk = inp.gamma_k.to(cuda).requires_grad_(True)
    qo, ko = qknr.qk_norm_rope(q, k, gq, gk, rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps,
                               norm="layer")
    torch.autograd.backward([qo, ko], [inp.dq_out.to(cuda), inp.dk_out.to(cuda)])
    ref = parity.gpu_run(inp, norm="layer")
    assert torch.equal(qo.detach().cpu(), ref["q_out"]) and torch.equal(q.grad.cpu(), ref["dq"])
    assert torch.equal(k.grad.cpu(), ref["dk"])
    for a, b in ((gq.grad, ref["dgamma_q"]), (gk.grad, ref["dgamma_k"])):
        scale = float(b.double().abs().max())
        assert float((a.cpu().double() - b.double()).abs().max()) / scale <= 1e-2


def test_no_pipeline_timeouts(cuda):
    assert qknr.pipeline_error() == 0
