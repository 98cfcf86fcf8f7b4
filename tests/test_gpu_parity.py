"""CUDA path vs the CPU oracle, through the C ABI, on seeded inputs.

Every element of every output is compared (the oracle runs in fp64, token
chunk by token chunk), at the five workload sizes in the launch geometry the
bench uses (the library picks it), and on small ragged shapes that sweep
head dims, rotary spans, dtypes, head counts and positions. Tolerances are
stated in parity.py. Also: bitwise determinism, in-place aliasing, position
ids and packing boundaries, guard bands around outputs, host-side error
codes with real device pointers, the autograd wrapper and non-default
streams.
"""
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


def with_positions(inp, pos_np):
    inp.pos = torch.from_numpy(np.ascontiguousarray(pos_np, dtype=np.int32))
    return inp


# ------------------------------------------------------------ full workloads
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_every_element(cuda, name):
    inp = workloads.make_inputs(name)
    got = parity.gpu_run(inp)
    st = parity.check(inp, got)
    print(name, st.summary())


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_tiny_more_seeds(cuda, k):
    w = workloads.WORKLOADS["tiny"]
    inp = workloads.make_inputs(w, seed=workloads.seed_for(w, k))
    parity.check(inp, parity.gpu_run(inp))


@pytest.mark.parametrize("k", [1, 2])
def test_bench_workload_more_seeds(cuda, k):
    w = workloads.WORKLOADS[workloads.BENCH_WORKLOAD]
    inp = workloads.make_inputs(w, seed=workloads.seed_for(w, k))
    parity.check(inp, parity.gpu_run(inp))


# ------------------------------------------------------------- shape sweep
EXTREME_POS = [0, 1, 65535, 2 ** 31 - 1, -1, -(2 ** 31), 1_000_000, 7]


def sweep_inputs(dtype, D, R, B=3, S=37, Hq=5, Hkv=3, seed=77, theta=1e4, eps=1e-6):
    inp = workloads.make_inputs("tiny", seed=seed, B=B, S=S, Hq=Hq, Hkv=Hkv, D=D,
                                rotary_dim=R, dtype=dtype, theta=theta, eps=eps,
                                qk_scale=2.0)
    rng = np.random.default_rng(seed)
    pos = rng.integers(0, 200_000, size=(B, S))
    flat = pos.reshape(-1)
    flat[:len(EXTREME_POS)] = EXTREME_POS[:flat.size]
    return with_positions(inp, pos)


SHAPES = [("bf16", 16, 16), ("bf16", 16, 0), ("bf16", 32, 16), ("bf16", 64, 32),
          ("bf16", 64, 64), ("bf16", 80, 80), ("bf16", 80, 16), ("bf16", 96, 48),
          ("bf16", 128, 0), ("bf16", 128, 32), ("bf16", 128, 128), ("bf16", 192, 64),
          ("bf16", 256, 256), ("bf16", 256, 32),
          ("f32", 8, 8), ("f32", 16, 8), ("f32", 24, 16), ("f32", 64, 64),
          ("f32", 128, 32), ("f32", 128, 128), ("f32", 256, 256), ("f32", 256, 0),
          # an odd number of 16-byte vectors per row: the last pass-through unit
          # has one vector (the plain-load kernels take these shapes)
          ("bf16", 8, 0), ("bf16", 40, 16), ("bf16", 72, 64), ("bf16", 72, 0),
          ("bf16", 120, 48), ("f32", 4, 0), ("f32", 12, 8), ("f32", 20, 16), ("f32", 12, 0)]


@pytest.mark.parametrize("dtype,D,R", SHAPES, ids=[f"{a}-D{b}-R{c}" for a, b, c in SHAPES])
def test_shape_sweep(cuda, dtype, D, R):
    inp = sweep_inputs(dtype, D, R)
    parity.check(inp, parity.gpu_run(inp))


@pytest.mark.parametrize("Hq,Hkv", [(1, 0), (0, 1), (0, 3), (7, 0), (1, 1), (33, 1), (3, 17)])
def test_head_counts(cuda, Hq, Hkv):
    inp = sweep_inputs("bf16", 128, 64, B=2, S=19, Hq=Hq, Hkv=Hkv)
    parity.check(inp, parity.gpu_run(inp))


@pytest.mark.parametrize("B,S", [(0, 5), (3, 0), (1, 1), (1, 2), (5, 1), (2, 4099)])
def test_batch_edges(cuda, B, S):
    inp = workloads.make_inputs("llama3-8b-qknorm", seed=5, B=B, S=S, Hq=4, Hkv=2)
    got = parity.gpu_run(inp)
    if B * S == 0:
        assert float(got["dgamma_q"].abs().sum()) == 0.0
        assert float(got["dgamma_k"].abs().sum()) == 0.0
    parity.check(inp, got)


def test_large_theta_and_eps(cuda):
    inp = sweep_inputs("f32", 64, 64, theta=1e7, eps=0.5)
    parity.check(inp, parity.gpu_run(inp))
    inp = sweep_inputs("bf16", 64, 64, theta=2.0, eps=0.0)
    parity.check(inp, parity.gpu_run(inp))


# -------------------------------------------------- exactness and aliasing
def _dev(inp, cuda):
    return {n: (None if getattr(inp, n) is None else getattr(inp, n).to(cuda))
            for n in ("q", "k", "gamma_q", "gamma_k", "dq_out", "dk_out", "pos")}


def _cfg(w):
    return dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)


def test_bitwise_deterministic(cuda):
    inp = workloads.make_inputs(workloads.BENCH_WORKLOAD)
    a = parity.gpu_run(inp)
    b = parity.gpu_run(inp)
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(a[n], b[n]), f"{n} differs between runs"


def test_in_place(cuda):
    inp = workloads.make_inputs("partial-rope-64k", B=1, S=3000)
    w = inp.w
    d = _dev(inp, cuda)
    qo, ko, rq, rk = qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"],
                                           **_cfg(w))
    dq, dk, dgq, dgk = qknr.qk_norm_rope_bwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], None,
                                             rq, rk, d["dq_out"], d["dk_out"], **_cfg(w))
    q2, k2 = d["q"].clone(), d["k"].clone()
    qknr.qk_norm_rope_fwd(q2, k2, d["gamma_q"], d["gamma_k"], q_out=q2, k_out=k2, **_cfg(w))
    dqo2, dko2 = d["dq_out"].clone(), d["dk_out"].clone()
    qknr.qk_norm_rope_bwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], None, rq, rk, dqo2,
                          dko2, dq=dqo2, dk=dko2, **_cfg(w))
    torch.cuda.synchronize()
    assert torch.equal(q2, qo) and torch.equal(k2, ko)
    assert torch.equal(dqo2, dq) and torch.equal(dko2, dk)


def test_explicit_positions_equal_default(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=3, S=700)
    a = parity.gpu_run(inp)
    w = inp.w
    pos = np.tile(np.arange(w.S, dtype=np.int32), (w.B, 1))
    b = parity.gpu_run(with_positions(inp, pos))
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(a[n], b[n]), n


def test_packing_boundaries_and_pass_through(cuda):
    """Exact identities of the kernel, checked bitwise against a host
    recomputation from the kernel's own rstd: at doc starts (position 0)
    every dim of the output is (x * gamma) * r rounded once to bf16, and
    in a partial rotary layout so is every dim >= R at every position;
    padding slots stay zero."""
    inp = workloads.make_inputs("bfd-packed", rotary_dim=32)
    w = inp.w
    got = parity.gpu_run(inp, fwd_only=True)
    starts = (inp.pos == 0) & inp.valid
    assert int(starts.sum()) == len(inp.doc_lengths)
    for x, g, name, rname in ((inp.q, inp.gamma_q, "q_out", "rstd_q"),
                              (inp.k, inp.gamma_k, "k_out", "rstd_k")):
        n = ((x.float() * g.float()) * got[rname].unsqueeze(-1)).to(torch.bfloat16)
        assert torch.equal(got[name][starts], n[starts]), f"{name} at doc starts"
        R = w.rotary_dim
        assert torch.equal(got[name][..., R:], n[..., R:]), f"{name} pass-through dims"
        assert not torch.equal(got[name][..., :R], n[..., :R])
    pad = ~inp.valid
    assert torch.all(got["q_out"][pad] == 0) and torch.all(got["k_out"][pad] == 0)


def test_guard_bands(cuda):
    """Outputs written inside canary-filled buffers: nothing outside changes."""
    inp = workloads.make_inputs("qwen2.5-0.5b", B=2, S=333)
    w = inp.w
    d = _dev(inp, cuda)
    pad = 4096

    def guarded(shape, dtype):
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * pad,), -7.0, dtype=dtype, device=cuda)
        return buf, buf[pad:pad + n].view(shape)

    bq, qo = guarded(d["q"].shape, d["q"].dtype)
    bk, ko = guarded(d["k"].shape, d["k"].dtype)
    brq, rq = guarded((w.B, w.S, w.Hq), torch.float32)
    brk, rk = guarded((w.B, w.S, w.Hkv), torch.float32)
    bdq, dq = guarded(d["q"].shape, d["q"].dtype)
    bdk, dk = guarded(d["k"].shape, d["k"].dtype)
    bgq, dgq = guarded((w.D,), torch.float32)
    bgk, dgk = guarded((w.D,), torch.float32)
    qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], q_out=qo, k_out=ko,
                          rstd_q=rq, rstd_k=rk, **_cfg(w))
    qknr.qk_norm_rope_bwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], None, rq, rk,
                          d["dq_out"], d["dk_out"], dq=dq, dk=dk, dgamma_q=dgq,
                          dgamma_k=dgk, **_cfg(w))
    torch.cuda.synchronize()
    for buf in (bq, bk, brq, brk, bdq, bdk, bgq, bgk):
        assert torch.all(buf[:pad] == -7.0) and torch.all(buf[-pad:] == -7.0)
    got = {"q_out": qo.cpu(), "k_out": ko.cpu(), "rstd_q": rq.cpu(), "rstd_k": rk.cpu(),
           "dq": dq.cpu(), "dk": dk.cpu(), "dgamma_q": dgq.cpu(), "dgamma_k": dgk.cpu()}
    parity.check(inp, got)


def test_error_codes_with_device_pointers(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=1, S=64)
    w = inp.w
    d = _dev(inp, cuda)
    flat = torch.empty(d["q"].numel() + 8, dtype=d["q"].dtype, device=cuda)
    misaligned = flat[1:1 + d["q"].numel()].view(d["q"].shape)
    with pytest.raises(qknr.QKNRError) as e:
        qknr.qk_norm_rope_fwd(misaligned, d["k"], d["gamma_q"], d["gamma_k"], **_cfg(w))
    assert e.value.status == qknr.QKNR_ERR_ALIGNMENT
    q_out = torch.empty_like(d["q"])
    with pytest.raises(qknr.QKNRError) as e:   # k_out on top of q_out
        qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], q_out=q_out,
                              k_out=q_out.view(-1)[:d["k"].numel()].view(d["k"].shape),
                              **_cfg(w))
    assert e.value.status == qknr.QKNR_ERR_INVALID_ARG
    with pytest.raises(qknr.QKNRError) as e:
        qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], rotary_dim=8,
                              theta=1e4, eps=1e-6)
    assert e.value.status == qknr.QKNR_ERR_UNSUPPORTED


def test_autograd_wrapper(cuda):
    inp = workloads.make_inputs("tiny")
    w = inp.w
    d = _dev(inp, cuda)
    q = d["q"].clone().requires_grad_()
    k = d["k"].clone().requires_grad_()
    gq = d["gamma_q"].clone().requires_grad_()
    gk = d["gamma_k"].clone().requires_grad_()
    qo, ko = qknr.qk_norm_rope(q, k, gq, gk, rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)
    ((qo * d["dq_out"]).sum() + (ko * d["dk_out"]).sum()).backward()
    got = parity.gpu_run(inp)
    assert torch.equal(qo.detach().cpu(), got["q_out"])
    assert torch.equal(q.grad.cpu(), got["dq"]) and torch.equal(k.grad.cpu(), got["dk"])
    # dgamma is summed with atomics in a run-dependent order: normwise check
    for a_, b_ in ((gq.grad.cpu(), got["dgamma_q"]), (gk.grad.cpu(), got["dgamma_k"])):
        assert float((a_ - b_).abs().max()) <= 1e-5 * float(b_.abs().max())


def test_side_stream_and_graph_capture(cuda):
    inp = workloads.make_inputs("qwen2.5-0.5b", B=2, S=512)
    w = inp.w
    d = _dev(inp, cuda)
    ref = parity.gpu_run(inp)
    s = torch.cuda.Stream()
    outs = {}
    with torch.cuda.stream(s):
        qo, ko, rq, rk = qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"],
                                               **_cfg(w))
        dq, dk, dgq, dgk = qknr.qk_norm_rope_bwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"],
                                                 None, rq, rk, d["dq_out"], d["dk_out"],
                                                 **_cfg(w))
    s.synchronize()
    assert torch.equal(qo.cpu(), ref["q_out"]) and torch.equal(dq.cpu(), ref["dq"])
    # the same calls captured in a CUDA graph and replayed
    g = torch.cuda.CUDAGraph()
    qo.zero_(); dq.zero_(); dgq.fill_(123.0)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        qknr.qk_norm_rope_fwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], q_out=qo, k_out=ko,
                              rstd_q=rq, rstd_k=rk, **_cfg(w))
        qknr.qk_norm_rope_bwd(d["q"], d["k"], d["gamma_q"], d["gamma_k"], None, rq, rk,
                              d["dq_out"], d["dk_out"], dq=dq, dk=dk, dgamma_q=dgq,
                              dgamma_k=dgk, **_cfg(w))
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(qo.cpu(), ref["q_out"]) and torch.equal(dq.cpu(), ref["dq"])
    assert float((dgq.cpu() - ref["dgamma_q"]).abs().max()) <= 1e-5 * float(ref["dgamma_q"].abs().max())


# ------------------------------------------------- simple (fallback) kernels
@pytest.fixture
def simple_kernels():
    import os
    os.environ["QKNR_SIMPLE_KERNELS"] = "1"
    yield
    del os.environ["QKNR_SIMPLE_KERNELS"]


@pytest.mark.parametrize("dtype,D,R", [("bf16", 64, 64), ("bf16", 128, 32), ("bf16", 80, 16),
                                       ("f32", 24, 16), ("f32", 128, 128)])
def test_simple_kernels_shape_sweep(cuda, simple_kernels, dtype, D, R):
    inp = sweep_inputs(dtype, D, R)
    parity.check(inp, parity.gpu_run(inp))


def test_simple_kernels_exact_identities(cuda, simple_kernels):
    test_packing_boundaries_and_pass_through(cuda)


def test_simple_kernels_bench_workload(cuda, simple_kernels):
    inp = workloads.make_inputs(workloads.BENCH_WORKLOAD)
    parity.check(inp, parity.gpu_run(inp))


def test_simple_and_pipelined_agree(cuda):
    """Both kernel families compute the same arithmetic; outputs agree to
    within the rounding of the fp32 sum-of-squares order (1 bf16 ulp)."""
    import os
    inp = workloads.make_inputs("partial-rope-64k", B=1, S=5000)
    a = parity.gpu_run(inp)
    os.environ["QKNR_SIMPLE_KERNELS"] = "1"
    try:
        b = parity.gpu_run(inp)
    finally:
        del os.environ["QKNR_SIMPLE_KERNELS"]
    for n in ("q_out", "k_out", "dq", "dk"):
        d = (a[n].double() - b[n].double()).abs()
        ulp = torch.from_numpy(parity.bf16_ulp(b[n].double().numpy()))
        assert float((d / torch.clamp(ulp, min=1e-5)).max()) <= 1.0, n
    torch.testing.assert_close(a["rstd_q"], b["rstd_q"], rtol=1e-5, atol=0)


def test_no_pipeline_timeouts(cuda):
    assert qknr.pipeline_error() == 0


@pytest.mark.parametrize("family", ["pipelined", "plain"])
def test_offsets_past_4gib_sampled(cuda, family, monkeypatch):
    """A q tensor of 4.3 GB (1,048,613 tokens x 16 heads x 128 dims, bf16):
    element offsets past 2^31 and byte offsets past 2^32 in every pointer
    the kernels form. The rows repeat one seeded 4,096-token block along the
    tokens; positions are s (up to 2^20), so no two tokens give the same
    output. Forward outputs, rstd, dq and dk of sampled tokens (the ends,
    both sides of the 2^31- and 2^32-byte offsets of q, random ones) against
    the oracle; dgamma sums over every row and is checked at the sizes
    above. Both kernel families."""
    if family == "plain":
        monkeypatch.setenv("QKNR_SIMPLE_KERNELS", "1")
    B0 = workloads.make_inputs("llama3-8b-qknorm", B=1, S=4096, Hq=16, Hkv=4, rotary_dim=64)
    w = B0.w
    T = 2 ** 20 + 37
    reps = -(-T // w.S)

    def big(t):
        return t.to(cuda).repeat(1, reps, 1, 1)[:, :T].contiguous()

    q, k, dqo, dko = big(B0.q), big(B0.k), big(B0.dq_out), big(B0.dk_out)
    gq, gk = B0.gamma_q.to(cuda), B0.gamma_k.to(cuda)
    assert q.numel() * q.element_size() > 2 ** 32
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta, eps=w.eps)
    qo, ko, rq, rk = qknr.qk_norm_rope_fwd(q, k, gq, gk, None, **cfg)
    dq, dk, _, _ = qknr.qk_norm_rope_bwd(q, k, gq, gk, None, rq, rk, dqo, dko, **cfg)
    torch.cuda.synchronize()
    tok_bytes = w.Hq * w.D * 2
    edges = [0, 1, T - 2, T - 1]
    for b in (2 ** 31, 2 ** 32):
        t = b // tok_bytes
        edges += [t - 1, t, t + 1]
    rng = np.random.default_rng(5)
    pick = np.unique(np.concatenate([edges, rng.choice(T, 96, replace=False)]))
    idx = torch.from_numpy(pick).to(cuda)
    base = torch.from_numpy(pick % w.S)
    orc = oracle.get()
    ref_q, ref_k, ref_rq, ref_rk = orc.fwd(B0.q[0, base], B0.k[0, base], B0.gamma_q, B0.gamma_k,
                                          pick.astype(np.int64), w.rotary_dim, w.theta, w.eps)
    ref_dq, ref_dk, _, _ = orc.bwd(B0.q[0, base], B0.k[0, base], B0.gamma_q, B0.gamma_k,
                                   pick.astype(np.int64), B0.dq_out[0, base], B0.dk_out[0, base],
                                   w.rotary_dim, w.theta, w.eps)

    def rows(t):
        return oracle.as_f64(t[0].index_select(0, idx).cpu())

    st = parity.Stats(w.dtype, w.D)
    st.elem("q_out", rows(qo), ref_q)
    st.elem("k_out", rows(ko), ref_k)
    st.elem("dq", rows(dq), ref_dq)
    st.elem("dk", rows(dk), ref_dk)
    st.rstd(rows(rq).reshape(-1), np.asarray(ref_rq).reshape(-1))
    st.rstd(rows(rk).reshape(-1), np.asarray(ref_rk).reshape(-1))
    st.check()
