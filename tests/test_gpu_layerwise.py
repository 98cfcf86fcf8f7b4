"""Layerwise QK-RMSNorm + RoPE under tensor parallelism (the qk_layerwise_*
entry points) against the oracle's layerwise functions (``lw_fwd`` /
``lw_bwd``: one statistic per token over all heads, gamma over the full
hidden vector).

One rank holding every head is checked element by element against the
oracle, for both kernel families (the pipelined kernels, and the plain-load
kernels that serve shapes the pipeline's shared-memory ring cannot hold). Tensor parallelism is emulated on one GPU: the heads are split into
W slices ("ranks"), each slice runs stats / dots on its own, the per-token
partial sums are added (the all-reduce a multi-GPU run makes over NCCL),
and each slice then normalises its heads; the concatenated outputs and the
per-slice dgamma must match the oracle on the full tensor. No kernel waits
on another slice, so this needs one GPU only.
"""
import os

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


def lw_inputs(name, seed=None, **over):
    inp = workloads.make_inputs(name, seed=seed, **over)
    gq, gk = workloads.layerwise_gamma(inp.w, 17 if seed is None else seed)
    return inp, gq, gk


def positions_of(inp):
    w = inp.w
    return oracle.positions(None if inp.pos is None else inp.pos.numpy(), w.B, w.S)


def run_ranks(inp, gq, gk, cuda, world=1, local=False):
    """fwd + bwd with the heads split into ``world`` even slices; the
    partial sums of the slices are added on the device between the calls.
    ``local`` (one slice only): no separate stats / dots calls, the fwd and
    bwd take the statistics in their own pass. Returns CPU results over all
    heads (rstd per token)."""
    w = inp.w
    assert w.Hq % world == 0 and w.Hkv % world == 0
    hq, hk, D = w.Hq // world, w.Hkv // world, w.D
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta)
    pos = None if inp.pos is None else inp.pos.to(cuda)
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    dqo, dko = inp.dq_out.to(cuda), inp.dk_out.to(cuda)
    gqd, gkd = gq.to(cuda), gk.to(cuda)
    sl = []
    for r in range(world):
        sq_, sk_ = slice(r * hq, (r + 1) * hq), slice(r * hk, (r + 1) * hk)
        sl.append(dict(q=q[:, :, sq_].contiguous(), k=k[:, :, sk_].contiguous(),
                       dqo=dqo[:, :, sq_].contiguous(), dko=dko[:, :, sk_].contiguous(),
                       gq=gqd[r * hq * D:(r + 1) * hq * D], gk=gkd[r * hk * D:(r + 1) * hk * D]))
    assert world == 1 or not local
    stats = [qknr.qk_layerwise_stats(s["q"], s["k"]) for s in sl]
    Sq = sum(s[0] for s in stats)
    Sk = sum(s[1] for s in stats)
    if local:
        Sq_in = Sk_in = None
    else:
        Sq_in, Sk_in = Sq, Sk
    fw = [qknr.qk_layerwise_norm_rope_fwd(s["q"], s["k"], s["gq"], s["gk"], pos, Sq_in, Sk_in,
                                          eps=w.eps, Hq_total=w.Hq, Hkv_total=w.Hkv, **cfg)
          for s in sl]
    dots = [qknr.qk_layerwise_bwd_dots(s["q"], s["k"], s["gq"], s["gk"], pos, f[2], f[3],
                                       s["dqo"], s["dko"], **cfg) for s, f in zip(sl, fw)]
    Pq = sum(d[0] for d in dots)
    Pk = sum(d[1] for d in dots)
    Pq_in, Pk_in = (None, None) if local else (Pq, Pk)
    bw = [qknr.qk_layerwise_norm_rope_bwd(s["q"], s["k"], s["gq"], s["gk"], pos, f[2], f[3],
                                          s["dqo"], s["dko"], Pq_in, Pk_in, Hq_total=w.Hq,
                                          Hkv_total=w.Hkv, **cfg) for s, f in zip(sl, fw)]
    torch.cuda.synchronize()
    cat = lambda xs, d: torch.cat(xs, dim=d).cpu()
    return {"q_out": cat([f[0] for f in fw], 2), "k_out": cat([f[1] for f in fw], 2),
            "rstd_q": fw[0][2].cpu(), "rstd_k": fw[0][3].cpu(),
            "rstd_q_all": [f[2].cpu() for f in fw],
            "dq": cat([b[0] for b in bw], 2), "dk": cat([b[1] for b in bw], 2),
            "dgamma_q": cat([b[2] for b in bw], 0), "dgamma_k": cat([b[3] for b in bw], 0),
            "sumsq_q": Sq.cpu(), "dot_q": Pq.cpu()}


def check_vs_oracle(inp, gq, gk, got):
    """Element bounds of parity.py (fp32 1e-5 max-abs; bf16 2e-2 max-abs where
    |ref| < 8 and one bf16 ulp everywhere); rstd to (H D) 2^-24 relative
    (an fp32 sum over the whole hidden vector); dgamma to its normwise
    tolerance."""
    w = inp.w
    o = oracle.get()
    m = positions_of(inp)
    T = w.B * w.S
    st_q = parity.Stats(w.dtype, max(w.Hq, 1) * w.D)
    st_k = parity.Stats(w.dtype, max(w.Hkv, 1) * w.D)
    dg = {}
    for name, x, g, dy, st, H in (("q", inp.q, gq, inp.dq_out, st_q, w.Hq),
                                  ("k", inp.k, gk, inp.dk_out, st_k, w.Hkv)):
        if H == 0:
            continue
        x3 = x.reshape(T, H, w.D)
        y, r = o.lw_fwd(x3, g, m, w.rotary_dim, w.theta, w.eps)
        dx, dgr = o.lw_bwd(x3, g, dy.reshape(T, H, w.D), m, w.rotary_dim, w.theta, w.eps)
        st.elem(f"{name}_out", got[f"{name}_out"].double().numpy().reshape(-1), y.reshape(-1))
        st.rstd(got[f"rstd_{name}"].double().numpy().reshape(-1), r)
        st.elem(f"d{name}", got[f"d{name}"].double().numpy().reshape(-1), dx.reshape(-1))
        dg[f"dgamma_{name}"] = (got[f"dgamma_{name}"].double().numpy(), dgr)
    st_q.check({k_: v for k_, v in dg.items() if k_ == "dgamma_q"})
    st_k.check({k_: v for k_, v in dg.items() if k_ == "dgamma_k"})


CASES = [
    ("tiny", dict()),
    ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=24, rotary_dim=16)),
    ("qwen2.5-0.5b", dict(B=2, S=129)),
    ("llama3-8b-qknorm", dict(B=1, S=97)),
    ("partial-rope-64k", dict(S=300)),
    ("bfd-packed", dict()),
]


@pytest.mark.parametrize("local", [False, True], ids=["two-phase", "one-pass"])
@pytest.mark.parametrize("name,over", CASES,
                         ids=[f"{n}-{'-'.join(f'{k}{v}' for k, v in o.items())}"
                              for n, o in CASES])
def test_layerwise_one_rank_vs_oracle(cuda, kernels, name, over, local):
    inp, gq, gk = lw_inputs(name, **over)
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, world=1, local=local))


@pytest.mark.parametrize("name,over", [("qwen2.5-0.5b", dict(B=2, S=300)),
                                       ("llama3-8b-qknorm", dict(B=1, S=150)),
                                       ("partial-rope-64k", dict(S=211)),
                                       ("tiny", dict(B=3, S=37, Hq=5, Hkv=3, D=24,
                                                     rotary_dim=16))])
def test_layerwise_one_pass_equals_two_phase(cuda, kernels, name, over):
    """The one-pass calls take the statistics with the same lane layout and
    order as qk_layerwise_stats / qk_layerwise_bwd_dots: bit for bit the same
    rstd, outputs and dx (dgamma, summed with atomics, to its tolerance)."""
    inp, gq, gk = lw_inputs(name, **over)
    two = run_ranks(inp, gq, gk, cuda)
    one = run_ranks(inp, gq, gk, cuda, local=True)
    for n in ("q_out", "k_out", "rstd_q", "rstd_k", "dq", "dk"):
        assert torch.equal(one[n], two[n]), n
    for n in ("dgamma_q", "dgamma_k"):
        ref = two[n].double()
        assert float((one[n].double() - ref).abs().max() / ref.abs().max()) <= 1e-5, n


@pytest.mark.parametrize("world", [2, 4, 8])
def test_layerwise_tp_slices_vs_oracle(cuda, kernels, world):
    inp, gq, gk = lw_inputs("llama3-8b-qknorm", B=2, S=65)
    got = run_ranks(inp, gq, gk, cuda, world=world)
    # every slice saved the same statistic (it used the summed totals)
    for r in got["rstd_q_all"][1:]:
        assert torch.equal(r, got["rstd_q_all"][0])
    check_vs_oracle(inp, gq, gk, got)


def test_layerwise_tp_matches_one_rank(cuda):
    # the slices change only the fp32 summation order of the statistics
    inp, gq, gk = lw_inputs("qwen2.5-0.5b", B=1, S=200, Hq=16, Hkv=4)
    one = run_ranks(inp, gq, gk, cuda, world=1)
    two = run_ranks(inp, gq, gk, cuda, world=2)
    rel = float(((one["sumsq_q"] - two["sumsq_q"]).abs() / one["sumsq_q"]).max())
    assert rel <= 16 * 64 * 2.0 ** -24
    for n in ("q_out", "k_out", "dq", "dk"):
        a, b = one[n].float(), two[n].float()
        # at most about one bf16 rounding apart
        assert bool(((a - b).abs() <= 2e-2 + b.abs() * 2.0 ** -7).all()), n


def test_layerwise_one_head_is_per_head(cuda):
    """With one head per tensor the layerwise statistic is the per-head one:
    the same values as qk_norm_rope_* (to rounding; different kernels)."""
    inp, _, _ = lw_inputs("llama3-8b-qknorm", B=2, S=50, Hq=1, Hkv=1, dtype="f32")
    w = inp.w
    got = run_ranks(inp, inp.gamma_q, inp.gamma_k, cuda)
    dense = parity.gpu_run(inp)
    for n in ("q_out", "k_out", "dq", "dk"):
        assert float((got[n] - dense[n]).abs().max()) <= 1e-5, n
    for n in ("rstd_q", "rstd_k"):
        a, b = got[n].reshape(-1), dense[n].reshape(-1)
        assert float(((a - b).abs() / b).max()) <= w.D * 2.0 ** -24, n
    for n in ("dgamma_q", "dgamma_k"):
        ref = dense[n].double()
        assert float((got[n].double() - ref).abs().max() / ref.abs().max()) <= 1e-5, n


@pytest.mark.parametrize("Hq,Hkv", [(4, 0), (0, 4), (33, 1)])
def test_layerwise_head_counts(cuda, kernels, Hq, Hkv):
    inp, gq, gk = lw_inputs("qwen2.5-0.5b", seed=5, B=2, S=41, Hq=Hq, Hkv=Hkv)
    got = run_ranks(inp, gq, gk, cuda)
    check_vs_oracle(inp, gq, gk, got)


def test_layerwise_autograd(cuda):
    inp, gq, gk = lw_inputs("qwen2.5-0.5b", B=2, S=65)
    w = inp.w
    q = inp.q.to(cuda).requires_grad_(True)
    k = inp.k.to(cuda).requires_grad_(True)
    gqd = gq.to(cuda).requires_grad_(True)
    gkd = gk.to(cuda).requires_grad_(True)
    qo, ko = qknr.qk_layerwise_norm_rope(q, k, gqd, gkd, rotary_dim=w.rotary_dim, theta=w.theta,
                                         eps=w.eps)
    torch.autograd.backward([qo, ko], [inp.dq_out.to(cuda), inp.dk_out.to(cuda)])
    got = run_ranks(inp, gq, gk, cuda)
    assert torch.equal(qo.detach().cpu(), got["q_out"])
    assert torch.equal(ko.detach().cpu(), got["k_out"])
    assert torch.equal(q.grad.cpu(), got["dq"]) and torch.equal(k.grad.cpu(), got["dk"])
    for a, b in ((gqd.grad, got["dgamma_q"]), (gkd.grad, got["dgamma_k"])):
        ref = b.double()
        rel = float((a.double().cpu() - ref).abs().max() / ref.abs().max())
        assert rel <= 1e-2   # dgamma is returned in gamma's dtype (bf16)


def test_layerwise_in_place(cuda):
    inp, gq, gk = lw_inputs("qwen2.5-0.5b", B=1, S=100)
    w = inp.w
    ref = run_ranks(inp, gq, gk, cuda)
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    gqd, gkd = gq.to(cuda), gk.to(cuda)
    sq, sk = qknr.qk_layerwise_stats(q, k)
    qknr.qk_layerwise_norm_rope_fwd(q, k, gqd, gkd, None, sq, sk, rotary_dim=w.rotary_dim,
                                    theta=w.theta, eps=w.eps, Hq_total=w.Hq, Hkv_total=w.Hkv,
                                    q_out=q, k_out=k)
    torch.cuda.synchronize()
    assert torch.equal(q.cpu(), ref["q_out"]) and torch.equal(k.cpu(), ref["k_out"])


def test_layerwise_errors(cuda):
    inp, gq, gk = lw_inputs("qwen2.5-0.5b", B=1, S=16)
    w = inp.w
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    gqd, gkd = gq.to(cuda), gk.to(cuda)
    sq, sk = qknr.qk_layerwise_stats(q, k)
    with pytest.raises(qknr.QKNRError):    # totals below the local head counts
        qknr.qk_layerwise_norm_rope_fwd(q, k, gqd, gkd, None, sq, sk, rotary_dim=64, theta=1e4,
                                        eps=1e-6, Hq_total=w.Hq - 1, Hkv_total=w.Hkv)
    with pytest.raises(ValueError):        # a per-head gamma is not a layerwise one
        qknr.qk_layerwise_norm_rope_fwd(q, k, gqd[:w.D], gkd, None, sq, sk, rotary_dim=64,
                                        theta=1e4, eps=1e-6, Hq_total=w.Hq, Hkv_total=w.Hkv)
    # the backward's dgamma partial sums must fit in shared memory
    big = torch.zeros(1, 4, 512, 128, dtype=torch.bfloat16, device=cuda)
    gbig = torch.ones(512 * 128, dtype=torch.bfloat16, device=cuda)
    r = torch.ones(4, device=cuda)
    with pytest.raises(qknr.QKNRError) as e:
        qknr.qk_layerwise_norm_rope_bwd(big, big[:, :, :0], gbig, gbig[:0], None, r, r, big,
                                        big[:, :, :0].contiguous(), r, r, rotary_dim=128,
                                        theta=1e4, Hq_total=512, Hkv_total=0)
    assert e.value.status == qknr.QKNR_ERR_UNSUPPORTED


@pytest.mark.parametrize("B,S", [(1, 1), (1, 3), (2, 5), (3, 41), (1, 4099)])
def test_layerwise_token_counts(cuda, B, S):
    # ragged last stages and CTAs with a single partial stage
    inp, gq, gk = lw_inputs("llama3-8b-qknorm", seed=9, B=B, S=S, Hq=6, Hkv=2)
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, local=True))


def test_layerwise_large_hidden_falls_back(cuda):
    # 72 heads of 256 fp32 elements per token: too big for the ring; the
    # plain-load kernels serve it
    inp, gq, gk = lw_inputs("tiny", seed=2, B=1, S=9, Hq=64, Hkv=8, D=256, rotary_dim=128)
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, local=True))


def test_layerwise_no_pipeline_timeouts(cuda):
    assert qknr.pipeline_error() == 0


@pytest.mark.parametrize("dtype,D,R", [("bf16", 128, 0), ("f32", 64, 0), ("f32", 64, 16),
                                       ("bf16", 64, 32), ("bf16", 72, 64), ("f32", 12, 8)])
def test_layerwise_rotary_spans_and_dtypes(cuda, kernels, dtype, D, R):
    # NoPE (no rotary span), partial spans, fp32 I/O; one rank and two slices
    inp, gq, gk = lw_inputs("tiny", seed=6, B=2, S=45, Hq=8, Hkv=4, D=D, rotary_dim=R,
                            dtype=dtype)
    for world in (1, 2):
        check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, world=world))
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, local=True))


def test_layerwise_extreme_positions(cuda, kernels):
    import numpy as np
    inp, gq, gk = lw_inputs("tiny", seed=3, B=2, S=40, Hq=6, Hkv=2, D=128, rotary_dim=64,
                            dtype="bf16", theta=1e4)
    rng = np.random.default_rng(3)
    pos = rng.integers(-2 ** 31, 2 ** 31 - 1, size=(2, 40))
    pos.reshape(-1)[:6] = [0, 1, -1, 2 ** 31 - 1, -(2 ** 31), 65535]
    inp.pos = torch.from_numpy(pos.astype(np.int32))
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, local=True))
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, world=2))


def test_layerwise_full_size_sampled(cuda):
    """The Llama-3-8B-shaped batch at full size (32,768 tokens, 40 heads), one
    pass each way as the bench times it; outputs, rstd and dX of 384 sampled
    tokens against the oracle (each token's statistic involves that token
    only). dgamma is a sum over every token and is checked at the smaller
    sizes above."""
    import numpy as np
    inp, gq, gk = lw_inputs("llama3-8b-qknorm")
    w = inp.w
    got = run_ranks(inp, gq, gk, cuda, local=True)
    T = w.B * w.S
    pick = np.sort(np.random.default_rng(11).choice(T, 384, replace=False))
    pick[:2] = [0, T - 1]
    m = positions_of(inp)[pick]
    o = oracle.get()
    for name, x, g, dy, H in (("q", inp.q, gq, inp.dq_out, w.Hq), ("k", inp.k, gk, inp.dk_out, w.Hkv)):
        st = parity.Stats(w.dtype, H * w.D)
        x3 = x.reshape(T, H, w.D)[pick]
        y, r = o.lw_fwd(x3, g, m, w.rotary_dim, w.theta, w.eps)
        dx, _ = o.lw_bwd(x3, g, dy.reshape(T, H, w.D)[pick], m, w.rotary_dim, w.theta, w.eps)
        st.elem(f"{name}_out", got[f"{name}_out"].reshape(T, H, w.D)[pick].double().numpy(), y)
        st.rstd(got[f"rstd_{name}"].reshape(T)[pick].double().numpy(), r)
        st.elem(f"d{name}", got[f"d{name}"].reshape(T, H, w.D)[pick].double().numpy(), dx)
        st.check()


@pytest.mark.parametrize("name,over,chunks", [("llama3-8b-qknorm", dict(B=2, S=97), 4),
                                              ("partial-rope-64k", dict(S=1000), 3),
                                              ("bfd-packed", dict(), 4),
                                              ("tiny", dict(B=3, S=37, Hq=6, Hkv=2, D=24,
                                                            rotary_dim=16), 7)])
def test_layerwise_chunked_schedule_vs_oracle(cuda, name, over, chunks):
    """The binding's chunked exchange schedule (stats of a chunk, its sums
    exchanged on a side stream, the chunk normalised once they are in, the
    next chunk's stats overlapping the exchange), for each of two emulated
    ranks on one GPU: the exchange adds the other slice's partial sums of the
    chunk's tokens, as an all-reduce over two ranks would. The concatenated
    outputs and the per-slice dgamma must match the oracle on the full
    tensor; the outputs equal the unchunked two-phase calls bit for bit."""
    inp, gq, gk = lw_inputs(name, **over)
    w = inp.w
    hq, hk, D = w.Hq // 2, w.Hkv // 2, w.D
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta)
    pos = None if inp.pos is None else inp.pos.to(cuda)
    q, k = inp.q.to(cuda), inp.k.to(cuda)
    dqo, dko = inp.dq_out.to(cuda), inp.dk_out.to(cuda)
    gqd, gkd = gq.to(cuda), gk.to(cuda)
    sl = []
    for r in range(2):
        sq_, sk_ = slice(r * hq, (r + 1) * hq), slice(r * hk, (r + 1) * hk)
        sl.append(dict(q=q[:, :, sq_].contiguous(), k=k[:, :, sk_].contiguous(),
                       dqo=dqo[:, :, sq_].contiguous(), dko=dko[:, :, sk_].contiguous(),
                       gq=gqd[r * hq * D:(r + 1) * hq * D], gk=gkd[r * hk * D:(r + 1) * hk * D]))
    stats = [qknr.qk_layerwise_stats(s["q"], s["k"]) for s in sl]

    def exchange_with(other):
        def ex(buf, span):
            t0, t1 = span
            buf[0] += other[0][t0:t1]
            buf[1] += other[1][t0:t1]
        return ex

    fw = [qknr.layerwise_chunked_fwd(s["q"], s["k"], s["gq"], s["gk"], pos, eps=w.eps,
                                     Hq_total=w.Hq, Hkv_total=w.Hkv,
                                     exchange=exchange_with(stats[1 - r]), chunks=chunks,
                                     min_chunk=1, min_chunk_bytes=0, **cfg)
          for r, s in enumerate(sl)]
    dots = [qknr.qk_layerwise_bwd_dots(s["q"], s["k"], s["gq"], s["gk"], pos, f[2], f[3],
                                       s["dqo"], s["dko"], **cfg) for s, f in zip(sl, fw)]
    bw = [qknr.layerwise_chunked_bwd(s["q"], s["k"], s["gq"], s["gk"], pos, f[2], f[3],
                                     s["dqo"], s["dko"], Hq_total=w.Hq, Hkv_total=w.Hkv,
                                     exchange=exchange_with(dots[1 - r]), chunks=chunks,
                                     min_chunk=1, min_chunk_bytes=0, **cfg)
          for r, (s, f) in enumerate(zip(sl, fw))]
    torch.cuda.synchronize()
    cat = lambda xs, d: torch.cat(xs, dim=d).cpu()
    got = {"q_out": cat([f[0] for f in fw], 2), "k_out": cat([f[1] for f in fw], 2),
           "rstd_q": fw[0][2].cpu(), "rstd_k": fw[0][3].cpu(),
           "dq": cat([b[0] for b in bw], 2), "dk": cat([b[1] for b in bw], 2),
           "dgamma_q": cat([b[2] for b in bw], 0), "dgamma_k": cat([b[3] for b in bw], 0)}
    assert torch.equal(fw[0][2], fw[1][2]) and torch.equal(fw[0][3], fw[1][3])
    check_vs_oracle(inp, gq, gk, got)
    two = run_ranks(inp, gq, gk, cuda, world=2)
    for n in ("q_out", "k_out", "dq", "dk"):
        assert torch.equal(got[n], two[n]), n


def test_layerwise_partial_last_stage_vs_oracle(cuda):
    """A shape whose CTA runs end in a partial stage (the tokens after the
    first tile not a multiple of the stage's tokens) and whose grid is below
    the SM count:
    the launch plan says so, and every element matches the oracle."""
    sms = torch.cuda.get_device_properties(cuda).multi_processor_count
    inp, gq, gk = lw_inputs("llama3-8b-qknorm", B=1, S=1500)
    w = inp.w
    for mode in ("bwd", "tok"):
        g = qknr.layerwise_geometry(mode, w.B, w.S, w.Hq, w.Hkv, w.D, w.rotary_dim,
                                    torch.bfloat16, sms)
        # after a first tile of first_tile tokens, whole tiles of TT, then
        # a partial one
        assert g["pipelined"] and g["grid"] < sms, (mode, g)
        assert g["tpc"] > g["TT"] and (g["tpc"] - g["first_tile"]) % g["TT"] != 0, (mode, g)
    for local in (False, True):
        check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, world=1, local=local))
    check_vs_oracle(inp, gq, gk, run_ranks(inp, gq, gk, cuda, world=2))


def test_layerwise_offsets_past_4gib_sampled(cuda):
    """One rank holding every head, q of 4.3 GB (1,048,613 tokens x 16 heads
    x 128 dims, bf16): offsets past 2^31 elements and 2^32 bytes. The rows
    repeat one seeded 4,096-token block along the tokens, positions are s,
    so every token's output differs. Outputs, rstd and dX of sampled tokens
    (the ends, both sides of the 2^31- and 2^32-byte offsets of q, random
    ones) against the oracle; dgamma is checked at the sizes above."""
    import numpy as np
    base_inp, gq, gk = lw_inputs("llama3-8b-qknorm", B=1, S=4096, Hq=16, Hkv=4, rotary_dim=64)
    w = base_inp.w
    T = 2 ** 20 + 37
    reps = -(-T // w.S)

    def big(t):
        return t.to(cuda).repeat(1, reps, 1, 1)[:, :T].contiguous()

    q, k = big(base_inp.q), big(base_inp.k)
    dqo, dko = big(base_inp.dq_out), big(base_inp.dk_out)
    assert q.numel() * q.element_size() > 2 ** 32
    cfg = dict(rotary_dim=w.rotary_dim, theta=w.theta, Hq_total=w.Hq, Hkv_total=w.Hkv)
    qo, ko, rq, rk = qknr.qk_layerwise_norm_rope_fwd(q, k, gq.to(cuda), gk.to(cuda), None, None,
                                                     None, eps=w.eps, **cfg)
    dq, dk, _, _ = qknr.qk_layerwise_norm_rope_bwd(q, k, gq.to(cuda), gk.to(cuda), None, rq, rk,
                                                   dqo, dko, None, None, **cfg)
    torch.cuda.synchronize()
    tok_bytes = w.Hq * w.D * 2
    edges = [0, 1, T - 2, T - 1]
    for b in (2 ** 31, 2 ** 32):
        t = b // tok_bytes
        edges += [t - 1, t, t + 1]
    pick = np.unique(np.concatenate([edges, np.random.default_rng(6).choice(T, 96,
                                                                           replace=False)]))
    idx = torch.from_numpy(pick).to(cuda)
    base = torch.from_numpy(pick % w.S)
    o = oracle.get()
    got = {"q_out": qo, "k_out": ko, "dq": dq, "dk": dk, "rstd_q": rq, "rstd_k": rk}
    for name, x, g, dy, H in (("q", base_inp.q, gq, base_inp.dq_out, w.Hq),
                              ("k", base_inp.k, gk, base_inp.dk_out, w.Hkv)):
        st = parity.Stats(w.dtype, H * w.D)
        y, r = o.lw_fwd(x[0, base], g, pick, w.rotary_dim, w.theta, w.eps)
        dx, _ = o.lw_bwd(x[0, base], g, dy[0, base], pick, w.rotary_dim, w.theta, w.eps)
        sel = lambda t: oracle.as_f64(t.reshape(T, -1).index_select(0, idx).cpu())
        st.elem(f"{name}_out", sel(got[f"{name}_out"]).reshape(y.shape), y)
        st.elem(f"d{name}", sel(got[f"d{name}"]).reshape(dx.shape), dx)
        st.rstd(sel(got[f"rstd_{name}"]).reshape(-1), np.asarray(r).reshape(-1))
        st.check()
