"""Pins for the CPU oracle: checks against what the mathematics fixes.

Each ``pin_*`` takes an ``oracle.Oracle`` handle and raises AssertionError if
the oracle disagrees with something that does not come from the oracle
itself: a library routine (``torch.nn.functional.rms_norm``, complex
multiplication, torch autograd), a closed form, an invariant of rotations or
of RMSNorm, or central finite differences. ``test_oracle.py`` runs them on
the real oracle; ``test_oracle_mutations.py`` runs them on copies of the
oracle with a planted mistake and requires at least one to fail.

Method sources: Chronicals (arXiv 2601.02609), abstract, contribution (1)
(fused QK-RoPE); "Fractional Rotation, Full Potential? ... Partial RoPE",
abstract (rotary on a fraction of dims); "QK-Normed MLA", abstract (one
inverse-RMS scalar per row).
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

TOL = 1e-11


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol * scale:.3e}"


def _rows(rng, n, D, scale=1.0):
    return rng.standard_normal((n, D)) * scale


def _gamma(rng, D):
    return 1.0 + 0.1 * rng.standard_normal(D)


def _torch_rmsnorm(x, gamma, eps):
    """Library RMSNorm (normalised over the last dim, weighted by gamma)."""
    xt = torch.as_tensor(np.asarray(x, dtype=np.float64))
    gt = torch.as_tensor(np.asarray(gamma, dtype=np.float64))
    return F.rms_norm(xt, (xt.shape[-1],), weight=gt, eps=eps).numpy()


def _complex_rope(n, m, R, theta):
    """Rotation of the first R dims written as complex multiplication:
    pair (i, i + R/2) is the complex number n_i + j n_{i+R/2}, multiplied by
    exp(j * m * theta^(-2i/R)) (the RoFormer form of RoPE)."""
    n = np.asarray(n, dtype=np.float64)
    if R == 0:
        return n.copy()
    half = R // 2
    freqs = np.power(float(theta), -2.0 * np.arange(half) / R)
    ang = np.asarray(m, dtype=np.float64)[:, None] * freqs[None, :]
    z = (n[:, :half] + 1j * n[:, half:R]) * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag, n[:, R:]], axis=1)


# --------------------------------------------------------------------- norm
def pin_rmsnorm_matches_library(orc):
    """rotary_dim = 0 reduces the forward to torch's RMSNorm (fp64)."""
    rng = np.random.default_rng(11)
    for D, eps, scale in [(16, 1e-6, 1.0), (64, 0.5, 0.7), (128, 1e-5, 4.0)]:
        x = _rows(rng, 9, D, scale)
        g = _gamma(rng, D)
        y, r = orc.fwd_rows(x, g, np.zeros(9, np.int64), 0, 1e4, eps)
        _close(y, _torch_rmsnorm(x, g, eps), what=f"rmsnorm D={D} eps={eps}")
        # inverse RMS read off the library norm at unit weight
        unit = _torch_rmsnorm(x, np.ones(D), eps)
        j = np.argmax(np.abs(x), axis=1)
        r_lib = unit[np.arange(9), j] / x[np.arange(9), j]
        _close(r, r_lib, what="rstd vs library")


def pin_unit_rms(orc):
    """gamma = 1: each output row has RMS sqrt(ms / (ms + eps)), any position."""
    rng = np.random.default_rng(12)
    D, R, eps = 32, 32, 0.25
    x = _rows(rng, 7, D, 0.8)
    m = rng.integers(-5000, 70000, 7)
    y, _ = orc.fwd_rows(x, np.ones(D), m, R, 1e6, eps)
    ms = np.mean(x * x, axis=1)
    _close(np.sqrt(np.mean(y * y, axis=1)), np.sqrt(ms / (ms + eps)),
           what="unit RMS")


def pin_scale_invariance(orc):
    """eps = 0: y(c x) = y(x) for c > 0."""
    rng = np.random.default_rng(13)
    D, R = 24, 16
    x = _rows(rng, 5, D)
    g = _gamma(rng, D)
    m = rng.integers(0, 4096, 5)
    y1, r1 = orc.fwd_rows(x, g, m, R, 1e4, 0.0)
    y2, r2 = orc.fwd_rows(7.0 * x, g, m, R, 1e4, 0.0)
    _close(y2, y1, what="scale invariance")
    _close(7.0 * r2, r1, what="rstd scales as 1/c")


# ------------------------------------------------------------------- rotary
def pin_rotation_matches_complex(orc):
    """Norm then rotation equals library RMSNorm followed by complex
    multiplication, for full and partial rotary spans and any position."""
    rng = np.random.default_rng(14)
    for D, R, theta in [(16, 16, 1e4), (64, 64, 1e6), (128, 32, 1e6),
                        (128, 128, 5e5), (48, 16, 10.0)]:
        n = 11
        x = _rows(rng, n, D, 2.0)
        g = _gamma(rng, D)
        m = np.concatenate([[0, 1, 65535, -3], rng.integers(0, 70000, n - 4)])
        eps = 1e-6
        y, _ = orc.fwd_rows(x, g, m, R, theta, eps)
        ref = _complex_rope(_torch_rmsnorm(x, g, eps), m, R, theta)
        _close(y, ref, tol=1e-10, what=f"complex rope D={D} R={R}")


def pin_frequency_progression(orc):
    """Recovered rotation angles at m = 1 form the geometric progression
    that starts at 1 and would reach 1/theta after R/2 steps."""
    D, R, theta = 24, 16, 1e4
    half = R // 2
    x = np.zeros((1, D))
    x[0, :half] = 1.0          # each pair starts on the real axis
    x[0, R:] = 1.0
    y, r = orc.fwd_rows(x, np.ones(D), np.array([1]), R, theta, 0.0)
    ang = np.arctan2(y[0, half:R], y[0, :half])
    ratio = theta ** (-1.0 / half)
    assert abs(ang[0] - 1.0) < 1e-14, f"first frequency {ang[0]} != 1"
    _close(ang[1:] / ang[:-1], np.full(half - 1, ratio), tol=1e-12,
           what="frequency ratio")
    assert abs(ang[-1] * ratio - 1.0 / theta) < 1e-15, "progression end"
    _close(y[0, R:], np.full(D - R, r[0]), what="pass-through at m=1")


def pin_pair_norm_preserved(orc):
    """Rotation preserves each pair's length (relative 1e-12)."""
    rng = np.random.default_rng(15)
    D, R = 128, 96
    half = R // 2
    x = _rows(rng, 6, D, 3.0)
    g = _gamma(rng, D)
    m = rng.integers(0, 65536, 6)
    y, _ = orc.fwd_rows(x, g, m, R, 5e5, 1e-5)
    n = _torch_rmsnorm(x, g, 1e-5)
    ly = np.hypot(y[:, :half], y[:, half:R])
    ln = np.hypot(n[:, :half], n[:, half:R])
    _close(ly, ln, tol=1e-12, what="pair norm")


def pin_relative_position(orc):
    """<rope(q, a), rope(k, b)> depends only on a - b."""
    rng = np.random.default_rng(16)
    D, R, theta = 64, 64, 1e4
    q = _rows(rng, 1, D)
    k = _rows(rng, 1, D)
    g = np.ones(D)
    for a, b, t in [(5, 2, 100), (0, 17, 9000), (300, 300, 65000), (7, 1, -7)]:
        yq1, _ = orc.fwd_rows(q, g, np.array([a]), R, theta, 0.0)
        yk1, _ = orc.fwd_rows(k, g, np.array([b]), R, theta, 0.0)
        yq2, _ = orc.fwd_rows(q, g, np.array([a + t]), R, theta, 0.0)
        yk2, _ = orc.fwd_rows(k, g, np.array([b + t]), R, theta, 0.0)
        s1 = float(yq1[0] @ yk1[0])
        s2 = float(yq2[0] @ yk2[0])
        assert abs(s1 - s2) < 1e-9 * max(1.0, abs(s1)), (a, b, t, s1, s2)


def pin_position_zero_identity(orc):
    """At position 0 the rotation is exactly the identity (bitwise)."""
    rng = np.random.default_rng(17)
    D = 32
    x = _rows(rng, 4, D)
    g = _gamma(rng, D)
    z = np.zeros(4, np.int64)
    y_rot, r1 = orc.fwd_rows(x, g, z, D, 1e4, 1e-6)
    y_nope, r2 = orc.fwd_rows(x, g, z, 0, 1e4, 1e-6)
    assert np.array_equal(y_rot, y_nope), "position 0 is not the identity"
    assert np.array_equal(r1, r2)


def pin_pass_through_untouched(orc):
    """Dims >= R equal the norm-only output bitwise, at any position."""
    rng = np.random.default_rng(18)
    D, R = 128, 32
    x = _rows(rng, 5, D)
    g = _gamma(rng, D)
    m = rng.integers(1, 65536, 5)
    y, _ = orc.fwd_rows(x, g, m, R, 1e6, 1e-6)
    y0, _ = orc.fwd_rows(x, g, m, 0, 1e6, 1e-6)
    assert np.array_equal(y[:, R:], y0[:, R:]), "pass-through dims changed"
    assert not np.allclose(y[:, :R], y0[:, :R]), "rotary dims not rotated"


def pin_inverse_rotation(orc):
    """eps = 0, gamma = 1: applying the op at -m to the output at m returns
    the normalised input."""
    rng = np.random.default_rng(19)
    D, R = 64, 48
    x = _rows(rng, 4, D)
    m = rng.integers(0, 65536, 4)
    g = np.ones(D)
    y, r = orc.fwd_rows(x, g, m, R, 1e6, 0.0)
    back, _ = orc.fwd_rows(y, g, -m, R, 1e6, 0.0)
    _close(back, x * r[:, None], what="inverse rotation")


def pin_closed_form(orc):
    """Two-dim rows, eps = 0, worked by hand: x = (3, 0) normalises to
    (sqrt 2, 0); the single pair turns by m * theta^0 = m radians."""
    s2 = math.sqrt(2.0)
    cases = [
        ((3.0, 0.0), (1.0, 1.0), 1, (s2 * math.cos(1), s2 * math.sin(1))),
        ((3.0, 0.0), (2.0, 1.0), 1, (2 * s2 * math.cos(1), 2 * s2 * math.sin(1))),
        ((0.0, -5.0), (1.0, 1.0), 2, (s2 * math.sin(2), -s2 * math.cos(2))),
        ((1.0, 1.0), (1.0, 3.0), 0, (1.0, 3.0)),
    ]
    for x, g, m, want in cases:
        y, r = orc.fwd_rows(np.array([x]), np.array(g), np.array([m]), 2,
                            123.0, 0.0)
        _close(y[0], np.array(want), tol=1e-14, what=f"closed form {x} m={m}")


# ----------------------------------------------------------------- backward
def _small_problem(rng, T=3, Hq=2, Hkv=1, D=8):
    q = rng.standard_normal((T, Hq, D)) * 1.5
    k = rng.standard_normal((T, Hkv, D)) * 1.5
    gq, gk = _gamma(rng, D), _gamma(rng, D)
    dqo = rng.standard_normal((T, Hq, D))
    dko = rng.standard_normal((T, Hkv, D))
    m = np.array([0, 5, 1000, 37, 2, 9][:T], dtype=np.int64)
    return q, k, gq, gk, dqo, dko, m


def pin_bwd_finite_differences(orc):
    """Every gradient element equals a central difference of
    L = <dq_out, q_out> + <dk_out, k_out> (fp64, h = 1e-6)."""
    rng = np.random.default_rng(20)
    for R, theta, eps in [(8, 1e4, 1e-6), (4, 1e2, 0.1)]:
        q, k, gq, gk, dqo, dko, m = _small_problem(rng)

        def loss(q_, k_, gq_, gk_):
            qo, ko, _, _ = orc.fwd(q_, k_, gq_, gk_, m, R, theta, eps)
            return float(np.sum(qo * dqo) + np.sum(ko * dko))

        dq, dk, dgq, dgk = orc.bwd(q, k, gq, gk, m, dqo, dko, R, theta, eps)
        h = 1e-6
        args = [q, k, gq, gk]
        grads = [dq, dk, dgq, dgk]
        for a_i, (arr, grad) in enumerate(zip(args, grads)):
            flat = arr.reshape(-1)
            fd = np.empty(flat.size)
            for j in range(flat.size):
                keep = flat[j]
                flat[j] = keep + h
                lp = loss(*args)
                flat[j] = keep - h
                lm = loss(*args)
                flat[j] = keep
                fd[j] = (lp - lm) / (2 * h)
            _close(grad.reshape(-1), fd, tol=2e-7,
                   what=f"finite differences arg {a_i} R={R}")


def torch_restatement(q, k, gq, gk, m, R, theta, eps):
    """The forward written with library pieces only: torch RMSNorm, then the
    rotation as complex multiplication (differentiable, fp64)."""
    def one(x, g):
        n = F.rms_norm(x, (x.shape[-1],), weight=g, eps=eps)
        if R == 0:
            return n
        half = R // 2
        freqs = float(theta) ** (-2.0 * torch.arange(half, dtype=torch.float64) / R)
        ang = m.to(torch.float64)[:, None] * freqs[None, :]
        rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
        z = torch.complex(n[..., :half], n[..., half:R]) * rot
        return torch.cat([z.real, z.imag, n[..., R:]], dim=-1)
    return one(q, gq), one(k, gk)


def pin_bwd_matches_autograd(orc):
    """Oracle gradients equal torch autograd through the library restatement."""
    rng = np.random.default_rng(21)
    for R, D in [(16, 16), (8, 32), (0, 8)]:
        T, Hq, Hkv = 6, 4, 2
        q, k, gq, gk, dqo, dko, _ = _small_problem(rng, T, Hq, Hkv, D)
        m = rng.integers(0, 70000, T)
        theta, eps = 5e5, 1e-5
        tq, tk = (torch.tensor(a, requires_grad=True) for a in (q, k))
        tgq, tgk = (torch.tensor(a, requires_grad=True) for a in (gq, gk))
        yq, yk = torch_restatement(tq, tk, tgq, tgk, torch.tensor(m), R, theta, eps)
        L = (yq * torch.tensor(dqo)).sum() + (yk * torch.tensor(dko)).sum()
        L.backward()
        qo, ko, _, _ = orc.fwd(q, k, gq, gk, m, R, theta, eps)
        _close(qo, yq.detach().numpy(), tol=1e-10, what="fwd vs restatement q")
        _close(ko, yk.detach().numpy(), tol=1e-10, what="fwd vs restatement k")
        dq, dk, dgq, dgk = orc.bwd(q, k, gq, gk, m, dqo, dko, R, theta, eps)
        _close(dq, tq.grad.numpy(), tol=1e-10, what=f"dq R={R}")
        _close(dk, tk.grad.numpy(), tol=1e-10, what=f"dk R={R}")
        _close(dgq, tgq.grad.numpy(), tol=1e-10, what=f"dgamma_q R={R}")
        _close(dgk, tgk.grad.numpy(), tol=1e-10, what=f"dgamma_k R={R}")


def pin_bwd_orthogonal_at_zero_eps(orc):
    """eps = 0: the output is invariant to scaling x, so dx is orthogonal to x."""
    rng = np.random.default_rng(22)
    D, R = 32, 16
    x = _rows(rng, 5, D, 2.0)
    dy = _rows(rng, 5, D)
    g = _gamma(rng, D)
    m = rng.integers(0, 65536, 5)
    dx, _ = orc.bwd_rows(x, g, dy, m, R, 1e4, 0.0)
    dots = np.sum(dx * x, axis=1)
    assert np.max(np.abs(dots)) < 1e-12 * np.max(np.abs(dx)) * np.max(np.abs(x)) * D


def pin_rows_match_tensors(orc):
    """Whole-tensor entry points equal per-row evaluation with each token's
    position and the right weight (gamma_q for Q heads, gamma_k for K)."""
    rng = np.random.default_rng(23)
    T, Hq, Hkv, D, R = 5, 3, 2, 16, 8
    q, k, gq, gk, dqo, dko, _ = _small_problem(rng, T, Hq, Hkv, D)
    m = rng.integers(0, 9000, T)
    qo, ko, rq, rk = orc.fwd(q, k, gq, gk, m, R, 1e4, 1e-6)
    yq, r1 = orc.fwd_rows(q.reshape(-1, D), gq, np.repeat(m, Hq), R, 1e4, 1e-6)
    yk, r2 = orc.fwd_rows(k.reshape(-1, D), gk, np.repeat(m, Hkv), R, 1e4, 1e-6)
    assert np.array_equal(qo.reshape(-1, D), yq) and np.array_equal(ko.reshape(-1, D), yk)
    assert np.array_equal(rq.reshape(-1), r1) and np.array_equal(rk.reshape(-1), r2)
    dq, dk, dgq, dgk = orc.bwd(q, k, gq, gk, m, dqo, dko, R, 1e4, 1e-6)
    dxq, tq = orc.bwd_rows(q.reshape(-1, D), gq, dqo.reshape(-1, D),
                           np.repeat(m, Hq), R, 1e4, 1e-6)
    dxk, tk = orc.bwd_rows(k.reshape(-1, D), gk, dko.reshape(-1, D),
                           np.repeat(m, Hkv), R, 1e4, 1e-6)
    assert np.array_equal(dq.reshape(-1, D), dxq) and np.array_equal(dk.reshape(-1, D), dxk)
    _close(dgq, tq.sum(axis=0), tol=1e-13, what="dgamma_q sum")
    _close(dgk, tk.sum(axis=0), tol=1e-13, what="dgamma_k sum")


def pin_gradients_nonzero(orc):
    """Gradients are real: every output is non-trivial for random inputs."""
    rng = np.random.default_rng(24)
    q, k, gq, gk, dqo, dko, m = _small_problem(rng, 4, 2, 2, 16)
    dq, dk, dgq, dgk = orc.bwd(q, k, gq, gk, m, dqo, dko, 16, 1e4, 1e-6)
    for name, a in [("dq", dq), ("dk", dk), ("dgamma_q", dgq), ("dgamma_k", dgk)]:
        assert np.linalg.norm(a) > 1e-3, f"{name} is (near) zero"
        assert np.count_nonzero(a) == a.size, f"{name} has exact zeros"


# ------------------------------------------------------------ rotation alone
def pin_rope_matches_complex(orc):
    """Rotation alone equals complex multiplication by exp(j m w_i) on the
    first R dims (a library routine), dims >= R copied."""
    rng = np.random.default_rng(31)
    for D, R in ((64, 64), (128, 32), (16, 0)):
        x = _rows(rng, 6, D, 2.0)
        m = rng.integers(-70000, 70000, 6)
        y = orc.rope_rows(x, m, R, 1e6)
        _close(y, _complex_rope(x, m, R, 1e6), tol=1e-12, what=f"rope D={D} R={R}")


def pin_rope_inverse(orc):
    """The inverse rotation is the transpose: it undoes the forward one, and
    equals the forward rotation at -m."""
    rng = np.random.default_rng(32)
    D, R = 32, 24
    x = _rows(rng, 5, D)
    m = rng.integers(0, 2 ** 31 - 1, 5)
    y = orc.rope_rows(x, m, R, 1e4)
    _close(orc.rope_rows(y, m, R, 1e4, inverse=True), x, tol=1e-12, what="inverse after fwd")
    _close(orc.rope_rows(x, m, R, 1e4, inverse=True), orc.rope_rows(x, -m, R, 1e4),
           tol=1e-15, what="inverse = fwd at -m")
    assert not np.allclose(orc.rope_rows(x, m, R, 1e4, inverse=True), y), "inverse == fwd"


def pin_rope_is_fwd_without_norm(orc):
    """With gamma = 1 and eps = 0 the fused forward is the rotation of x * r,
    so dividing by r recovers the rotation alone."""
    rng = np.random.default_rng(33)
    D, R = 48, 32
    x = _rows(rng, 4, D, 3.0)
    m = rng.integers(0, 9000, 4)
    y, r = orc.fwd_rows(x, np.ones(D), m, R, 5e5, 0.0)
    _close(orc.rope_rows(x, m, R, 5e5), y / r[:, None], tol=1e-12, what="rope vs fwd / r")


# ----------------------------------------------------- mean-centred variant
def pin_ln_matches_library(orc):
    """rotary_dim = 0: the mean-centred forward is torch's layer_norm with the
    weight and no bias (fp64); with a rotary span it is that, rotated as a
    complex multiplication."""
    rng = np.random.default_rng(41)
    for D, R, eps in ((16, 0, 1e-5), (64, 64, 1e-6), (48, 16, 0.3)):
        x = _rows(rng, 7, D, 2.5) + rng.standard_normal((7, 1)) * 3.0
        g = _gamma(rng, D)
        m = rng.integers(0, 50000, 7)
        y, r = orc.ln_fwd_rows(x, g, m, R, 1e4, eps)
        xt = torch.as_tensor(x)
        ln = F.layer_norm(xt, (D,), weight=torch.as_tensor(g), eps=eps).numpy()
        _close(y, _complex_rope(ln, m, R, 1e4), what=f"layer_norm D={D} R={R}")
        var = x.var(axis=1)
        _close(r, 1.0 / np.sqrt(var + eps), tol=1e-13, what="ln rstd")


def pin_ln_shift_invariance(orc):
    """Adding a constant to every element of a row leaves the mean-centred
    output unchanged."""
    rng = np.random.default_rng(42)
    D, R = 32, 32
    x = _rows(rng, 5, D)
    g = _gamma(rng, D)
    m = rng.integers(0, 1000, 5)
    y0, _ = orc.ln_fwd_rows(x, g, m, R, 1e4, 1e-6)
    y1, _ = orc.ln_fwd_rows(x + 7.25, g, m, R, 1e4, 1e-6)
    _close(y1, y0, tol=1e-11, what="shift invariance")


def pin_ln_bwd_finite_differences(orc):
    """Central differences of sum(y * dy) for every element of dx and dgamma."""
    rng = np.random.default_rng(43)
    n, D, R, eps = 3, 8, 4, 1e-3
    x = _rows(rng, n, D, 1.5) + 0.7
    g = _gamma(rng, D)
    dy = _rows(rng, n, D)
    m = rng.integers(0, 100, n)
    dx, dgr = orc.ln_bwd_rows(x, g, dy, m, R, 1e4, eps)

    def loss(xx, gg):
        y, _ = orc.ln_fwd_rows(xx, gg, m, R, 1e4, eps)
        return float(np.sum(y * dy))

    h = 1e-6
    num = np.zeros_like(x)
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        num[idx] = (loss(xp, g) - loss(xm, g)) / (2 * h)
    _close(dx, num, tol=1e-7, what="ln dx finite differences")
    numg = np.zeros(D)
    for d in range(D):
        gp, gm = g.copy(), g.copy()
        gp[d] += h
        gm[d] -= h
        numg[d] = (loss(x, gp) - loss(x, gm)) / (2 * h)
    _close(dgr.sum(axis=0), numg, tol=1e-7, what="ln dgamma finite differences")


def pin_ln_bwd_matches_autograd(orc):
    """torch autograd through layer_norm and a complex-multiplication rotation."""
    rng = np.random.default_rng(44)
    n, D, R, eps = 6, 32, 16, 1e-5
    x = _rows(rng, n, D, 2.0) - 1.0
    g = _gamma(rng, D)
    dy = _rows(rng, n, D)
    m = rng.integers(0, 9000, n)
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    ln = F.layer_norm(xt, (D,), weight=gt, eps=eps)
    half = R // 2
    ang = torch.tensor(m, dtype=torch.float64)[:, None] * torch.pow(
        torch.tensor(1e4, dtype=torch.float64), -2.0 * torch.arange(half, dtype=torch.float64) / R)
    z = torch.complex(ln[:, :half], ln[:, half:R]) * torch.polar(torch.ones_like(ang), ang)
    y = torch.cat([z.real, z.imag, ln[:, R:]], dim=1)
    (y * torch.tensor(dy)).sum().backward()
    dx, dgr = orc.ln_bwd_rows(x, g, dy, m, R, 1e4, eps)
    _close(dx, xt.grad.numpy(), tol=1e-12, what="ln dx vs autograd")
    _close(dgr.sum(axis=0), gt.grad.numpy(), tol=1e-12, what="ln dgamma vs autograd")


# ----------------------------------------------------------- layerwise variant
def pin_lw_matches_library(orc):
    """Layerwise forward: torch rms_norm over each token's whole hidden vector
    (H * D, weight over the hidden), then complex-multiplication RoPE on each
    head row."""
    rng = np.random.default_rng(51)
    for H, D, R in ((3, 8, 8), (4, 16, 0), (2, 32, 16)):
        T = 6
        x = rng.standard_normal((T, H, D)) * 2.0
        g = 1.0 + 0.1 * rng.standard_normal(H * D)
        m = rng.integers(0, 40000, T)
        y, r = orc.lw_fwd(x, g, m, R, 1e4, 1e-6)
        xt = torch.as_tensor(x.reshape(T, H * D))
        n = F.rms_norm(xt, (H * D,), weight=torch.as_tensor(g), eps=1e-6).numpy().reshape(T, H, D)
        want = _complex_rope(n.reshape(T * H, D), np.repeat(m, H), R, 1e4).reshape(T, H, D)
        _close(y, want, what=f"layerwise H={H} D={D} R={R}")
        _close(r, 1.0 / np.sqrt((x.reshape(T, -1) ** 2).mean(axis=1) + 1e-6), tol=1e-13,
               what="layerwise rstd")


def pin_lw_one_head_is_per_head(orc):
    """With one head the layerwise form is the per-head form."""
    rng = np.random.default_rng(52)
    T, D, R = 7, 32, 32
    x = rng.standard_normal((T, 1, D))
    g = _gamma(rng, D)
    m = rng.integers(0, 9000, T)
    y, r = orc.lw_fwd(x, g, m, R, 1e4, 1e-5)
    y1, r1 = orc.fwd_rows(x.reshape(T, D), g, m, R, 1e4, 1e-5)
    _close(y.reshape(T, D), y1, tol=1e-13, what="layerwise H=1 vs per head")
    _close(r, r1, tol=1e-13, what="layerwise H=1 rstd")
    dy = rng.standard_normal((T, 1, D))
    dx, dg = orc.lw_bwd(x, g, dy, m, R, 1e4, 1e-5)
    dx1, t1 = orc.bwd_rows(x.reshape(T, D), g, dy.reshape(T, D), m, R, 1e4, 1e-5)
    _close(dx.reshape(T, D), dx1, tol=1e-12, what="layerwise H=1 dx")
    _close(dg, t1.sum(axis=0), tol=1e-12, what="layerwise H=1 dgamma")


def pin_lw_bwd_matches_autograd(orc):
    """Layerwise backward against torch autograd through rms_norm over the
    hidden vector and complex-multiplication RoPE per head."""
    rng = np.random.default_rng(53)
    T, H, D, R, eps = 4, 3, 16, 8, 1e-4
    x = rng.standard_normal((T, H, D)) * 1.5
    g = 1.0 + 0.1 * rng.standard_normal(H * D)
    dy = rng.standard_normal((T, H, D))
    m = rng.integers(0, 5000, T)
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    n = F.rms_norm(xt.reshape(T, H * D), (H * D,), weight=gt, eps=eps).reshape(T, H, D)
    half = R // 2
    ang = torch.tensor(m, dtype=torch.float64)[:, None, None] * torch.pow(
        torch.tensor(1e4, dtype=torch.float64), -2.0 * torch.arange(half, dtype=torch.float64) / R)
    z = torch.complex(n[..., :half], n[..., half:R]) * torch.polar(torch.ones_like(ang), ang)
    y = torch.cat([z.real, z.imag, n[..., R:]], dim=-1)
    (y * torch.tensor(dy)).sum().backward()
    dx, dg = orc.lw_bwd(x, g, dy, m, R, 1e4, eps)
    _close(dx, xt.grad.numpy(), tol=1e-12, what="layerwise dx vs autograd")
    _close(dg, gt.grad.numpy(), tol=1e-12, what="layerwise dgamma vs autograd")


ALL_PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
