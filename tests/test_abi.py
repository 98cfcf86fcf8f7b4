"""The C ABI library: it loads, exports every symbol include/qknr.h declares,
and rejects bad arguments on the host before touching the GPU.

No GPU is needed: every call here either fails validation, which happens
before any CUDA runtime call, or is an empty problem (B = 0) that returns
before one, or is a host-only plan query. The pointers are fake addresses
that are never dereferenced.
"""
import ctypes
import os
import re

import pytest

import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qknr.h")

OK, INVALID, ALIGN, UNSUP, CUDA = range(5)
F32, BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qknr.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"#define QKNR_API.*", "", src)
    return re.findall(r"QKNR_API\s+[\w\s\*]*?\b(\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("qk_norm_rope_fwd", "qk_norm_rope_bwd", "qknr_strerror", "qknr_last_cuda_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in qknr.h but not exported"


def test_library_is_sm100a_only():
    assert "arch=compute_100a,code=sm_100a" in " ".join(qbuild.NVCC_FLAGS)
    assert "sm_90" not in " ".join(qbuild.NVCC_FLAGS)


def test_strerror_covers_every_status(lib):
    for s in range(5):
        assert len(qknr.qknr_strerror(s)) > 5
    assert qknr.qknr_strerror(99) == "unknown status"


# fake, 256-aligned, well separated device addresses (never dereferenced)
def P(i, off=0):
    return ctypes.c_void_p(0x7f0000000000 + i * (1 << 32) + off)


def fwd(lib, B=2, S=8, Hq=4, Hkv=2, D=64, R=64, theta=1e4, eps=1e-6, dt=BF16, **ptrs):
    p = dict(q=P(1), k=P(2), gq=P(3), gk=P(4), pos=None, qo=P(5), ko=P(6), rq=P(7), rk=P(8))
    p.update(ptrs)
    return lib.qk_norm_rope_fwd(p["q"], p["k"], p["gq"], p["gk"], p["pos"], p["qo"], p["ko"],
                                p["rq"], p["rk"], B, S, Hq, Hkv, D, R, theta, eps, dt, None)


def bwd(lib, B=2, S=8, Hq=4, Hkv=2, D=64, R=64, theta=1e4, eps=1e-6, dt=BF16, **ptrs):
    p = dict(q=P(1), k=P(2), gq=P(3), gk=P(4), pos=None, rq=P(7), rk=P(8), dqo=P(9),
             dko=P(10), dq=P(11), dk=P(12), dgq=P(13), dgk=P(14))
    p.update(ptrs)
    return lib.qk_norm_rope_bwd(p["q"], p["k"], p["gq"], p["gk"], p["pos"], p["rq"], p["rk"],
                                p["dqo"], p["dko"], p["dq"], p["dk"], p["dgq"], p["dgk"],
                                B, S, Hq, Hkv, D, R, theta, eps, dt, None)


@pytest.mark.parametrize("call", [fwd, bwd], ids=["fwd", "bwd"])
@pytest.mark.parametrize("kw,want", [
    (dict(B=-1), INVALID), (dict(S=-3), INVALID), (dict(Hq=-1), INVALID),
    (dict(D=0), INVALID), (dict(D=63), INVALID), (dict(R=66), INVALID),
    (dict(R=-2), INVALID), (dict(R=31), INVALID), (dict(theta=0.0), INVALID),
    (dict(theta=float("inf")), INVALID), (dict(theta=float("nan")), INVALID),
    (dict(eps=-1e-6), INVALID), (dict(eps=float("nan")), INVALID), (dict(dt=7), INVALID),
    (dict(D=512, R=512), UNSUP), (dict(D=72, R=72), UNSUP), (dict(D=64, R=8), UNSUP),
])
def test_shape_validation(lib, call, kw, want):
    assert call(lib, **kw) == want


@pytest.mark.parametrize("dt,D,R", [(BF16, 72, 64), (BF16, 72, 0), (BF16, 8, 0),
                                    (BF16, 40, 16), (F32, 12, 8), (F32, 20, 16), (F32, 4, 0)])
def test_sixteen_byte_rows_accepted(lib, dt, D, R):
    # D * elem_bytes a multiple of 16 is enough: an odd vector count per row
    # runs the plain-load kernels (empty problems launch nothing; the plan
    # query makes no CUDA call)
    assert fwd(lib, B=0, D=D, R=R, dt=dt) == OK
    assert bwd(lib, B=0, D=D, R=R, dt=dt, dgq=None, dgk=None) == OK
    plan = (ctypes.c_int64 * 15)()
    for kind in range(4):
        assert lib.qk_norm_rope_plan(kind, 2, 8, 4, 2, D, R, dt, 0, 148, 0,
                                     ctypes.cast(plan, ctypes.c_void_p)) == OK
        assert plan[0] == 0 and plan[13] == 256
    assert lib.qk_layerwise_stats(P(1), P(2), P(7), P(8), 0, 8, 4, 2, D, dt, None) == OK


@pytest.mark.parametrize("dt,D", [(BF16, 4), (BF16, 12), (F32, 2), (F32, 6)])
def test_rows_not_whole_vectors_rejected(lib, dt, D):
    assert fwd(lib, D=D, R=0, dt=dt) == UNSUP
    assert bwd(lib, D=D, R=0, dt=dt) == UNSUP


@pytest.mark.parametrize("call", [fwd, bwd], ids=["fwd", "bwd"])
def test_null_and_alignment(lib, call):
    assert call(lib, q=None) == INVALID
    assert call(lib, k=None) == INVALID
    assert call(lib, gq=None) == INVALID
    assert call(lib, rq=None) == INVALID
    assert call(lib, q=P(1, 8)) == ALIGN          # vectors need 16 bytes
    assert call(lib, gk=P(4, 4)) == ALIGN
    assert call(lib, rk=P(8, 2)) == ALIGN         # fp32 arrays need 4 bytes
    assert call(lib, pos=P(15, 1)) == ALIGN


def test_fwd_overlap_rules(lib):
    # B*S*Hq*D*2 bytes = 2*8*4*64*2 = 8 KiB per q tensor
    assert fwd(lib, qo=P(1, 4096)) == INVALID          # partial overlap with q
    assert fwd(lib, ko=P(5)) == INVALID                # k_out on top of q_out
    assert fwd(lib, rq=P(5, 64)) == INVALID            # rstd inside q_out
    assert fwd(lib, qo=P(2), ko=P(1)) == INVALID       # outputs swapped onto inputs


def test_bwd_overlap_rules(lib):
    assert bwd(lib, dq=P(9, 16)) == INVALID            # partial overlap with dq_out
    assert bwd(lib, dgq=P(11, 32)) == INVALID          # dgamma inside dq
    assert bwd(lib, dgq=P(13), dgk=P(13)) == INVALID   # both dgammas on one buffer
    assert bwd(lib, dq=P(1)) == INVALID                # dq on top of q


def test_zero_heads_allow_null_pointers(lib):
    # Hkv = 0: K pointers may be NULL, but an invalid D still fails first
    assert fwd(lib, Hkv=0, k=None, gk=None, ko=None, rk=None, D=63) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 2, 1, 16)
    with pytest.raises(ValueError):
        qknr.qk_norm_rope_fwd(q, q, q[0, 0, 0], q[0, 0, 0], rotary_dim=16, theta=1e4, eps=1e-6)


def fwd_strided(lib, qts, kts, B=2, S=8, Hq=4, Hkv=2, D=64, R=64, dt=BF16, **ptrs):
    p = dict(q=P(1), k=P(2), gq=P(3), gk=P(4), pos=None, qo=P(5), ko=P(6), rq=P(7), rk=P(8))
    p.update(ptrs)
    return lib.qk_norm_rope_fwd_strided(p["q"], p["k"], qts, kts, p["gq"], p["gk"], p["pos"],
                                        p["qo"], p["ko"], p["rq"], p["rk"], B, S, Hq, Hkv, D, R,
                                        1e4, 1e-6, dt, None)


def bwd_strided(lib, qts, kts, dqts, dkts, B=2, S=8, Hq=4, Hkv=2, D=64, R=64, dt=BF16, **ptrs):
    p = dict(q=P(1), k=P(2), gq=P(3), gk=P(4), pos=None, rq=P(7), rk=P(8), dqo=P(9),
             dko=P(10), dq=P(11), dk=P(12), dgq=P(13), dgk=P(14))
    p.update(ptrs)
    return lib.qk_norm_rope_bwd_strided(p["q"], p["k"], qts, kts, p["gq"], p["gk"], p["pos"],
                                        p["rq"], p["rk"], p["dqo"], p["dko"], p["dq"], p["dk"],
                                        dqts, dkts, p["dgq"], p["dgk"], B, S, Hq, Hkv, D, R,
                                        1e4, 1e-6, dt, None)


def test_strided_validation(lib):
    ts = (4 + 2 * 2) * 64                       # a fused QKV row: Hq + 2 Hkv heads
    assert fwd_strided(lib, 4 * 64 - 8, ts) == INVALID       # token step shorter than its rows
    assert fwd_strided(lib, ts, 2 * 64 - 1) == INVALID
    assert fwd_strided(lib, ts + 4, ts) == ALIGN              # 8-byte step (bf16)
    assert fwd_strided(lib, ts, ts, dt=F32, D=64, R=64, q=P(1, 8)) == ALIGN
    assert fwd_strided(lib, ts, ts, D=63) == INVALID          # shape checks still apply
    # q_out over a strided q's bytes (fwd outputs are dense)
    assert fwd_strided(lib, ts, ts, qo=P(1, 64)) == INVALID
    assert bwd_strided(lib, ts, ts, ts, 2 * 64 - 2) == INVALID      # dk step < Hkv * D
    assert bwd_strided(lib, ts, ts, ts + 4, ts) == ALIGN
    # strided dq and dk whose rows overlap (dk 64 bytes into dq's rows)
    assert bwd_strided(lib, ts, ts, ts, ts, dk=P(11, 64)) == INVALID
    # dq on top of the strided q
    assert bwd_strided(lib, ts, ts, ts, ts, dq=P(1)) == INVALID
    # a strided dq may not alias dq_out
    assert bwd_strided(lib, ts, ts, ts, ts, dq=P(9)) == INVALID


def test_nope_and_rope_only_validation(lib):
    # qk_norm_fwd(q, k, gq, gk, qo, ko, rq, rk, B, S, Hq, Hkv, D, eps, dtype, stream)
    def norm_fwd(D=64, eps=1e-6, q=P(1), rq=P(7)):
        return lib.qk_norm_fwd(q, P(2), P(3), P(4), P(5), P(6), rq, P(8), 2, 8, 4, 2, D, eps,
                               BF16, None)

    assert norm_fwd(D=63) == INVALID
    assert norm_fwd(eps=-1.0) == INVALID
    assert norm_fwd(q=None) == INVALID
    assert norm_fwd(rq=None) == INVALID              # the norm saves rstd
    assert norm_fwd(q=P(1, 8)) == ALIGN
    assert lib.qk_norm_bwd(P(1), P(2), P(3), P(4), P(7), P(8), P(9), P(10), P(9, 16), P(12),
                           P(13), P(14), 2, 8, 4, 2, 64, 1e-6, BF16, None) == INVALID

    # qk_rope_apply(q, k, pos, qo, ko, B, S, Hq, Hkv, D, R, theta, inverse, dtype, stream)
    def rope(D=64, R=64, theta=1e4, q=P(1), qo=P(5), pos=None):
        return lib.qk_rope_apply(q, P(2), pos, qo, P(6), 2, 8, 4, 2, D, R, theta, 1, BF16, None)

    assert rope(D=63) == INVALID
    assert rope(R=66) == INVALID
    assert rope(theta=0.0) == INVALID
    assert rope(D=64, R=8) == UNSUP
    assert rope(q=None) == INVALID
    assert rope(qo=None) == INVALID
    assert rope(qo=P(1, 4096)) == INVALID            # partial overlap with q
    assert rope(q=P(1, 8)) == ALIGN
    assert rope(pos=P(15, 2)) == ALIGN


def test_rms_stats_validation(lib):
    def stats(D=64, eps=1e-6, q=P(1), rq=P(7), rk=P(8)):
        return lib.qk_rms_stats(q, P(2), rq, rk, 2, 8, 4, 2, D, eps, BF16, None)

    assert stats(D=63) == INVALID
    assert stats(eps=float("nan")) == INVALID
    assert stats(q=None) == INVALID
    assert stats(rq=None) == INVALID
    assert stats(rq=P(7, 2)) == ALIGN
    assert stats(rk=P(7, 64)) == INVALID             # the two statistics overlap


def test_layernorm_entries_validate_like_rmsnorm(lib):
    def ln_fwd(D=64, R=64, eps=1e-6, q=P(1)):
        return lib.qk_layernorm_rope_fwd(q, P(2), P(3), P(4), None, P(5), P(6), P(7), P(8),
                                         2, 8, 4, 2, D, R, 1e4, eps, BF16, None)

    assert ln_fwd(D=63) == INVALID
    assert ln_fwd(R=8) == UNSUP
    assert ln_fwd(eps=-1.0) == INVALID
    assert ln_fwd(q=None) == INVALID
    assert ln_fwd(q=P(1, 8)) == ALIGN
    assert lib.qk_layernorm_rope_bwd(P(1), P(2), P(3), P(4), None, P(7), P(8), P(9), P(10),
                                     P(9, 16), P(12), P(13), P(14), 2, 8, 4, 2, 64, 64, 1e4,
                                     1e-6, BF16, None) == INVALID


def test_layerwise_validation(lib):
    def stats(D=64, q=P(1), sq=P(7), sk=P(8), Hq=4):
        return lib.qk_layerwise_stats(q, P(2), sq, sk, 2, 8, Hq, 2, D, BF16, None)

    assert stats(D=63) == INVALID
    assert stats(D=512) == UNSUP
    assert stats(q=None) == INVALID
    assert stats(sq=P(7, 2)) == ALIGN
    assert stats(sk=P(7, 32)) == INVALID            # the two sums overlap
    assert stats(sq=P(1, 64)) == INVALID            # a sum written over q

    def fwd(Hq_total=8, Hkv_total=4, qo=P(5), rq=P(9), eps=1e-6, R=64):
        return lib.qk_layerwise_norm_rope_fwd(P(1), P(2), P(3), P(4), None, P(7), P(8), qo,
                                              P(6), rq, P(10), 2, 8, 4, 2, Hq_total, Hkv_total,
                                              64, R, 1e4, eps, BF16, None)

    assert fwd(Hq_total=3) == INVALID               # total below the local head count
    assert fwd(Hkv_total=1) == INVALID
    assert fwd(eps=-1.0) == INVALID
    assert fwd(R=8) == UNSUP
    assert fwd(qo=P(5, 8)) == ALIGN
    assert fwd(qo=P(1, 256)) == INVALID             # q_out partly over q
    assert fwd(rq=P(7)) == INVALID                  # rstd written over the sums
    assert fwd(rq=None) == INVALID
    # no sums: only a rank holding every head may take the statistic itself
    assert lib.qk_layerwise_norm_rope_fwd(P(1), P(2), P(3), P(4), None, None, None, P(5), P(6),
                                          P(9), P(10), 2, 8, 4, 2, 8, 2, 64, 64, 1e4, 1e-6,
                                          BF16, None) == INVALID

    def dots(dq=P(11)):
        return lib.qk_layerwise_bwd_dots(P(1), P(2), P(3), P(4), None, P(7), P(8), dq, P(12),
                                         P(13), P(14), 2, 8, 4, 2, 64, 64, 1e4, BF16, None)

    assert dots(dq=None) == INVALID
    assert dots(dq=P(13)) == INVALID                # upstream gradient under dot_q

    def bwd(Hq=4, dgq=P(17), dq=P(15)):
        return lib.qk_layerwise_norm_rope_bwd(P(1), P(2), P(3), P(4), None, P(7), P(8), P(11),
                                              P(12), P(13), P(14), dq, P(16), dgq, P(18), 2, 8,
                                              Hq, 2, 512, 2, 128, 128, 1e4, BF16, None)

    assert bwd(Hq=511) == UNSUP                     # dgamma partials exceed shared memory
    assert bwd(dq=P(11, 16)) == INVALID             # dq partly over dq_out
    assert bwd(dgq=P(17, 2)) == ALIGN
    assert bwd(dq=None) == INVALID
    assert lib.qk_layerwise_norm_rope_bwd(P(1), P(2), P(3), P(4), None, P(7), P(8), P(11),
                                          P(12), None, None, P(15), P(16), P(17), P(18), 2, 8,
                                          4, 2, 4, 4, 128, 128, 1e4, BF16, None) == INVALID


def test_wait_selftest_validation(lib):
    # bad family or limit: refused before any CUDA call
    assert lib.qknr_wait_selftest(2, 1000, None) == INVALID
    assert lib.qknr_wait_selftest(0, 0, None) == INVALID
    assert lib.qknr_wait_selftest(1, 1 << 40, None) == INVALID


def test_plan_query_validation(lib):
    plan = (ctypes.c_int64 * 15)()
    pp = ctypes.cast(plan, ctypes.c_void_p)
    assert lib.qk_norm_rope_plan(4, 2, 8, 4, 2, 64, 64, BF16, 0, 148, 0, pp) == INVALID
    assert lib.qk_norm_rope_plan(0, 2, 8, 4, 2, 64, 64, BF16, 4, 148, 0, pp) == INVALID
    assert lib.qk_norm_rope_plan(0, 2, 8, 4, 2, 64, 64, BF16, 0, 0, 0, pp) == INVALID
    assert lib.qk_norm_rope_plan(0, 2, 8, 4, 2, 64, 64, BF16, 0, 148, 0, None) == INVALID
    assert lib.qk_norm_rope_plan(0, 2, 8, 4, 2, 63, 0, BF16, 0, 148, 0, pp) == INVALID
    assert lib.qk_norm_rope_plan(1, 2, 8, 4, 2, 64, 8, BF16, 0, 148, 0, pp) == UNSUP
    # the bench shapes: pipelined, one CTA per SM at most
    assert lib.qk_norm_rope_plan(1, 1, 65536, 32, 8, 128, 32, BF16, 0, 148, 0, pp) == OK
    assert plan[0] == 1 and plan[11] == 148 and plan[13] == (plan[3] + plan[4]) * 32
    assert plan[14] == plan[7]  # the backward runs whole tiles
    # the forward starts each CTA on half a tile, unless tensor copies
    # (strided inputs) move whole boxes
    assert lib.qk_norm_rope_plan(0, 1, 65536, 32, 8, 128, 32, BF16, 0, 148, 0, pp) == OK
    assert plan[0] == 1 and plan[14] == plan[7] // 2 and plan[7] >= 2
    assert lib.qk_norm_rope_plan(0, 1, 65536, 32, 8, 128, 32, BF16, 3, 148, 0, pp) == OK
    assert plan[6] == 3 and plan[14] == plan[7]


def test_layerwise_bwd_acc_validation(lib):
    # the accumulating backward checks its arguments exactly like the backward
    def bwd(fn, Hq=4, dgq=P(17), dq=P(15)):
        return fn(P(1), P(2), P(3), P(4), None, P(7), P(8), P(11), P(12), P(13), P(14), dq,
                  P(16), dgq, P(18), 2, 8, Hq, 2, 512, 2, 128, 128, 1e4, BF16, None)

    for fn in (lib.qk_layerwise_norm_rope_bwd, lib.qk_layerwise_norm_rope_bwd_acc):
        assert bwd(fn, Hq=511) == UNSUP
        assert bwd(fn, dq=P(11, 16)) == INVALID
        assert bwd(fn, dgq=P(17, 2)) == ALIGN
        assert bwd(fn, dq=None) == INVALID
