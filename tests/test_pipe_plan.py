"""Launch plans of the per-head pipelined kernels (``qk_norm_rope_plan``),
checked on the CPU for many shapes: what the kernels rely on must hold for
every plan the library hands them.

* A stage holds TT tokens of every section the kernel copies or writes into
  it (Q and K rows; backward: dQ_out and dK_out rows and the rstd blocks;
  the (cos, sin) table of R/2 angle pairs a token), and the ring of NS
  stages fits the shared memory an SM gives one block.
* The CTAs' token runs cover the T tokens exactly once; each run is cut
  into a first tile of ``first_tile`` tokens, then tiles of TT, the last
  one what remains, every tile inside the run and at most TT tokens.
* Backward: every tile starts its Q and K rstd blocks on a 16-byte boundary
  (the blocks arrive by bulk copy).
* The forward starts each CTA on half a tile unless its inputs are strided
  (tensor copies move whole boxes); the backward runs whole tiles.
"""
import ctypes
import random

import pytest
import torch

import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

SMEM_OPTIN = 232448   # B200: 227 KB of shared memory per block, opt-in
STATIC_RESERVE = 8192  # barriers, angle steps, gamma and dgamma tables


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qknr.load_library()


def tiles(t_lo, t_hi, TT, first):
    """The tile schedule a CTA runs over [t_lo, t_hi)."""
    n = t_hi - t_lo
    if n <= 0:
        return []
    h = first if n > TT else TT
    out = [(t_lo, min(h, n))]
    t = t_lo + h
    while t < t_hi:
        out.append((t, min(TT, t_hi - t)))
        t += TT
    return out


def check_plan(kind, B, S, Hq, Hkv, D, R, dtype, strided=0, sms=148):
    p = qknr.launch_plan(kind, B, S, Hq, Hkv, D, R, dtype, strided, sms)
    if not p["pipelined"]:
        return None
    e = 4 if dtype == torch.float32 else 2
    bwd = kind.endswith("bwd")
    T = B * S
    TT, NS, stage, tpc, grid = p["TT"], p["NS"], p["stage_bytes"], p["tpc"], p["grid"]
    rowb = D * e
    # sections of a stage, each rounded up to 128 bytes
    up = lambda x: (x + 127) // 128 * 128
    need = up(TT * Hq * rowb) + up(TT * Hkv * rowb)
    if bwd:
        need += up(TT * Hq * rowb) + up(TT * Hkv * rowb)
    need += up(TT * (R // 2) * 8)
    if bwd:
        need += up(TT * Hq * 4) + up(TT * Hkv * 4)
    assert 1 <= TT <= 32 and stage % 128 == 0 and stage >= need, (p, need)
    assert NS >= 2 and p["smem"] == NS * stage and p["smem"] + STATIC_RESERVE <= SMEM_OPTIN
    assert p["threads"] == (p["consumer_warps"] + p["producer_warps"]) * 32 <= 1024
    # token runs and tiles
    assert 1 <= grid <= sms and (grid - 1) * tpc < T <= grid * tpc, p
    first = p["first_tile"]
    if bwd or (p["tmap"] != 0):
        assert first == TT
    else:
        assert first == (TT // 2 if TT >= 2 else TT)
    covered = 0
    for c in range(grid):
        t_lo, t_hi = c * tpc, min(T, (c + 1) * tpc)
        prev = t_lo
        for t0, na in tiles(t_lo, t_hi, TT, first):
            assert t0 == prev and 1 <= na <= TT and t0 + na <= t_hi
            if bwd:
                assert (t0 * Hq * 4) % 16 == 0 and (t0 * Hkv * 4) % 16 == 0, (t0, p)
            prev = t0 + na
            covered += na
        assert prev == t_hi
    assert covered == T
    return p


SHAPES = [(8, 2048, 14, 2, 64, 64, torch.bfloat16), (4, 8192, 32, 8, 128, 128, torch.bfloat16),
          (1, 65536, 32, 8, 128, 32, torch.bfloat16), (5, 4096, 32, 8, 128, 128, torch.bfloat16),
          (1, 32, 4, 2, 16, 16, torch.float32), (3, 37, 5, 3, 24, 16, torch.float32),
          (2, 4099, 7, 1, 64, 64, torch.bfloat16), (1, 1, 1, 1, 256, 256, torch.bfloat16),
          (1, 1000, 3, 17, 128, 0, torch.bfloat16)]


@pytest.mark.parametrize("kind", ["fwd", "bwd", "ln_fwd", "ln_bwd"])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"{s[2]}x{s[3]}x{s[4]}-R{s[5]}-T{s[0] * s[1]}"
                                               for s in SHAPES])
def test_plan_of_listed_shapes(lib, kind, shape):
    check_plan(kind, *shape)


def test_strided_forward_plans_whole_tiles(lib):
    p = check_plan("fwd", 1, 65536, 32, 8, 128, 32, torch.bfloat16, strided=3)
    assert p is not None and p["tmap"] == 3


def test_plan_of_random_shapes(lib):
    rng = random.Random(23)
    planned = 0
    for _ in range(300):
        dt = rng.choice([torch.bfloat16, torch.float32])
        e = 4 if dt == torch.float32 else 2
        D = rng.choice([d for d in (8, 16, 24, 32, 48, 64, 96, 128, 192, 256) if d * e % 32 == 0])
        R = rng.choice([r for r in range(0, D + 1, 2) if (r // 2) * e % 16 == 0])
        Hq, Hkv = rng.randint(0, 40), rng.randint(0, 9)
        if Hq + Hkv == 0:
            continue
        B, S = rng.randint(1, 4), rng.randint(1, 5000)
        kind = rng.choice(["fwd", "bwd", "ln_fwd", "ln_bwd"])
        planned += check_plan(kind, B, S, Hq, Hkv, D, R, dt, sms=rng.choice([148, 132, 7])) \
            is not None
    assert planned > 200
