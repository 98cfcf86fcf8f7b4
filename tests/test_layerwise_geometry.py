"""Host-side replay of the layerwise pipelined kernels' launch geometry.

`qk_layerwise_geometry` returns the plan the backward and dots launches use
(no CUDA call). For many shapes this test replays, in plain Python, the
kernels' assignment of work — CTA token runs, stages of TT tokens, consumer
warp (token group, head-block set), lane (row slot, unit) — and checks that
every (token, head row, unit) is processed exactly once, that every stage
section, copy and table stays inside its shared-memory region, and that the
shared memory fits the SM. No GPU is needed.
"""
import random

import pytest
import torch

import qk_rmsnorm_rope_norm_b200 as qknr
from qk_rmsnorm_rope_norm_b200 import build as qbuild

# dynamic shared memory a CTA may take beside the kernel's static tables
# (a 64-bit angle step per rotary pair, 128 of them, and 32 int32 positions)
SMEM_LIMIT = 227 * 1024 - (128 * 8 + 32 * 4)
MAX_CONSUMER_WARPS = 15
MAX_BLOCKS_PER_WARP = 2
TX_LIMIT = (1 << 20) - 1  # bytes one mbarrier phase may count


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qknr.load_library()


def ceil_div(a, b):
    return -(-a // b)


def replay(mode, B, S, Hq, Hkv, D, R, dtype, sms=148):
    """Checks the plan for one shape; returns it (or None for the plain-load
    kernels)."""
    g = qknr.layerwise_geometry(mode, B, S, Hq, Hkv, D, R, dtype, sms)
    if not g["pipelined"]:
        return None
    e = 4 if dtype == torch.float32 else 2
    V = 16 // e
    Dv2 = D // (2 * V)
    rowb = D * e
    H = Hq + Hkv
    T = B * S
    lpr, TT, NS, stage = g["lpr"], g["TT"], g["NS"], g["stage_bytes"]
    G, NTG, HB = g["G"], g["NTG"], g["HB"]
    assert g["first_tile"] == TT  # the head-block pipeline runs whole tiles
    slots = 32 // lpr
    # lane layout and warp split
    assert lpr & (lpr - 1) == 0 and lpr >= Dv2 and (lpr == 1 or lpr // 2 < Dv2)
    assert HB == ceil_div(H, slots)
    assert G * NTG <= MAX_CONSUMER_WARPS and g["threads"] == (G * NTG + 1) * 32
    assert ceil_div(HB, G) <= MAX_BLOCKS_PER_WARP
    assert 1 <= TT <= 32 and TT % NTG == 0
    # stage sections: Q rows, K rows, dQ_out rows, dK_out rows, angles, scalars
    assert g["off_k"] == TT * Hq * rowb
    assert g["off_dq"] == TT * H * rowb
    assert g["off_dk"] == TT * (2 * Hq + Hkv) * rowb
    assert g["off_cs"] == 2 * TT * H * rowb
    assert g["off_sc"] == g["off_cs"] + TT * (R // 2) * 8
    assert g["off_pos"] == g["off_sc"] + 16 * TT
    assert g["off_pos"] + 4 * TT <= stage and stage % 128 == 0
    for k in ("off_k", "off_dq", "off_dk", "off_cs", "off_sc", "off_pos"):
        assert g[k] % 16 == 0, k
    # who fills the (cos, sin) tables: the consumer warps for few rows a
    # token, and only when a warp owns one head block (the kernel instance
    # that carries the fill)
    narrow = R > 0 and H * rowb < 32 * R
    assert g["cs_by_consumers"] == int(narrow and ceil_div(HB, G) == 1), g
    assert 2 * TT * H * rowb <= TX_LIMIT
    # ring, partial-sum table, gamma table
    assert NS >= 2 and g["off_parts"] == 128 + NS * stage
    assert g["off_gamma"] >= g["off_parts"] + NS * TT * G * 8 and g["off_gamma"] % 128 == 0
    assert g["smem"] >= g["off_gamma"] + H * rowb and g["smem"] <= SMEM_LIMIT
    assert NS * stage >= H * D * 4  # the backward's dgamma sums reuse the ring
    # CTA runs
    grid, tpc = g["grid"], g["tpc"]
    assert 1 <= grid <= sms and (grid - 1) * tpc < T <= grid * tpc
    # every (token, head row, unit) exactly once
    seen = set()
    for cta in range(grid):
        t_lo, t_hi = cta * tpc, min(T, (cta + 1) * tpc)
        for i in range(ceil_div(t_hi - t_lo, TT)):
            t0 = t_lo + i * TT
            na = min(TT, t_hi - t0)
            assert 1 <= na <= TT and t0 + na <= T
            for w in range(G * NTG):
                tg, wb = divmod(w, G)
                for j in range(tg, na, NTG):
                    for nb in range(MAX_BLOCKS_PER_WARP):
                        b = wb + nb * G
                        if b >= HB:
                            break
                        for lane in range(32):
                            slot, u = divmod(lane, lpr)
                            h = b * slots + slot
                            if u >= Dv2 or h >= H:
                                continue
                            key = (t0 + j, h, u)
                            assert key not in seen, key
                            seen.add(key)
    assert len(seen) == T * H * Dv2
    return g


SHAPES = [
    # B, S, Hq, Hkv, D, R, dtype
    (2, 129, 14, 2, 64, 64, torch.bfloat16),    # Qwen2.5-0.5B heads
    (1, 97, 32, 8, 128, 128, torch.bfloat16),   # Llama-3-8B heads
    (1, 300, 32, 8, 128, 32, torch.bfloat16),   # partial rotary
    (3, 37, 5, 3, 24, 16, torch.float32),
    (1, 32, 4, 2, 16, 16, torch.float32),
    (2, 41, 4, 0, 64, 64, torch.bfloat16),
    (2, 41, 0, 4, 64, 64, torch.bfloat16),
    (2, 41, 33, 1, 64, 64, torch.bfloat16),
    (1, 7, 64, 8, 128, 128, torch.bfloat16),
    (1, 1, 8, 2, 128, 0, torch.bfloat16),
    (5, 3, 1, 1, 256, 256, torch.bfloat16),
    (1, 4099, 6, 2, 128, 128, torch.bfloat16),
]


@pytest.mark.parametrize("mode", ["dots", "bwd"])
@pytest.mark.parametrize("shape", SHAPES, ids=[f"{s[2]}x{s[3]}x{s[4]}-R{s[5]}-T{s[0] * s[1]}"
                                               for s in SHAPES])
def test_plan_of_listed_shapes(lib, mode, shape):
    B, S, Hq, Hkv, D, R, dt = shape
    replay(mode, B, S, Hq, Hkv, D, R, dt)


def test_plan_of_random_shapes(lib):
    rng = random.Random(7)
    planned = 0
    for _ in range(60):
        dt = rng.choice([torch.bfloat16, torch.float32])
        e = 4 if dt == torch.float32 else 2
        D = rng.choice([d for d in (16, 24, 32, 48, 64, 96, 128, 192, 256) if d * e % 32 == 0])
        R = rng.choice([r for r in range(0, D + 1, 2) if (r // 2) * e % 16 == 0])
        Hq, Hkv = rng.randint(0, 40), rng.randint(0, 9)
        if Hq + Hkv == 0 or (Hq + Hkv) * D * 4 > 200 * 1024:
            continue
        B, S = rng.randint(1, 3), rng.randint(1, 90)
        sms = rng.choice([148, 132, 7])
        for mode in ("dots", "bwd"):
            planned += replay(mode, B, S, Hq, Hkv, D, R, dt, sms) is not None
    assert planned > 40


def test_bench_shapes_use_every_sm(lib):
    # the tokens are split evenly, so the bench shapes keep all 148 SMs busy
    for shape in ((8, 2048, 14, 2, 64, 64), (4, 8192, 32, 8, 128, 128)):
        g = qknr.layerwise_geometry("bwd", *shape, torch.bfloat16, 148)
        assert g["pipelined"] and g["grid"] == 148


def test_geometry_rejects_bad_arguments(lib):
    with pytest.raises(qknr.QKNRError):
        qknr.layerwise_geometry("bwd", 1, 8, 4, 2, 63, 0)       # odd head size
    with pytest.raises(qknr.QKNRError):
        qknr.layerwise_geometry("bwd", 1, 8, 400, 8, 256, 256)  # dgamma sums too large
    with pytest.raises(qknr.QKNRError):
        qknr.layerwise_geometry("bwd", 1, 8, 4, 2, 64, 64, sms=0)
    g = qknr.layerwise_geometry("bwd", 1, 9, 64, 8, 256, 128, torch.float32)
    assert g["pipelined"] == 0  # too large for the ring: the plain-load kernels


def replay_tok(B, S, Hq, Hkv, D, R, dtype, sms=148):
    """The statistics / forward pipeline: CTA token runs, stages of TT
    tokens, whole tokens dealt round-robin to the consumer warps (continuing
    across stages), every row of a token covered by the warp's lanes, the
    producer's (cos, sin) work split, and the shared-memory sections."""
    g = qknr.layerwise_geometry("tok", B, S, Hq, Hkv, D, R, dtype, sms)
    if not g["pipelined"]:
        return None
    e = 4 if dtype == torch.float32 else 2
    V = 16 // e
    Dv2 = D // (2 * V)
    rowb = D * e
    H = Hq + Hkv
    T = B * S
    lpr, TT, NS, stage, ncw = g["lpr"], g["TT"], g["NS"], g["stage_bytes"], g["NTG"]
    slots = 32 // lpr
    assert g["G"] == 1 and ncw <= MAX_CONSUMER_WARPS and g["threads"] == (ncw + 1) * 32
    assert 1 <= TT <= 32
    assert g["off_k"] == TT * Hq * rowb and g["off_cs"] == TT * H * rowb
    assert g["off_sc"] == g["off_cs"] + TT * (R // 2) * 8
    assert g["off_pos"] == g["off_sc"] + 8 * TT
    assert g["off_pos"] + 4 * TT <= stage and stage % 128 == 0
    for k in ("off_k", "off_cs", "off_sc"):
        assert g[k] % 16 == 0, k
    assert g["off_pos"] % 4 == 0
    # the consumer warps fill their tokens' (cos, sin) tables for few rows
    # a token, the producer warp otherwise
    assert g["cs_by_consumers"] == int(R > 0 and H * rowb < 32 * R), g
    assert TT * H * rowb <= TX_LIMIT
    assert NS >= 2 and g["off_gamma"] == 128 + NS * stage
    assert g["smem"] >= g["off_gamma"] + H * rowb and g["smem"] <= SMEM_LIMIT
    # the producer's (cos, sin) table: every (token, angle pair) exactly once,
    # inside the token's hp float4 entries
    hp = R // 4
    if hp:
        tpp = 32 // hp if hp <= 32 else 0
        for na in {TT, max(1, TT - 1), 1}:
            cells = set()
            for lane in range(32):
                if tpp:
                    if lane >= tpp * hp:
                        continue
                    jo, P = divmod(lane, hp)
                    pairs, toks = [P], range(jo, na, tpp)
                else:
                    pairs, toks = range(lane, hp, 32), range(na)
                for P in pairs:
                    pw = P // (V // 2)
                    dst = (P - pw * (V // 2)) * (hp // (V // 2)) + pw
                    assert 0 <= dst < hp
                    for j in toks:
                        assert (j, dst) not in cells
                        cells.add((j, dst))
            assert len(cells) == na * hp
    # CTA runs, stages, token dealing, rows of a token
    grid, tpc = g["grid"], g["tpc"]
    assert 1 <= grid <= sms and (grid - 1) * tpc < T <= grid * tpc
    seen = set()
    # each CTA's first tile holds half a tile (whole when TT == 1), later
    # tiles TT, the last what remains; a run of at most TT is one tile
    h0 = g["first_tile"]
    assert h0 == (TT // 2 if TT >= 2 else TT)
    for cta in range(grid):
        t_lo, t_hi = cta * tpc, min(T, (cta + 1) * tpc)
        h = h0 if t_hi - t_lo > TT else TT
        starts = [t_lo] + list(range(t_lo + h, t_hi, TT)) if t_hi - t_lo > h else [t_lo]
        pc = 0
        for i, t0 in enumerate(starts):
            na = min(h if i == 0 else TT, t_hi - t0)
            assert 1 <= na <= TT and t0 + na <= T
            for w in range(ncw):
                j = (w - pc) % ncw
                for jj in range(j, na, ncw):
                    for p in range(0, H, slots):
                        for lane in range(32):
                            slot, u = divmod(lane, lpr)
                            h = p + slot
                            if u >= Dv2 or h >= H:
                                continue
                            key = (t0 + jj, h, u)
                            assert key not in seen, key
                            seen.add(key)
            pc = (pc + na) % ncw
    assert len(seen) == T * H * Dv2
    return g


@pytest.mark.parametrize("shape", SHAPES, ids=[f"{s[2]}x{s[3]}x{s[4]}-R{s[5]}-T{s[0] * s[1]}"
                                               for s in SHAPES])
def test_token_plan_of_listed_shapes(lib, shape):
    assert replay_tok(*shape) is not None


def test_token_plan_of_random_shapes(lib):
    rng = random.Random(11)
    planned = 0
    for _ in range(60):
        dt = rng.choice([torch.bfloat16, torch.float32])
        e = 4 if dt == torch.float32 else 2
        D = rng.choice([d for d in (16, 24, 32, 48, 64, 96, 128, 192, 256) if d * e % 32 == 0])
        R = rng.choice([r for r in range(0, D + 1, 2) if (r // 2) * e % 16 == 0])
        Hq, Hkv = rng.randint(0, 40), rng.randint(0, 9)
        if Hq + Hkv == 0:
            continue
        B, S = rng.randint(1, 3), rng.randint(1, 90)
        planned += replay_tok(B, S, Hq, Hkv, D, R, dt, rng.choice([148, 132, 7])) is not None
    assert planned > 40


def test_token_plan_of_bench_shapes(lib):
    # the bench shapes take the token pipeline and keep every SM busy
    for shape in ((8, 2048, 14, 2, 64, 64), (4, 8192, 32, 8, 128, 128),
                  (1, 65536, 32, 8, 128, 32)):
        g = qknr.layerwise_geometry("tok", *shape, torch.bfloat16, 148)
        assert g["pipelined"] and g["grid"] == 148
    # an odd number of 16-byte vectors per row runs the plain-load kernels
    assert not qknr.layerwise_geometry("tok", 1, 64, 4, 2, 72, 64, torch.bfloat16)["pipelined"]
