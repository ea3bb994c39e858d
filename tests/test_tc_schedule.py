"""CPU replay of the tensor-core kernel's schedule against its shared-memory
plan (no GPU): for several layer shapes, token counts, union sizes and pair
distributions, the index arithmetic k_tc uses (gate/up tiles and their TMA
boxes, the scale copies, tensor-memory columns, the down tiles on tensor
cores, the down chunks on CUDA cores) is restated here and every coordinate,
byte range and column is checked against the buffer it lands in. The plan
comes from the library (moe_plan_query), so a plan change that breaks a
bound fails here before any kernel runs."""
import random

import pytest

from mxfp4_weight_streaming_fp8_b200 import moe

SMEM_LIMIT = 232448  # the B200 opt-in per-block limit
G = 148
UNITS_MAX, ACC_COLS, SF_COL, DOWN_PAIRS, DOWN_ROWS = 16, 32, 64, 16, 9

SHAPES = [(2560, 768, 256, 8), (256, 128, 16, 2), (512, 256, 40, 6), (384, 128, 12, 4), (128, 128, 8, 8),
          (1024, 512, 64, 8), (2560, 768, 257, 8), (640, 384, 300, 3),
          (2560, 384, 256, 8), (2560, 384, 257, 8), (2560, 256, 256, 8)]  # the Ling layer's parts (I/2, I/3)


def sw128(r, k, groups):
    """Byte offset of K element k of row r in a K-major 128-byte-swizzled operand."""
    kc, col, rr = k >> 7, k & 127, r & 7
    return kc * groups * 1024 + (r >> 3) * 1024 + rr * 128 + ((((col >> 4) ^ rr) & 7) << 4) + (col & 15)


def random_pairs(rng, E, K, M, shared):
    """Pair counts per union entry for M tokens of K distinct experts each."""
    counts = {}
    for _ in range(M):
        for e in rng.sample(range(E), K):
            counts[e] = counts.get(e, 0) + 1
    parts = [counts[e] for e in sorted(counts)]
    return ([M] if shared else []) + parts


def replay(H, I, E, K, MM, M, parts, shared, down):
    flags = (moe.MOE_FLAG_SHARED_EXPERT if shared else 0) | down
    st, pl = moe.plan_query(H, I, E, K, MM, flags=flags, sm_count=G, smem_limit=SMEM_LIMIT)
    t = pl["tc"]
    if not t["ok"]:
        return False
    assert t["smem"] <= SMEM_LIMIT
    end = t["smem"] - 1024  # the carve-out starts at a 1024-byte aligned base
    Eall, KCH, upe = E + int(shared), H // 128, I // 4
    U, NP = len(parts), sum(parts)
    assert U <= t["max_union"] and NP <= t["max_pairs"]
    ks, tu_max, ns = t["ks"], t["tu_max"], t["ns_gu"]
    assert KCH % ks == 0 and t["slot_gu"] == tu_max * ks * 1024
    # the MMA reads 16 units (128 rows) of the last slot: rows past tu_max
    # must stay inside the carve-out
    assert t["o_ring_gu"] + (ns - 1) * t["slot_gu"] + UNITS_MAX * ks * 1024 <= end
    assert t["nb_max"] >= max(8, M) and t["nb_max"] % 8 == 0 and t["nb_max"] <= ACC_COLS
    assert t["o_bx"] + KCH * (t["nb_max"] // 8) * 1024 <= end
    # tensor memory: two accumulators, two tiles' scale factors, the token scale factors
    assert SF_COL + 8 * KCH + 4 <= t["tmem_cols"] <= 512
    # gate/up tiles (round robin over the CTAs)
    T = U * upe
    rounds = max(1, -(-T // (G * tu_max)))
    tu = -(-T // (G * rounds))
    ntile = -(-T // tu)
    assert tu <= tu_max and ntile <= G * 64  # kTcMaxTiles tiles per CTA
    for tt in range(ntile):
        f0, f1 = tt * tu, min(T, tt * tu + tu)
        f, nrun = f0, 0
        while f < f1:
            u, j = f // upe, f % upe
            n = min(f1 - f, upe - j)
            g0 = f - f0
            nrun += 1
            assert 1 <= n <= UNITS_MAX and g0 + n <= tu_max
            e = Eall - 1  # the largest expert id
            # 5-D box: quads e*I/2 + j .. + n-1 (gate rows 4j.., up rows I+4j..)
            assert e * (I // 2) + j + n - 1 < Eall * (I // 2)
            assert e * 2 * I + I + 4 * (j + n - 1) + 3 < Eall * 2 * I
            # scale copies: 4n rows of H/32 bytes, 16-byte aligned
            assert ((e * 2 * I + 4 * j) * (H // 32)) % 16 == 0 and (4 * n * (H // 32)) % 16 == 0
            assert (4 * tu_max + 4 * g0 + 4 * n) * (H // 32) <= t["sc_bytes"]
            f += n
        assert nrun <= 2  # a tile has at most 16 units and an entry I/4 >= 32
        assert (f1 - f0) * ks * 512 + 8 * (f1 - f0) * (H // 32) < (1 << 20)  # expect_tx bound
    if t["mma_down"]:
        dkch = I // 128
        assert t["dkch"] == dkch and dkch <= KCH and t["bd_bytes"] == dkch * 4096
        assert 128 * (I // 32) <= t["sc_bytes"]
        assert t["o_bd"] % 1024 == 0 and t["o_bd"] + 2 * t["bd_bytes"] <= end
        assert t["o_dtoff"] + (t["max_union"] + 1) * 4 <= end
        RB = H // 128
        for p in parts:
            groups = -(-p // DOWN_PAIRS)
            for g in range(groups):
                npt = min(DOWN_PAIRS, p - DOWN_PAIRS * g)
                nn = 2 * npt  # hi and lo rows (one with the FP8 intermediate)
                N = max(8, -(-nn // 8) * 8)
                assert N <= ACC_COLS
                for n in (0, nn - 1):
                    for k in (0, I - 4):
                        o = sw128(n, k, 4)
                        assert o % 4 == 0 and o + 4 <= t["bd_bytes"]
            for R in (0, RB - 1):
                row0 = (Eall - 1) * H + R * 128
                assert row0 + 128 <= Eall * H
                assert (row0 * (I // 32)) % 16 == 0 and row0 * (I // 32) + 128 * (I // 32) <= Eall * H * (I // 32)
    else:
        # CUDA-core down: each CTA's output rows of every entry, codes then scales
        assert t["ns_d"] >= 1
        for b in (0, G - 1):
            r0, nrd = H * b // G, H * (b + 1) // G - H * b // G
            if nrd == 0:
                continue
            codes = nrd * I // 2
            for e in (0, Eall - 1):
                row = e * H + r0
                sa = row * (I // 32)
                sa0 = sa & ~15
                sn = ((sa + nrd * (I // 32) + 15) & ~15) - sa0
                assert codes + sn <= t["slot_d"]
        assert -(-H // G) == t["rpc_max"]
        assert -(-t["rpc_max"] // DOWN_ROWS) >= 1
    return True


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("down", [moe.MOE_FLAG_TC_DOWN_MMA, moe.MOE_FLAG_TC_DOWN_CUDA])
def test_tensor_core_schedule_stays_in_bounds(shape, down):
    H, I, E, K = shape
    rng = random.Random(hash((shape, down)) & 0xFFFF)
    planned = 0
    for MM in (1, 2, 4, 8, 16, 32):
        for shared in (False, True):
            for trial in range(3):
                M = MM if trial == 0 else rng.randint(1, MM)
                parts = random_pairs(rng, E, K, M, shared)
                planned += replay(H, I, E, K, MM, M, parts, shared, down)
    # I > H (or I > 1024) forbids the tensor-core down; every other shape plans
    if down == moe.MOE_FLAG_TC_DOWN_MMA and I > H:
        assert planned == 0
    else:
        assert planned > 0
