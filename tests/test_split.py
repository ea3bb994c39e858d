"""Intra-expert split of one layer over G GPUs (CPU only: the oracle and the
host-side rules of the C ABI).

Part g keeps rows [g*I/G, (g+1)*I/G) of every expert's gate and up
projections and the same columns of its down projection. h_n depends on row n
of gate and up alone and the down product sums over n, so the parts' fp64
sums add up to the whole layer's sum before the bf16 round. The tests pin
that reading of the split (and the slicing in tests/cases.py that the GPU
tests use) against the unsplit oracle, check that a wrong slicing is caught,
and check the library's argument rules without a GPU.
"""
import ctypes

import numpy as np
import pytest

import oracle
from cases import Layer, bits, part_arrays
from mxfp4_weight_streaming_fp8_b200 import moe

INVALID_ARG, UNSUPPORTED = 1, 2  # moe_status codes


def _sum_parts(L, G):
    return sum(L.oracle_part(g, G)["y64"] for g in range(G))


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("shared", [False, True])
def test_parts_add_up_to_the_whole_layer(G, shared):
    L = Layer(256, 128, 16, 4, 3, seed=5, device="cpu", shared=shared)
    whole = L.oracle()
    parts = [L.oracle_part(g, G) for g in range(G)]
    total = sum(p["y64"] for p in parts)
    scale = np.abs(whole["y64"]).max()
    assert scale > 0
    assert np.max(np.abs(total - whole["y64"])) <= 1e-12 * scale
    for p in parts:  # routing is not split: every part sees the same ids
        assert np.array_equal(p["ids"], whole["ids"])
        assert np.array_equal(p["q"], whole["q"])
        assert np.abs(p["y64"]).max() > 0
    # rounding the sum gives the whole layer's bf16 y
    def rnd(y):
        return np.array([[oracle.bf16_round(v) for v in row] for row in y], dtype=np.uint16)
    yb = rnd(total)
    assert np.array_equal(yb, rnd(whole["y64"]))
    if "y_bf16" in whole:
        assert np.array_equal(yb, whole["y_bf16"])


def test_a_wrong_slicing_does_not_add_up():
    """Down columns of part g+1 paired with the gate/up rows of part g (an
    off-by-one-part slicing) must not reproduce the layer."""
    G = 2
    L = Layer(256, 128, 16, 4, 2, seed=6, device="cpu")
    whole = L.oracle()
    xb = bits(L.x)
    ids = whole["ids"]
    per = L.expert_slices(ids)
    Ip = L.I // G
    total = 0.0
    for g in range(G):
        sl = [[None] * L.E for _ in range(4)]
        for e in range(L.E):
            if per[0][e] is None:
                continue
            a = part_arrays(*(per[t][e] for t in range(4)), L.I, g, G)
            b = part_arrays(*(per[t][e] for t in range(4)), L.I, (g + 1) % G, G)
            for t, v in enumerate((a[0], a[1], b[2], b[3])):
                sl[t][e] = v
        total = total + oracle.moe_decode(xb, L.wr, *sl, L.H, Ip, L.E, L.K)["y64"]
    assert np.max(np.abs(total - whole["y64"])) > 1e-3 * np.abs(whole["y64"]).max()


def test_part_arrays_take_whole_scale_blocks():
    w = [np.arange(2 * 128 * 4, dtype=np.uint8).reshape(256, 4), np.arange(256, dtype=np.uint8).reshape(256, 1),
         np.arange(64 * 64, dtype=np.uint16).astype(np.uint8).reshape(64, 64),
         np.arange(64 * 4, dtype=np.uint8).reshape(64, 4)]
    a = part_arrays(*w, 128, 1, 2)
    assert a[0].shape == (128, 4) and a[0][0, 0] == w[0][64, 0] and a[0][64, 0] == w[0][192, 0]
    assert a[2].shape == (64, 32) and a[2][0, 0] == w[2][0, 32]
    assert a[3].shape == (64, 2) and a[3][0, 0] == w[3][0, 2]


def test_split_rules_without_gpu():
    # the plan of part g is the plan of the I/G-wide layer
    st, whole = moe.plan_query(2560, 768, 256, 8, 4)
    st2, part = moe.plan_query(2560, 768, 256, 8, 4, shard=(1, 2))
    assert st == st2 == moe.MOE_OK
    assert whole["tc"]["dkch"] == 6 and part["tc"]["dkch"] == 3
    assert moe.plan_query(2560, 768, 256, 8, 1, shard=(0, 0))[0] == moe.MOE_OK  # 0 parts: the whole layer
    assert moe.plan_query(2560, 768, 256, 8, 1, shard=(0, 24))[0] == moe.MOE_OK  # I/G = 32
    for shard in [(2, 2), (-1, 2), (0, -1), (0, 5), (0, 48), (0, 129)]:
        assert moe.plan_query(2560, 768, 256, 8, 1, shard=shard)[0] == INVALID_ARG, shard
    # the FP8 intermediate's per-token scale spans all of I
    f8 = moe.MOE_FLAG_FP8_INTERMEDIATE
    assert moe.plan_query(2560, 768, 256, 8, 1, flags=f8, shard=(0, 2))[0] == UNSUPPORTED
    assert moe.plan_query(2560, 768, 256, 8, 1, flags=f8, shard=(0, 1))[0] == moe.MOE_OK
    # no context: the static entry has no part
    cfg = moe.moe_config(256, 128, 16, 4, 1, 0, 0, 0, 2)
    z = ctypes.c_void_p(0)
    assert moe.lib().moe_decode_static(ctypes.byref(cfg), *([z] * 6), 0, *([z] * 6)) == UNSUPPORTED


def test_round_bf16_argument_checks_without_gpu():
    L = moe.lib()
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 24)
    assert L.moe_round_bf16(None, b, 4, None) == INVALID_ARG
    assert L.moe_round_bf16(a, None, 4, None) == INVALID_ARG
    assert L.moe_round_bf16(a, b, -1, None) == INVALID_ARG
    assert L.moe_round_bf16(ctypes.c_void_p((1 << 20) + 2), b, 4, None) == INVALID_ARG
    assert L.moe_round_bf16(a, ctypes.c_void_p((1 << 24) + 1), 4, None) == INVALID_ARG
    # overlap: 4 floats at a, 4 bf16 starting 8 bytes into them
    assert L.moe_round_bf16(a, ctypes.c_void_p((1 << 20) + 8), 4, None) == INVALID_ARG
    assert L.moe_round_bf16(a, b, 0, None) == moe.MOE_OK  # nothing to do, no launch


@pytest.mark.parametrize("G,MM,flags", [(2, 1, 0), (2, 4, 0), (2, 32, 0), (3, 4, 0), (6, 32, 0), (4, 1, 0),
                                        (2, 32, moe.MOE_FLAG_SHARED_EXPERT), (2, 4, moe.MOE_FLAG_SPLITK_DOWN)])
def test_a_part_is_planned_as_the_narrow_layer(G, MM, flags):
    """Every part of the Ling layer gets exactly the launch plan of the layer
    of width I/G (the kernels see only the narrow layer)."""
    for g in range(G):
        st, part = moe.plan_query(2560, 768, 256, 8, MM, flags=flags, shard=(g, G))
        st2, narrow = moe.plan_query(2560, 768 // G, 256, 8, MM, flags=flags)
        assert st == st2 and part == narrow
