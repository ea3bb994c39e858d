"""The C-ABI library builds, loads and exports every entry point include/moe.h
declares; host-side argument checks work without a GPU."""
import ctypes
import os
import re

import pytest

from mxfp4_weight_streaming_fp8_b200 import build as libbuild
from mxfp4_weight_streaming_fp8_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return moe.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("moe_create", "moe_load_experts", "moe_decode", "moe_sync_status", "moe_query",
                 "moe_destroy", "moe_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in moe.STATUS_NAMES.items():
        assert moe.status_string(code) == name


def test_create_rejects_bad_config_without_gpu(L):
    out = ctypes.c_void_p()
    assert L.moe_create(None, ctypes.byref(out)) == 1
    bad = [moe.moe_config(100, 64, 16, 2, 1, 0, 0),   # H not a multiple of 32
           moe.moe_config(256, 48, 16, 2, 1, 0, 0),   # I not a multiple of 32
           moe.moe_config(256, 64, 16, 17, 1, 0, 0),  # top_k > E
           moe.moe_config(256, 64, 16, 2, 33, 0, 0),  # max_tokens > 32
           moe.moe_config(256, 64, 2000, 2, 1, 0, 0),  # E > 1024
           moe.moe_config(256, 64, 16, 2, 1, 0x200, 0)]  # unknown flag
    for c in bad:
        assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 1
        assert not out.value


def test_null_context_calls(L):
    assert L.moe_decode(None, None, 1, None, None, None, None, None, None, None) == 1
    assert L.moe_sync_status(None, None) == 1
    buf = ctypes.create_string_buffer(64)
    assert L.moe_query(None, buf, 64) == 1
    assert L.moe_debug_set_wait(None, 0, 0) == 1
    L.moe_destroy(None)


@pytest.mark.parametrize("shape", [(256, 64, 16, 2, 1), (96, 32, 5, 3, 3), (160, 96, 12, 4, 7),
                                   (544, 224, 40, 6, 5), (2560, 768, 256, 8, 1), (2560, 768, 256, 8, 4),
                                   (2560, 768, 256, 8, 32), (256, 64, 16, 4, 32), (128, 64, 8, 8, 3),
                                   (32, 32, 1, 1, 1), (4096, 1024, 512, 8, 8)])
def test_persistent_kernel_plan_fits(L, shape):
    """Host-only launch plan (no CUDA call): shared-memory carving fits the
    227 KB opt-in limit, the router rows of a CTA fit their staging area, and
    every ring holds at least two slots big enough for one CTA's slice."""
    st, pl = moe.plan_query(*shape)
    assert st == 0 and pl["ok"], pl
    H, I, E, K, MM = shape
    G = pl["grid"]
    assert G == 148 and pl["smem"] <= 232448
    assert pl["o_ring_d"] - pl["o_ring_gu"] >= pl["router_bytes_per_cta"]
    assert pl["router_bytes_per_cta"] == -(-E // G) * H * 4
    nr, nrd = -(-I // G), -(-H // G)
    assert pl["slot_gu"] >= nr * H + 2 * (nr * H // 32 + 30)
    assert pl["slot_d"] >= nrd * I // 2 + nrd * I // 32 + 30
    assert pl["ns_gu"] >= min(2, min(E, MM * K)) and pl["ns_d"] >= min(2, min(E, MM * K))
    assert pl["o_act"] % 16 == 0 and pl["o_ring_gu"] % 128 == 0 and pl["o_ring_d"] % 128 == 0


def test_shared_expert_flag_without_gpu(L):
    """The shared-expert flag is a persistent-kernel option: with the split
    path it is refused before any CUDA call. Its plan has one more union
    entry and one more pair per token, and still fits."""
    out = ctypes.c_void_p()
    c = moe.moe_config(256, 64, 16, 2, 1, moe.MOE_FLAG_SHARED_EXPERT | moe.MOE_FLAG_SPLIT_KERNELS, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 2 and not out.value
    c = moe.moe_config(256, 64, 16, 2, 1, moe.MOE_FLAG_FP8_INTERMEDIATE | moe.MOE_FLAG_SPLIT_KERNELS, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 2 and not out.value
    # an unknown flag bit is refused as an invalid argument (0x10..0x100 are kernel choices)
    c = moe.moe_config(256, 64, 16, 2, 1, moe.MOE_FLAG_SHARED_EXPERT | moe.MOE_FLAG_PRE_RMSNORM | 0x200, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 1 and not out.value
    for shape in [(2560, 768, 256, 8, 1), (2560, 768, 256, 8, 32), (128, 64, 8, 8, 3), (256, 64, 16, 2, 1)]:
        st0, base = moe.plan_query(*shape)
        st, pl = moe.plan_query(*shape, flags=moe.MOE_FLAG_SHARED_EXPERT)
        assert st == 0 and pl["ok"], pl
        H, I, E, K, MM = shape
        assert pl["ns_gu"] >= min(2, min(E, MM * K) + 1) and pl["ns_d"] >= min(2, min(E, MM * K) + 1)
        # dsm grows by one row block per token
        assert pl["o_dsm"] >= base["o_dsm"]
        assert pl["smem"] <= 232448
        # slot 0 of each ring fills during routing: the router rows, the
        # gathered logits and the staged x start one slot in and still fit
        staged = max(pl["router_bytes_per_cta"], MM * E * 4)
        assert pl["o_ring_d"] - pl["o_ring_gu"] >= pl["slot_gu"] + staged
        if pl["x_staged"]:
            assert MM * H * 2 + pl["slot_d"] <= pl["ns_d"] * pl["slot_d"]


def test_fp8_intermediate_flag_without_gpu(L):
    """The FP8-intermediate option changes no buffer: its plan equals the
    plain one, alone and with a shared expert; the split path refuses it."""
    F8, SH = moe.MOE_FLAG_FP8_INTERMEDIATE, moe.MOE_FLAG_SHARED_EXPERT
    for shape in [(2560, 768, 256, 8, 1), (2560, 768, 256, 8, 32), (512, 1056, 16, 2, 5), (256, 64, 16, 2, 1)]:
        for base_flags in (0, SH):
            st0, base = moe.plan_query(*shape, flags=base_flags)
            st, pl = moe.plan_query(*shape, flags=base_flags | F8)
            assert st == st0 == 0 and pl == base
    out = ctypes.c_void_p()
    c = moe.moe_config(256, 64, 16, 2, 1, F8 | moe.MOE_FLAG_SPLIT_KERNELS, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 2 and not out.value


def test_splitk_flag_rules_without_gpu(L):
    out = ctypes.c_void_p()
    SK = moe.MOE_FLAG_SPLITK_DOWN
    for flags, mt in ((SK | moe.MOE_FLAG_SPLIT_KERNELS, 1), (SK | moe.MOE_FLAG_FP8_INTERMEDIATE, 1), (SK, 5)):
        c = moe.moe_config(256, 64, 16, 2, mt, flags, 0)
        assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 2 and not out.value
    for shape in [(2560, 768, 256, 8, 1), (2560, 768, 256, 8, 4), (256, 64, 16, 2, 1), (128, 64, 8, 8, 3)]:
        for extra in (0, moe.MOE_FLAG_SHARED_EXPERT):
            st, pl = moe.plan_query(*shape, flags=SK | extra)
            assert st == 0 and pl["ok"] and pl["smem"] <= 232448, (shape, pl)


def test_plan_rejects_what_does_not_fit(L):
    st, pl = moe.plan_query(8192, 4096, 1024, 32, 32)
    assert st == 2 and not pl["ok"]


def test_lm_head_entry_points_reject_bad_arguments_without_a_gpu(L):
    """The LM head entry points validate arguments before touching CUDA."""
    import ctypes
    out = ctypes.c_void_p()
    assert L.moe_lm_create(0, 256, 1, 0, ctypes.byref(out)) == 1       # vocab < 1
    assert L.moe_lm_create(1000, 100, 1, 0, ctypes.byref(out)) == 1    # hidden % 64
    assert L.moe_lm_create(1000, 256, 17, 0, ctypes.byref(out)) == 1   # max_tokens > 16
    assert L.moe_lm_create(1000, 256, 1, 0, None) == 1
    assert L.moe_lm_load(None, None) == 1
    assert L.moe_lm_head(None, None, 1, None, None) == 1
    assert L.moe_lm_sync_status(None, None) == 1
    assert L.moe_lm_read_weights(None, None, None, None) == 1
    buf = ctypes.create_string_buffer(64)
    assert L.moe_lm_query(None, buf, 64) == 1
    L.moe_lm_destroy(None)


def _regions(t):
    """(start, end, name) of the tensor-core kernel's shared-memory regions."""
    NP, UMAX = t["max_pairs"], t["max_union"]
    regs = {"ring_gu": (t["o_ring_gu"], max(t["ns_gu"] * t["slot_gu"], t["wr_bytes_max"])),
            "bx": (t["o_bx"], t["bx_bytes"]), "sc": (t["o_sc"], 2 * t["sc_bytes"]),
            "ring_d": (t["o_ring_d"], t["ns_d"] * t["slot_d"]),
            "ids": (t["o_ids"], NP * 4), "w": (t["o_w"], NP * 4), "pm": (t["o_pm"], NP * 4),
            "ppos": (t["o_ppos"], NP * 4), "union": (t["o_union"], UMAX * 4), "poff": (t["o_poff"], (UMAX + 1) * 4)}
    if t["mma_down"]:
        regs.update(bd=(t["o_bd"], 2 * t["bd_bytes"]), dsc=(t["o_dsc"], 4 * 16 * 4),
                    dtoff=(t["o_dtoff"], (UMAX + 1) * 4))
    else:
        regs["dsm"] = (t["o_dsm"], NP * t["rpc_max"] * 4)
    return sorted((o, o + s, n) for n, (o, s) in regs.items() if s > 0)


@pytest.mark.parametrize("MM", [1, 2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("extra", [0, moe.MOE_FLAG_SHARED_EXPERT])
def test_tensor_core_plan_and_kernel_choice(L, MM, extra):
    """The tensor-core kernel's plan at the Ling shape: chosen from
    MOE_TC_MIN_TOKENS tokens on, its down projection on tensor cores from
    MOE_TC_DOWN_MMA_MIN_TOKENS, non-overlapping shared-memory regions inside
    the opt-in limit, a gate/up ring of at least two 16 KB slots when the
    down projection shares it, and the B operand buffers large enough for
    the routing scratch they hold until routing ends."""
    st, pl = moe.plan_query(2560, 768, 256, 8, MM, flags=extra, sm_count=148, smem_limit=232448)
    assert st == 0 and pl["ok"]
    assert pl["variant"] == ("tc" if MM >= moe.MOE_TC_MIN_TOKENS else "fused")
    t = pl["tc"]
    assert t["ok"] and t["smem"] <= 232448
    assert t["mma_down"] == int(MM >= moe.MOE_TC_DOWN_MMA_MIN_TOKENS)
    if t["mma_down"]:
        assert t["tu_max"] == 16 and t["ks"] == 1 and t["slot_gu"] == 16384 and t["ns_gu"] >= 2
        assert t["ns_d"] == 0 and t["dkch"] == 768 // 128 and t["bd_bytes"] == 6 * 4096
        assert t["o_bd"] % 1024 == 0
        if t["o_lg"] == t["o_bd"]:
            assert MM * 256 * 4 + 256 * 4 <= 2 * t["bd_bytes"]
    regs = _regions(t)
    for a, b in zip(regs, regs[1:]):
        assert a[1] <= b[0], (a, b)
    assert regs[-1][1] <= t["smem"] - 1024


def test_tensor_core_down_flags_without_gpu(L):
    out = ctypes.c_void_p()
    both = moe.MOE_FLAG_TC_DOWN_MMA | moe.MOE_FLAG_TC_DOWN_CUDA
    c = moe.moe_config(2560, 768, 256, 8, 4, both, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 1 and not out.value
    c = moe.moe_config(2560, 768, 256, 8, 4, moe.MOE_FLAG_TENSOR_CORES | moe.MOE_FLAG_SPLITK_DOWN, 0)
    assert L.moe_create(ctypes.byref(c), ctypes.byref(out)) == 1 and not out.value
    # forced either way on the plan
    st, pl = moe.plan_query(2560, 768, 256, 8, 1, flags=moe.MOE_FLAG_TC_DOWN_MMA)
    assert st == 0 and pl["tc"]["mma_down"] == 1
    st, pl = moe.plan_query(2560, 768, 256, 8, 32, flags=moe.MOE_FLAG_TC_DOWN_CUDA)
    assert st == 0 and pl["tc"]["mma_down"] == 0 and pl["tc"]["ns_d"] >= 2
    # I > H: a down tile's scale factors would not fit a gate/up tile's
    # tensor-memory columns, so the default keeps the CUDA-core down and a
    # forced tensor-core down has no plan
    st, pl = moe.plan_query(512, 768, 64, 8, 8)
    assert pl["tc"]["ok"] and pl["tc"]["mma_down"] == 0
    st, pl = moe.plan_query(512, 768, 64, 8, 8, flags=moe.MOE_FLAG_TC_DOWN_MMA)
    assert not pl["tc"]["ok"]
