"""The intra-expert split on one GPU, through the C ABI.

Each part (a context created with shard=(g, G)) is compared with the oracle
of that part: the layer of width I/G made of every expert's gate/up rows
[g*I/G, (g+1)*I/G) and the same down columns, whose fp64 sum the part's fp32
output must match within the per-token bound. Then the parts' outputs,
added in fp32 (what the all-reduce between GPUs computes) and rounded with
moe_round_bf16, are compared with the whole layer's oracle. The parts run one
after another on the same GPU; no part waits on another.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from cases import Layer, compare
from mxfp4_weight_streaming_fp8_b200 import moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from mxfp4_weight_streaming_fp8_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _run_parts(L, G, flags=0, max_tokens=None, variant=None):
    if L.shared:
        flags |= moe.MOE_FLAG_SHARED_EXPERT
    parts = []
    for g in range(G):
        ctx = moe.MoELayer(L.H, L.I, L.E, L.K, max_tokens or max(1, L.M), flags=flags, shard=(g, G))
        q = ctx.query()
        assert q["shard"] == [g, G] and q["inter"] == L.I // G and q["inter_full"] == L.I and q["y"] == "f32", q
        if variant is not None:
            assert q["variant"] == variant, q
        ctx.load_experts(L.wr_d, *L.experts)
        got = L.run(ctx)
        assert got["y"].dtype == torch.float32
        parts.append(got)
        ctx.close()
    return parts


def _check(L, G, parts, tokens=None):
    """Every part against its oracle, then the rounded sum against the layer."""
    worst = 0.0
    for g, got in enumerate(parts):
        worst = max(worst, compare(L, got, L.oracle_part(g, G, tokens=tokens), tokens=tokens))
    total = parts[0]["y"].clone()
    for got in parts[1:]:
        total += got["y"]
    y = moe.round_bf16(total)
    torch.cuda.synchronize()
    whole = dict(parts[0], y=y)
    return max(worst, compare(L, whole, L.oracle(tokens=tokens), tokens=tokens))


@pytest.mark.parametrize("G", [2, 4])
def test_ling_m1_parts(G):
    L = Layer(2560, 768, 256, 8, 1, seed=0, mode="gap")
    worst = _check(L, G, _run_parts(L, G, variant="fused"))
    print(f"Ling M=1, {G} parts: worst y error {worst:.3f} of the bound")


@pytest.mark.parametrize("mode", ["natural", "distinct"])
def test_ling_m4_parts_on_tensor_cores(mode):
    L = Layer(2560, 768, 256, 8, 4, seed=1, mode=mode)
    worst = _check(L, 2, _run_parts(L, 2, variant="tc"))
    print(f"Ling M=4 {mode}, 2 parts (k_tc, I/G = 384): worst y error {worst:.3f} of the bound")


def test_ling_m32_parts_sampled():
    L = Layer(2560, 768, 256, 8, 32, seed=2, mode="zipf")
    parts = _run_parts(L, 2, variant="tc")
    worst = _check(L, 2, parts, tokens=[0, 9, 17, 31])
    print(f"Ling M=32 zipf, 2 parts: worst y error {worst:.3f} of the bound")


@pytest.mark.parametrize("flags,shared", [(moe.MOE_FLAG_CUDA_CORES, False), (moe.MOE_FLAG_CUDA_CORES, True),
                                          (moe.MOE_FLAG_TENSOR_CORES, True),
                                          (moe.MOE_FLAG_SPLIT_KERNELS, False), (moe.MOE_FLAG_SPLITK_DOWN, False)])
def test_small_layer_every_token(flags, shared):
    M = 32 if flags != moe.MOE_FLAG_SPLITK_DOWN else 4
    L = Layer(512, 256, 24, 4, M, seed=3, mode="natural", shared=shared)
    G = 2
    worst = _check(L, G, _run_parts(L, G, flags=flags))
    print(f"512x256 M={M} flags={flags:#x} shared={shared}, 2 parts: worst {worst:.3f}")


def test_narrowest_parts():
    """I/G = 32: one E8M0 block of W2 per part."""
    L = Layer(256, 128, 16, 2, 3, seed=4, mode="gap")
    worst = _check(L, 4, _run_parts(L, 4))
    print(f"256x128, 4 parts of width 32: worst {worst:.3f}")


def test_round_bf16_matches_the_oracle_rounding():
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-30, 30, 3000),
                           [0.0, -0.0, 1.0, -1.0, 3.3895313892515355e38, 1e-40, -1e-45, 65504.0]])
    # exact midpoints between neighbouring bf16 values (ties go to even)
    hi = rng.integers(0x0080, 0x7F00, 400).astype(np.uint32)
    mids = ((hi << 16) | 0x8000).view(np.float32)
    v = np.concatenate([vals.astype(np.float32), mids, -mids])
    y32 = torch.from_numpy(v).cuda()
    y = moe.round_bf16(y32)
    torch.cuda.synchronize()
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = np.array([oracle.bf16_round(float(a)) for a in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_part_needs_a_copy_and_an_f32_output():
    L = Layer(256, 128, 16, 2, 2, seed=5, mode="gap")
    ctx = moe.MoELayer(L.H, L.I, L.E, L.K, 2, shard=(1, 2))
    p = [moe._ptr(t) for t in (L.wr_d, *L.experts)]
    assert moe.lib().moe_load_experts(ctx._ctx, *p, moe.MOE_LOAD_BORROW) == 1  # INVALID_ARG
    ctx.load_experts(L.wr_d, *L.experts)
    # an fp32 y that overlaps x is refused before any launch
    buf = torch.zeros(2 * L.H * 2 + 2 * L.H * 4, dtype=torch.uint8, device="cuda")  # room for x and y
    x = buf[:2 * L.H * 2].view(torch.bfloat16).view(2, L.H)
    x.copy_(L.x_d)
    y_alias = ctypes.c_void_p(buf.data_ptr() + 2 * L.H * 2 - 16)
    assert moe.lib().moe_decode(ctx._ctx, moe._ptr(x), 2, y_alias, None, None, None, None, None, None) == 1
    ctx.close()
