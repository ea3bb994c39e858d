"""The tensor-core kernel (k_tc: tcgen05 block-scaled gate/up, CUDA-core
down) against the CPU oracle, element by element, through the C ABI.

k_tc needs H and I to be multiples of 128 (MOE_FLAG_TENSOR_CORES selects
it; by default it runs from MOE_TC_MIN_TOKENS tokens on). These cases
cover small layers that still span several tiles, K-chunk stages and ragged
unions, one K-chunk per stage (H/128 odd), the Ling-shaped layer at M=1, 4
and 32 with every token checked, the shared expert, the FP8 intermediate, a
context sized for more tokens than a call uses, and agreement with the
CUDA-core kernel (MOE_FLAG_CUDA_CORES).
"""
import numpy as np
import pytest
import torch

from cases import Layer, compare, bits
from mxfp4_weight_streaming_fp8_b200 import moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from mxfp4_weight_streaming_fp8_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _ctx(L, flags=0, max_tokens=None):
    ctx = L.make_ctx(flags | moe.MOE_FLAG_TENSOR_CORES, max_tokens=max_tokens)
    assert ctx.query()["variant"] == "tc", ctx.query()
    return ctx


@pytest.mark.parametrize("shape,M,mode", [((256, 128, 16, 2), 1, "natural"), ((256, 128, 16, 2), 3, "gap"),
                                          ((512, 256, 40, 6), 5, "gap"), ((384, 128, 12, 4), 4, "natural"),
                                          ((128, 128, 8, 8), 3, "natural"), ((1024, 512, 64, 8), 7, "zipf")])
def test_small_layers(shape, M, mode):
    H, I, E, K = shape
    L = Layer(H, I, E, K, M, seed=41, mode=mode)
    got = L.run(_ctx(L))
    worst = compare(L, got, L.oracle(), check_ids=(mode != "natural" or K < E))
    print(f"k_tc {shape} M={M}: worst y error {worst:.3f} of the bound")


def test_ling_m1():
    L = Layer(2560, 768, 256, 8, 1, seed=0, mode="gap")
    ctx = _ctx(L)
    got = L.run(ctx)
    worst = compare(L, got, L.oracle())
    print(f"k_tc Ling M=1: worst y error {worst:.3f} of the bound")
    again = L.run(ctx)
    assert torch.equal(got["y"], again["y"])


@pytest.mark.parametrize("mode,U", [("distinct", 32), ("shared", 8), ("natural", None)])
def test_ling_m4_verify(mode, U):
    L = Layer(2560, 768, 256, 8, 4, seed=1, mode=mode)
    got = L.run(_ctx(L))
    if U is not None:
        assert len(set(got["ids"].ravel().tolist())) == U
    compare(L, got, L.oracle())


@pytest.mark.slow
@pytest.mark.parametrize("mode", ["zipf", "shared"])
def test_ling_m32_every_token(mode):
    """All 32 tokens' y against the oracle at the Ling shape."""
    L = Layer(2560, 768, 256, 8, 32, seed=2, mode=mode)
    got = L.run(_ctx(L))
    worst = compare(L, got, L.oracle())
    print(f"k_tc Ling M=32 {mode}: worst y error {worst:.3f} of the bound")


def test_context_larger_than_call():
    L = Layer(2560, 768, 256, 8, 3, seed=3, mode="natural")
    got = L.run(_ctx(L, max_tokens=32))
    compare(L, got, L.oracle())


@pytest.mark.parametrize("shape,M,mode", [((256, 128, 16, 2), 2, "natural"), ((2560, 768, 256, 8), 1, "gap"),
                                          ((2560, 768, 256, 8), 4, "natural")])
def test_shared_expert(shape, M, mode):
    H, I, E, K = shape
    L = Layer(H, I, E, K, M, seed=21, mode=mode, shared=True)
    ctx = _ctx(L)
    assert ctx.query()["shared_expert"] is True
    got = L.run(ctx)
    compare(L, got, L.oracle())


@pytest.mark.slow
def test_shared_expert_m32_every_token():
    L = Layer(2560, 768, 256, 8, 32, seed=22, mode="zipf", shared=True)
    got = L.run(_ctx(L))
    compare(L, got, L.oracle())


@pytest.mark.parametrize("M,mode", [(1, "gap"), (4, "natural"), (6, "shared")])
def test_fp8_intermediate(M, mode):
    from test_gpu_parity import _check_a8
    L = Layer(2560, 768, 256, 8, M, seed=31, mode=mode, a8=True)
    ctx = _ctx(L)
    assert ctx.query()["fp8_intermediate"] is True
    got = L.run(ctx)
    _check_a8(L, got)


@pytest.mark.slow
def test_fp8_intermediate_m32_every_token():
    from test_gpu_parity import _check_a8
    L = Layer(2560, 768, 256, 8, 32, seed=32, mode="zipf", a8=True)
    got = L.run(_ctx(L))
    _check_a8(L, got)


def test_agrees_with_cuda_core_kernel():
    L = Layer(2560, 768, 256, 8, 4, seed=8, mode="gap")
    a = L.run(_ctx(L))
    ctx_b = L.make_ctx(moe.MOE_FLAG_CUDA_CORES)
    assert ctx_b.query()["variant"] == "fused"
    b = L.run(ctx_b)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["ids"], b["ids"])
    ya, yb = a["y"].float(), b["y"].float()
    assert torch.all((ya - yb).abs() <= 4e-3 * ya.norm(dim=1, keepdim=True))


def test_forced_timeout_is_reported_and_recovers():
    L = Layer(256, 128, 16, 2, 1, seed=0, mode="natural")
    ctx = _ctx(L)
    good = L.run(ctx)["y"].clone()
    assert ctx.set_wait(20000, force_stall=True) == moe.MOE_OK
    y = torch.empty_like(L.x_d)
    assert ctx.decode_raw(L.x_d, 1, y) == moe.MOE_OK
    assert ctx.sync_status() == 6  # MOE_ERR_TIMEOUT
    assert ctx.set_wait(0, force_stall=False) == moe.MOE_OK
    again = L.run(ctx)["y"]
    assert torch.equal(again, good)


def test_back_to_back_and_graph_replay():
    """Programmatic dependent launches between contexts and replay of a
    captured graph give the results of separate calls."""
    Ls = [Layer(2560, 768, 256, 8, 1, seed=9, layer=l, mode="gap") for l in range(3)]
    ctxs = [_ctx(L) for L in Ls]
    ys = [torch.empty_like(L.x_d) for L in Ls]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for L, c, y in zip(Ls, ctxs, ys):
            assert c.decode_raw(L.x_d, 1, y, stream=s) == moe.MOE_OK
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for L, c, y in zip(Ls, ctxs, ys):
            assert c.decode_raw(L.x_d, 1, y) == moe.MOE_OK
    for y in ys:
        y.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    for L, c, y in zip(Ls, ctxs, ys):
        assert c.sync_status() == moe.MOE_OK
        assert torch.equal(L.run(c)["y"], y)


@pytest.mark.parametrize("shape,M,mode", [((2560, 768, 256, 8), 1, "gap"), ((2560, 768, 256, 8), 4, "natural"),
                                          ((512, 256, 40, 6), 5, "gap")])
def test_copy_repack_matches_borrowed(shape, M, mode):
    """MOE_LOAD_COPY_REPACK: the context's re-tiled copy gives the same bits
    as the borrowed weights (the MMAs see the same operands), matches the
    oracle, and keeps working after the caller's arrays are overwritten."""
    H, I, E, K = shape
    L = Layer(H, I, E, K, M, seed=51, mode=mode)
    a = L.run(_ctx(L))
    ctx = moe.MoELayer(H, I, E, K, M, flags=moe.MOE_FLAG_TENSOR_CORES)
    ctx.load_experts(L.wr_d, *L.experts, repack=True)
    b = L.run(ctx)
    assert torch.equal(a["y"], b["y"])
    compare(L, b, L.oracle())
    # the context owns its copy: clobbering the caller's arrays changes nothing
    for t in L.experts:
        t.zero_()
    L.wr_d.zero_()
    c = L.run(ctx)
    assert torch.equal(b["y"], c["y"])


def test_copy_repack_cuda_core_kernel():
    L = Layer(2560, 768, 256, 8, 2, seed=52, mode="natural")
    ctx = moe.MoELayer(2560, 768, 256, 8, 2, flags=moe.MOE_FLAG_CUDA_CORES)
    ctx.load_experts(L.wr_d, *L.experts, repack=True)
    got = L.run(ctx)
    compare(L, got, L.oracle())


# ---- the down projection on tensor cores (MOE_FLAG_TC_DOWN_MMA; the default
#      from MOE_TC_DOWN_MMA_MIN_TOKENS tokens of max_tokens on)

def _ctx_down(L, mma, flags=0, max_tokens=None):
    f = flags | moe.MOE_FLAG_TENSOR_CORES | (moe.MOE_FLAG_TC_DOWN_MMA if mma else moe.MOE_FLAG_TC_DOWN_CUDA)
    ctx = L.make_ctx(f, max_tokens=max_tokens)
    q = ctx.query()
    assert q["variant"] == "tc" and q["down"] == ("tensor_cores" if mma else "cuda_cores"), q
    return ctx


@pytest.mark.parametrize("shape,M,mode", [((256, 128, 16, 2), 3, "gap"), ((512, 256, 40, 6), 5, "gap"),
                                          ((128, 128, 8, 8), 3, "natural"), ((1024, 512, 64, 8), 7, "zipf"),
                                          ((384, 128, 12, 4), 4, "shared")])
def test_mma_down_small_layers(shape, M, mode):
    """Tiles of 128 output rows over several row blocks, pair groups of one
    to many pairs, ragged unions."""
    H, I, E, K = shape
    L = Layer(H, I, E, K, M, seed=61, mode=mode)
    got = L.run(_ctx_down(L, True))
    worst = compare(L, got, L.oracle(), check_ids=(mode != "natural" or K < E))
    print(f"k_tc down on tensor cores {shape} M={M}: worst y error {worst:.3f} of the bound")


@pytest.mark.parametrize("M,mode", [(1, "gap"), (4, "distinct"), (8, "zipf"), (16, "shared")])
def test_mma_down_ling(M, mode):
    L = Layer(2560, 768, 256, 8, M, seed=62, mode=mode)
    ctx = _ctx_down(L, True)
    got = L.run(ctx)
    compare(L, got, L.oracle())
    assert torch.equal(L.run(ctx)["y"], got["y"])  # repeatable


def test_mma_down_is_default_from_min_tokens():
    L = Layer(2560, 768, 256, 8, 1, seed=63, mode="gap")
    ctx = L.make_ctx(moe.MOE_FLAG_TENSOR_CORES, max_tokens=moe.MOE_TC_DOWN_MMA_MIN_TOKENS)
    assert ctx.query()["down"] == "tensor_cores"
    compare(L, L.run(ctx), L.oracle())
    ctx = L.make_ctx(moe.MOE_FLAG_TENSOR_CORES, max_tokens=moe.MOE_TC_DOWN_MMA_MIN_TOKENS - 1)
    assert ctx.query()["down"] == "cuda_cores"
    # without a kernel flag the library picks the tensor-core kernel from
    # MOE_TC_MIN_TOKENS tokens of max_tokens on
    assert L.make_ctx(0, max_tokens=moe.MOE_TC_MIN_TOKENS).query()["variant"] == "tc"
    assert L.make_ctx(0, max_tokens=moe.MOE_TC_MIN_TOKENS - 1).query()["variant"] == "fused"


def test_mma_down_agrees_with_cuda_core_down():
    L = Layer(2560, 768, 256, 8, 8, seed=64, mode="zipf")
    a, b = L.run(_ctx_down(L, True)), L.run(_ctx_down(L, False))
    assert np.array_equal(a["ids"], b["ids"])
    ya, yb = a["y"].float(), b["y"].float()
    assert torch.all((ya - yb).abs() <= 4e-3 * yb.norm(dim=1, keepdim=True))


@pytest.mark.parametrize("M,mode", [(2, "gap"), (12, "zipf")])
def test_mma_down_shared_expert_and_fp8_intermediate(M, mode):
    from test_gpu_parity import _check_a8
    L = Layer(2560, 768, 256, 8, M, seed=65, mode=mode, shared=True)
    compare(L, L.run(_ctx_down(L, True, moe.MOE_FLAG_SHARED_EXPERT)), L.oracle())
    L = Layer(2560, 768, 256, 8, M, seed=66, mode=mode, a8=True)
    _check_a8(L, L.run(_ctx_down(L, True, moe.MOE_FLAG_FP8_INTERMEDIATE)))
