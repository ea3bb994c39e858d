"""moe_decode_static, the entry point that allocates nothing.

It is for callers that cannot allocate device memory, such as a plugin whose
host runtime owns all device memory, or a serving loop that must never call
cudaMalloc. Its scratch is one fixed device array in the library. This test
calls it through the C ABI twice in a row and checks each output against
moe_decode's on the same inputs: bit-exact FP8 codes and expert ids, and y
within the per-token bound the parity tests use.

This file sorts last, so a run that stops at the first failure has already
run every other test. It also passes on its own in a fresh process, where
its first call does the device set-up.
"""
import numpy as np
import pytest
import torch

from cases import Layer, Y_TOL
from mxfp4_weight_streaming_fp8_b200 import moe

pytestmark = pytest.mark.gpu


def _static_call(L):
    dev = L.dev
    M, K = L.M, L.K
    y = torch.full_like(L.x_d, float("nan"))
    ids = torch.full((M, K), -1, dtype=torch.int32, device=dev)
    w = torch.zeros((M, K), dtype=torch.float32, device=dev)
    xq = torch.zeros((M, L.H), dtype=torch.uint8, device=dev)
    xs = torch.zeros((M,), dtype=torch.float32, device=dev)
    st = moe.decode_static(L.H, L.I, L.E, L.K, L.wr_d, *L.experts, L.x_d, M, y, None, ids, w, xq, xs)
    assert st == moe.MOE_OK, moe.status_string(st)
    torch.cuda.synchronize()
    return dict(y=y, ids=ids.cpu().numpy(), w=w.cpu().numpy(), q=xq.cpu().numpy(), s=xs.cpu().numpy())


@pytest.mark.parametrize("shape,mode", [((2560, 768, 256, 8, 4), "gap"), ((256, 64, 16, 2, 1), "natural")])
def test_static_entry_matches_moe_decode_on_two_calls(shape, mode):
    from mxfp4_weight_streaming_fp8_b200 import build
    build.build()
    H, I, E, K, M = shape
    L = Layer(H, I, E, K, M, seed=13, mode=mode)
    # the existing entry point (moe_create + moe_decode) running the same kernels
    ref = L.run(L.make_ctx(moe.MOE_FLAG_SPLIT_KERNELS))
    yref = ref["y"].float()
    bound = Y_TOL * yref.norm(dim=1, keepdim=True)
    for call in range(2):
        got = _static_call(L)
        assert np.array_equal(got["q"], ref["q"]), f"call {call}: E4M3 codes differ"
        assert np.array_equal(got["s"], ref["s"]), f"call {call}: activation scales differ"
        assert np.array_equal(got["ids"], ref["ids"]), f"call {call}: expert ids differ"
        assert np.all(np.abs(got["w"] - ref["w"]) <= 1e-6), f"call {call}: routing weights differ"
        err = (got["y"].float() - yref).abs()
        assert torch.all(err <= bound), f"call {call}: y differs by {err.max().item():.3e}"


def test_static_entry_rejects_what_does_not_fit():
    L = Layer(256, 64, 16, 2, 1, seed=0, mode="natural")
    y = torch.empty_like(L.x_d)
    # E*M*4 + M*H + M*K*4*I far above the 4 MiB scratch: rejected, nothing launched
    big_x = torch.zeros((32, 8192), dtype=torch.bfloat16, device=L.dev)
    big_y = torch.zeros_like(big_x)
    st = moe.decode_static(8192, 4096, 16, 8, L.wr_d, *L.experts, big_x, 32, big_y)
    assert st == 2  # MOE_ERR_UNSUPPORTED
    assert moe.decode_static(256, 64, 16, 2, L.wr_d, *L.experts, L.x_d, 0, y) == moe.MOE_OK  # M = 0: no-op
    assert moe.decode_static(256, 64, 16, 2, L.wr_d, *L.experts, L.x_d, 1, L.x_d) == 1  # y aliases x
