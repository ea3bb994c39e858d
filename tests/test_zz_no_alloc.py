"""moe_decode_static, the entry point that allocates nothing.

It is for callers that cannot allocate device memory, such as a plugin whose
host runtime owns all device memory, or a serving loop that must never call
cudaMalloc. Its scratch is one fixed device array in the library, shared by
every call and keeping whatever the last call left in it.

The tests call it through the C ABI on layers of different shapes in turn
(the 4-token Ling-shaped layer, the tiny layer, then the Ling layer again),
so a call that wrongly reused state left in the array by the previous call
would show. Each call is checked against the CPU oracle with the bound every
parity test uses (bit-exact FP8 codes and expert ids, y within 2e-3 of each
token's norm), and against moe_decode on the same inputs: identical codes
and ids, y within the same bound.

This file sorts last, so a run that stops at the first failure has already
run every other test. It also passes on its own in a fresh process, where
its first call does the device set-up.
"""
import numpy as np
import pytest
import torch

from cases import Layer, Y_TOL, compare
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


def test_static_entry_matches_oracle_across_interleaved_shapes():
    from mxfp4_weight_streaming_fp8_b200 import build
    build.build()
    ling = Layer(2560, 768, 256, 8, 4, seed=13, mode="gap")
    tiny = Layer(256, 64, 16, 2, 1, seed=13, mode="natural")
    refs = {id(ling): ling.oracle(), id(tiny): tiny.oracle()}
    viaapi = {id(L): L.run(L.make_ctx(0)) for L in (ling, tiny)}
    for call, L in enumerate((ling, tiny, ling, tiny)):
        got = _static_call(L)
        compare(L, got, refs[id(L)])
        other = viaapi[id(L)]
        assert np.array_equal(got["q"], other["q"]), f"call {call}: E4M3 codes differ from moe_decode"
        assert np.array_equal(got["ids"], other["ids"]), f"call {call}: expert ids differ from moe_decode"
        yo = other["y"].float()
        err = (got["y"].float() - yo).abs()
        assert torch.all(err <= Y_TOL * yo.norm(dim=1, keepdim=True)), f"call {call}: y far from moe_decode"


def test_static_entry_rejects_what_does_not_fit():
    L = Layer(256, 64, 16, 2, 1, seed=0, mode="natural")
    y = torch.empty_like(L.x_d)
    # H=2560, I=4096, top-8, M=32: the gate/up kernel's f16 activations
    # (M*H*2 = 160 KB) fit its shared memory, but the per-pair SwiGLU output
    # alone (M*top_k*I*4 = 4 MiB) fills the 4 MiB scratch array, so the call
    # is rejected by the scratch check before anything is launched
    big_x = torch.zeros((32, 2560), dtype=torch.bfloat16, device=L.dev)
    big_y = torch.zeros_like(big_x)
    st = moe.decode_static(2560, 4096, 16, 8, L.wr_d, *L.experts, big_x, 32, big_y)
    assert st == 2  # MOE_ERR_UNSUPPORTED
    assert moe.decode_static(256, 64, 16, 2, L.wr_d, *L.experts, L.x_d, 0, y) == moe.MOE_OK  # M = 0: no-op
    assert moe.decode_static(256, 64, 16, 2, L.wr_d, *L.experts, L.x_d, 1, L.x_d) == 1  # y aliases x
