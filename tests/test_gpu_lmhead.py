"""FP8 LM head through the C ABI against the CPU oracle.

The BF16 matrix is drawn on the device from a seeded generator and the
oracle quantises its own copy of the rows it checks, so no expected value
comes from the CUDA path. Codes and scales must match bit for bit. Logits
are fp32 sums of exact products: each must be within 1e-4 of the sum of
|products| of its row (about 40 fp32 roundings' worth at H = 2560).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_weight_streaming_fp8_b200 import moe

pytestmark = pytest.mark.gpu

REL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from mxfp4_weight_streaming_fp8_b200 import build
    build.build()
    assert torch.cuda.is_available()


def bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def make_w(V, H, seed, dev="cuda:0"):
    g = torch.Generator(device=dev).manual_seed(seed)
    w = (torch.randn(V, H, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    if V > 3:
        w[1] = 0                                   # all-zero row
        w[2] = 0
        w[2, H // 3] = 3.0                         # one non-zero element
        w[3] *= 1000                               # a row with large values
    return w


def make_x(M, H, seed, dev="cuda:0"):
    g = torch.Generator(device=dev).manual_seed(seed + 1000)
    return torch.randn(M, H, generator=g, device=dev).to(torch.bfloat16)


def check_rows(lm, w, x, rows, logits):
    codes, scales = lm.weights()
    torch.cuda.synchronize()
    wb = bits(w[rows])
    oc, os_ = oracle.lm_quantize(wb)
    gc = codes[rows].cpu().numpy()
    gs = scales[rows].cpu().numpy()
    assert np.array_equal(gc, oc), "E4M3 codes differ"
    assert np.array_equal(gs, os_), "row scales differ"
    xb = bits(x)
    ref = oracle.lm_head(oc, os_, xb)
    absx = bits(x.float().abs().to(torch.bfloat16))
    bound = REL * oracle.lm_head(oc & 0x7F, os_, absx)
    got = logits[:, rows].cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= bound + 1e-30), f"max err {err.max():.3e}, ratio {(err / (bound + 1e-30)).max():.2f}"


@pytest.mark.parametrize("V,H,M", [(1000, 256, 1), (1000, 256, 3), (777, 128, 16), (5, 64, 2)])
def test_lm_head_small_every_row(V, H, M):
    w, x = make_w(V, H, seed=V + H), make_x(M, H, seed=V)
    lm = moe.LMHead(V, H, max_tokens=16)
    assert lm.query()["kernel"] == "k_lm_head"
    lm.load(w)
    logits = lm(x)
    assert lm.sync_status() == moe.MOE_OK
    check_rows(lm, w, x, list(range(V)), logits)


@pytest.mark.parametrize("M", [1, 4])
def test_lm_head_ling_vocab_sampled(M):
    V, H = 157184, 2560
    w, x = make_w(V, H, seed=11), make_x(M, H, seed=12)
    lm = moe.LMHead(V, H, max_tokens=8)
    lm.load(w)
    logits = lm(x)
    assert lm.sync_status() == moe.MOE_OK
    rng = np.random.default_rng(M)
    G = torch.cuda.get_device_properties(0).multi_processor_count
    edges = sorted({V * b // G for b in range(0, G, 13)} | {V * b // G - 1 for b in range(1, G, 17)})
    rows = sorted(set(rng.integers(0, V, 48).tolist()) | {0, 1, 2, 3, V - 1} | set(edges))
    check_rows(lm, w, x, rows, logits)
    assert torch.isfinite(logits).all()


def test_lm_head_repeatable_and_m0():
    V, H = 3000, 512
    w, x = make_w(V, H, seed=3), make_x(2, H, seed=4)
    lm = moe.LMHead(V, H, max_tokens=2)
    lm.load(w)
    a = lm(x).clone()
    b = lm(x)
    assert torch.equal(a, b)
    y = torch.full((1, V), 7.0, device="cuda:0")
    assert lm.head_raw(x, 0, y) == moe.MOE_OK
    torch.cuda.synchronize()
    assert torch.all(y == 7.0)


def test_lm_head_errors():
    V, H = 100, 128
    lm = moe.LMHead(V, H, max_tokens=2)
    x = make_x(2, H, seed=5)
    out = torch.empty((2, V), device="cuda:0")
    assert lm.head_raw(x, 1, out) == 5          # not loaded
    lm.load(make_w(V, H, seed=6))
    assert lm.head_raw(x, 3, out) == 1          # M > max_tokens
    xs = torch.empty(2 * H + 8, dtype=torch.bfloat16, device="cuda:0")
    assert lm.head_raw(xs[1:H + 1], 1, out) == 1  # misaligned x
    with pytest.raises(moe.MoEError):
        moe.LMHead(V, 100, max_tokens=1)        # hidden not a multiple of 64
