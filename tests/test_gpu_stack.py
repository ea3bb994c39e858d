"""Stacked layers with RMSNorm between them (unit weight, eps 1e-6), checked
layer by layer with teacher forcing: the oracle takes each layer's GPU input
(the previous layer's bf16 output), normalises it itself, and the GPU's
normalised input, FP8 codes, expert ids and output are compared against it.
Rounding compounds over layers, so the stack is not compared end to end."""
import numpy as np
import pytest
import torch

import oracle
from cases import Y_TOL, bits
from mxfp4_weight_streaming_fp8_b200 import moe, synth

pytestmark = pytest.mark.gpu


def _bf16_ulp_diff(a_bits, b_bits):
    """|difference| in units in the last place between bf16 bit patterns of the same sign."""
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    sa = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    sb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(sa - sb)


@pytest.mark.parametrize("M,kernel", [(1, 0), (3, 0), (1, moe.MOE_FLAG_TENSOR_CORES),
                                      (5, moe.MOE_FLAG_TENSOR_CORES)])
def test_three_layer_stack_teacher_forced(M, kernel):
    """kernel 0: the library's choice (the CUDA-core kernel below 4 tokens);
    MOE_FLAG_TENSOR_CORES: the tensor-core kernel (its one-token routing at
    M=1, the per-warp token routing with the RMSNorm factor at M=5)."""
    H, I, E, K, seed = 2560, 768, 256, 8, 21
    dev = torch.device("cuda:0")
    x_in = synth.gen_x(seed, M, H)  # bf16, layer 0 input (not normalised)
    for l in range(3):
        flags = (moe.MOE_FLAG_PRE_RMSNORM if l > 0 else 0) | kernel
        xin_bits = bits(x_in)
        # the oracle's view of this layer's routing input
        xr_bits = oracle.rmsnorm(xin_bits, 1e-6) if l > 0 else xin_bits
        xr = torch.from_numpy(xr_bits.view(np.int16)).view(torch.bfloat16)
        wr = synth.force_router(xr, synth.gen_router(seed, l, E, H), K, "gap", seed=seed, layer=l)
        ex = synth.layer_experts_torch(seed, l, E, H, I, dev)
        ctx = moe.MoELayer(H, I, E, K, M, flags=flags)
        if kernel:
            assert ctx.query()["variant"] == "tc"
        ctx.load_experts(torch.from_numpy(wr).to(dev), *ex)
        out = ctx.decode(x_in.to(dev), routing=True)
        y, ids, w, xq, xs = out[:5]
        torch.cuda.synchronize()
        assert ctx.sync_status() == moe.MOE_OK
        if l > 0:
            xn_gpu = bits(out[5])
            d = _bf16_ulp_diff(xn_gpu, xr_bits)
            assert d.max() <= 1, f"layer {l}: normalised input off by {d.max()} ulp"
            print(f"layer {l}: normalised input, {int((d > 0).sum())} of {d.size} elements 1 ulp off")
        else:
            xn_gpu = xin_bits
        # teacher forcing: everything downstream is checked on the GPU's own normalised input
        logits = oracle.router_logits(xn_gpu, wr)
        rid, _ = oracle.topk(logits, K)
        per = [[None] * E for _ in range(4)]
        for e in sorted(set(rid.ravel().tolist())):
            parts = synth.expert_np(seed, l, e, H, I)
            for t in range(4):
                per[t][e] = parts[t]
        ref = oracle.moe_decode(xn_gpu, wr, *per, H, I, E, K)
        assert np.array_equal(xq.cpu().numpy(), ref["q"]), f"layer {l}: E4M3 codes differ"
        assert np.array_equal(ids.cpu().numpy(), ref["ids"]), f"layer {l}: expert ids differ"
        yg = y.float().cpu().numpy().astype(np.float64)
        bound = Y_TOL * np.linalg.norm(ref["y64"], axis=1, keepdims=True)
        assert np.all(np.abs(yg - ref["y64"]) <= bound), f"layer {l}: y out of bound"
        x_in = y.cpu()
        ctx.close()


def test_rmsnorm_flag_rules():
    with pytest.raises(moe.MoEError) as ei:
        moe.MoELayer(256, 64, 16, 2, 1, flags=moe.MOE_FLAG_PRE_RMSNORM | moe.MOE_FLAG_SPLIT_KERNELS)
    assert ei.value.status == 2
    ctx = moe.MoELayer(256, 64, 16, 2, 1)
    x = torch.zeros((1, 256), dtype=torch.bfloat16, device="cuda:0")
    y = torch.empty_like(x)
    xn = torch.empty_like(x)
    ex = synth.layer_experts_torch(0, 0, 16, 256, 64, "cuda:0")
    ctx.load_experts(torch.zeros((16, 256), device="cuda:0"), *ex)
    assert ctx.decode_raw(x, 1, y, xnorm=xn) == 1  # xnorm only with the RMSNorm flag
