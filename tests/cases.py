"""Shared helpers for the GPU parity tests: build a seeded layer on the device,
run the CUDA path through the C ABI, run the oracle on the same inputs, and
compare.

The tolerance on y is a per-token bound: every element must satisfy
|y_gpu - y_oracle_fp64| <= 2e-3 * ||y_oracle[m]||_2. FP8 activation codes and
expert ids must match bit for bit. Where ids are compared, the oracle's fp64
gap at rank k must be at least 1e-5, because closer pairs can legitimately
reorder under fp32.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mxfp4_weight_streaming_fp8_b200 import moe, synth

Y_TOL = 2e-3      # per-token relative-to-norm bound on y
W_TOL = 1e-5      # routing weights (fp32 softmax vs fp64)
GAP_MIN = 1e-5    # fp64 logit gap needed to demand identical ids


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class Layer:
    """Seeded inputs of one MoE layer, on the device and (lazily) on the CPU."""

    def __init__(self, H, I, E, K, M, seed=0, layer=0, mode="gap", device="cuda:0", shared=False, a8=False):
        self.H, self.I, self.E, self.K, self.M = H, I, E, K, M
        self.seed, self.layer = seed, layer
        self.shared = shared  # expert E (the last of E + 1) is a shared expert
        self.a8 = a8          # FP8 intermediate (MOE_FLAG_FP8_INTERMEDIATE)
        self.x = synth.gen_x(seed, M, H, layer=layer)
        self.wr = synth.force_router(self.x, synth.gen_router(seed, layer, E, H), K, mode, seed=seed,
                                     layer=layer) if M > 0 else synth.gen_router(seed, layer, E, H)
        self.dev = torch.device(device)
        self.experts = synth.layer_experts_torch(seed, layer, E + int(shared), H, I, self.dev)
        self.wr_d = torch.from_numpy(self.wr).to(self.dev)
        self.x_d = self.x.to(self.dev)

    def expert_slices(self, ids):
        per = [[None] * self.E for _ in range(4)]
        for e in sorted(set(int(i) for i in np.asarray(ids).ravel())):
            parts = synth.expert_np(self.seed, self.layer, e, self.H, self.I)
            for t in range(4):
                per[t][e] = parts[t]
        return per

    def oracle(self, tokens=None, a8=None):
        """Oracle outputs for the given token subset (default all); a8
        overrides the layer's FP8-intermediate setting."""
        a8 = self.a8 if a8 is None else a8
        xb = bits(self.x)
        if tokens is not None:
            xb = xb[list(tokens)]
        logits = oracle.router_logits(xb, self.wr)
        ids, _ = oracle.topk(logits, self.K)
        per = self.expert_slices(ids)
        if a8:
            sh = synth.expert_np(self.seed, self.layer, self.E, self.H, self.I) if self.shared else None
            return oracle.moe_decode_a8(xb, self.wr, *per, self.H, self.I, self.E, self.K, shared=sh)
        if self.shared:
            sh = synth.expert_np(self.seed, self.layer, self.E, self.H, self.I)
            return oracle.moe_decode_shared(xb, self.wr, *per, sh, self.H, self.I, self.E, self.K)
        return oracle.moe_decode(xb, self.wr, *per, self.H, self.I, self.E, self.K)

    def oracle_part(self, g, G, tokens=None):
        """Oracle outputs of part g of an intra-expert split over G: the
        layer of width I/G made of each expert's part (part_arrays); its y64
        is the part's fp64 sum before any rounding."""
        assert not self.a8
        xb = bits(self.x)
        if tokens is not None:
            xb = xb[list(tokens)]
        logits = oracle.router_logits(xb, self.wr)
        ids, _ = oracle.topk(logits, self.K)
        per = self.expert_slices(ids)
        for e in range(self.E):
            if per[0][e] is not None:
                parts = part_arrays(*(per[t][e] for t in range(4)), self.I, g, G)
                for t in range(4):
                    per[t][e] = parts[t]
        Ip = self.I // G
        if self.shared:
            sh = part_arrays(*synth.expert_np(self.seed, self.layer, self.E, self.H, self.I), self.I, g, G)
            return oracle.moe_decode_shared(xb, self.wr, *per, sh, self.H, Ip, self.E, self.K)
        return oracle.moe_decode(xb, self.wr, *per, self.H, Ip, self.E, self.K)

    def make_ctx(self, flags=0, max_tokens=None):
        if self.shared:
            flags |= moe.MOE_FLAG_SHARED_EXPERT
        if self.a8:
            flags |= moe.MOE_FLAG_FP8_INTERMEDIATE
        ctx = moe.MoELayer(self.H, self.I, self.E, self.K, max_tokens or max(1, self.M), flags=flags,
                           device=self.dev.index or 0)
        ctx.load_experts(self.wr_d, *self.experts)
        return ctx

    def run(self, ctx):
        out = ctx.decode(self.x_d, routing=True)
        y, ids, w, xq, xs = out[:5]
        torch.cuda.synchronize()
        st = ctx.sync_status()
        assert st == moe.MOE_OK, moe.status_string(st)
        res = dict(y=y, ids=ids.cpu().numpy(), w=w.cpu().numpy(), q=xq.cpu().numpy(), s=xs.cpu().numpy())
        if len(out) > 5:
            res["xn"] = out[5]
        return res


def part_arrays(w13c, w13s, w2c, w2s, I, g, G):
    """Part g of G of one expert's arrays (the layouts of synth.expert_np):
    gate rows [g*I/G, (g+1)*I/G), the up rows I + the same, and the same
    columns of the down projection (codes two per byte, scales one per 32)."""
    Ip = I // G
    rows = np.r_[g * Ip:(g + 1) * Ip, I + g * Ip:I + (g + 1) * Ip]
    return (np.ascontiguousarray(w13c[rows]), np.ascontiguousarray(w13s[rows]),
            np.ascontiguousarray(w2c[:, g * Ip // 2:(g + 1) * Ip // 2]),
            np.ascontiguousarray(w2s[:, g * Ip // 32:(g + 1) * Ip // 32]))


def min_gap(logits: np.ndarray, k: int) -> float:
    """Smallest fp64 gap among each token's k+1 largest logits."""
    s = -np.sort(-logits, axis=1)[:, :k + 1]
    if s.shape[1] < 2:
        return np.inf
    return float(np.min(s[:, :-1] - s[:, 1:]))


def compare(layer: Layer, got: dict, ref: dict, tokens=None, check_ids=True):
    """Assert parity; returns the worst y error as a fraction of the bound."""
    t = list(range(layer.M)) if tokens is None else list(tokens)
    assert np.array_equal(got["q"][t], ref["q"]), "E4M3 activation codes differ"
    assert np.array_equal(got["s"][t], ref["s"]), "activation scales differ"
    if check_ids:
        gap = min_gap(ref["logits"], layer.K)
        if gap >= GAP_MIN:
            assert np.array_equal(got["ids"][t], ref["ids"]), "expert ids differ"
            assert np.all(np.abs(got["w"][t] - ref["weights"]) <= W_TOL), "routing weights differ"
    y = got["y"].float().cpu().numpy().astype(np.float64)[t]
    norm = np.linalg.norm(ref["y64"], axis=1, keepdims=True)
    bound = Y_TOL * norm
    err = np.abs(y - ref["y64"])
    worst = float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
    assert np.all(err <= bound), f"y error {err.max():.3e} exceeds bound {bound.min():.3e} (ratio {worst:.2f})"
    return worst
