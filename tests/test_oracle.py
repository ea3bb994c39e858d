"""Pins for the CPU oracle, against things other than the oracle itself.

Sources: the format tables of OCP MX v1.0 (E2M1, E8M0) and OFP8 (E4M3), kept
as fixtures under tests/golden; torch's independent float8 conversions; numpy
and scipy library routines where a step reduces to one; a hand-derived
2-expert example; one-hot probes that read single weights back out of the
packed layout; brute-force dense evaluation; and invariants.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from mxfp4_weight_streaming_fp8_b200 import synth


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- formats
def test_e2m1_table_matches_mx_spec(oracle_mod):
    for code, val in read_golden("e2m1_values.txt"):
        got = oracle_mod.e2m1_value(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_e8m0_all_bytes(oracle_mod):
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64)
    for b in range(256):
        v = oracle_mod.e8m0_value(b)
        if b == 255:
            assert math.isnan(v)
        else:
            assert v == 2.0 ** (b - 127)
            assert v == lib_vals[b].item()


def test_e4m3_points_match_ofp8_spec(oracle_mod):
    for code, val in read_golden("e4m3_points.txt"):
        got = oracle_mod.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_decode_matches_torch_float8(oracle_mod):
    lib_vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        a, b = oracle_mod.e4m3_value(c), lib_vals[c].item()
        assert (math.isnan(a) and math.isnan(b)) or a == b, hex(c)


def test_e4m3_roundtrip_and_monotone(oracle_mod):
    prev = -1.0
    for c in range(0x7F):
        v = oracle_mod.e4m3_value(c)
        assert oracle_mod.e4m3_encode(v) == c
        assert oracle_mod.e4m3_encode(-v) == (c | 0x80)
        assert v > prev
        prev = v


def test_e4m3_midpoints_round_to_even(oracle_mod):
    for c in range(0x7E):
        lo, hi = oracle_mod.e4m3_value(c), oracle_mod.e4m3_value(c + 1)
        mid = (lo + hi) / 2  # at most 5 significant bits: exact in fp32
        assert np.float32(mid) == mid
        even = c if c % 2 == 0 else c + 1
        assert oracle_mod.e4m3_encode(mid) == even
        assert oracle_mod.e4m3_encode(np.nextafter(np.float32(mid), np.float32(0))) == c
        assert oracle_mod.e4m3_encode(np.nextafter(np.float32(mid), np.float32(1e9))) == c + 1


def test_e4m3_saturates_and_nan(oracle_mod):
    for v in (448.0, 449.0, 463.9, 464.0, 500.0, 1e30, float("inf")):
        assert oracle_mod.e4m3_encode(v) == 0x7E
        assert oracle_mod.e4m3_encode(-v) == 0xFE
    assert oracle_mod.e4m3_encode(float("nan")) == 0x7F
    assert oracle_mod.e4m3_encode(-1e-12) == 0x80


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    # torch's fp32 -> float8_e4m3fn conversion is RNE for |v| < 448
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(3000) * 60, rng.uniform(-447.9, 447.9, 3000),
                        rng.standard_normal(1000) * 0.01]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.e4m3_encode(float(a)) for a in v], np.uint8)
    assert np.array_equal(got, ref)


def test_bf16_round_matches_torch(oracle_mod):
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.standard_normal(4000), rng.standard_normal(1000) * 1e-30,
                        rng.standard_normal(1000) * 1e30]).astype(np.float32)
    ref = bf16_bits(torch.from_numpy(v).to(torch.bfloat16))
    got = np.array([oracle_mod.bf16_round(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, ref)
    for bits in (0x0000, 0x3F80, 0xBF80, 0x7F7F, 0x0001):
        assert oracle_mod.bf16_round(oracle_mod.bf16_value(bits)) == bits


# ---------------------------------------------------------------- A1 quantiser
def test_quantize_matches_torch_float8(oracle_mod):
    x = synth.gen_x(5, 4, 512)
    q, s = oracle_mod.quantize(bf16_bits(x))
    xf = x.float()
    amax = xf.abs().amax(dim=1, keepdim=True)
    inv = torch.tensor(448.0, dtype=torch.float32) / amax  # IEEE fp32 division
    v = xf * inv
    v = torch.clamp(v, -448.0, 448.0)  # saturation: only the amax element can round past 448
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    assert np.array_equal(s, (amax / torch.tensor(448.0)).numpy().ravel())


def test_quantize_amax_and_pow2_invariance(oracle_mod):
    x = synth.gen_x(6, 3, 256)
    bits = bf16_bits(x)
    q, s = oracle_mod.quantize(bits)
    for m in range(3):
        j = int(np.argmax(np.abs(x[m].float().numpy())))
        assert q[m, j] in (0x7E, 0xFE)
    for p in (-3, 1, 4):
        q2, s2 = oracle_mod.quantize(bf16_bits(x * (2.0 ** p)))
        assert np.array_equal(q, q2)
        assert np.array_equal(s2, s * np.float32(2.0 ** p))


def test_quantize_zero_token(oracle_mod):
    q, s = oracle_mod.quantize(np.zeros((2, 64), np.uint16))
    assert not q.any() and np.all(s == 1.0)


# ---------------------------------------------------------------- A2-A4 routing
def test_router_logits_match_matmul(oracle_mod):
    x = synth.gen_x(7, 3, 256)
    wr = synth.gen_router(7, 0, 16, 256)
    got = oracle_mod.router_logits(bf16_bits(x), wr)
    ref = x.double().numpy() @ wr.astype(np.float64).T
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-13)


def _brute_topk(l, k):
    # expert e is kept iff fewer than k experts beat it (higher, or equal and lower index)
    E = len(l)
    kept = [e for e in range(E) if sum(1 for f in range(E) if l[f] > l[e] or (l[f] == l[e] and f < e)) < k]
    return sorted(kept, key=lambda e: (-l[e], e))


def test_topk_brute_force_and_softmax(oracle_mod):
    rng = np.random.default_rng(3)
    for trial in range(50):
        E = int(rng.integers(2, 12))
        k = int(rng.integers(1, E + 1))
        l = np.round(rng.standard_normal((2, E)), 1)  # rounding plants ties
        ids, w = oracle_mod.topk(l, k)
        for m in range(2):
            assert list(ids[m]) == _brute_topk(list(l[m]), k)
            sel = l[m, ids[m]]
            ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
            assert np.allclose(w[m], ref, rtol=1e-14, atol=0)
            assert abs(w[m].sum() - 1.0) < 1e-15


def test_topk_ties_take_lower_index(oracle_mod):
    l = np.array([[1.0, 3.0, 3.0, 0.5, 3.0, 2.0]])
    ids, w = oracle_mod.topk(l, 3)
    assert list(ids[0]) == [1, 2, 4]
    ids, w = oracle_mod.topk(l, 4)
    assert list(ids[0]) == [1, 2, 4, 5]
    ids, w = oracle_mod.topk(np.zeros((1, 8)), 2)
    assert list(ids[0]) == [0, 1] and np.allclose(w, 0.5)


def test_union_structure(oracle_mod):
    ids = np.array([[5, 2, 9], [2, 7, 5], [0, 9, 2]], np.int32)
    uid, off, tok, slot = oracle_mod.union(ids, 10)
    assert list(uid) == [0, 2, 5, 7, 9]
    pairs = [[(int(tok[p]), int(slot[p])) for p in range(off[u], off[u + 1])] for u in range(5)]
    assert pairs == [[(2, 0)], [(0, 1), (1, 0), (2, 2)], [(0, 0), (1, 2)], [(1, 1)], [(0, 2), (2, 1)]]
    assert off[-1] == ids.size


# ---------------------------------------------------------------- A5-A8 experts
def _const_expert(H, I, c13, s13, c2, s2):
    return (np.full((2 * I, H // 2), c13, np.uint8), np.full((2 * I, H // 32), s13, np.uint8),
            np.full((H, I // 2), c2, np.uint8), np.full((H, I // 32), s2, np.uint8))


def test_hand_two_expert_example(oracle_mod):
    g = {r[0]: r[1] for r in read_golden("hand_2expert.txt")}
    H, I, E, k = int(g["H"]), int(g["I"]), int(g["E"]), int(g["k"])
    x = np.full((1, H), int(g["x_bf16_all"], 16), np.uint16)
    wr = np.stack([np.full(H, float(g["router_row0_all"]), np.float32),
                   np.full(H, float(g["router_row1_all"]), np.float32)])
    e0 = _const_expert(H, I, int(g["w13_codes_all"], 16), int(g["w13_scales_all"]),
                       int(g["w2_codes_expert0"], 16), int(g["w2_scales_all"]))
    e1 = _const_expert(H, I, int(g["w13_codes_all"], 16), int(g["w13_scales_all"]),
                       int(g["w2_codes_expert1"], 16), int(g["w2_scales_all"]))
    out = oracle_mod.moe_decode(x, wr, *[[e0[i], e1[i]] for i in range(4)], H, I, E, k)
    assert np.all(out["q"] == 0x7E)
    s = float(np.float32(1.0) / np.float32(448.0))
    assert out["s"][0] == np.float32(s)
    assert float(np.float32(1.0 / 7.0)) * 2.0 ** -6 == s
    gval = 224.0 * float(np.float32(1.0 / 7.0))
    h = gval * gval / (1.0 + math.exp(-gval))
    w0, w1 = 1 / (1 + math.exp(-0.75)), 1 / (1 + math.exp(0.75))
    assert list(out["ids"][0]) == [0, 1]
    assert np.allclose(out["logits"][0], [0.5, -0.25], rtol=0, atol=1e-15)
    assert np.allclose(out["weights"][0], [w0, w1], rtol=1e-14)
    assert np.allclose(out["y64"][0], (w0 - w1) * 32 * h, rtol=1e-13)
    hv, d = oracle_mod.expert(out["q"][0], out["s"][0], *e0, H, I)
    assert np.allclose(hv, h, rtol=1e-13) and np.allclose(d, 32 * h, rtol=1e-13)


def _onehot_x(H, j):
    x = np.zeros((1, H), np.uint16)
    x[0, j] = 0x3F80  # 1.0
    return x


@pytest.mark.parametrize("j", [0, 1, 32, 33, 63, 100])
def test_onehot_probe_reads_packed_gate_element(oracle_mod, j):
    """x one-hot at column j: g_n = s * 448 * W13[n][j] with s = fl32(1/448),
    so the gate/up outputs read single packed weights; this pins nibble order
    (even column in bits 3:0) and the per-32 scale index."""
    H, I = 128, 32
    rng = np.random.default_rng(j)
    w13c = rng.integers(0, 256, (2 * I, H // 2), dtype=np.uint8)
    w13s = rng.integers(124, 131, (2 * I, H // 32), dtype=np.uint8)
    w2c, w2s = np.zeros((H, I // 2), np.uint8), np.full((H, I // 32), 127, np.uint8)
    q, s = oracle_mod.quantize(_onehot_x(H, j))
    assert q[0, j] == 0x7E and s[0] == np.float32(1 / 448)
    hv, _ = oracle_mod.expert(q[0], s[0], w13c, w13s, w2c, w2s, H, I)
    scale448 = float(s[0]) * 448.0
    E2M1 = [float(r[1]) for r in read_golden("e2m1_values.txt")]
    for n in range(I):
        def elem(row):
            byte = int(w13c[row, j // 2])
            code = (byte & 0xF) if j % 2 == 0 else (byte >> 4)
            return E2M1[code] * 2.0 ** (int(w13s[row, j // 32]) - 127)
        gv, uv = elem(n) * scale448, elem(I + n) * scale448
        ref = gv / (1 + math.exp(-gv)) * uv
        assert math.isclose(hv[n], ref, rel_tol=1e-13, abs_tol=1e-300)


def test_onehot_probe_down_orientation(oracle_mod):
    """H != I. Only gate/up row n0 is non-zero, so h is zero except h[n0];
    then d[r] = W2[r][n0] * h[n0] must hold for every r (W2 is [H][I])."""
    H, I, n0 = 96, 64, 37
    w13c = np.zeros((2 * I, H // 2), np.uint8)
    w13c[n0, :] = 0x22
    w13c[I + n0, :] = 0x22
    w13s = np.full((2 * I, H // 32), 127, np.uint8)
    rng = np.random.default_rng(9)
    w2c = rng.integers(0, 256, (H, I // 2), dtype=np.uint8)
    w2s = rng.integers(120, 130, (H, I // 32), dtype=np.uint8)
    x = np.full((1, H), 0x3F80, np.uint16)
    q, s = oracle_mod.quantize(x)
    hv, d = oracle_mod.expert(q[0], s[0], w13c, w13s, w2c, w2s, H, I)
    assert np.count_nonzero(hv) == 1 and hv[n0] > 0
    E2M1 = [float(r[1]) for r in read_golden("e2m1_values.txt")]
    for r in range(H):
        byte = int(w2c[r, n0 // 2])
        code = (byte & 0xF) if n0 % 2 == 0 else (byte >> 4)
        ref = E2M1[code] * 2.0 ** (int(w2s[r, n0 // 32]) - 127) * hv[n0]
        assert d[r] == ref


def _tiny_layer(seed=0, H=256, I=64, E=16, M=1, mode="natural", k=2):
    x = synth.gen_x(seed, M, H)
    wr = synth.force_router(x, synth.gen_router(seed, 0, E, H), k, mode, seed=seed)
    ex = [synth.expert_np(seed, 0, e, H, I) for e in range(E)]
    per = [[ex[e][i] for e in range(E)] for i in range(4)]
    return bf16_bits(x), wr, per


@pytest.mark.parametrize("M,k,mode", [(1, 2, "natural"), (3, 4, "gap"), (4, 2, "distinct")])
def test_dense_brute_force_equals_sparse(oracle_mod, M, k, mode):
    H, I, E = 256, 64, 16
    x, wr, per = _tiny_layer(M=M, k=k, mode=mode)
    out = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)
    dense = oracle_mod.moe_dense(x, wr, *per, H, I, E, k)
    scale = np.linalg.norm(out["y64"], axis=1, keepdims=True)
    assert np.all(np.abs(out["y64"] - dense) <= 1e-12 * scale)


def test_invariant_zero_codes_give_zero(oracle_mod):
    H, I, E, k = 256, 64, 16, 2
    x, wr, per = _tiny_layer()
    for zero_code in (0x00, 0x88):  # +0 and -0 in both nibbles
        z13 = [np.full_like(a, zero_code) for a in per[0]]
        out = oracle_mod.moe_decode(x, wr, z13, per[1], per[2], per[3], H, I, E, k)
        assert not out["y64"].any()
        z2 = [np.full_like(a, zero_code) for a in per[2]]
        out = oracle_mod.moe_decode(x, wr, per[0], per[1], z2, per[3], H, I, E, k)
        assert not out["y64"].any()


def _shared_expert(seed=7, H=256, I=64):
    return [np.asarray(a) for a in synth.expert_np(seed, 0, 0, H, I)]


@pytest.mark.parametrize("M,k,mode", [(1, 2, "natural"), (3, 4, "gap")])
def test_shared_expert_zero_w2_is_routed_only(oracle_mod, M, k, mode):
    # A shared expert whose down weights are all zero adds nothing: the
    # result is the routed-only step bit for bit, ids and weights included.
    H, I, E = 256, 64, 16
    x, wr, per = _tiny_layer(M=M, k=k, mode=mode)
    sh = _shared_expert()
    sh[2] = np.zeros_like(sh[2])
    base = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)
    out = oracle_mod.moe_decode_shared(x, wr, *per, sh, H, I, E, k)
    for key in ("q", "s", "logits", "ids"):
        assert np.array_equal(out[key], base[key])
    assert np.array_equal(out["weights"], base["weights"])
    assert np.array_equal(out["y64"], base["y64"])


def test_shared_expert_alone_is_one_expert_at_weight_one(oracle_mod):
    # With every routed expert's down weights zero, the layer output is the
    # shared expert applied to the quantised token, with weight exactly 1.
    H, I, E, k, M = 256, 64, 16, 2, 3
    x, wr, per = _tiny_layer(M=M, k=k, mode="gap")
    z2 = [np.zeros_like(a) for a in per[2]]
    sh = _shared_expert()
    out = oracle_mod.moe_decode_shared(x, wr, per[0], per[1], z2, per[3], sh, H, I, E, k)
    q, s = oracle_mod.quantize(x)
    for m in range(M):
        _, d = oracle_mod.expert(q[m], s[m], *sh, H, I)
        assert np.array_equal(out["y64"][m], d)
        assert np.any(d != 0)


def test_shared_expert_is_additive_and_scales(oracle_mod):
    # Raising every E8M0 down scale of the shared expert by one doubles its
    # contribution exactly, and leaves the routed part untouched.
    H, I, E, k, M = 256, 64, 16, 4, 2
    x, wr, per = _tiny_layer(M=M, k=k, mode="gap")
    sh = _shared_expert()
    base = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)["y64"]
    one = oracle_mod.moe_decode_shared(x, wr, *per, sh, H, I, E, k)["y64"]
    sh2 = list(sh)
    sh2[3] = sh[3] + 1
    two = oracle_mod.moe_decode_shared(x, wr, *per, sh2, H, I, E, k)["y64"]
    scale = np.abs(one).max() + np.abs(base).max()
    assert np.all(np.abs((two - base) - 2 * (one - base)) <= 1e-13 * scale)
    assert np.any(one != base)


def test_invariant_w2_scale_doubles_output(oracle_mod):
    H, I, E, k = 256, 64, 16, 2
    x, wr, per = _tiny_layer()
    base = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)["y64"]
    s2 = [a + 1 for a in per[3]]
    dbl = oracle_mod.moe_decode(x, wr, per[0], per[1], per[2], s2, H, I, E, k)["y64"]
    assert np.array_equal(dbl, 2 * base)


def test_invariant_expert_permutation(oracle_mod):
    H, I, E, k = 256, 64, 16, 4
    x, wr, per = _tiny_layer(M=2, k=k, mode="gap")
    base = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)
    perm = synth.permutation(11, 0, E)
    per_p = [[t[p] for p in perm] for t in per]
    out = oracle_mod.moe_decode(x, wr[perm], *per_p, H, I, E, k)
    assert np.allclose(out["y64"], base["y64"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(perm[out["ids"]], base["ids"])


def test_sum_of_weights_is_one(oracle_mod):
    x, wr, per = _tiny_layer(M=4, k=8, mode="gap")
    out = oracle_mod.moe_decode(x, wr, *per, 256, 64, 16, 8)
    assert np.all(np.abs(out["weights"].sum(axis=1) - 1.0) < 1e-15)


def test_nan_scale_is_rejected(oracle_mod):
    x, wr, per = _tiny_layer()
    bad = [a.copy() for a in per[1]]
    for a in bad:
        a[0, 0] = 0xFF
    with pytest.raises(ValueError):
        oracle_mod.moe_decode(x, wr, per[0], bad, per[2], per[3], 256, 64, 16, 16)


# ---------------------------------------------------------------- A9 RMSNorm
def test_rmsnorm_matches_torch_and_closed_form(oracle_mod):
    y = synth.gen_x(12, 3, 256) * 3.0
    got = oracle_mod.rmsnorm(bf16_bits(y), 1e-6)
    yd = y.double()
    ref = torch.nn.functional.rms_norm(yd, (256,), eps=1e-6)
    ref_bits = bf16_bits(ref.to(torch.bfloat16))
    # fp64 -> bf16 in torch may round through fp32; compare values within 1 bf16 ulp
    gv = torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).double()
    rv = torch.from_numpy(ref_bits.view(np.int16)).view(torch.bfloat16).double()
    assert torch.all((gv - rv).abs() <= rv.abs() * 2 ** -8)
    const = np.full((1, 64), 0x4040, np.uint16)  # 3.0 everywhere -> 3/sqrt(9+eps) ~ 1
    assert np.all(oracle_mod.rmsnorm(const, 1e-6) == 0x3F80)


# ---------------------------------------------------------------- FP8 LM head
def _f8_codes(v32: torch.Tensor) -> np.ndarray:
    """torch's own float32 -> float8_e4m3fn conversion (round to nearest even)."""
    return v32.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_lm_quantize_hand_row(oracle_mod):
    # row [1, 2, 3, 4]: amax 4, inv = 448/4 = 112 -> 112, 224, 336, 448.
    # OFP8 E4M3: 112 = 1.75*2^6 -> 0x6E; 224 = 1.75*2^7 -> 0x76; 336 = 1.3125*2^8
    # lies halfway between 1.25 and 1.375 and rounds to the even 1.25 -> 0x7A;
    # 448 = 1.75*2^8 -> 0x7E. Scale fl32(4/448).
    w = bf16_bits(torch.tensor([[1.0, 2.0, 3.0, 4.0], [0.0, 0.0, 0.0, 0.0]], dtype=torch.bfloat16))
    codes, scales = oracle_mod.lm_quantize(w)
    assert codes[0].tolist() == [0x6E, 0x76, 0x7A, 0x7E]
    assert codes[1].tolist() == [0, 0, 0, 0] and scales[1] == 1.0
    assert scales[0] == np.float32(4.0) / np.float32(448.0)
    # x = [1, -1, 0.5, 2]: 112 - 224 + 0.5*320 + 2*448 = 944 (in units of the scale)
    x = bf16_bits(torch.tensor([[1.0, -1.0, 0.5, 2.0]], dtype=torch.bfloat16))
    lg = oracle_mod.lm_head(codes, scales, x)
    assert lg[0, 0] == 944.0 * float(scales[0]) and lg[0, 1] == 0.0


def test_lm_quantize_matches_torch_float8(oracle_mod):
    g = torch.Generator().manual_seed(5)
    w = torch.randn(37, 96, generator=g) * torch.logspace(-3, 3, 37).unsqueeze(1)
    w[3] = 0.0
    w[7] = 0.0
    w[7, 11] = -0.75
    wb = w.to(torch.bfloat16)
    codes, scales = oracle_mod.lm_quantize(bf16_bits(wb))
    w32 = wb.float()
    amax = w32.abs().amax(dim=1)
    for v in range(w.shape[0]):
        if amax[v] == 0:
            assert np.all(codes[v] == 0) and scales[v] == 1.0
            continue
        inv = torch.tensor(448.0, dtype=torch.float32) / amax[v]
        assert np.array_equal(codes[v], _f8_codes(w32[v] * inv)), v
        assert scales[v] == (amax[v] / torch.tensor(448.0)).item()


def test_lm_head_one_hot_reads_a_column(oracle_mod):
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 256, (23, 64)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01  # no NaN codes
    scales = (2.0 ** rng.integers(-8, 8, 23)).astype(np.float32) * np.float32(1.5)
    dec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    for h in (0, 17, 63):
        x = np.zeros((1, 64), np.float32)
        x[0, h] = 1.0
        lg = oracle_mod.lm_head(codes, scales, bf16_bits(torch.from_numpy(x).to(torch.bfloat16)))
        assert np.array_equal(lg[0], dec[:, h] * scales.astype(np.float64)), h


def test_lm_head_linear_and_homogeneous(oracle_mod):
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 0x7E, (19, 128)).astype(np.uint8)
    scales = rng.uniform(0.5, 2.0, 19).astype(np.float32)
    x = torch.randn(2, 128, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    a, b = x.clone(), x.clone()
    a[:, 64:] = 0
    b[:, :64] = 0
    la = oracle_mod.lm_head(codes, scales, bf16_bits(a))
    lb = oracle_mod.lm_head(codes, scales, bf16_bits(b))
    lx = oracle_mod.lm_head(codes, scales, bf16_bits(x))
    assert np.allclose(la + lb, lx, rtol=1e-12, atol=1e-9)
    l2 = oracle_mod.lm_head(codes, scales, bf16_bits(x * 2))
    assert np.array_equal(l2, 2 * lx)


# ------------------------------------------------- FP8 intermediate (A8 down)
def _mx_decode_np(codes: np.ndarray, scales: np.ndarray, K: int) -> np.ndarray:
    """Dequantise packed MXFP4 rows [R][K/2] + [R][K/32] with numpy and the
    OCP E2M1 table fixture (low nibble = even element)."""
    table = np.zeros(16, np.float64)
    for code, val in read_golden("e2m1_values.txt"):
        table[int(code)] = float(val)
    c = np.asarray(codes, np.uint8).reshape(-1, K // 2)
    el = np.empty((c.shape[0], K), np.float64)
    el[:, 0::2] = table[c & 0xF]
    el[:, 1::2] = table[c >> 4]
    sc = 2.0 ** (np.asarray(scales, np.float64).reshape(-1, K // 32) - 127.0)
    return el * np.repeat(sc, 32, axis=1)


def test_quantize_f32_hand_and_torch(oracle_mod):
    q, s = oracle_mod.quantize_f32(np.array([1.0, 2.0, 3.0, 4.0], np.float32))
    assert q.tolist() == [0x6E, 0x76, 0x7A, 0x7E] and s == np.float32(4.0) / np.float32(448.0)
    q, s = oracle_mod.quantize_f32(np.zeros(5, np.float32))
    assert not q.any() and s == 1.0
    g = torch.Generator().manual_seed(11)
    for scale in (1e-6, 0.03, 1.0, 700.0):
        v = (torch.randn(300, generator=g) * scale).float()
        v[7] = 0.0
        v[9] = v[10] * 1e-4  # deep in the subnormal range after scaling
        q, s = oracle_mod.quantize_f32(v.numpy())
        amax = v.abs().max()
        inv = torch.tensor(448.0, dtype=torch.float32) / amax
        ref = torch.clamp(v * inv, -448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q, ref), scale
        assert s == (amax / torch.tensor(448.0)).item()


def test_expert_a8_is_the_dequantised_down_projection(oracle_mod):
    # The A8 expert = SwiGLU output h (fp64 from the plain expert, rounded to
    # fp32), quantised by torch's float8 conversion, then W2 (dequantised by
    # numpy from the MX table) times the dequantised h in fp64.
    H, I = 256, 64
    x = synth.gen_x(12, 2, H)
    q, s = oracle_mod.quantize(bf16_bits(x))
    ex = synth.expert_np(12, 0, 3, H, I)
    w2 = _mx_decode_np(ex[2], ex[3], I)  # [H][I]
    for m in range(2):
        h, _ = oracle_mod.expert(q[m], s[m], *ex, H, I)
        hq, hs, d = oracle_mod.expert_a8(q[m], s[m], *ex, H, I)
        h32 = torch.from_numpy(h.astype(np.float32))
        amax = h32.abs().max()
        inv = torch.tensor(448.0, dtype=torch.float32) / amax
        ref = torch.clamp(h32 * inv, -448.0, 448.0).to(torch.float8_e4m3fn)
        assert np.array_equal(hq, ref.view(torch.uint8).numpy())
        assert hs == (amax / torch.tensor(448.0)).item()
        hd = ref.to(torch.float64).numpy() * hs
        want = w2 @ hd
        assert np.all(np.abs(d - want) <= 1e-12 * np.abs(w2) @ np.abs(hd))
        # E4M3 rounding bound on every element, and the largest maps to 448
        err = np.abs(hd - h.astype(np.float32).astype(np.float64))
        assert np.all(err <= 2.0 ** -4 * np.abs(h) * (1 + 1e-6) + hs * 2.0 ** -10)
        assert hq[int(np.argmax(np.abs(h)))] & 0x7F == 0x7E


def test_moe_decode_a8_invariants(oracle_mod):
    H, I, E, k, M = 256, 64, 16, 4, 3
    x, wr, per = _tiny_layer(M=M, k=k, mode="gap")
    plain = oracle_mod.moe_decode(x, wr, *per, H, I, E, k)
    a8 = oracle_mod.moe_decode_a8(x, wr, *per, H, I, E, k)
    for key in ("q", "s", "logits", "ids", "weights"):
        assert np.array_equal(a8[key], plain[key])
    # quantising h moves y by a few percent of its norm: visible, not larger
    rel = np.linalg.norm(a8["y64"] - plain["y64"]) / np.linalg.norm(plain["y64"])
    assert 2e-3 < rel < 0.1, rel
    # zero down codes give zero; +1 on every down scale doubles y exactly
    z2 = [np.zeros_like(a) for a in per[2]]
    assert not oracle_mod.moe_decode_a8(x, wr, per[0], per[1], z2, per[3], H, I, E, k)["y64"].any()
    s2 = [a + 1 for a in per[3]]
    dbl = oracle_mod.moe_decode_a8(x, wr, per[0], per[1], per[2], s2, H, I, E, k)["y64"]
    assert np.array_equal(dbl, 2 * a8["y64"])
    # the shared expert adds its own A8 output with weight 1
    sh = _shared_expert()
    withsh = oracle_mod.moe_decode_a8(x, wr, *per, H, I, E, k, shared=sh)["y64"]
    qv, sv = oracle_mod.quantize(x)
    for m in range(M):
        _, _, d = oracle_mod.expert_a8(qv[m], sv[m], *sh, H, I)
        assert np.all(np.abs(withsh[m] - a8["y64"][m] - d) <= 1e-13 * (np.abs(a8["y64"][m]) + np.abs(d)))
