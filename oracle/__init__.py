"""Python access to the C++ CPU oracle (``moe_oracle.cpp``) through ctypes.

TEST INFRASTRUCTURE ONLY. The test suite, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only callers;
the product path (``mxfp4_weight_streaming_fp8_b200``) never imports this
package and shares no code with it.

Each wrapper takes numpy arrays with the layouts documented in
``moe_oracle.h`` and returns numpy arrays. The library is built by
``oracle.build.build()`` (g++, no fast-math).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build, LIB_PATH

_lib = None

_u8p = ctypes.POINTER(ctypes.c_uint8)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u8pp = ctypes.POINTER(_u8p)


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            build()
        L = ctypes.CDLL(LIB_PATH)
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e8m0_value.restype = ctypes.c_double
        L.oracle_e8m0_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_encode.restype = ctypes.c_int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_bf16_value.restype = ctypes.c_double
        L.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_round.restype = ctypes.c_uint16
        L.oracle_bf16_round.argtypes = [ctypes.c_double]
        L.oracle_quantize.argtypes = [ctypes.c_int, ctypes.c_int, _u16p, _u8p, _f32p]
        L.oracle_router_logits.argtypes = [ctypes.c_int] * 3 + [_u16p, _f32p, _f64p]
        L.oracle_topk.argtypes = [ctypes.c_int] * 3 + [_f64p, _i32p, _f64p]
        L.oracle_union.argtypes = [ctypes.c_int] * 3 + [_i32p] * 5
        L.oracle_expert.argtypes = [ctypes.c_int, ctypes.c_int, _u8p, ctypes.c_float,
                                    _u8p, _u8p, _u8p, _u8p, _f64p, _f64p]
        L.oracle_moe_decode.argtypes = ([ctypes.c_int] * 5 + [_u16p, _f32p] + [_u8pp] * 4 +
                                        [_u8p, _f32p, _f64p, _i32p, _f64p, _f64p, _u16p])
        L.oracle_moe_dense.argtypes = [ctypes.c_int] * 5 + [_u16p, _f32p] + [_u8pp] * 4 + [_f64p]
        L.oracle_rmsnorm.argtypes = [ctypes.c_int, ctypes.c_int, _u16p, ctypes.c_double, _u16p]
        L.oracle_moe_decode_shared.argtypes = ([ctypes.c_int] * 5 + [_u16p, _f32p] + [_u8pp] * 4 + [_u8p] * 4 +
                                               [_u8p, _f32p, _f64p, _i32p, _f64p, _f64p])
        L.oracle_quantize_f32.argtypes = [ctypes.c_int, _f32p, _u8p, _f32p]
        L.oracle_expert_a8.argtypes = [ctypes.c_int, ctypes.c_int, _u8p, ctypes.c_float] + [_u8p] * 4 + [
            _u8p, _f32p, _f64p]
        L.oracle_moe_decode_a8.argtypes = ([ctypes.c_int] * 5 + [_u16p, _f32p] + [_u8pp] * 4 + [_u8p] * 4 +
                                           [_u8p, _f32p, _f64p, _i32p, _f64p, _f64p])
        L.oracle_lm_quantize.argtypes = [ctypes.c_int, ctypes.c_int, _u16p, _u8p, _f32p]
        L.oracle_lm_head.argtypes = [ctypes.c_int] * 3 + [_u8p, _f32p, _u16p, _f64p]
        _lib = L
    return _lib


def _p(a, ptype):
    return a.ctypes.data_as(ptype)


def _check(rc, what):
    if rc < 0:
        raise ValueError(f"oracle {what} failed with code {rc}")
    return rc


# ---- element formats ------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e8m0_value(b: int) -> float:
    return lib().oracle_e8m0_value(int(b))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(v))


def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(int(bits))


def bf16_round(v: float) -> int:
    return lib().oracle_bf16_round(float(v))


# ---- steps ----------------------------------------------------------------
def quantize(x_bits: np.ndarray):
    """A1. x_bits: uint16 [M,H] bf16 patterns -> (codes uint8 [M,H], s float32 [M])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, H = x.shape
    q = np.zeros((M, H), np.uint8)
    s = np.zeros(M, np.float32)
    _check(lib().oracle_quantize(M, H, _p(x, _u16p), _p(q, _u8p), _p(s, _f32p)), "quantize")
    return q, s


def router_logits(x_bits: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    w = np.ascontiguousarray(router_w, dtype=np.float32)
    M, H = x.shape
    E = w.shape[0]
    out = np.zeros((M, E), np.float64)
    _check(lib().oracle_router_logits(M, H, E, _p(x, _u16p), _p(w, _f32p), _p(out, _f64p)), "logits")
    return out


def topk(logits: np.ndarray, k: int):
    lg = np.ascontiguousarray(logits, dtype=np.float64)
    M, E = lg.shape
    ids = np.zeros((M, k), np.int32)
    w = np.zeros((M, k), np.float64)
    _check(lib().oracle_topk(M, E, k, _p(lg, _f64p), _p(ids, _i32p), _p(w, _f64p)), "topk")
    return ids, w


def union(ids: np.ndarray, E: int):
    """A4 -> (union_ids [U], pair_off [U+1], pair_tok [M*k], pair_slot [M*k])."""
    iv = np.ascontiguousarray(ids, dtype=np.int32)
    M, k = iv.shape
    uid = np.zeros(M * k, np.int32)
    off = np.zeros(M * k + 1, np.int32)
    tok = np.zeros(M * k, np.int32)
    slot = np.zeros(M * k, np.int32)
    U = _check(lib().oracle_union(M, E, k, _p(iv, _i32p), _p(uid, _i32p), _p(off, _i32p),
                                  _p(tok, _i32p), _p(slot, _i32p)), "union")
    return uid[:U].copy(), off[:U + 1].copy(), tok, slot


def expert(q_m, s_m, w13c, w13s, w2c, w2s, H, I):
    """A5-A7 for one token: returns (h [I], d [H]) in fp64."""
    q = np.ascontiguousarray(q_m, dtype=np.uint8)
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (w13c, w13s, w2c, w2s)]
    h = np.zeros(I, np.float64)
    d = np.zeros(H, np.float64)
    _check(lib().oracle_expert(H, I, _p(q, _u8p), float(s_m), *[_p(a, _u8p) for a in arrs],
                               _p(h, _f64p), _p(d, _f64p)), "expert")
    return h, d


def _expert_ptrs(per_expert, E):
    """Array of E uint8* (NULL where the entry is None); keeps arrays alive."""
    keep = []
    arr = (_u8p * E)()
    for e in range(E):
        a = per_expert[e] if per_expert is not None else None
        if a is None:
            arr[e] = _u8p()
        else:
            c = np.ascontiguousarray(a, dtype=np.uint8)
            keep.append(c)
            arr[e] = _p(c, _u8p)
    return arr, keep


def moe_decode(x_bits, router_w, w13c, w13s, w2c, w2s, H, I, E, k):
    """A1-A8. w13c etc: sequences of E per-expert arrays (None for unused).

    Returns dict with q, s, logits, ids, weights, y64, y_bf16.
    """
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(router_w, dtype=np.float32)
    M = x.shape[0]
    ptrs = [_expert_ptrs(t, E) for t in (w13c, w13s, w2c, w2s)]
    out = dict(q=np.zeros((M, H), np.uint8), s=np.zeros(M, np.float32),
               logits=np.zeros((M, E), np.float64), ids=np.zeros((M, k), np.int32),
               weights=np.zeros((M, k), np.float64), y64=np.zeros((M, H), np.float64),
               y_bf16=np.zeros((M, H), np.uint16))
    _check(lib().oracle_moe_decode(
        H, I, E, k, M, _p(x, _u16p), _p(wr, _f32p), *[p[0] for p in ptrs],
        _p(out["q"], _u8p), _p(out["s"], _f32p), _p(out["logits"], _f64p),
        _p(out["ids"], _i32p), _p(out["weights"], _f64p), _p(out["y64"], _f64p),
        _p(out["y_bf16"], _u16p)), "moe_decode")
    return out


def moe_decode_shared(x_bits, router_w, w13c, w13s, w2c, w2s, shared, H, I, E, k):
    """A1-A8 plus one always-active shared expert; shared = (w13c, w13s, w2c,
    w2s) arrays of one expert. Returns dict with q, s, logits, ids, weights,
    y64."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(router_w, dtype=np.float32)
    M = x.shape[0]
    ptrs = [_expert_ptrs(t, E) for t in (w13c, w13s, w2c, w2s)]
    sh = [np.ascontiguousarray(a, dtype=np.uint8) for a in shared]
    out = dict(q=np.zeros((M, H), np.uint8), s=np.zeros(M, np.float32),
               logits=np.zeros((M, E), np.float64), ids=np.zeros((M, k), np.int32),
               weights=np.zeros((M, k), np.float64), y64=np.zeros((M, H), np.float64))
    _check(lib().oracle_moe_decode_shared(
        H, I, E, k, M, _p(x, _u16p), _p(wr, _f32p), *[p[0] for p in ptrs], *[_p(a, _u8p) for a in sh],
        _p(out["q"], _u8p), _p(out["s"], _f32p), _p(out["logits"], _f64p), _p(out["ids"], _i32p), _p(out["weights"], _f64p), _p(out["y64"], _f64p)), "moe_decode_shared")
    return out


def quantize_f32(v):
    """A1 rule on one fp32 vector: (codes uint8 [n], scale float)."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    q = np.zeros(a.shape[0], np.uint8)
    s = np.zeros(1, np.float32)
    _check(lib().oracle_quantize_f32(a.shape[0], _p(a, _f32p), _p(q, _u8p), _p(s, _f32p)), "quantize_f32")
    return q, float(s[0])


def expert_a8(q_m, s_m, w13c, w13s, w2c, w2s, H, I):
    """A5-A7 with the FP8 intermediate: returns (hq [I] uint8, hs, d [H])."""
    q = np.ascontiguousarray(q_m, dtype=np.uint8)
    arrs = [np.ascontiguousarray(a, dtype=np.uint8) for a in (w13c, w13s, w2c, w2s)]
    hq = np.zeros(I, np.uint8)
    hs = np.zeros(1, np.float32)
    d = np.zeros(H, np.float64)
    _check(lib().oracle_expert_a8(H, I, _p(q, _u8p), float(s_m), *[_p(a, _u8p) for a in arrs],
                                  _p(hq, _u8p), _p(hs, _f32p), _p(d, _f64p)), "expert_a8")
    return hq, float(hs[0]), d


def moe_decode_a8(x_bits, router_w, w13c, w13s, w2c, w2s, H, I, E, k, shared=None):
    """A1-A8 with the FP8 intermediate for every expert; shared = (w13c,
    w13s, w2c, w2s) of one shared expert or None. Returns dict with q, s,
    logits, ids, weights, y64."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(router_w, dtype=np.float32)
    M = x.shape[0]
    ptrs = [_expert_ptrs(t, E) for t in (w13c, w13s, w2c, w2s)]
    sh = [np.ascontiguousarray(a, dtype=np.uint8) for a in shared] if shared is not None else None
    shp = [_p(a, _u8p) for a in sh] if sh is not None else [_u8p()] * 4
    out = dict(q=np.zeros((M, H), np.uint8), s=np.zeros(M, np.float32),
               logits=np.zeros((M, E), np.float64), ids=np.zeros((M, k), np.int32),
               weights=np.zeros((M, k), np.float64), y64=np.zeros((M, H), np.float64))
    _check(lib().oracle_moe_decode_a8(
        H, I, E, k, M, _p(x, _u16p), _p(wr, _f32p), *[p[0] for p in ptrs], *shp,
        _p(out["q"], _u8p), _p(out["s"], _f32p), _p(out["logits"], _f64p), _p(out["ids"], _i32p),
        _p(out["weights"], _f64p), _p(out["y64"], _f64p)), "moe_decode_a8")
    return out


def moe_dense(x_bits, router_w, w13c, w13s, w2c, w2s, H, I, E, k):
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(router_w, dtype=np.float32)
    M = x.shape[0]
    ptrs = [_expert_ptrs(t, E) for t in (w13c, w13s, w2c, w2s)]
    y = np.zeros((M, H), np.float64)
    _check(lib().oracle_moe_dense(H, I, E, k, M, _p(x, _u16p), _p(wr, _f32p),
                                  *[p[0] for p in ptrs], _p(y, _f64p)), "moe_dense")
    return y


def rmsnorm(y_bits, eps=1e-6):
    y = np.ascontiguousarray(y_bits, dtype=np.uint16)
    M, H = y.shape
    out = np.zeros((M, H), np.uint16)
    _check(lib().oracle_rmsnorm(M, H, _p(y, _u16p), float(eps), _p(out, _u16p)), "rmsnorm")
    return out


def lm_quantize(w_bits: np.ndarray):
    """FP8 LM head weights: uint16 bf16 [V,H] -> (codes uint8 [V,H], scales float32 [V])."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    V, H = w.shape
    codes = np.zeros((V, H), np.uint8)
    scales = np.zeros(V, np.float32)
    _check(lib().oracle_lm_quantize(V, H, _p(w, _u16p), _p(codes, _u8p), _p(scales, _f32p)), "lm_quantize")
    return codes, scales


def lm_head(codes: np.ndarray, scales: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """fp64 logits [M,V] of the FP8 LM head for bf16 activations x [M,H]."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(scales, dtype=np.float32)
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    V, H = c.shape
    M = x.shape[0]
    out = np.zeros((M, V), np.float64)
    _check(lib().oracle_lm_head(V, H, M, _p(c, _u8p), _p(s, _f32p), _p(x, _u16p), _p(out, _f64p)), "lm_head")
    return out
