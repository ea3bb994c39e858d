"""Seeded synthetic inputs for the W4A8 MoE decode step.

This module only draws inputs. It holds none of the step's arithmetic: no
FP8/MXFP4 encoding or decoding, no top-k, no expert math. Both the CUDA path
and the CPU oracle receive what it produces.

Every value comes from a counter-based hash, so any slice can be regenerated
on its own. Word i of the stream for key K is SplitMix64's output function
applied to K + (i+1)*0x9E3779B97F4A7C15. SplitMix64 is the generator Steele,
Lea and Flood published (OOPSLA 2014), with the finaliser constants Vigna
uses. Each stream is keyed by (seed, layer, tensor, expert).

There are two bit-identical implementations of the integer hash: numpy
uint64 on the CPU, and torch int64 on any device (wrapping multiply, with
logical shifts built from arithmetic shifts and a mask). The CPU tests pin
them to each other.

Distributions, as configured for the benchmark workloads:
  x         bf16 RNE(fp32(N(0,1)))  (Box-Muller from one 64-bit word)
  router_w  fp32 N(0, 0.02)         (0.02 is the standard deviation)
  codes     uniform bytes, so both E2M1 nibbles are uniform over 0..15
  scales    E8M0 bytes uniform over {lo..hi}; the default {121..125} gives
            exponents -6..-2
Routing structure is forced on the router weights. Each expert row gets a
combination of the token vectors, solved from their Gram matrix in fp64, so
the logits land on chosen targets. The modes are "natural" (no change),
"gap", "distinct", "shared" and "zipf"; force_router() documents each one.
"""
from __future__ import annotations

import math

import numpy as np
import torch

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
C1 = 0xBF58476D1CE4E5B9
C2 = 0x94D049BB133111EB

# tensor ids inside a stream key
T_X, T_ROUTER, T_W13C, T_W13S, T_W2C, T_W2S, T_PERM, T_JITTER = range(1, 9)


def _signed(v: int) -> int:
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix_int(z: int) -> int:
    """SplitMix64 output function on a Python int (exact, mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * C1) & MASK64
    z = ((z ^ (z >> 27)) * C2) & MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, layer: int, tensor: int, expert: int = 0) -> int:
    k = mix_int(seed + GAMMA)
    k = mix_int(k ^ (layer + 1))
    k = mix_int(k ^ (tensor * 0x100000001B3))
    k = mix_int(k ^ (expert + 1))
    return k


# ---- numpy (CPU) implementation --------------------------------------------
def _mix_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(C1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(C2)
    return z ^ (z >> np.uint64(31))


def words_np(key: int, start: int, count: int) -> np.ndarray:
    """Words start..start+count-1 of stream `key` as uint64."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix_np(np.uint64(key) + i * np.uint64(GAMMA))


# ---- torch implementation (int64 two's complement) -------------------------
def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix_t(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _signed(C1)
    z = (z ^ _lsr(z, 27)) * _signed(C2)
    return z ^ _lsr(z, 31)


def words_torch(keys: torch.Tensor, start: int, count: int) -> torch.Tensor:
    """keys: int64 [n] (signed views of the 64-bit keys) -> int64 [n, count]."""
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=keys.device)
    z = keys.view(-1, 1) + i.view(1, -1) * _signed(GAMMA)
    return _mix_t(z)


# ---- byte streams -----------------------------------------------------------
def _scale_bytes(raw: np.ndarray | torch.Tensor, lo: int, hi: int):
    n = hi - lo + 1
    if isinstance(raw, np.ndarray):
        return (lo + ((raw.astype(np.uint16) * n) >> 8)).astype(np.uint8)
    return (lo + ((raw.to(torch.int32) * n) >> 8)).to(torch.uint8)


def expert_sizes(H: int, I: int):
    """Bytes per expert of (w13 codes, w13 scales, w2 codes, w2 scales)."""
    return (2 * I * H // 2, 2 * I * H // 32, H * I // 2, H * I // 32)


def expert_np(seed: int, layer: int, e: int, H: int, I: int, scale_lo=121, scale_hi=125):
    """One expert's MXFP4 tensors on the CPU:
    (w13c [2I,H/2], w13s [2I,H/32], w2c [H,I/2], w2s [H,I/32]), all uint8."""
    shapes = [(2 * I, H // 2), (2 * I, H // 32), (H, I // 2), (H, I // 32)]
    out = []
    for t, shp in zip((T_W13C, T_W13S, T_W2C, T_W2S), shapes):
        nbytes = shp[0] * shp[1]
        nw = (nbytes + 7) // 8
        raw = words_np(stream_key(seed, layer, t, e), 0, nw).view(np.uint8)[:nbytes]
        if t in (T_W13S, T_W2S):
            raw = _scale_bytes(raw, scale_lo, scale_hi)
        out.append(raw.reshape(shp).copy())
    return tuple(out)


def layer_experts_torch(seed: int, layer: int, E: int, H: int, I: int, device,
                        scale_lo=121, scale_hi=125, chunk_bytes=1 << 28):
    """All E experts of one layer on `device`:
    (w13c [E,2I,H/2], w13s [E,2I,H/32], w2c [E,H,I/2], w2s [E,H,I/32]) uint8."""
    shapes = [(2 * I, H // 2), (2 * I, H // 32), (H, I // 2), (H, I // 32)]
    out = []
    for t, shp in zip((T_W13C, T_W13S, T_W2C, T_W2S), shapes):
        nbytes = shp[0] * shp[1]
        nw = (nbytes + 7) // 8
        dst = torch.empty((E, nbytes), dtype=torch.uint8, device=device)
        per = max(1, chunk_bytes // max(1, nw * 8 * 4))
        for e0 in range(0, E, per):
            e1 = min(E, e0 + per)
            keys = torch.tensor([_signed(stream_key(seed, layer, t, e)) for e in range(e0, e1)],
                                dtype=torch.int64, device=device)
            raw = words_torch(keys, 0, nw).view(torch.uint8).view(e1 - e0, nw * 8)[:, :nbytes]
            if t in (T_W13S, T_W2S):
                raw = _scale_bytes(raw, scale_lo, scale_hi)
            dst[e0:e1].copy_(raw)
        out.append(dst.view(E, *shp))
    return tuple(out)


# ---- Gaussian draws (CPU, fp64) ----------------------------------------------
def normal_np(key: int, count: int) -> np.ndarray:
    """count N(0,1) draws, fp64: Box-Muller on the two 32-bit halves of a word."""
    w = words_np(key, 0, count)
    hi = (w >> np.uint64(32)).astype(np.float64)
    lo = (w & np.uint64(0xFFFFFFFF)).astype(np.float64)
    u1 = (hi + 1.0) / 4294967296.0
    u2 = lo / 4294967296.0
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def gen_x(seed: int, M: int, H: int, layer: int = 0) -> torch.Tensor:
    """Activations x [M,H] bf16 = RNE(fp32(N(0,1))) on the CPU."""
    z = normal_np(stream_key(seed, layer, T_X), M * H).astype(np.float32)
    return torch.from_numpy(z.reshape(M, H)).to(torch.bfloat16)


def gen_router(seed: int, layer: int, E: int, H: int, std: float = 0.02) -> np.ndarray:
    """Router weights [E,H] fp32 ~ N(0, std)."""
    z = normal_np(stream_key(seed, layer, T_ROUTER), E * H) * std
    return z.astype(np.float32).reshape(E, H)


def permutation(seed: int, layer: int, n: int, salt: int = 0) -> np.ndarray:
    """Seeded permutation of 0..n-1 (argsort of hash words)."""
    w = words_np(stream_key(seed, layer, T_PERM, salt), 0, n)
    return np.argsort(w, kind="stable")


def zipf_bias(seed: int, layer: int, E: int, s: float = 1.1) -> np.ndarray:
    """log p_e with p_e proportional to rank_e^-s over a seeded expert order."""
    perm = permutation(seed, layer, E, salt=1)
    rank = np.empty(E, np.float64)
    rank[perm] = np.arange(1, E + 1, dtype=np.float64)
    return -s * np.log(rank)


def _enforce_gap(T: np.ndarray, k: int, gap: float) -> np.ndarray:
    """Raise the top-k entries of each row of T as needed so that the k+1
    leading values are strictly decreasing with steps >= gap; the (k+1)-th and
    everything below it are untouched, so the top-k set is unchanged."""
    T = T.copy()
    M, E = T.shape
    kk = min(k, E - 1)
    for m in range(M):
        order = np.argsort(-T[m], kind="stable")
        for j in range(kk - 1, -1, -1):
            lo = T[m, order[j + 1]]
            if T[m, order[j]] < lo + gap:
                T[m, order[j]] = lo + gap
    return T


def force_router(x: torch.Tensor, router_w: np.ndarray, k: int, mode: str = "gap",
                 seed: int = 0, layer: int = 0, gap: float = 1e-3,
                 zipf_s: float = 1.1) -> np.ndarray:
    """Return router weights (fp32 [E,H]) whose fp64 logits against x hit the
    mode's targets. Input construction only: both sides recompute the logits
    from the returned weights.

    modes:
      natural  - unchanged
      gap      - consecutive gaps among each token's k+1 largest logits >= gap
      distinct - the M tokens select M*k distinct experts (needs M*k <= E)
      shared   - all tokens select the same k experts
      zipf     - log-prior log p_e (Zipf(s) over a seeded expert order) added
                 to every token's logits, then the gap rule
    """
    if mode == "natural":
        return router_w
    X = x.to(torch.float64).cpu().numpy()  # bf16 values exactly
    W = router_w.astype(np.float64)
    M, H = X.shape
    E = W.shape[0]
    L0 = X @ W.T
    if mode == "gap":
        T = _enforce_gap(L0, k, gap)
    elif mode == "zipf":
        T = _enforce_gap(L0 + zipf_bias(seed, layer, E, zipf_s)[None, :], k, gap)
    elif mode in ("distinct", "shared"):
        if mode == "distinct" and M * k > E:
            raise ValueError("distinct routing needs M*k <= E")
        perm = permutation(seed, layer, E, salt=2)
        T = L0.copy()
        jit = words_np(stream_key(seed, layer, T_JITTER), 0, M * k).astype(np.float64)
        jit = (jit / 2.0 ** 64).reshape(M, k)
        for m in range(M):
            chosen = perm[m * k:(m + 1) * k] if mode == "distinct" else perm[:k]
            rest = np.setdiff1d(np.arange(E), chosen)
            top_rest = L0[m, rest].max()
            for j, e in enumerate(chosen):
                T[m, e] = top_rest + 0.25 + 0.3 * (k - 1 - j) + 0.1 * jit[m, j]
    else:
        raise ValueError(f"unknown routing mode {mode!r}")
    D = T - L0  # [M,E]
    G = X @ X.T  # [M,M]
    A = np.linalg.solve(G, D)  # [M,E]
    W2 = W + A.T @ X
    return W2.astype(np.float32)
