"""The seeded input generator: published SplitMix64 values, numpy/torch
bit-identity, distributions, and the forced routing structures (checked on
the oracle's own fp64 logits)."""
import numpy as np
import torch

from mxfp4_weight_streaming_fp8_b200 import synth


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with 0: the first outputs of the reference generator
    # (state += 0x9E3779B97F4A7C15, then the output mix).
    w = synth.words_np(0, 0, 3)
    assert [int(v) for v in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_numpy_and_torch_streams_identical():
    keys = [synth.stream_key(0, l, t, e) for l in (0, 31) for t in (synth.T_W13C, synth.T_W2S) for e in (0, 255)]
    kt = torch.tensor([synth._signed(k) for k in keys], dtype=torch.int64)
    wt = synth.words_torch(kt, 1000, 4096).numpy().view(np.uint64)
    for i, k in enumerate(keys):
        assert np.array_equal(wt[i], synth.words_np(k, 1000, 4096))


def test_layer_generator_matches_expert_slices():
    H, I, E = 256, 64, 16
    full = synth.layer_experts_torch(3, 2, E, H, I, "cpu", chunk_bytes=1 << 16)
    for e in (0, 7, 15):
        part = synth.expert_np(3, 2, e, H, I)
        for a, b in zip(full, part):
            assert np.array_equal(a[e].numpy(), b)


def test_distributions():
    H, I = 2560, 768
    w13c, w13s, w2c, w2s = synth.expert_np(0, 0, 0, H, I)
    assert set(np.unique(w13s)) == {121, 122, 123, 124, 125}
    nib = np.concatenate([w13c.ravel() & 0xF, w13c.ravel() >> 4])
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.9 * nib.size / 16 and counts.max() < 1.1 * nib.size / 16
    x = synth.gen_x(0, 8, H).float()
    assert abs(x.mean()) < 0.05 and abs(x.std() - 1) < 0.05
    wr = synth.gen_router(0, 0, 256, H)
    assert abs(wr.std() - 0.02) < 5e-4


def _logits(oracle_mod, x, wr):
    bits = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    return oracle_mod.router_logits(bits, wr)


def test_forced_gap(oracle_mod):
    H, E, k = 2560, 256, 8
    x = synth.gen_x(0, 4, H)
    wr = synth.force_router(x, synth.gen_router(0, 0, E, H), k, "gap")
    l = _logits(oracle_mod, x, wr)
    for m in range(4):
        top = np.sort(l[m])[::-1][:k + 1]
        assert np.all(np.diff(top) <= -0.9e-3)


def test_forced_distinct_and_shared(oracle_mod):
    H, E, k, M = 2560, 256, 8, 4
    x = synth.gen_x(0, M, H)
    wr = synth.force_router(x, synth.gen_router(0, 0, E, H), k, "distinct")
    ids, _ = oracle_mod.topk(_logits(oracle_mod, x, wr), k)
    assert len(set(ids.ravel().tolist())) == M * k
    wr = synth.force_router(x, synth.gen_router(0, 0, E, H), k, "shared")
    ids, _ = oracle_mod.topk(_logits(oracle_mod, x, wr), k)
    assert len(set(ids.ravel().tolist())) == k


def test_forced_zipf_skews_popularity(oracle_mod):
    H, E, k, M = 2560, 256, 8, 32
    x = synth.gen_x(0, M, H)
    wr = synth.force_router(x, synth.gen_router(0, 0, E, H), k, "zipf")
    ids, _ = oracle_mod.topk(_logits(oracle_mod, x, wr), k)
    U = len(set(ids.ravel().tolist()))
    assert U < M * k * 0.8  # popular experts are shared between tokens
