"""The seeded input recipe: determinism, shapes, dtype rounding, mask counts."""
import numpy as np

import workloads as W


def test_seeded_and_deterministic():
    w = W.WORKLOADS["gated_bf16_n4k"].with_shape(B=2, H=3)
    a = W.make_all(w)
    b = W.make_all(w)
    for key in ("u", "k", "w", "v"):
        assert np.array_equal(a[key], b[key])
    assert a["u"].shape == (2, 3, 4096) and a["k"].shape == (3, 4096)


def test_dtype_rounding_is_idempotent():
    for name in ("gated_bf16_n4k", "fp16_n32k"):
        w = W.WORKLOADS[name].with_shape(B=1, H=2, N=1024)
        u = W.make_input(w)
        assert np.array_equal(W.round_to(u, w.dtype), u)


def test_mask_has_exact_sparsity():
    w = W.WORKLOADS["sparse_bf16_n8k"]
    m = W.make_mask(w)
    assert m.shape == (1, 8192 // 32)
    assert int((m == 0).sum()) == 192


def test_partial_filter_length_scales():
    w = W.WORKLOADS["partial_bf16_n8k"]
    assert w.L == 2048
    r = w.with_shape(B=1, H=2, N=4096)
    assert r.L == 1024


def test_dna_input_takes_four_values_per_channel():
    w = W.WORKLOADS["dna_bf16_n1m"].with_shape(H=3, N=4096)
    u = W.make_input(w)
    for h in range(3):
        assert len(np.unique(u[0, h])) <= 4


def test_sample_points_cover_edges():
    w = W.WORKLOADS["fp32_n1k"]
    s, t = W.sample_points(w, nseq=4, nrand=5)
    assert len(s) == len(t) == 4 * 8
    assert set([0, 1, w.N - 1]).issubset(set(t.tolist()))


def test_channel_shards_own_streams_share_symbols_and_mask():
    base = W.WORKLOADS["dna_bf16_n1m"].with_shape(H=4, N=4096)
    s0, s1 = W.shard_of(base, 0), W.shard_of(base, 1)
    assert np.array_equal(W.make_input(s0), W.make_input(base))     # shard 0 is the workload
    u0, u1 = W.make_input(s0), W.make_input(s1)
    assert not np.array_equal(u0, u1)                              # own projection
    # the symbol stream is shared: positions that carry one symbol on shard 0
    # (equal columns across all channels) carry one symbol on shard 1 too
    key0 = [tuple(u0[0, :, t]) for t in range(base.N)]
    key1 = [tuple(u1[0, :, t]) for t in range(base.N)]
    first = {}
    for t, kk in enumerate(key0):
        first.setdefault(kk, t)
    for t, kk in enumerate(key0):
        assert key1[t] == key1[first[kk]]
    sp = W.WORKLOADS["sparse_bf16_n8k"].with_shape(B=1, H=2)
    assert np.array_equal(W.make_mask(W.shard_of(sp, 3)), W.make_mask(sp))
    assert not np.array_equal(W.make_filter(W.shard_of(sp, 3)), W.make_filter(sp))
