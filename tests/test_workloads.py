"""The seeded input generator: determinism, bf16 rounding and layout."""
import os

import numpy as np
import torch

from content_routed_block_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -2.0, 0.0, 3.4e38], np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(W.to_bf16_bits(x), want)
    back = torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(W.bf16_bits_to_float32(want), back)


def test_zorder_matches_quadtree_golden():
    grid = np.loadtxt(os.path.join(GOLDEN, "zorder_4x4.txt"), dtype=np.int64)
    r, c = np.meshgrid(np.arange(4), np.arange(4), indexing="ij")
    np.testing.assert_array_equal(W.morton_rc(r, c, 2), grid)
    g = W.zorder_sequence_to_grid(4)
    np.testing.assert_array_equal(grid.ravel()[g], np.arange(16))


def test_zorder_is_recursive_quadrants():
    side = 128
    g = W.zorder_sequence_to_grid(side)
    assert sorted(g.tolist()) == list(range(side * side))
    # each run of 4**L consecutive tokens is one aligned 2**L x 2**L square
    for L in (1, 3, 5):
        run = 4 ** L
        blk = g[:run * 7].reshape(7, run)
        rr, cc = blk // side, blk % side
        assert ((rr.max(1) - rr.min(1)) == 2 ** L - 1).all()
        assert ((cc.max(1) - cc.min(1)) == 2 ** L - 1).all()


def test_generators_are_deterministic_and_headwise():
    w = W.CONFIGS[1].with_(N=256, Hq=4, Hkv=2)
    a, b = W.make_inputs(w), W.make_inputs(w)
    for n in "qkv":
        np.testing.assert_array_equal(a[n], b[n])
    sub = W.make_inputs(w, q_heads=[3], kv_heads=[1])
    np.testing.assert_array_equal(sub["q"][:, 0], a["q"][:, 3])
    np.testing.assert_array_equal(sub["k"][:, 0], a["k"][:, 1])


def test_clustered_structure():
    w = W.CONFIGS[2].with_(N=4096, Hq=4, Hkv=2)
    x = W.make_inputs(w)
    k = W.bf16_bits_to_float32(x["k"]).astype(np.float64)
    blocks = k.reshape(1, 2, 64, 64, 64)
    within = blocks.std(axis=3).mean()
    assert 0.25 < within < 0.35            # sigma_within = 0.3
    sub = W.make_inputs(w, q_heads=[1], kv_heads=[0])
    np.testing.assert_array_equal(sub["q"][:, 0], x["q"][:, 1])


def test_needle_structure():
    w = W.CONFIGS[3].with_(B=1, Hq=2, Hkv=2, N=8192, needles=8)
    x = W.make_inputs(w)
    q = W.bf16_bits_to_float32(x["q"])[0, 0]
    k = W.bf16_bits_to_float32(x["k"])[0, 0]
    # a query equal to a quarter of a key exists for each needle, 4096+ later
    found = 0
    for t in range(4096, 8192):
        hits = np.flatnonzero((np.abs(k[:4096] - 4 * q[t]) == 0).all(axis=1))
        for p in hits:
            assert t - p >= 4096
            found += 1
    assert found == 8


def test_image_fields_are_smooth_and_unit_scale():
    w = W.CONFIGS[4].with_(B=1, Hq=1, Hkv=1, N=64 * 64)
    x = W.make_inputs(w)
    f = W.bf16_bits_to_float32(x["k"])[0, 0].astype(np.float64)
    assert 0.85 < f.std() < 1.2
    # neighbouring tokens in Z-order are strongly correlated
    cor = np.mean(np.sum(f[:-1] * f[1:], axis=1)) / np.mean(np.sum(f * f, axis=1))
    assert cor > 0.8
