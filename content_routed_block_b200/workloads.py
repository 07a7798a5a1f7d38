"""Seeded synthetic inputs for content-routed block-sparse attention.

This module is shared by the CUDA path (bench, GPU tests) and by the oracle's
tests. It holds none of the method's arithmetic: it only draws Q, K, V with
the shapes, value distributions and structure of the workloads the method is
evaluated on, rounds them to bf16 (round-to-nearest-even) and returns the raw
bf16 bit patterns as ``uint16`` arrays, so both sides consume the same bytes.

Workloads (all seeded with ``numpy.random.default_rng``; every tensor is drawn
from its own child stream ``[seed, tag, b, head]`` so that any head can be
regenerated alone):

* ``iid``       -- Q, K, V iid N(0, 1).
* ``clustered`` -- per (batch, KV head) ``centres`` Gaussian centres N(0, I);
  each key block takes one centre uniformly at random and its keys are
  centre + N(0, 0.3^2); query i is a copy of a uniformly drawn earlier key
  j in [0, i-1] of its KV group (query 0 copies key 0) plus N(0, 0.5^2);
  V iid N(0, 1).  Routing is non-trivial because block means mix the
  targets of several queries.
* ``needles``   -- iid N(0, 1) background; per (batch, head) 64 distinct
  needle positions p in [0, N-4096-1]; K[p] is scaled by 4, V[p] is redrawn,
  and one distinct query position t in [p+4096, N-1] gets Q[t] = the
  unscaled K[p].  An isolated needle is diluted 1:Bk in its block mean, the
  adversarial case for summary routing (jonsmirl/ssa README, "Algorithm and
  complexity", the paragraph on the retrieval law).
* ``image``     -- per (batch, head, channel) white noise on a side x side
  grid, circularly filtered by a Gaussian of sigma = 4 px truncated at 4 sigma
  (separable, periodic boundary), rescaled to unit variance by the filter's
  exact gain, plus N(0, 0.1^2) noise; Q, K, V are independent fields; tokens
  are laid out in quadtree Z-order (SingleZombie/LLSA README, "Preprocessing
  for Non-Sequential Data": reorder so that similar tokens are adjacent).
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import math

import numpy as np

__all__ = [
    "Workload", "CONFIGS", "make_inputs", "to_bf16_bits", "bf16_bits_to_float32",
    "morton_rc", "zorder_sequence_to_grid",
]

# child-stream tags: one per drawn tensor family
_TAG_Q, _TAG_K, _TAG_V, _TAG_CLUSTER, _TAG_NEEDLE, _TAG_IMG = 1, 2, 3, 4, 5, 6


@dataclass(frozen=True)
class Workload:
    """Shapes and method parameters of one synthetic workload."""
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    block_k: int
    block_q: int
    top_k: int
    window: int
    causal: bool
    kind: str = "iid"          # iid | clustered | needles | image
    seed: int = 0
    centres: int = 64          # clustered only
    needles: int = 64          # needles only
    needle_gap: int = 4096     # needles only: minimum query-after-key distance
    consensus: bool = False    # one route per (batch, KV head, query block), voted by its heads
    beta: float = 0.0          # weight of the second-cumulant routing term
    tree_fanout: int = 0       # two-level routing: key blocks per super-block (0: flat)
    tree_beam: int = 0         # two-level routing: super-blocks kept per query block

    @property
    def n_kblocks(self) -> int:
        return self.N // self.block_k

    @property
    def n_qblocks(self) -> int:
        return self.N // self.block_q

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five evaluation workloads.  Query block = key block everywhere (one
# block size, as LLSA's single ``block_size`` argument and the first
# workload's stated "query block 64").
CONFIGS = {
    1: Workload("iid-1k", B=1, Hq=2, Hkv=2, N=1024, D=64, block_k=64, block_q=64,
                top_k=4, window=128, causal=True, kind="iid", seed=0),
    2: Workload("gqa-clustered-32k", B=1, Hq=14, Hkv=2, N=32768, D=64, block_k=64,
                block_q=64, top_k=16, window=512, causal=True, kind="clustered",
                seed=1, centres=64),
    3: Workload("needles-8k-d128", B=4, Hq=16, Hkv=16, N=8192, D=128, block_k=64,
                block_q=64, top_k=8, window=256, causal=True, kind="needles", seed=2),
    4: Workload("image-zorder-16k", B=2, Hq=16, Hkv=16, N=16384, D=64, block_k=16,
                block_q=16, top_k=8, window=0, causal=False, kind="image", seed=3),
    5: Workload("gqa-clustered-1m", B=1, Hq=14, Hkv=2, N=1048576, D=64, block_k=64,
                block_q=64, top_k=16, window=1024, causal=True, kind="clustered",
                seed=4, centres=1024),
}


# ----------------------------------------------------------------------------
# bf16 conversions (bit level, no dependency on torch)
# ----------------------------------------------------------------------------
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_float32(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Z-order layout of an image grid
# ----------------------------------------------------------------------------
def morton_rc(r: np.ndarray, c: np.ndarray, bits: int) -> np.ndarray:
    """Z-order index of grid cell (r, c): at every level the row bit sits
    above the column bit, i.e. quadrants are numbered (top-left, top-right,
    bottom-left, bottom-right) recursively."""
    r = np.asarray(r, dtype=np.int64)
    c = np.asarray(c, dtype=np.int64)
    z = np.zeros(np.broadcast(r, c).shape, dtype=np.int64)
    for lvl in range(bits):
        z |= ((c >> lvl) & 1) << (2 * lvl)
        z |= ((r >> lvl) & 1) << (2 * lvl + 1)
    return z


def zorder_sequence_to_grid(side: int) -> np.ndarray:
    """``g[z]`` = raster index (r*side + c) of the token at sequence position z."""
    bits = int(round(math.log2(side)))
    assert 1 << bits == side, "grid side must be a power of two"
    r, c = np.meshgrid(np.arange(side), np.arange(side), indexing="ij")
    z = morton_rc(r, c, bits).ravel()
    g = np.empty(side * side, dtype=np.int64)
    g[z] = (r * side + c).ravel()
    return g


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------
def _rng(w: Workload, tag: int, b: int, h: int) -> np.random.Generator:
    return np.random.default_rng([w.seed, tag, b, h])


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def _iid(w: Workload, tag: int, H: int, heads) -> np.ndarray:
    out = np.empty((w.B, len(heads), w.N, w.D), dtype=np.uint16)
    for b in range(w.B):
        for o, h in enumerate(heads):
            out[b, o] = to_bf16_bits(_normal(_rng(w, tag, b, h), (w.N, w.D)))
    return out


def _clustered_keys(w: Workload, b: int, g: int) -> np.ndarray:
    rng = _rng(w, _TAG_CLUSTER, b, g)
    centres = _normal(rng, (w.centres, w.D))                 # sigma_center = 1
    assign = rng.integers(0, w.centres, size=w.n_kblocks)
    k = np.repeat(centres[assign], w.block_k, axis=0)
    k += np.float32(0.3) * _normal(rng, (w.N, w.D))           # sigma_within = 0.3
    return k


def _clustered_queries(w: Workload, k32: np.ndarray, b: int, h: int) -> np.ndarray:
    rng = _rng(w, _TAG_Q, b, h)
    i = np.arange(w.N, dtype=np.float64)
    j = np.floor(rng.random(w.N) * i).astype(np.int64)       # uniform in [0, i-1]
    j = np.minimum(j, np.maximum(np.arange(w.N) - 1, 0))
    q = k32[j]
    q += np.float32(0.5) * _normal(rng, (w.N, w.D))
    return q


def _needles(w: Workload, b: int, h: int):
    rng = _rng(w, _TAG_NEEDLE, b, h)
    q = _normal(rng, (w.N, w.D))
    k = _normal(rng, (w.N, w.D))
    v = _normal(rng, (w.N, w.D))
    hi = w.N - w.needle_gap                                   # p in [0, hi-1]
    assert hi >= w.needles, "sequence too short for the requested needles"
    pos = rng.choice(hi, size=w.needles, replace=False)
    used = set()
    for p in pos:
        while True:
            t = int(rng.integers(p + w.needle_gap, w.N))
            if t not in used:
                used.add(t)
                break
        q[t] = k[p]
        k[p] = np.float32(4.0) * k[p]
        v[p] = _normal(rng, (w.D,))
    return q, k, v


def _gauss_taps(sigma: float) -> np.ndarray:
    rad = int(round(4 * sigma))
    t = np.arange(-rad, rad + 1, dtype=np.float64)
    wts = np.exp(-0.5 * (t / sigma) ** 2)
    return wts / wts.sum()


def _image_field(w: Workload, tag: int, b: int, h: int, side: int, order: np.ndarray,
                 sigma: float = 4.0) -> np.ndarray:
    rng = _rng(w, _TAG_IMG * 16 + tag, b, h)
    z = _normal(rng, (side, side, w.D)).astype(np.float64)
    taps = _gauss_taps(sigma)
    # periodic (circular) separable filter, applied as one 2-D FFT product
    ker = np.zeros(side)
    rad = (len(taps) - 1) // 2
    for o, wt in zip(range(-rad, rad + 1), taps):
        ker[o % side] += wt
    kf = np.fft.fft2(np.outer(ker, ker))
    f = np.real(np.fft.ifft2(np.fft.fft2(z, axes=(0, 1)) * kf[:, :, None], axes=(0, 1)))
    # std of the filtered unit white noise = sqrt(sum of squared 2-D weights)
    #                                      = sum of squared 1-D weights
    gain = float((ker ** 2).sum())
    f = f / gain + 0.1 * _normal(rng, (side, side, w.D)).astype(np.float64)
    return f.reshape(side * side, w.D)[order].astype(np.float32)


def make_inputs(w: Workload, q_heads=None, kv_heads=None) -> dict:
    """Draw Q, K, V for workload ``w`` as bf16 bit patterns.

    Returns ``{"q": uint16[B, len(q_heads), N, D], "k": uint16[B, len(kv_heads), N, D],
    "v": ...}``.  ``q_heads`` / ``kv_heads`` default to all heads; passing a
    subset regenerates exactly those heads' bytes.
    """
    q_heads = list(range(w.Hq)) if q_heads is None else list(q_heads)
    kv_heads = list(range(w.Hkv)) if kv_heads is None else list(kv_heads)
    assert w.Hq % w.Hkv == 0 and w.N % w.block_k == 0 and w.N % w.block_q == 0
    grp = w.Hq // w.Hkv
    if w.kind == "iid":
        return {"q": _iid(w, _TAG_Q, w.Hq, q_heads), "k": _iid(w, _TAG_K, w.Hkv, kv_heads),
                "v": _iid(w, _TAG_V, w.Hkv, kv_heads)}
    if w.kind == "clustered":
        q = np.empty((w.B, len(q_heads), w.N, w.D), dtype=np.uint16)
        k = np.empty((w.B, len(kv_heads), w.N, w.D), dtype=np.uint16)
        need = sorted(set(kv_heads) | {h // grp for h in q_heads})
        for b in range(w.B):
            for g in need:
                k32 = _clustered_keys(w, b, g)
                if g in kv_heads:
                    k[b, kv_heads.index(g)] = to_bf16_bits(k32)
                for o, h in enumerate(q_heads):
                    if h // grp == g:
                        q[b, o] = to_bf16_bits(_clustered_queries(w, k32, b, h))
        return {"q": q, "k": k, "v": _iid(w, _TAG_V, w.Hkv, kv_heads)}
    if w.kind == "needles":
        assert grp == 1, "needle workload pairs query head h with KV head h"
        heads = sorted(set(q_heads) | set(kv_heads))
        q = np.empty((w.B, len(q_heads), w.N, w.D), dtype=np.uint16)
        k = np.empty((w.B, len(kv_heads), w.N, w.D), dtype=np.uint16)
        v = np.empty_like(k)
        for b in range(w.B):
            for h in heads:
                qq, kk, vv = _needles(w, b, h)
                if h in q_heads:
                    q[b, q_heads.index(h)] = to_bf16_bits(qq)
                if h in kv_heads:
                    o = kv_heads.index(h)
                    k[b, o] = to_bf16_bits(kk)
                    v[b, o] = to_bf16_bits(vv)
        return {"q": q, "k": k, "v": v}
    if w.kind == "image":
        side = int(round(math.sqrt(w.N)))
        assert side * side == w.N
        order = zorder_sequence_to_grid(side)
        out = {}
        for name, tag, heads in (("q", 0, q_heads), ("k", 1, kv_heads), ("v", 2, kv_heads)):
            a = np.empty((w.B, len(heads), w.N, w.D), dtype=np.uint16)
            for b in range(w.B):
                for o, h in enumerate(heads):
                    a[b, o] = to_bf16_bits(_image_field(w, tag, b, h, side, order))
            out[name] = a
        return out
    raise ValueError(f"unknown workload kind {w.kind!r}")
