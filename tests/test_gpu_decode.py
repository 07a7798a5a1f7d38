"""Parity of the decode path (one query per head against the cached keys)
with the float64 oracle's decode step.

Selections are compared bit-exactly except at the oracle's counted near-ties
(fp64 scores within 1e-4 relative), where the GPU's choice must be one the
oracle enumerates itself; outputs against the oracle's read over that
selection; the block-mean cache against fp64 means.  No expected value comes
from the CUDA path.
"""
import numpy as np
import pytest
import torch

import oracle as O
from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, make_inputs
from parity_utils import MAX_ABS, MEAN_ABS, LSE_ABS, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


def W(name, **kw):
    base = dict(B=2, Hq=4, Hkv=2, N=2048, D=64, block_k=64, block_q=64, top_k=4, window=100,
                causal=True, kind="iid", seed=29)
    base.update(kw)
    return Workload(name, **base)


class Cache:
    """A workload's Q, K, V: K/V as the decode cache (capacity N), Q as the
    queries of successive positions."""

    def __init__(self, w, x=None):
        self.w = w
        self.p = ssa.params_of(w)
        self.op = O.Params.of(w)
        x = x if x is not None else make_inputs(w)
        self.qu16 = x["q"]                                   # upcast per query on demand
        self.k64, self.v64 = (O.upcast_bf16(x[n]) for n in "kv")
        self.qd, self.kd, self.vd = (to_dev(x[n]) for n in "qkv")
        self.ksum = ssa.block_summary(self.kd, w.block_k, self.p)   # every complete block
        self.ws = torch.empty(max(ssa.decode_workspace_size(self.p), 1), dtype=torch.uint8,
                              device="cuda")

    def step(self, n_ctx):
        q = self.qd[:, :, n_ctx - 1].contiguous()
        out = ssa.decode(q, self.kd, self.vd, n_ctx, self.ksum, self.p, workspace=self.ws)
        ssa.check_error()
        return [(t.float() if t.dtype == torch.bfloat16 else t).cpu().numpy() if t is not None
                else None for t in out]


def check_step(c, n_ctx, o, lse, idx, cnt):
    """Routing (near-tie aware) and the read of every (b, head) at one step."""
    op = c.op
    i = n_ctx - 1
    nb = i // op.block_k
    mu = O.block_summary(c.k64[:, :, :nb * op.block_k], op.block_k) if nb else None
    errs, alt = [], 0
    for b in range(op.B):
        for h in range(op.Hq):
            g = h // op.group
            q = O.upcast_bf16(c.qu16[b, h, i])
            if nb:
                own, _, _ = O.route_row(q, mu[b, g], np.arange(nb), op.top_k)
            else:
                own = np.zeros(0, dtype=np.int64)
            n = int(cnt[b, h])
            got = idx[b, h, :n]
            assert n == len(own), (n_ctx, b, h, n, len(own))
            assert (idx[b, h, n:] == -1).all()
            if np.array_equal(got, own):
                chosen = own
            else:
                acc = O.acceptable_selections(q, mu[b, g], np.arange(nb), op.top_k)
                match = [a for a in acc if np.array_equal(a, got)]
                assert match, f"step {n_ctx} {(b, h)}: {got.tolist()} != {own.tolist()}"
                chosen = match[0]
                alt += 1
            o_ref, l_ref = O.decode_attend(q, c.k64[b, g], c.v64[b, g], i, chosen, op)
            errs.append(np.abs(o[b, h].astype(np.float64) - o_ref))
            assert abs(float(lse[b, h]) - l_ref) <= LSE_ABS, (n_ctx, b, h)
    e = np.stack(errs)
    assert np.isfinite(o).all()
    assert e.max() <= MAX_ABS, (n_ctx, e.max())
    assert e.mean() <= MEAN_ABS, (n_ctx, e.mean())
    return alt


SHAPES = [
    W("gqa2"),
    W("gqa7-clustered", B=1, Hq=14, Hkv=2, N=4096, top_k=8, window=256, kind="clustered",
      centres=16),
    W("d128", B=1, Hq=2, Hkv=1, N=1024, D=128, top_k=3, window=96),
    W("bk16-k40", B=1, Hq=2, Hkv=2, N=2048, block_k=16, block_q=16, top_k=40, window=40),
    W("window-only", B=1, Hq=2, Hkv=1, N=512, top_k=0, window=77),
    W("window1", B=1, Hq=2, Hkv=2, N=1024, top_k=5, window=1),
    W("dense", B=1, Hq=2, Hkv=1, N=512, top_k=8, window=64),
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_decode_steps_match_oracle(w):
    c = Cache(w)
    N, bk = w.N, w.block_k
    steps = sorted({1, 2, bk - 1, bk, bk + 1, 2 * bk, 2 * bk + 1, 5 * bk + 3, N // 2 + 7,
                    N - 1, N})
    for n_ctx in steps:
        check_step(c, n_ctx, *c.step(n_ctx))


def test_decode_loop_maintains_the_block_mean_cache():
    # a prefill of n0 tokens leaves the cache valid for the blocks before the
    # newest admissible one; every later step writes the block that becomes
    # admissible at it
    w = W("loop", B=1, Hq=4, Hkv=2, N=1024, top_k=4, window=64, block_k=32, block_q=32)
    c = Cache(w)
    n0, n1, bk = 200, 520, w.block_k
    valid = (n0 - 1) // bk - 1
    c.ksum[:, :, max(valid, 0):] = float("nan")       # not yet valid
    for n_ctx in range(n0, n1 + 1):
        out = c.step(n_ctx)
        if n_ctx % 37 == 0 or n_ctx in (n0, n1):
            check_step(c, n_ctx, *out)
    nb = (n1 - 1) // bk
    want = O.block_summary(c.k64[:, :, :nb * bk], bk)
    got = c.ksum[:, :, :nb].cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5)
    assert torch.isnan(c.ksum[:, :, nb:]).all()          # nothing beyond was written


def test_decode_million_token_cache_sampled():
    w = CONFIGS[5]
    c = Cache(w)
    for n_ctx in (w.N, w.N - 4097, 300_001):
        check_step(c, n_ctx, *c.step(n_ctx))


def _tied_cache(w, period_blocks, seed):
    """Keys whose block means repeat every ``period_blocks`` blocks (a
    constant cache for period 1): small integer keys, so every block mean is
    exact in fp32 whatever the summation order, and equal means give exactly
    equal scores on both sides."""
    from content_routed_block_b200.workloads import to_bf16_bits
    rng = np.random.default_rng(seed)
    span = period_blocks * w.block_k
    base = rng.integers(-2, 3, size=(w.B, w.Hkv, span, w.D)).astype(np.float32)
    k = np.tile(base, (1, 1, w.N // span + 1, 1))[:, :, :w.N]
    x = make_inputs(w)
    x["k"] = to_bf16_bits(k)
    return x


def test_decode_selection_when_ties_defeat_the_fast_paths():
    # Each routing split normally passes at most 64 keys to a sort; these
    # caches push both kernels onto their merge paths and the result must not
    # change.  (a) A constant cache: every score of a split ties, so all of a
    # split's candidates (111 of them here: 8 KV heads give 37 splits of
    # 4096 blocks) reach the split's threshold.  (b) Block means that repeat
    # with the split length (32 blocks): every split holds the same scores, so
    # about 7 keys of each of 16 splits reach the merge threshold.  Exact ties
    # go to the lower block index on both sides.
    wa = W("tied-constant", B=1, Hq=8, Hkv=8, N=4096 * 16 + 16, block_k=16, block_q=16,
           top_k=8, window=32)
    ca = Cache(wa, _tied_cache(wa, 1, 5))
    for n_ctx in (wa.N, wa.N - 700):
        check_step(ca, n_ctx, *ca.step(n_ctx))
    wb = W("tied-periodic", B=1, Hq=2, Hkv=1, N=512 * 16 + 16, block_k=16, block_q=16,
           top_k=8, window=32)
    cb = Cache(wb, _tied_cache(wb, 32, 6))
    for n_ctx in (wb.N, wb.N - 16 * 32):
        check_step(cb, n_ctx, *cb.step(n_ctx))
