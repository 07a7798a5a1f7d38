"""Parity of the backward of the read (selection held fixed) with the float64
oracle's ``attend_backward``.

The forward runs on the GPU; its lists are checked against the oracle's
(near-tie aware) and the oracle differentiates over the oracle-side lists
equal to them.  The upstream gradient g is a seeded bf16 tensor drawn here.

Tolerance, element by element, from the arithmetic.  The GPU forms
delta_i = g_i . o_i from the forward's output rounded to bf16 (unit roundoff
2^-8), so its delta is off by at most
    E_i = 2^-8 sum_d |g_id| |o_id|        (o the oracle's output),
which moves dS_ij by at most P_ij E_i.  Hence
    |err dq_id| <= scale E_i sum_j P_ij |k_jd|   (the oracle's read with values |k|)
    |err dk_jd| <= scale sum_i P_ij E_i |q_id|   (the oracle's dv for upstream E_i |q_i|)
and dv does not depend on delta.  Each bound gets a slack of 1e-4 of the
largest reference entry for fp32 arithmetic (scores, exponentials and sums
over up to a few thousand terms).

The default (tensor-core) form feeds P and dS to bf16 MMAs as two bf16 parts
each, hi + lo, which leaves a relative rounding of at most 2^-16 per term --
below the fp32 arithmetic the slack covers -- so the same bounds apply to it
and to the CUDA-core form (SSA_BWD=simt).  The tensor-core form sums every
gradient in a fixed order (no atomics), so two runs agree bit for bit; the
CUDA-core form adds dk and dv atomically, so only its tolerance is checked.
"""
import numpy as np
import pytest
import torch

import oracle as O
from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, to_bf16_bits
from parity_utils import Case, check_route_rows, to_dev

pytestmark = pytest.mark.gpu

SLACK = 1e-4       # fp32 arithmetic, relative to the largest reference entry
U_BF16 = 2.0 ** -8  # unit roundoff of bf16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


def W(name, **kw):
    base = dict(B=1, Hq=4, Hkv=2, N=1024, D=64, block_k=64, block_q=64, top_k=4, window=100,
                causal=True, kind="clustered", centres=16, seed=53)
    base.update(kw)
    return Workload(name, **base)


SHAPES = [
    W("gqa2"),
    W("b2-mha", B=2, Hq=2, Hkv=2, N=512, top_k=3, window=64, kind="iid"),
    W("d128", Hq=2, Hkv=1, N=768, D=128, top_k=3, window=96),
    W("bk16", Hq=2, Hkv=1, N=512, block_k=16, block_q=16, top_k=6, window=40),
    W("bk32-bq64", Hq=2, Hkv=1, N=1024, block_k=32, block_q=64, top_k=8, window=70),
    W("bk128-bq128", Hq=2, Hkv=1, N=1024, block_k=128, block_q=128, top_k=3, window=130),
    W("window-only", Hq=2, Hkv=1, N=512, top_k=0, window=77),
    W("window1", Hq=2, Hkv=2, N=512, top_k=3, window=1),
    W("noncausal-image", Hq=2, Hkv=2, N=1024, block_k=16, block_q=16, top_k=8, window=0,
      causal=False, kind="image"),
    W("consensus", Hq=4, Hkv=2, top_k=5, consensus=True),
    W("tree", Hq=4, Hkv=2, N=2048, top_k=4, tree_fanout=4, tree_beam=2),
]


def upstream(w, seed):
    rng = np.random.default_rng(seed)
    u16 = to_bf16_bits(rng.standard_normal((w.B, w.Hq, w.N, w.D)).astype(np.float32))
    return u16, to_dev(u16), O.upcast_bf16(u16)


def oracle_lists(case, idx_g, cnt_g):
    """The oracle's lists equal to the GPU's (per query head)."""
    op = case.op
    if op.consensus or op.tree_fanout:
        # consensus / tree lists: every row checked elsewhere; here they are
        # the oracle's own when they match it exactly
        ref = O.forward(case.q64, case.k64, case.v64, op)
        if op.consensus:
            np.testing.assert_array_equal(idx_g, ref["idx"])
            return O.expand_consensus(ref["idx"], ref["cnt"], op)
        np.testing.assert_array_equal(idx_g, ref["idx"])
        return ref["idx"], ref["cnt"]
    r_idx, r_cnt, _ = check_route_rows(case, idx_g, cnt_g, case.all_rows())
    return r_idx, r_cnt


def delta_bounds(case, g64, r_idx, r_cnt, blocks=None):
    """Bounds on |err dq| and |err dk| from the bf16 rounding of the forward
    output (see the module docstring), all from oracle quantities.  With
    ``blocks`` only those query blocks' rows of the dq bound are filled and
    the dk bound sums over them alone."""
    op = case.op
    todo = blocks if blocks is not None else case.all_rows()
    o, _ = O.attend_masked_dense(case.q64, case.k64, case.v64, r_idx, r_cnt, op, blocks=todo)
    rab, _ = O.attend_masked_dense(case.q64, case.k64, np.abs(case.k64), r_idx, r_cnt, op,
                                   blocks=todo)
    s = op.softmax_scale
    bq = op.block_q
    E = np.zeros(case.q64.shape[:-1])
    bound_dq = np.zeros_like(case.q64)
    for t, (b, h, qb) in enumerate(todo):
        sl = slice(qb * bq, (qb + 1) * bq)
        E[b, h, sl] = U_BF16 * (np.abs(g64[b, h, sl]) * np.abs(o[t])).sum(axis=-1)
        bound_dq[b, h, sl] = s * E[b, h, sl, None] * rab[t]
    _, _, pe = O.attend_backward(case.q64, case.k64, case.v64, E[..., None] * np.abs(case.q64),
                                 r_idx, r_cnt, op, blocks=todo)
    return bound_dq, s * pe


def assert_grad_close(got, want, what, bound=None):
    slack = SLACK * max(float(np.abs(want).max()), 1e-6)
    err = np.abs(got - want)
    lim = slack + (bound if bound is not None else 0.0)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} entries over the bound; worst excess "
                           f"{float((err - lim).max()):.3e}, max err {float(err.max()):.3e}")


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_backward_matches_oracle(w):
    case = Case(w)
    p = case.p
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    _, g_d, g64 = upstream(w, 7)
    dq, dk, dv = ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, idx, cnt, p)
    ssa.check_error()
    r_idx, r_cnt = oracle_lists(case, idx.cpu().numpy(), cnt.cpu().numpy())
    want = O.attend_backward(case.q64, case.k64, case.v64, g64, r_idx, r_cnt, case.op)
    bq, bk = delta_bounds(case, g64, r_idx, r_cnt)
    for got, ref, bound, name in zip((dq, dk, dv), want, (bq, bk, None), ("dq", "dk", "dv")):
        assert_grad_close(got.cpu().numpy().astype(np.float64), ref, f"{w.name} {name}", bound)


def test_backward_rejects_bad_lists_through_the_error_word():
    w = SHAPES[0]
    case = Case(w)
    p = case.p
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    _, g_d, _ = upstream(w, 9)
    bad = idx.clone()
    bad[0, 0, 5, 0] = w.N // w.block_k + 3          # out of range
    ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, bad, cnt, p)
    with pytest.raises(ssa.SsaError):
        ssa.check_error()
    ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, idx, cnt, p)
    ssa.check_error()                               # the context is still usable


def test_backward_full_size_sampled():
    w = CONFIGS[2]
    case = Case(w)
    p, op = case.p, case.op
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    _, g_d, g64 = upstream(w, 11)
    dq, dk, dv = ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, idx, cnt, p)
    ssa.check_error()
    idx_g, cnt_g = idx.cpu().numpy(), cnt.cpu().numpy()
    # dq on sampled query blocks
    rows = case.sample_rows(6, seed=2)
    r_idx, r_cnt, _ = check_route_rows(case, idx_g, cnt_g, rows)
    want = O.attend_backward(case.q64, case.k64, case.v64, g64, r_idx, r_cnt, op, blocks=rows)
    bound_dq, _ = delta_bounds(case, g64, r_idx, r_cnt, blocks=rows)
    got = dq.cpu().numpy()
    for b, h, qb in rows:
        sl = slice(qb * op.block_q, (qb + 1) * op.block_q)
        assert_grad_close(got[b, h, sl].astype(np.float64), want[0][b, h, sl], f"dq {(b, h, qb)}",
                          bound_dq[b, h, sl])
    # dk / dv of one key block of KV head 1: every query block that reads it
    c, g = 300, 1
    heads = range(g * op.group, (g + 1) * op.group)
    lo, hi = c * op.block_k, (c + 1) * op.block_k - 1
    contrib = [(0, h, qb) for h in heads for qb in range(op.n_qblocks)
               if c in idx_g[0, h, qb, :cnt_g[0, h, qb]]
               or (qb * op.block_q <= hi + op.window - 1 and (qb + 1) * op.block_q - 1 >= lo)]
    r_idx, r_cnt, _ = check_route_rows(case, idx_g, cnt_g, contrib)
    _, wdk, wdv = O.attend_backward(case.q64, case.k64, case.v64, g64, r_idx, r_cnt, op,
                                    blocks=contrib)
    _, bound_dk = delta_bounds(case, g64, r_idx, r_cnt, blocks=contrib)
    assert_grad_close(dk[0, g, lo:hi + 1].cpu().numpy().astype(np.float64), wdk[0, g, lo:hi + 1],
                      "dk block 300", bound_dk[0, g, lo:hi + 1])
    assert_grad_close(dv[0, g, lo:hi + 1].cpu().numpy().astype(np.float64), wdv[0, g, lo:hi + 1],
                      "dv block 300")


def _with_form(form, fn):
    import os
    old = os.environ.get("SSA_BWD")
    if form is None:
        os.environ.pop("SSA_BWD", None)
    else:
        os.environ["SSA_BWD"] = form
    try:
        return fn()
    finally:
        if old is None:
            os.environ.pop("SSA_BWD", None)
        else:
            os.environ["SSA_BWD"] = old


@pytest.mark.parametrize("w", [SHAPES[0], SHAPES[3], SHAPES[8]], ids=lambda w: w.name)
def test_cuda_core_form_matches_oracle(w):
    # the CUDA-core form, kept for comparison, under the same bounds
    case = Case(w)
    p = case.p
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    _, g_d, g64 = upstream(w, 7)
    dq, dk, dv = _with_form("simt", lambda: ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d,
                                                         idx, cnt, p))
    ssa.check_error()
    r_idx, r_cnt = oracle_lists(case, idx.cpu().numpy(), cnt.cpu().numpy())
    want = O.attend_backward(case.q64, case.k64, case.v64, g64, r_idx, r_cnt, case.op)
    bq, bk = delta_bounds(case, g64, r_idx, r_cnt)
    for got, ref, bound, name in zip((dq, dk, dv), want, (bq, bk, None), ("dq", "dk", "dv")):
        assert_grad_close(got.cpu().numpy().astype(np.float64), ref, f"simt {w.name} {name}", bound)


@pytest.mark.parametrize("w", [SHAPES[0], SHAPES[2], SHAPES[8], SHAPES[9], CONFIGS[2]],
                         ids=lambda w: w.name)
def test_tensor_core_backward_is_bit_reproducible(w):
    # every gradient is summed by one CTA in a fixed order: two runs (with a
    # different call in between) agree bit for bit
    case = Case(w)
    p = case.p
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    _, g_d, _ = upstream(w, 5)
    first = ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, idx, cnt, p)
    _, g2, _ = upstream(w, 6)
    ssa.backward(case.qd, case.kd, case.vd, o, lse, g2, idx, cnt, p)
    second = ssa.backward(case.qd, case.kd, case.vd, o, lse, g_d, idx, cnt, p)
    ssa.check_error()
    for name, a, b in zip(("dq", "dk", "dv"), first, second):
        assert torch.equal(a, b), f"{w.name}: {name} differs between two runs"
