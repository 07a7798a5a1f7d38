"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Per-kernel checks isolate each step: K1 summaries against fp64 means, K2
selections against the oracle's top-k (bit-exact except at counted near-ties,
where the GPU's choice must be one the oracle itself enumerates as
acceptable), K3 fed the oracle's own selections against the oracle's attend.
Then the whole forward on small shapes (every row) and on the five workloads
at full size: every row's list against the oracle's route, outputs on
sampled query blocks and on every near-tie row.
"""
import numpy as np
import pytest
import torch

import oracle as O
from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, make_inputs
from parity_utils import (Case, assert_close, check_forward, check_route_every_row,
                          check_route_rows, gpu_rows, oracle_attend_rows, output_rows, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


def W(name, **kw):
    base = dict(B=1, Hq=2, Hkv=2, N=1024, D=64, block_k=64, block_q=64, top_k=4, window=128,
                causal=True, kind="iid", seed=11)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    CONFIGS[1],
    W("ragged-gqa2", B=2, Hq=4, Hkv=2, N=1216, top_k=4, window=200),
    W("d128-gqa8", Hq=8, Hkv=1, D=128, top_k=3, window=96),
    W("window1", N=640, top_k=2, window=1),
    W("sliding-k0", N=640, top_k=0, window=100),
    W("dense-causal", N=768, top_k=12, window=64),
    W("bk16", N=512, block_k=16, block_q=16, top_k=5, window=40),
    W("bk32-bq64", N=768, block_k=32, block_q=64, top_k=6, window=70),
    W("bq128-bk16", N=1024, block_k=16, block_q=128, top_k=8, window=130),
    W("bk128", N=1024, block_k=128, block_q=128, top_k=2, window=128),
    W("bk128-bq32", N=1024, block_k=128, block_q=32, top_k=2, window=50),
    W("noncausal-bk16", B=1, Hq=2, Hkv=2, N=1024, block_k=16, block_q=16, top_k=8, window=0,
      causal=False, kind="image"),
    W("noncausal-k64", N=4096, top_k=64, window=0, causal=False),
    W("k40", N=4096, top_k=40, window=64, Hq=2, Hkv=1),
    W("tiny", N=64, Hq=1, Hkv=1, block_k=16, block_q=16, top_k=2, window=20),
    W("gqa7-clustered", Hq=14, Hkv=2, N=2048, top_k=8, window=256, kind="clustered", centres=16),
    W("needles-d128", Hq=2, Hkv=2, N=5120, D=128, top_k=4, window=256, kind="needles",
      needles=4),
]


# ------------------------------------------------------------------ error path
def test_bounded_wait_reports_timeout_and_context_survives():
    ssa.probe_wait_timeout(2000)
    with pytest.raises(ssa.SsaError) as e:
        ssa.check_error()
    assert e.value.status == 5
    ssa.check_error()                       # the word was cleared
    check_forward(Case(CONFIGS[1]))         # and the context still works


# ------------------------------------------------------------------ K1
@pytest.mark.parametrize("D,block", [(64, 16), (64, 32), (64, 64), (128, 64), (128, 128)])
def test_block_summary_matches_fp64_means(D, block):
    w = W("pool", B=2, Hq=3, Hkv=3, N=1024, D=D)
    x = make_inputs(w)["q"]
    p = ssa.params_of(w)
    g = ssa.block_summary(to_dev(x), block, p).cpu().numpy().astype(np.float64)
    ref = O.block_summary(O.upcast_bf16(x), block)
    np.testing.assert_allclose(g, ref, rtol=0, atol=1e-5)


def test_block_summary_exact_on_integer_inputs():
    rng = np.random.default_rng(5)
    vals = rng.integers(-64, 65, size=(1, 2, 2048, 64)).astype(np.float32)
    from content_routed_block_b200.workloads import to_bf16_bits
    x = to_bf16_bits(vals)
    p = ssa.make_params(1, 2, 2, 2048, 64, 64, 64, 4, 64, True)
    g = ssa.block_summary(to_dev(x), 64, p).cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(g, O.block_summary(vals.astype(np.float64), 64))


# ------------------------------------------------------------------ K2
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_route_matches_oracle(w):
    case = Case(w)
    p = case.p
    ks = ssa.block_summary(case.kd, w.block_k, p)
    qs = ssa.block_summary(case.qd, w.block_q, p)
    idx, cnt = ssa.route(qs, ks, p)
    ssa.check_error()
    check_route_rows(case, idx.cpu().numpy(), cnt.cpu().numpy(), case.all_rows())


def test_route_equal_scores_take_lowest_indices():
    w = W("flat", N=2048, Hq=2, Hkv=1, top_k=7, window=64)
    x = make_inputs(w)
    x["k"][:] = x["k"][:, :, :1, :]            # every key row equal -> every score equal
    case = Case(w, x)
    p = case.p
    ks = ssa.block_summary(case.kd, 64, p)
    qs = ssa.block_summary(case.qd, 64, p)
    idx, cnt = ssa.route(qs, ks, p)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for qb in range(32):
        n = min(7, qb)
        assert cnt[0, 0, qb] == n and cnt[0, 1, qb] == n
        assert idx[0, 0, qb, :n].tolist() == list(range(n))
        assert idx[0, 1, qb, :n].tolist() == list(range(n))


# ------------------------------------------------------------------ K3
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attend_with_oracle_selection(w):
    case = Case(w)
    op = case.op
    r = O.route(case.qsum64, case.ksum64, op)
    idx = torch.from_numpy(r.idx).cuda()
    cnt = torch.from_numpy(r.cnt).cuda()
    o, lse = ssa.attend(case.qd, case.kd, case.vd, idx, cnt, case.p)
    ssa.check_error()
    rows = case.all_rows()
    o_ref, l_ref = oracle_attend_rows(case, r.idx, r.cnt, rows)
    assert_close(gpu_rows(o, rows, op.block_q), o_ref, gpu_rows(lse, rows, op.block_q), l_ref,
                 what=w.name)


# ------------------------------------------------------------------ whole path
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_small_every_row(w):
    check_forward(Case(w))


def _route_properties_all_rows(case, idx, cnt):
    op = case.op
    qb = np.arange(op.n_qblocks)
    if op.causal:
        n_adm = np.minimum((qb * op.block_q) // op.block_k, op.n_kblocks)
    else:
        n_adm = np.full(op.n_qblocks, op.n_kblocks)
    want = np.minimum(op.top_k, n_adm)
    assert (cnt == want[None, None, :]).all()
    if op.top_k == 0:
        return
    e = np.arange(op.top_k)
    valid = e[None, None, None, :] < cnt[..., None]
    assert (idx[~valid] == -1).all()
    sel = np.where(valid, idx, -1)
    assert (sel[valid] >= 0).all()
    lim = n_adm[None, None, :, None]
    assert (np.where(valid, sel < lim, True)).all()
    d = np.diff(sel, axis=-1)
    vpair = valid[..., 1:]
    assert (np.where(vpair, d > 0, True)).all()


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_forward_full_size_every_row_routed_like_the_oracle(cfg):
    # every row's list against the oracle's fp64 route (exact outside counted
    # near-ties); outputs on one random, the first and the last query block of
    # every (b, head) and on every near-tie row, through the oracle's
    # block-gathered read
    case = Case(CONFIGS[cfg])
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    idx_g, cnt_g = idx.cpu().numpy(), cnt.cpu().numpy()
    _route_properties_all_rows(case, idx_g, cnt_g)
    r_idx, r_cnt, alt, near = check_route_every_row(case, idx_g, cnt_g)
    rows = output_rows(case, near, seed=cfg)
    print(f"{case.w.name}: {near.size} rows, {int(near.sum())} counted near-ties, "
          f"{alt} GPU near-tie alternatives, outputs on {len(rows)} query blocks")
    o_ref, l_ref = O.attend_gathered_blocks(case.q64, case.k64, case.v64, r_idx, r_cnt, case.op,
                                            rows)
    assert_close(gpu_rows(o, rows, case.op.block_q), o_ref, gpu_rows(lse, rows, case.op.block_q),
                 l_ref, what=case.w.name)
    assert torch.isfinite(o).all()


def test_forward_is_deterministic():
    case = Case(CONFIGS[1].with_(N=2048, Hq=4, Hkv=2, top_k=6))
    a = ssa.forward(case.qd, case.kd, case.vd, case.p)
    b = ssa.forward(case.qd, case.kd, case.vd, case.p)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_attend_without_lse_matches_with_lse():
    case = Case(CONFIGS[1])
    r = O.route(case.qsum64, case.ksum64, case.op)
    idx, cnt = torch.from_numpy(r.idx).cuda(), torch.from_numpy(r.cnt).cuda()
    o1, _ = ssa.attend(case.qd, case.kd, case.vd, idx, cnt, case.p, with_lse=True)
    o2, l2 = ssa.attend(case.qd, case.kd, case.vd, idx, cnt, case.p, with_lse=False)
    assert l2 is None and torch.equal(o1, o2)


def test_out_of_range_block_is_reported_not_read():
    case = Case(CONFIGS[1])
    r = O.route(case.qsum64, case.ksum64, case.op)
    bad = r.idx.copy()
    bad[0, 1, 9, 0] = case.op.n_kblocks + 5
    o, _ = ssa.attend(case.qd, case.kd, case.vd, torch.from_numpy(bad).cuda(),
                      torch.from_numpy(r.cnt).cuda(), case.p)
    with pytest.raises(ssa.SsaError) as e:
        ssa.check_error()
    assert e.value.status == 6
    # rows of other query tiles are untouched by the bad entry
    rows = [(0, 0, qb) for qb in range(16)]
    o_ref, _ = oracle_attend_rows(case, r.idx, r.cnt, rows)
    assert_close(gpu_rows(o, rows, 64), o_ref, what="other rows")


def test_forward_host_roundtrip():
    case = Case(CONFIGS[1])
    qh, kh, vh = (t.cpu().pin_memory() for t in (case.qd, case.kd, case.vd))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    ssa.forward_host(qh, kh, vh, case.p, oh)
    torch.cuda.synchronize()
    o, _, _, _ = ssa.forward(case.qd, case.kd, case.vd, case.p)
    assert torch.equal(oh, o.cpu())


# ------------------------------------------------------------------ router forms
def _route_with(form, case, in_kernel_split=False):
    import os
    old = os.environ.get("SSA_ROUTER")
    os.environ["SSA_ROUTER"] = form
    try:
        p = case.p
        ks = ssa.block_summary(case.kd, case.w.block_k, p)
        qs = ssa.block_summary(case.qd, case.w.block_q, p)
        idx, cnt = ssa.route(qs, ks, p, in_kernel_split=in_kernel_split)
        ssa.check_error()
        return idx, cnt
    finally:
        if old is None:
            os.environ.pop("SSA_ROUTER", None)
        else:
            os.environ["SSA_ROUTER"] = old


@pytest.mark.parametrize("w", [w for w in SMALL if w.top_k > 0] + [CONFIGS[c] for c in (2, 3, 4, 5)],
                         ids=lambda w: w.name)
def test_tensor_core_router_equals_fp32_router(w):
    # the tensor-core router ranks on the same fp32 scores as the FMA router
    # (bf16 prefilter with a proven bound + exact rescoring): bit-identical lists
    # The tensor-core form runs twice: with the key image split once into
    # scratch (ssa_route_with_workspace, as in the forward) and split by each
    # CTA (ssa_route, no scratch).
    case = Case(w)
    i1, c1 = _route_with("fp32", case)
    i2, c2 = _route_with("tc", case)
    i3, c3 = _route_with("tc", case, in_kernel_split=True)
    assert torch.equal(c1, c2) and torch.equal(c1, c3)
    assert torch.equal(i1, i2) and torch.equal(i1, i3)


def test_tensor_core_router_on_flat_and_tied_scores():
    # all-equal keys (every candidate inside the bound: all rescored) and
    # integer-valued summaries with many exact ties
    w = W("flat-tc", N=8192, Hq=2, Hkv=1, top_k=16, window=64)
    x = make_inputs(w)
    x["k"][:] = x["k"][:, :, :1, :]
    case = Case(w, x)
    i1, c1 = _route_with("fp32", case)
    i2, c2 = _route_with("tc", case)
    i3, c3 = _route_with("tc", case, in_kernel_split=True)
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
    assert torch.equal(i1, i3) and torch.equal(c1, c3)
    idx = i2.cpu().numpy()
    for qb in (5, 40, 127):
        n = min(16, qb)
        assert idx[0, 0, qb, :n].tolist() == list(range(n))
    from content_routed_block_b200.workloads import to_bf16_bits
    rng = np.random.default_rng(9)
    xi = {n: to_bf16_bits(rng.integers(-2, 3, size=s).astype(np.float32))
          for n, s in (("q", (1, 2, 8192, 64)), ("k", (1, 1, 8192, 64)), ("v", (1, 1, 8192, 64)))}
    case = Case(w, xi)
    i1, c1 = _route_with("fp32", case)
    i2, c2 = _route_with("tc", case)
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
    check_route_rows(case, i2.cpu().numpy(), c2.cpu().numpy(), case.sample_rows(40, seed=1))


def test_non_finite_key_block_is_reported_and_the_oracle_refuses_it():
    # non-finite inputs are outside the method's domain: the oracle refuses
    # to route them, and the GPU path reports them through the error word
    # (pool kernel) without hanging; the context stays usable
    case = Case(CONFIGS[1])
    x = {n: case.u16[n].copy() for n in "qkv"}
    x["k"][0, 1, 3 * 64 + 5, 7] = 0x7FC0            # a bf16 NaN in key block 3 of KV head 1
    bad = Case(CONFIGS[1], x)
    with pytest.raises(ValueError):
        O.route(bad.qsum64, bad.ksum64, bad.op)
    o, _, idx, cnt = ssa.forward(bad.qd, bad.kd, bad.vd, bad.p)
    with pytest.raises(ssa.SsaError) as e:
        ssa.check_error()
    assert e.value.status == 6
    # KV head 1's routing never picks the NaN block; head 0 is unaffected
    idx = idx.cpu().numpy()
    assert not (idx[0, 1] == 3).any()
    rows = [(0, 0, qb) for qb in range(case.op.n_qblocks)]
    r_idx, r_cnt, _ = check_route_rows(case, idx, cnt.cpu().numpy(), rows)
    o_ref, l_ref = oracle_attend_rows(case, r_idx, r_cnt, rows)
    assert_close(gpu_rows(o, rows, 64), o_ref, what="the finite head")
    check_forward(Case(CONFIGS[1]))


def _band_inputs(N, seed):
    """Keys 10 + integer offsets whose sum over each 64-row block is a planted
    j_c in [-6, 6]; every query row is 0 or 2 (heads 0) / 0 or 4 (head 1) with
    a block mean of exactly 1 (2).  Block means are multiples of 1/64 that
    bf16 does not hold (so both split parts are non-zero), and every score is
    exactly (640 + j_c / 64) * {1, 2} in fp32 as in fp64: the order is known
    exactly, every candidate lies within the tensor-core bound E_c of the
    k-th score, and equal j_c are exact ties."""
    from content_routed_block_b200.workloads import to_bf16_bits
    rng = np.random.default_rng(seed)
    D, nb = 64, N // 64
    k = np.full((1, 1, N, D), 10.0, np.float32)
    for c in range(nb):
        j = int(rng.integers(-6, 7))
        off = np.zeros(64 * D, np.float32)
        pos = rng.choice(64 * D, size=80 + abs(j), replace=False)
        off[pos[:40]] += 1.0
        off[pos[40:80]] -= 1.0
        off[pos[80:]] += np.sign(j)
        k[0, 0, c * 64:(c + 1) * 64] += off.reshape(64, D)
    q = np.zeros((1, 2, N, D), np.float32)
    q[0, 0, 0::2] = 2.0
    q[0, 1, 1::2] = 4.0
    v = rng.standard_normal((1, 1, N, D)).astype(np.float32)
    return {"q": to_bf16_bits(q), "k": to_bf16_bits(k), "v": to_bf16_bits(v)}


def test_tensor_core_router_with_every_candidate_inside_its_bound():
    # the filter / queue / rescoring path with whole rows inside the bound and
    # many exact ties: both routers must give the exact lexicographic order
    # (no near-tie allowance: the fp32 scores here are exact)
    w = W("band-tc", N=16384, Hq=2, Hkv=1, top_k=16, window=64)
    case = Case(w, _band_inputs(16384, seed=13))
    i1, c1 = _route_with("fp32", case)
    i2, c2 = _route_with("tc", case)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    r = O.route_flat_all(case.qsum64, case.ksum64, case.op)
    np.testing.assert_array_equal(c2.cpu().numpy(), r.cnt)
    np.testing.assert_array_equal(i2.cpu().numpy(), r.idx)
    # the planted scores are what the construction says
    mu = case.ksum64[0, 0]
    s = mu @ case.qsum64[0, 0, 5]
    assert np.all(np.abs(s * 64 - np.round(s * 64)) == 0) and np.ptp(s) <= 12 / 64


def test_tensor_core_router_on_near_duplicate_blocks():
    # blocks that copy another block's keys with one bf16 step changed in one
    # element: fp32 scores within the tensor-core bound of each other and not
    # exact; the two routers must agree bit for bit, and with the oracle
    # outside counted near-ties
    w = W("dup-tc", N=16384, Hq=2, Hkv=1, top_k=16, window=64, kind="clustered", centres=8)
    x = make_inputs(w)
    kk = x["k"].reshape(1, 1, 256, 64, 64)
    rng = np.random.default_rng(17)
    for c in rng.choice(np.arange(1, 256), size=120, replace=False):
        src = int(rng.integers(0, 256))
        kk[0, 0, c] = kk[0, 0, src]
        t, d = int(rng.integers(64)), int(rng.integers(64))
        kk[0, 0, c, t, d] = kk[0, 0, c, t, d] + np.uint16(1)   # one bf16 step
    case = Case(w, x)
    i1, c1 = _route_with("fp32", case)
    i2, c2 = _route_with("tc", case)
    assert torch.equal(c1, c2) and torch.equal(i1, i2)
    _, _, alt, near = check_route_every_row(case, i2.cpu().numpy(), c2.cpu().numpy())
    print(f"near-duplicate blocks: {int(near.sum())} counted near-ties, {alt} alternatives")
