"""Pins for the float64 oracle against facts fixed outside it.

Each test checks the oracle against something other than itself: a
hand-derived worked example (tests/golden), a library routine in a special
case the method reduces to (torch SDPA in float64 on the CPU), closed forms,
or invariants (set semantics, the lower-index tie rule, weights summing to 1,
the append law of the softmax read, causality).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _params(**kw):
    base = dict(B=1, Hq=1, Hkv=1, N=8, D=2, block_k=2, block_q=2, top_k=1,
                window=2, causal=True, scale=0.0)
    base.update(kw)
    return O.Params(**base)


def _worked_inputs():
    k = np.array([[1, 0], [1, 0], [0, 1], [0, 1], [-1, 0], [-1, 0], [0, -1], [0, -1]],
                 dtype=np.float64)
    q = np.tile(np.array([[0.0, 2.0]]), (8, 1))
    v = np.stack([np.arange(8.0), np.ones(8)], axis=1)
    return q[None, None], k[None, None], v[None, None]


def _read_worked_golden():
    rows = []
    with open(os.path.join(GOLDEN, "worked_example_4block.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kk, i, expr = line.split(maxsplit=2)
            rows.append((int(kk), int(i), expr))
    return rows


# ---------------------------------------------------------------- worked example
@pytest.mark.parametrize("form", ["dense", "gathered"])
def test_worked_example_matches_hand_derivation(form):
    q, k, v = _worked_inputs()
    E = math.exp(math.sqrt(2.0))
    rows = _read_worked_golden()
    assert len(rows) == 26
    by_k = {}
    for kk, i, expr in rows:
        by_k.setdefault(kk, []).append((i, eval(expr, {"E": E})))
    for kk, items in by_k.items():
        p = _params(top_k=kk)
        out = O.forward(q, k, v, p, form=form)
        for i, want in items:
            assert out["o"][0, 0, i, 0] == pytest.approx(want, abs=1e-12), (kk, i)
        np.testing.assert_allclose(out["o"][0, 0, :, 1], 1.0, atol=1e-14)


def test_worked_example_routing_and_tie_rule():
    q, k, v = _worked_inputs()
    p1 = O.forward(q, k, v, _params(top_k=1))
    assert p1["idx"][0, 0, :, 0].tolist() == [-1, 0, 1, 1]
    assert p1["cnt"][0, 0].tolist() == [0, 1, 1, 1]
    p2 = O.forward(q, k, v, _params(top_k=2))
    # qb3 scores (0, 2, 0): block 1, then the tie between blocks 0 and 2 goes to 0
    assert p2["idx"][0, 0, 3].tolist() == [0, 1]
    assert p2["idx"][0, 0, 2].tolist() == [0, 1]
    assert p2["idx"][0, 0, 1].tolist() == [0, -1]
    assert p2["cnt"][0, 0].tolist() == [0, 1, 2, 2]
    # block means are the hand values
    np.testing.assert_array_equal(p2["ksum"][0, 0], [[1, 0], [0, 1], [-1, 0], [0, -1]])


# ---------------------------------------------------------------- summaries
def test_block_summary_closed_form():
    # rows K[t, :] = t (exact in binary): the mean of block c is c*Bk + (Bk-1)/2
    for bk in (1, 2, 16, 64):
        n = bk * 5
        x = np.tile(np.arange(n, dtype=np.float64)[:, None], (1, 3))[None, None]
        s = O.block_summary(x, bk)
        want = np.arange(5) * bk + (bk - 1) / 2
        np.testing.assert_array_equal(s[0, 0, :, 0], want)


def test_block_summary_rejects_ragged():
    with pytest.raises(ValueError):
        O.block_summary(np.zeros((1, 1, 10, 2)), 4)


# ---------------------------------------------------------------- routing
def _route_property_check(qsum, ksum, r, p):
    """Selection property written pairwise: every selected admissible block
    beats every unselected one in (score desc, index asc)."""
    for b in range(p.B):
        for h in range(p.Hq):
            mu = ksum[b, h // p.group]
            for qb in range(p.n_qblocks):
                if p.causal:
                    adm = [c for c in range(p.n_kblocks) if (c + 1) * p.block_k <= qb * p.block_q]
                else:
                    adm = list(range(p.n_kblocks))
                c_n = int(r.cnt[b, h, qb])
                sel = r.idx[b, h, qb, :c_n].tolist()
                assert c_n == min(p.top_k, len(adm))
                assert (r.idx[b, h, qb, c_n:] == -1).all()
                assert sel == sorted(sel) and len(set(sel)) == c_n
                assert set(sel) <= set(adm)
                s = {c: float(np.dot(qsum[b, h, qb], mu[c])) for c in adm}
                for a in sel:
                    for u in set(adm) - set(sel):
                        assert (s[a] > s[u]) or (s[a] == s[u] and a < u), (qb, a, u)


@pytest.mark.parametrize("causal", [True, False])
def test_route_selection_property_with_planted_ties(causal):
    # entries in {-1, 0, 1} with Bk = 2 make block means multiples of 1/2 and
    # scores multiples of 1/4: exact ties are frequent, so the lower-index rule
    # is exercised many times
    rng = np.random.default_rng(7)
    p = _params(B=2, Hq=4, Hkv=2, N=48, D=3, block_k=2, block_q=4, top_k=3,
                window=3, causal=causal)
    q = rng.integers(-1, 2, size=(2, 4, 48, 3)).astype(np.float64)
    k = rng.integers(-1, 2, size=(2, 2, 48, 3)).astype(np.float64)
    qs, ks = O.block_summary(q, 4), O.block_summary(k, 2)
    r = O.route(qs, ks, p)
    _route_property_check(qs, ks, r, p)
    ties = 0
    for b in range(2):
        for h in range(4):
            for qb in range(p.n_qblocks):
                sc = ks[b, h // 2] @ qs[b, h, qb]
                ties += len(sc) - len(np.unique(sc))
    assert ties > 20


def test_route_all_equal_keys_pick_lowest_indices():
    p = _params(N=64, D=4, block_k=4, block_q=4, top_k=5, window=4)
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 1, 64, 4))
    k = np.ones((1, 1, 64, 4))
    r = O.route(O.block_summary(q, 4), O.block_summary(k, 4), p)
    for qb in range(16):
        n = min(5, qb)
        assert r.idx[0, 0, qb, :n].tolist() == list(range(n))
        assert r.cnt[0, 0, qb] == n


def test_route_brute_force_tiny():
    # brute force: enumerate every subset of the admissible blocks of the right
    # size; the chosen one is the unique subset that beats its complement
    import itertools
    rng = np.random.default_rng(3)
    p = _params(N=24, D=2, block_k=3, block_q=3, top_k=3, window=1)
    q = rng.standard_normal((1, 1, 24, 2))
    k = rng.standard_normal((1, 1, 24, 2))
    qs, ks = O.block_summary(q, 3), O.block_summary(k, 3)
    r = O.route(qs, ks, p)
    for qb in range(8):
        adm = list(range(qb))
        s = ks[0, 0, :qb] @ qs[0, 0, qb]
        n = min(3, qb)
        best = max(itertools.combinations(adm, n), key=lambda sub: sorted(s[list(sub)])[::-1])
        assert sorted(best) == r.idx[0, 0, qb, :n].tolist()


@pytest.mark.parametrize("causal,bq,bk,k,chunk", [
    (True, 4, 2, 3, 5), (False, 4, 2, 3, 7), (True, 2, 4, 5, 3), (True, 4, 4, 40, 4),
    (False, 2, 2, 1, 100), (True, 8, 2, 6, 2)])
def test_route_flat_all_equals_the_per_row_route(causal, bq, bk, k, chunk):
    # integer entries make exact ties frequent; chunks smaller than the row
    # count cross chunk boundaries; k = 40 exceeds every row's admissible set
    rng = np.random.default_rng(11)
    p = _params(B=2, Hq=4, Hkv=2, N=64, D=3, block_k=bk, block_q=bq, top_k=k,
                window=0 if not causal else 3, causal=causal)
    q = rng.integers(-1, 2, size=(2, 4, 64, 3)).astype(np.float64)
    kk = rng.integers(-1, 2, size=(2, 2, 64, 3)).astype(np.float64)
    qs, ks = O.block_summary(q, bq), O.block_summary(kk, bk)
    a = O.route(qs, ks, p)
    b = O.route_flat_all(qs, ks, p, chunk=chunk)
    np.testing.assert_array_equal(a.idx, b.idx)
    np.testing.assert_array_equal(a.cnt, b.cnt)
    np.testing.assert_array_equal(a.kth, b.kth)
    np.testing.assert_array_equal(a.next, b.next)
    _route_property_check(qs, ks, b, p)


def test_route_flat_all_brute_force_and_restriction():
    # independent of the per-row route: for every row, the selection is the
    # first top_k of a full Python sort of (-score, index); restricted to one
    # (b, head) the other heads stay empty
    rng = np.random.default_rng(4)
    p = _params(B=1, Hq=3, Hkv=1, N=96, D=4, block_k=4, block_q=4, top_k=4, window=2)
    q = rng.integers(-2, 3, size=(1, 3, 96, 4)).astype(np.float64)
    kk = rng.integers(-2, 3, size=(1, 1, 96, 4)).astype(np.float64)
    qs, ks = O.block_summary(q, 4), O.block_summary(kk, 4)
    r = O.route_flat_all(qs, ks, p, chunk=8)
    for h in range(3):
        for qb in range(p.n_qblocks):
            cand = [(-float(ks[0, 0, c] @ qs[0, h, qb]), c) for c in range(qb)]
            want = sorted(c for _, c in sorted(cand)[:4])
            assert r.idx[0, h, qb, :r.cnt[0, h, qb]].tolist() == want
    only = O.route_flat_all(qs, ks, p, heads=[(0, 1)])
    np.testing.assert_array_equal(only.idx[0, 1], r.idx[0, 1])
    assert (only.cnt[0, 0] == 0).all() and (only.idx[0, 2] == -1).all()


def test_route_flat_all_rejects_non_finite_summaries():
    p = _params(N=16, D=2, block_k=2, block_q=2, top_k=2, window=2)
    qs = np.zeros((1, 1, 8, 2))
    ks = np.zeros((1, 1, 8, 2))
    ks[0, 0, 3, 1] = np.nan
    with pytest.raises(ValueError):
        O.route_flat_all(qs, ks, p)


# ---------------------------------------------------------------- attend: special cases
def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask=None, causal=False, gqa=False):
    t = [torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v)]
    m = None if mask is None else torch.from_numpy(mask)
    return F.scaled_dot_product_attention(t[0], t[1], t[2], attn_mask=m, is_causal=causal,
                                          enable_gqa=gqa).numpy()


@pytest.mark.parametrize("D,Hq,Hkv,bk", [(16, 2, 2, 8), (32, 4, 2, 16), (64, 6, 2, 32)])
def test_dense_causal_when_topk_covers_every_block(D, Hq, Hkv, bk):
    N = 8 * bk
    p = _params(B=2, Hq=Hq, Hkv=Hkv, N=N, D=D, block_k=bk, block_q=bk, top_k=N // bk,
                window=bk)
    q, k, v = _rand((2, Hq, N, D), 1), _rand((2, Hkv, N, D), 2), _rand((2, Hkv, N, D), 3)
    out = O.forward(q, k, v, p)
    want = _sdpa(q, k, v, causal=True, gqa=Hq != Hkv)
    np.testing.assert_allclose(out["o"], want, atol=1e-12, rtol=0)


def test_dense_noncausal_when_topk_covers_every_block():
    N, D, bk = 128, 16, 16
    p = _params(B=1, Hq=2, Hkv=1, N=N, D=D, block_k=bk, block_q=bk, top_k=N // bk,
                window=0, causal=False)
    q, k, v = _rand((1, 2, N, D), 4), _rand((1, 1, N, D), 5), _rand((1, 1, N, D), 6)
    out = O.forward(q, k, v, p)
    want = _sdpa(q, k, v, gqa=True)
    np.testing.assert_allclose(out["o"], want, atol=1e-12, rtol=0)


@pytest.mark.parametrize("W", [1, 5, 16, 40])
def test_sliding_window_when_topk_is_zero(W):
    N, D = 96, 8
    p = _params(B=1, Hq=1, Hkv=1, N=N, D=D, block_k=16, block_q=16, top_k=0, window=W)
    q, k, v = _rand((1, 1, N, D), 8), _rand((1, 1, N, D), 9), _rand((1, 1, N, D), 10)
    out = O.forward(q, k, v, p)
    # textbook sliding-window attention: query i sees the W most recent keys
    band = np.zeros((N, N), dtype=bool)
    for i in range(N):
        band[i, max(0, i - W + 1):i + 1] = True
    want = _sdpa(q, k, v, mask=band)
    np.testing.assert_allclose(out["o"], want, atol=1e-12, rtol=0)


def test_explicit_scale_is_used():
    N, D = 64, 8
    p = _params(B=1, Hq=1, Hkv=1, N=N, D=D, block_k=8, block_q=8, top_k=8, window=8,
                scale=0.37)
    q, k, v = _rand((1, 1, N, D), 11), _rand((1, 1, N, D), 12), _rand((1, 1, N, D), 13)
    out = O.forward(q, k, v, p)
    t = [torch.from_numpy(a) for a in (q, k, v)]
    want = F.scaled_dot_product_attention(*t, is_causal=True, scale=0.37).numpy()
    np.testing.assert_allclose(out["o"], want, atol=1e-12, rtol=0)


# ---------------------------------------------------------------- attend: invariants
@pytest.mark.parametrize("causal", [True, False])
def test_weights_are_a_distribution_on_the_key_set(causal):
    # V = identity makes O the attention-weight matrix itself
    N, D = 48, 4
    p = _params(B=1, Hq=1, Hkv=1, N=N, D=D, block_k=4, block_q=4, top_k=3,
                window=5 if causal else 0, causal=causal)
    q, k = _rand((1, 1, N, D), 14), _rand((1, 1, N, D), 15)
    v = np.eye(N)[None, None]
    out = O.forward(q, k, v, p)
    wts = out["o"][0, 0]
    np.testing.assert_allclose(wts.sum(axis=1), 1.0, atol=1e-14)
    assert (wts >= 0).all()
    scale = 1 / math.sqrt(D)
    for i in range(N):
        qb = i // 4
        sel = out["idx"][0, 0, qb, :out["cnt"][0, 0, qb]]
        # key set written from the definition: routed blocks' keys, plus the
        # causal window, cut at i
        member = np.zeros(N, dtype=bool)
        for c in sel:
            member[c * 4:(c + 1) * 4] = True
        if causal:
            member[max(0, i - 4):i + 1] = True
            member[i + 1:] = False
        assert (wts[i, ~member] == 0).all()
        assert (wts[i, member] > 0).all()
        logits = k[0, 0] @ q[0, 0, i] * scale
        j0 = np.flatnonzero(member)[0]
        np.testing.assert_allclose(wts[i, member] / wts[i, j0],
                                   np.exp(logits[member] - logits[j0]), rtol=1e-12)


def test_key_set_is_a_set_and_obeys_cardinality_bound():
    # routed block overlapping the window must be counted once, and
    # |S_i| <= W + k*Bk (jonsmirl/ssa README, "Mathematical status": union with
    # a fixed carrier has a uniform W + C cardinality bound)
    p = _params(N=256, D=4, block_k=16, block_q=16, top_k=4, window=40)
    rng = np.random.default_rng(0)
    for i in rng.integers(0, 256, size=60):
        qb = i // 16
        sel = rng.choice(max(qb, 1), size=min(4, qb), replace=False) if qb else np.zeros(0, int)
        s = O.key_set(int(i), np.sort(sel), p)
        assert len(s) == len(np.unique(s))
        assert len(s) <= p.window + p.top_k * p.block_k
        assert s.max() <= i and (s >= max(0, i - 39)).sum() >= min(40, i + 1)


def test_append_law_of_the_read():
    # jonsmirl/ssa README, "Mathematical status": appending a fresh item of mass
    # a to an old mass Z moves the read by a/(Z+a) times the fresh value's
    # displacement from the old read, and the potential by log(1 + a/Z).
    # With Bk = 1, non-causal, every block is one key; selecting one more block
    # appends exactly one item.
    N, D = 32, 6
    p2 = _params(N=N, D=D, block_k=1, block_q=1, top_k=2, window=0, causal=False)
    p3 = _params(N=N, D=D, block_k=1, block_q=1, top_k=3, window=0, causal=False)
    q, k, v = _rand((1, 1, N, D), 21), _rand((1, 1, N, D), 22), _rand((1, 1, N, 5), 23)
    idx2 = np.full((1, 1, N, 2), -1, np.int32)
    idx3 = np.full((1, 1, N, 3), -1, np.int32)
    rng = np.random.default_rng(5)
    extra = np.zeros(N, int)
    for i in range(N):
        trio = rng.choice(N, size=3, replace=False)
        idx2[0, 0, i] = np.sort(trio[:2])
        idx3[0, 0, i] = np.sort(trio)
        extra[i] = trio[2]
    cnt2 = np.full((1, 1, N), 2, np.int32)
    cnt3 = np.full((1, 1, N), 3, np.int32)
    o2, l2 = O.attend_gathered(q, k, v, idx2, cnt2, p2)
    o3, l3 = O.attend_gathered(q, k, v, idx3, cnt3, p3)
    scale = 1 / math.sqrt(D)
    for i in range(N):
        ell = float(k[0, 0, extra[i]] @ q[0, 0, i]) * scale
        a_over_z = math.exp(ell - l2[0, 0, i])             # a / Z
        assert l3[0, 0, i] == pytest.approx(l2[0, 0, i] + math.log1p(a_over_z), abs=1e-12)
        frac = a_over_z / (1 + a_over_z)                   # a / (Z + a)
        want = o2[0, 0, i] + frac * (v[0, 0, extra[i]] - o2[0, 0, i])
        np.testing.assert_allclose(o3[0, 0, i], want, atol=1e-12)


def test_future_keys_do_not_move_past_outputs():
    N, D = 128, 8
    p = _params(B=1, Hq=2, Hkv=1, N=N, D=D, block_k=8, block_q=16, top_k=3, window=10)
    q, k, v = _rand((1, 2, N, D), 31), _rand((1, 1, N, D), 32), _rand((1, 1, N, D), 33)
    base = O.forward(q, k, v, p)
    for cut in (15, 47, 96):
        k2, v2 = k.copy(), v.copy()
        k2[:, :, cut + 1:] = _rand(k2[:, :, cut + 1:].shape, cut)
        v2[:, :, cut + 1:] = _rand(v2[:, :, cut + 1:].shape, cut + 1)
        out = O.forward(q, k2, v2, p)
        # every query at or before the cut is unchanged, bit for bit
        np.testing.assert_array_equal(out["o"][:, :, :cut + 1], base["o"][:, :, :cut + 1])


def test_masked_dense_and_gathered_forms_agree():
    N, D = 192, 16
    p = _params(B=2, Hq=4, Hkv=2, N=N, D=D, block_k=16, block_q=32, top_k=3, window=23)
    q, k, v = _rand((2, 4, N, D), 41), _rand((2, 2, N, D), 42), _rand((2, 2, N, D), 43)
    a = O.forward(q, k, v, p, form="dense")
    b = O.forward(q, k, v, p, form="gathered")
    np.testing.assert_allclose(a["o"], b["o"], atol=1e-12, rtol=0)
    np.testing.assert_allclose(a["lse"], b["lse"], atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal,bq,bk,W", [(True, 32, 16, 23), (True, 16, 32, 40),
                                            (False, 16, 16, 0), (True, 16, 16, 1)])
def test_block_gathered_form_agrees_with_masked_dense(causal, bq, bk, W):
    N, D = 192, 16
    p = _params(B=2, Hq=4, Hkv=2, N=N, D=D, block_k=bk, block_q=bq, top_k=3, window=W,
                causal=causal)
    q, k, v = _rand((2, 4, N, D), 51), _rand((2, 2, N, D), 52), _rand((2, 2, N, D), 53)
    r = O.forward(q, k, v, p, form="dense")
    blocks = [(b, h, qb) for b in range(2) for h in range(4) for qb in range(N // bq)]
    o, l = O.attend_gathered_blocks(q, k, v, r["idx"], r["cnt"], p, blocks)
    o_ref = np.stack([r["o"][b, h, qb * bq:(qb + 1) * bq] for b, h, qb in blocks])
    l_ref = np.stack([r["lse"][b, h, qb * bq:(qb + 1) * bq] for b, h, qb in blocks])
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(l, l_ref, atol=1e-12, rtol=0)


def test_lse_against_dense_logsumexp():
    N, D = 64, 8
    p = _params(N=N, D=D, block_k=8, block_q=8, top_k=8, window=8)
    q, k, v = _rand((1, 1, N, D), 51), _rand((1, 1, N, D), 52), _rand((1, 1, N, D), 53)
    out = O.forward(q, k, v, p)
    t = torch.from_numpy(q[0, 0]) @ torch.from_numpy(k[0, 0]).T / math.sqrt(D)
    t = t.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(out["lse"][0, 0], torch.logsumexp(t, dim=1).numpy(), atol=1e-12)


def test_near_tie_rows_flags_only_close_scores():
    r = O.RouteResult(idx=None, cnt=None,
                      kth=np.array([1.0, 1.0, -2.0, 5.0, np.nan]),
                      next=np.array([0.99995, 0.9, -2.0001, np.nan, np.nan]))
    assert O.near_tie_rows(r).tolist() == [True, False, True, False, False]


def test_bf16_upcast_is_exact():
    u = np.array([0x3F80, 0xBF80, 0x0000, 0x7F7F, 0x0001, 0x4049], dtype=np.uint16)
    want = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.upcast_bf16(u), want)


def test_acceptable_selections_cover_near_ties():
    # scores 3, 2, 1.99999, 1.99998, 0 with k = 2: block 0 is sure, then any
    # one of the three band blocks 1, 2, 3
    mu = np.array([[3.0], [2.0], [1.99999], [1.99998], [0.0]])
    q = np.array([1.0])
    cand = np.arange(5)
    acc = O.acceptable_selections(q, mu, cand, 2)
    assert [a.tolist() for a in acc] == [[0, 1], [0, 2], [0, 3]]
    sel, kth, nxt = O.route_row(q, mu, cand, 2)
    assert sel.tolist() == [0, 1]
    # no near tie: exactly the lexicographic selection
    acc = O.acceptable_selections(q, mu[[0, 1, 4]], np.arange(3), 2)
    assert [a.tolist() for a in acc] == [[0, 1]]


# ---------------------------------------------------------------- consensus route
def _read_consensus_votes():
    cases = []
    with open(os.path.join(GOLDEN, "consensus_votes.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, heads, want = (x.strip() for x in line.split("|"))
            sels = [[int(c) for c in h.split()] for h in heads.split(";")]
            cases.append((int(k), sels, [int(c) for c in want.split()]))
    return cases


def test_consensus_votes_match_hand_derivation():
    cases = _read_consensus_votes()
    assert len(cases) == 7
    for k, sels, want in cases:
        assert O.consensus_row(sels, k).tolist() == want, (k, sels)


def test_consensus_brute_force_tiny():
    # brute force: among all subsets of the voted blocks of the right size, the
    # consensus is the unique one whose every member beats every non-member in
    # (votes desc, index asc)
    import itertools
    rng = np.random.default_rng(5)
    for trial in range(300):
        g = int(rng.integers(1, 5))
        k = int(rng.integers(1, 5))
        sels = [sorted(rng.choice(9, size=int(rng.integers(0, k + 1)), replace=False).tolist())
                for _ in range(g)]
        votes = {}
        for s in sels:
            for c in s:
                votes[c] = votes.get(c, 0) + 1
        voted = sorted(votes)
        m = min(k, len(voted))
        ok = [sub for sub in itertools.combinations(voted, m)
              if all((votes[a], -a) > (votes[u], -u) for a in sub for u in set(voted) - set(sub))]
        assert len(ok) == 1
        assert O.consensus_row(sels, k).tolist() == list(ok[0]), (sels, k)


def _gqa_inputs(p, seed, same_heads=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((p.B, p.Hq, p.N, p.D))
    if same_heads:
        q = np.repeat(q[:, ::p.group], p.group, axis=1)
    k = rng.standard_normal((p.B, p.Hkv, p.N, p.D))
    v = rng.standard_normal((p.B, p.Hkv, p.N, p.D))
    return q, k, v


def test_consensus_with_groups_of_one_is_the_per_head_route():
    p = _params(B=2, Hq=3, Hkv=3, N=96, D=4, block_k=8, block_q=8, top_k=3, window=8,
                consensus=True)
    q, k, v = _gqa_inputs(p, 21)
    out = O.forward(q, k, v, p)
    r = out["route"]
    np.testing.assert_array_equal(out["idx"], r.idx)
    np.testing.assert_array_equal(out["cnt"], r.cnt)
    per_head = O.forward(q, k, v, O.Params(**{**p.__dict__, "consensus": False}))
    np.testing.assert_array_equal(out["o"], per_head["o"])


def test_consensus_of_identical_heads_is_their_own_route():
    p = _params(B=1, Hq=6, Hkv=2, N=128, D=4, block_k=8, block_q=8, top_k=4, window=10,
                consensus=True)
    q, k, v = _gqa_inputs(p, 22, same_heads=True)
    out = O.forward(q, k, v, p)
    per_head = O.forward(q, k, v, O.Params(**{**p.__dict__, "consensus": False}))
    for kv in range(2):
        for h in range(kv * 3, kv * 3 + 3):
            np.testing.assert_array_equal(out["idx"][:, kv], per_head["idx"][:, h])
    np.testing.assert_allclose(out["o"], per_head["o"], atol=1e-13, rtol=0)


def test_consensus_differs_from_per_head_routes_when_heads_disagree():
    # not a tautology: with independent queries the shared list replaces many
    # heads' own choices, and the outputs move
    p = _params(B=1, Hq=4, Hkv=1, N=256, D=8, block_k=16, block_q=16, top_k=3, window=16,
                consensus=True)
    q, k, v = _gqa_inputs(p, 23)
    out = O.forward(q, k, v, p)
    own = out["route"].idx
    shared = O.expand_consensus(out["idx"], out["cnt"], p)[0]
    assert (own != shared).any(axis=-1).mean() > 0.3
    per_head = O.forward(q, k, v, O.Params(**{**p.__dict__, "consensus": False}))
    assert np.abs(out["o"] - per_head["o"]).max() > 1e-3


@pytest.mark.parametrize("D,Hq,Hkv,bk", [(16, 4, 2, 8), (32, 6, 2, 16)])
def test_consensus_dense_causal_when_topk_covers_every_block(D, Hq, Hkv, bk):
    N = 8 * bk
    p = _params(B=2, Hq=Hq, Hkv=Hkv, N=N, D=D, block_k=bk, block_q=bk, top_k=N // bk,
                window=bk, consensus=True)
    q, k, v = _rand((2, Hq, N, D), 4), _rand((2, Hkv, N, D), 5), _rand((2, Hkv, N, D), 6)
    out = O.forward(q, k, v, p)
    want = _sdpa(q, k, v, causal=True, gqa=True)
    np.testing.assert_allclose(out["o"], want, atol=1e-12, rtol=0)


@pytest.mark.parametrize("form", ["dense", "gathered"])
def test_consensus_worked_example_matches_hand_derivation(form):
    q0, k, v = _worked_inputs()
    q1 = np.tile(np.array([[2.0, 0.0]]), (8, 1))[None, None]
    q = np.concatenate([q0, q1], axis=1)
    p = _params(Hq=2, Hkv=1, top_k=1, consensus=True)
    out = O.forward(q, k, v, p, form=form)
    assert out["route"].idx[0, :, :, 0].tolist() == [[-1, 0, 1, 1], [-1, 0, 0, 0]]
    assert out["idx"][0, 0, :, 0].tolist() == [-1, 0, 0, 0]
    E = math.exp(math.sqrt(2.0))
    n = 0
    with open(os.path.join(GOLDEN, "consensus_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            h, i, expr = line.split(maxsplit=2)
            assert out["o"][0, int(h), int(i), 0] == pytest.approx(eval(expr, {"E": E}),
                                                                 abs=1e-12)
            assert out["o"][0, int(h), int(i), 1] == pytest.approx(1.0, abs=1e-12)
            n += 1
    assert n == 16


# ---------------------------------------------------------------- second-cumulant score
def test_block_covariance_and_second_moment_match_numpy():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((2, 3, 48, 5))
    cov = O.block_covariance(x, 8)
    m2 = O.block_second_moment(x, 8)
    for b in range(2):
        for h in range(3):
            for c in range(6):
                xb = x[b, h, c * 8:(c + 1) * 8]
                np.testing.assert_allclose(cov[b, h, c], np.cov(xb.T, bias=True), atol=1e-13)
                np.testing.assert_allclose(m2[b, h, c], xb.T @ xb / 8, atol=1e-13)
    # a block of one row has no spread
    assert np.abs(O.block_covariance(x, 1)).max() == 0.0


def test_second_cumulant_route_matches_hand_derivation():
    k = np.array([[0, 0], [0, 0], [1, 0], [-1, 0], [0.5, 0], [0.5, 0], [0, 1], [0, 1]],
                 dtype=np.float64)[None, None]
    q = np.zeros((1, 1, 8, 2))
    q[0, 0, 6] = (2.0, 0.0)
    v = np.stack([np.arange(8.0), np.ones(8)], axis=1)[None, None]
    n = 0
    with open(os.path.join(GOLDEN, "second_cumulant_route.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            beta, kk, want = float(parts[0]), int(parts[1]), [int(c) for c in parts[2:]]
            p = _params(top_k=kk, beta=beta)
            out = O.forward(q, k, v, p)
            assert out["idx"][0, 0, 3, :kk].tolist() == want, (beta, kk)
            n += 1
    assert n == 9


def test_block_score_is_the_mean_of_per_query_scores():
    # brute force over the block's queries of r_c(q_i) = <q_i, mu_c> + (beta/2) q_i^T Sigma_c q_i
    rng = np.random.default_rng(32)
    D, Bk, Bq = 6, 4, 8
    k = rng.standard_normal((1, 1, 64, D))
    q = rng.standard_normal((1, 1, 64, D))
    mu, cov = O.block_summary(k, Bk), O.block_covariance(k, Bk)
    qbar, qm2 = O.block_summary(q, Bq), O.block_second_moment(q, Bq)
    cand = np.arange(16)
    for beta in (0.0, 0.7, -1.3):
        for qb in range(8):
            got = O.block_scores(qbar[0, 0, qb], mu[0, 0], cand, beta, qm2[0, 0, qb], cov[0, 0])
            rows = q[0, 0, qb * Bq:(qb + 1) * Bq]
            want = np.zeros(16)
            for c in cand:
                kc = k[0, 0, c * Bk:(c + 1) * Bk]
                sig = (kc - kc.mean(0)).T @ (kc - kc.mean(0)) / Bk
                want[c] = np.mean([qi @ kc.mean(0) + 0.5 * beta * qi @ sig @ qi for qi in rows])
            np.testing.assert_allclose(got, want, atol=1e-12)


def test_second_cumulant_with_zero_beta_or_no_spread_is_the_mean_route():
    rng = np.random.default_rng(33)
    p0 = _params(B=1, Hq=2, Hkv=1, N=128, D=4, block_k=8, block_q=8, top_k=3, window=8)
    q, k, v = rng.standard_normal((1, 2, 128, 4)), rng.standard_normal((1, 1, 128, 4)), \
        rng.standard_normal((1, 1, 128, 4))
    base = O.forward(q, k, v, p0)
    # keys constant inside each block: Sigma_c = 0 for every beta
    kc = np.repeat(k[:, :, ::8], 8, axis=2)
    flat0 = O.forward(q, kc, v, p0)
    flat1 = O.forward(q, kc, v, O.Params(**{**p0.__dict__, "beta": 2.5}))
    np.testing.assert_array_equal(flat0["idx"], flat1["idx"])
    # and a nonzero beta moves some selections on spread blocks
    moved = O.forward(q, k, v, O.Params(**{**p0.__dict__, "beta": 4.0}))
    assert (moved["idx"] != base["idx"]).any()


# ---------------------------------------------------------------- decode step
@pytest.mark.parametrize("kk", [0, 1, 2, 4])
def test_decode_steps_match_hand_derivation(kk):
    # in the 4-block example the decode admissible set of every position equals
    # its query block's, so the hand-derived prefill values hold per step
    q, k, v = _worked_inputs()
    E = math.exp(math.sqrt(2.0))
    want = {i: eval(expr, {"E": E}) for k_, i, expr in _read_worked_golden() if k_ == kk}
    assert len(want) == (2 if kk == 4 else 8)
    p = _params(top_k=kk)
    for i, val in want.items():
        o, lse, idx, cnt = O.decode_step(q[:, :, i], k, v, i + 1, p)
        assert o[0, 0, 0] == pytest.approx(val, abs=1e-12), (kk, i)
        assert o[0, 0, 1] == pytest.approx(1.0, abs=1e-12)


def test_decode_step_equals_prefill_with_query_blocks_of_one():
    rng = np.random.default_rng(41)
    p = _params(B=2, Hq=4, Hkv=2, N=96, D=8, block_k=8, block_q=1, top_k=3, window=10)
    q, k, v = _rand((2, 4, 96, 8), 42), _rand((2, 2, 96, 8), 43), _rand((2, 2, 96, 8), 44)
    full = O.forward(q, k, v, p)                       # masked-dense form, Bq = 1
    for i in list(range(0, 96, 7)) + [95]:
        o, lse, idx, cnt = O.decode_step(q[:, :, i], k, v, i + 1, p)
        np.testing.assert_allclose(o, full["o"][:, :, i], atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse, full["lse"][:, :, i], atol=1e-12, rtol=0)
        np.testing.assert_array_equal(idx, full["idx"][:, :, i])
        # the cache beyond n_ctx is never read
        k2, v2 = k.copy(), v.copy()
        k2[:, :, i + 1:] = rng.standard_normal(k2[:, :, i + 1:].shape) * 50
        v2[:, :, i + 1:] = 7.0
        o2, _, _, _ = O.decode_step(q[:, :, i], k2, v2, i + 1, p)
        np.testing.assert_array_equal(o2, o)


def test_decode_step_dense_and_sliding_window_limits():
    N, D, bk = 160, 16, 16
    q, k, v = _rand((1, 4, N, D), 45), _rand((1, 2, N, D), 46), _rand((1, 2, N, D), 47)
    i = N - 1
    dense = _params(B=1, Hq=4, Hkv=2, N=N, D=D, block_k=bk, block_q=1, top_k=N // bk, window=bk)
    o, _, _, _ = O.decode_step(q[:, :, i], k, v, N, dense)
    want = _sdpa(q[:, :, i:i + 1], k, v, gqa=True)[:, :, 0]
    np.testing.assert_allclose(o, want, atol=1e-12, rtol=0)
    W = 37
    win = _params(B=1, Hq=4, Hkv=2, N=N, D=D, block_k=bk, block_q=1, top_k=0, window=W)
    o, _, _, _ = O.decode_step(q[:, :, i], k, v, N, win)
    want = _sdpa(q[:, :, i:i + 1], k[:, :, i - W + 1:], v[:, :, i - W + 1:], gqa=True)[:, :, 0]
    np.testing.assert_allclose(o, want, atol=1e-12, rtol=0)


# ---------------------------------------------------------------- two-level (tree) routing
def _tree_worked_inputs():
    k = np.array([[1, 0], [1, 0], [4, 0], [-4, 0], [0, 1], [0, 0], [2, 0], [0, 0]],
                 dtype=np.float64)[None, None]
    q = np.tile(np.array([[1.0, 0.0]]), (8, 1))[None, None]
    return q, k


def _lst(tok):
    return [] if tok == "-" else [int(x) for x in tok.split(",")]


def test_tree_route_matches_hand_derivation():
    q, k = _tree_worked_inputs()
    ksum = O.block_summary(k, 1)
    qsum = O.block_summary(q, 1)
    ksum2 = O.tree_summary(k, 1, 2)
    assert ksum2[0, 0].tolist() == [[1, 0], [0, 0], [0, 0.5], [1, 0]]
    n = 0
    with open(os.path.join(GOLDEN, "tree_route.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            causal, qb, beam, kk, sup, sel = line.split()
            causal = bool(int(causal))
            p = _params(N=8, block_k=1, block_q=1, top_k=int(kk), causal=causal,
                        window=1 if causal else 0, tree_fanout=2, tree_beam=int(beam))
            r = O.route(qsum, ksum, p, rows=[(0, 0, int(qb))], ksum2=ksum2)
            row = (0, 0, int(qb))
            assert r.sup_idx[row][:r.sup_cnt[row]].tolist() == _lst(sup), line
            assert r.idx[row][:r.cnt[row]].tolist() == _lst(sel), line
            n += 1
    assert n == 10


def test_tree_summary_is_the_mean_of_its_child_block_means():
    rng = np.random.default_rng(41)
    k = rng.standard_normal((2, 3, 16 * 22, 5))          # 22 blocks of 16: 5 super-blocks of 4
    got = O.tree_summary(k, 16, 4)
    assert got.shape == (2, 3, 5, 5)
    mu = O.block_summary(k, 16)
    for s in range(5):
        np.testing.assert_allclose(got[:, :, s], mu[:, :, 4 * s:4 * s + 4].mean(axis=2),
                                   atol=1e-14)
        np.testing.assert_allclose(got[:, :, s], k[:, :, 64 * s:64 * s + 64].mean(axis=2),
                                   atol=1e-14)


def _tree_case(causal, N=16 * 22, D=6, bk=16, F=4, beam=2, top_k=3, Hq=2, Hkv=1, seed=43):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, Hq, N, D))
    k = rng.standard_normal((1, Hkv, N, D)) + rng.standard_normal((1, Hkv, N // bk, 1, D)).repeat(
        bk, axis=2).reshape(1, Hkv, N, D)
    p = _params(Hq=Hq, Hkv=Hkv, N=N, D=D, block_k=bk, block_q=bk, top_k=top_k, causal=causal,
                window=bk if causal else 0, tree_fanout=F, tree_beam=beam)
    return p, q, k


@pytest.mark.parametrize("causal", [True, False])
def test_tree_keeping_every_super_block_is_the_flat_route(causal):
    p, q, k = _tree_case(causal, beam=64, top_k=4)
    ksum, qsum = O.block_summary(k, p.block_k), O.block_summary(q, p.block_q)
    tree = O.route(qsum, ksum, p, ksum2=O.tree_summary(k, p.block_k, p.tree_fanout))
    flat = O.route(qsum, ksum, O.Params(**{**p.__dict__, "tree_fanout": 0, "tree_beam": 0}))
    np.testing.assert_array_equal(tree.idx, flat.idx)
    np.testing.assert_array_equal(tree.cnt, flat.cnt)
    assert (tree.cnt > 0).any()


def test_tree_with_fanout_one_keeps_the_flat_top_k():
    p, q, k = _tree_case(True, F=1, beam=5, top_k=3)
    ksum, qsum = O.block_summary(k, p.block_k), O.block_summary(q, p.block_q)
    tree = O.route(qsum, ksum, p, ksum2=O.tree_summary(k, p.block_k, 1))
    flat = O.route(qsum, ksum, O.Params(**{**p.__dict__, "tree_fanout": 0, "tree_beam": 0}))
    np.testing.assert_array_equal(tree.idx, flat.idx)
    # the upper level alone is the flat top-beam
    flat5 = O.route(qsum, ksum, O.Params(**{**p.__dict__, "tree_fanout": 0, "tree_beam": 0,
                                            "top_k": 5}))
    np.testing.assert_array_equal(tree.sup_idx, flat5.idx)


def _top_set_brute(keys_of, items, m):
    """The one m-subset of ``items`` whose every member's (score, -index) key
    beats every non-member's, found by enumerating all m-subsets."""
    import itertools
    found = []
    for sub in itertools.combinations(items, m):
        rest = [c for c in items if c not in sub]
        if all(keys_of(a) > keys_of(b) for a in sub for b in rest):
            found.append(sorted(sub))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("causal", [True, False])
def test_tree_route_matches_brute_force_on_tiny_integer_inputs(causal):
    from fractions import Fraction
    rng = np.random.default_rng(47 + causal)
    bk, F, N, D, beam, top_k = 4, 2, 52, 3, 2, 3            # 13 blocks: 6 super-blocks + 1
    # small integers: exact in float64 and full of exact ties
    k = rng.integers(-2, 3, size=(1, 1, N, D)).astype(np.float64)
    q = rng.integers(-2, 3, size=(1, 1, N, D)).astype(np.float64)
    p = _params(N=N, D=D, block_k=bk, block_q=bk, top_k=top_k, causal=causal,
                window=bk if causal else 0, tree_fanout=F, tree_beam=beam)
    r = O.route(O.block_summary(q, bk), O.block_summary(k, bk), p,
                ksum2=O.tree_summary(k, bk, F))
    kk, qq = k[0, 0].astype(int).tolist(), q[0, 0].astype(int).tolist()

    def mean_rows(x, lo, hi):
        return [Fraction(sum(x[t][d] for t in range(lo, hi)), hi - lo) for d in range(D)]

    nb = N // bk
    for qb in range(N // bk):
        qbar = mean_rows(qq, qb * bk, qb * bk + bk)
        n_adm = min(qb, nb) if causal else nb             # Bq = Bk: c + 1 <= qb
        score_blk = lambda c: sum(a * b for a, b in zip(qbar, mean_rows(kk, c * bk, c * bk + bk)))
        score_sup = lambda s: sum(a * b for a, b in
                                  zip(qbar, mean_rows(kk, s * F * bk, (s + 1) * F * bk)))
        sups = list(range(n_adm // F))
        kept = _top_set_brute(lambda s: (score_sup(s), -s), sups, min(beam, len(sups)))
        cand = [s * F + j for s in kept for j in range(F)] + list(range(len(sups) * F, n_adm))
        sel = _top_set_brute(lambda c: (score_blk(c), -c), cand, min(top_k, len(cand)))
        assert r.sup_idx[0, 0, qb][:r.sup_cnt[0, 0, qb]].tolist() == kept, qb
        assert r.idx[0, 0, qb][:r.cnt[0, 0, qb]].tolist() == sel, qb


def test_tree_acceptable_selections_hold_the_route_and_its_tie_alternatives():
    q, k = _tree_worked_inputs()
    p = _params(N=8, block_k=1, block_q=1, top_k=2, causal=False, window=0, tree_fanout=2,
                tree_beam=1)
    mu, mu2 = O.block_summary(k, 1)[0, 0], O.tree_summary(k, 1, 2)[0, 0]
    qbar = np.array([1.0, 0.0])
    acc = [(a.tolist(), b.tolist()) for a, b in O.acceptable_tree_selections(qbar, mu, mu2, 8, p)]
    # S0 and S3 tie exactly: both beams are acceptable; inside S0, blocks 0
    # and 1 are both taken; inside S3, block 6 and then 7 (score 0, alone)
    assert ([0], [0, 1]) in acc and ([3], [6, 7]) in acc
    assert len(acc) == 2
    sup, sel, _, _ = O.route_tree_row(qbar, mu, mu2, 8, p)
    assert (sup.tolist(), sel.tolist()) == ([0], [0, 1])


def test_tree_forward_attends_over_the_tree_selection():
    p, q, k = _tree_case(True, N=16 * 12, beam=1, top_k=2)
    v = np.random.default_rng(5).standard_normal(k.shape)
    out = O.forward(q, k, v, p)
    r = out["route"]
    assert r.sup_idx is not None and out["ksum2"].shape[2] == 3
    o2, l2 = O.attend_gathered(q, k, v, r.idx, r.cnt, p)
    np.testing.assert_allclose(out["o"], o2, atol=1e-12)
    np.testing.assert_allclose(out["lse"], l2, atol=1e-12)
    # every selected block is a candidate of the row's kept super-blocks
    for qb in range(p.n_qblocks):
        n_adm = len(O.admissible_blocks(qb, p))
        cand = O.tree_candidates(r.sup_idx[0, 0, qb][:r.sup_cnt[0, 0, qb]], n_adm, p.tree_fanout)
        assert set(r.idx[0, 0, qb][:r.cnt[0, 0, qb]].tolist()) <= set(cand.tolist())


# ---------------------------------------------------------------- backward (fixed selection)
def _bwd_case(causal, seed=61, B=1, Hq=4, Hkv=2, N=96, D=5, bk=8, top_k=3, W=10):
    rng = np.random.default_rng(seed)
    p = _params(B=B, Hq=Hq, Hkv=Hkv, N=N, D=D, block_k=bk, block_q=bk, top_k=top_k,
                causal=causal, window=W if causal else 0)
    q = rng.standard_normal((B, Hq, N, D))
    k = rng.standard_normal((B, Hkv, N, D))
    v = rng.standard_normal((B, Hkv, N, D))
    do = rng.standard_normal((B, Hq, N, D))
    r = O.route(O.block_summary(q, bk), O.block_summary(k, bk), p)
    return p, q, k, v, do, r.idx, r.cnt


def _torch_masked_attention(p, q, k, v, idx, cnt):
    """The read as a torch graph: the allowed (query, key) pairs built here
    from the lists and the window, a -inf mask, softmax, weights @ V."""
    B, Hq, N, D = q.shape
    g = p.Hq // p.Hkv
    allow = torch.zeros((B, Hq, N, N), dtype=torch.bool)
    for b in range(B):
        for h in range(Hq):
            for qb in range(N // p.block_q):
                r0, r1 = qb * p.block_q, (qb + 1) * p.block_q
                for c in idx[b, h, qb, :cnt[b, h, qb]]:
                    allow[b, h, r0:r1, c * p.block_k:(c + 1) * p.block_k] = True
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    if p.causal:
        allow |= ((j > i - p.window) & (j <= i))[None, None]
        allow &= (j <= i)[None, None]
    kk = k.repeat_interleave(g, dim=1)
    vv = v.repeat_interleave(g, dim=1)
    s = (q @ kk.transpose(-1, -2)) * p.softmax_scale
    s = s.masked_fill(~allow, float("-inf"))
    return torch.softmax(s, dim=-1) @ vv


@pytest.mark.parametrize("causal", [True, False])
def test_backward_matches_torch_autograd(causal):
    p, q, k, v, do, idx, cnt = _bwd_case(causal)
    dq, dk, dv = O.attend_backward(q, k, v, do, idx, cnt, p)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = _torch_masked_attention(p, tq, tk, tv, idx, cnt)
    o.backward(torch.tensor(do))
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    # the forward of that graph is the oracle's read
    o_ref, _ = O.attend_masked_dense(q, k, v, idx, cnt, p)
    np.testing.assert_allclose(o.detach().numpy(), o_ref, atol=1e-12)


def test_backward_dense_case_matches_sdpa_autograd():
    # every block routed and W >= Bq: the read is dense causal GQA attention
    p, q, k, v, do, _, _ = _bwd_case(True, top_k=12, W=8)
    r = O.route(O.block_summary(q, 8), O.block_summary(k, 8), p)
    dq, dk, dv = O.attend_backward(q, k, v, do, r.idx, r.cnt, p)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(2, dim=1),
                                       tv.repeat_interleave(2, dim=1), is_causal=True)
    o.backward(torch.tensor(do))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.numpy(), atol=1e-11)


def test_backward_matches_central_differences():
    p, q, k, v, do, idx, cnt = _bwd_case(True, N=48, Hq=2, Hkv=1, D=3, bk=8, top_k=2, W=6,
                                         seed=67)
    dq, dk, dv = O.attend_backward(q, k, v, do, idx, cnt, p)

    def loss(q_, k_, v_):
        o, _ = O.attend_masked_dense(q_, k_, v_, idx, cnt, p)
        return float((o * do).sum())

    rng = np.random.default_rng(3)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            pos = tuple(int(rng.integers(n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[pos] += eps
            xm[pos] -= eps
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            a_p = [xp if t is x else t for t in args]
            a_m = [xm if t is x else t for t in args]
            fd = (loss(*a_p) - loss(*a_m)) / (2 * eps)
            assert fd == pytest.approx(grad[pos], abs=2e-7), (name, pos)


def test_backward_shift_invariants():
    # a common shift of every key adds the same logit to a row: no change,
    # so the key gradients of a KV head sum to zero; a common shift of every
    # value shifts every read by it, so the value gradients of a KV head sum
    # to the upstream gradients of its query heads
    p, q, k, v, do, idx, cnt = _bwd_case(True, seed=71)
    _, dk, dv = O.attend_backward(q, k, v, do, idx, cnt, p)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    g = p.group
    for kv in range(p.Hkv):
        want = do[:, kv * g:(kv + 1) * g].sum(axis=(1, 2))
        np.testing.assert_allclose(dv[:, kv].sum(axis=1), want, atol=1e-11)


def test_backward_restricted_to_blocks_sums_to_the_whole():
    p, q, k, v, do, idx, cnt = _bwd_case(True, seed=73)
    dq, dk, dv = O.attend_backward(q, k, v, do, idx, cnt, p)
    blocks = [(0, h, qb) for h in range(p.Hq) for qb in range(p.n_qblocks)]
    a = O.attend_backward(q, k, v, do, idx, cnt, p, blocks=blocks[::2])
    b = O.attend_backward(q, k, v, do, idx, cnt, p, blocks=blocks[1::2])
    np.testing.assert_allclose(a[0] + b[0], dq, atol=1e-12)
    np.testing.assert_allclose(a[1] + b[1], dk, atol=1e-12)
    np.testing.assert_allclose(a[2] + b[2], dv, atol=1e-12)
