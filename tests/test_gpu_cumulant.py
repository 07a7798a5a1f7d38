"""Parity of the second-cumulant routing path (SSA's full score
<q, mu_c> + (beta/2) q^T Sigma_c q, a query block scoring by the mean of its
queries' scores) with the float64 oracle.

Features are compared entry by entry; selections bit-exactly except at the
oracle's counted near-ties (fp64 scores within 1e-4 relative), where the GPU's
choice must be one the oracle enumerates itself; outputs against the oracle's
attend over the oracle-side selection.  No expected value comes from the CUDA
path.
"""
import numpy as np
import pytest
import torch

import oracle as O
from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload
from parity_utils import Case, assert_close, gpu_rows, oracle_attend_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


def W(name, **kw):
    base = dict(B=1, Hq=2, Hkv=1, N=1024, D=64, block_k=64, block_q=64, top_k=4, window=128,
                causal=True, kind="iid", seed=23, beta=0.5)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    W("iid-beta0.5"),
    W("iid-beta-neg", beta=-0.3, Hq=2, Hkv=2),
    W("clustered-gqa7", Hq=14, Hkv=2, N=2048, top_k=8, window=256, kind="clustered",
      centres=16, beta=2.0),
    W("d128", D=128, N=768, top_k=3, window=96, beta=1.0),
    W("bk16", N=512, block_k=16, block_q=16, top_k=5, window=40, beta=4.0),
    W("bk32-bq64-k40", N=4096, block_k=32, block_q=64, top_k=40, window=70, beta=0.25),
    W("noncausal-image", Hq=2, Hkv=2, N=1024, block_k=16, block_q=16, top_k=8, window=0,
      causal=False, kind="image", beta=1.5),
    W("consensus", Hq=4, Hkv=2, N=1024, top_k=6, window=128, consensus=True, beta=0.8),
]


class CumOracle:
    """fp64 second-cumulant summaries of one case, computed per row on demand."""

    def __init__(self, case):
        self.case = case
        self._kcov = {}

    def kcov(self, b, g):
        """[NB, D, D] covariances of KV head g's key blocks."""
        if (b, g) not in self._kcov:
            self._kcov[(b, g)] = O.block_covariance(self.case.k64[b, g], self.case.op.block_k)
        return self._kcov[(b, g)]

    def q2(self, b, h, qb):
        op = self.case.op
        rows = self.case.q64[b, h, qb * op.block_q:(qb + 1) * op.block_q]
        return rows.T @ rows / op.block_q

    def select(self, b, h, qb):
        case, op = self.case, self.case.op
        g = h // op.group
        args = (case.qsum64[b, h, qb], case.ksum64[b, g], O.admissible_blocks(qb, op), op.top_k)
        kw = dict(beta=op.beta, q2=self.q2(b, h, qb), sigma=self.kcov(b, g))
        own, _, _ = O.route_row(*args, **kw)
        return own, (lambda: O.acceptable_selections(*args, **kw))


def check_cumulant_rows(case, idx_g, cnt_g, rows, co=None):
    """As parity_utils.check_route_rows, with the second-cumulant scores."""
    co = co or CumOracle(case)
    op = case.op
    idx = np.full((op.B, op.Hq, op.n_qblocks, op.top_k), -1, np.int32)
    cnt = np.zeros((op.B, op.Hq, op.n_qblocks), np.int32)
    alt = 0
    for b, h, qb in rows:
        own, accepted = co.select(b, h, qb)
        n = int(cnt_g[b, h, qb])
        g = idx_g[b, h, qb, :n]
        assert n == len(own), f"row {(b, h, qb)}: count {n} != {len(own)}"
        assert (idx_g[b, h, qb, n:] == -1).all(), f"row {(b, h, qb)}: bad padding"
        if np.array_equal(g, own):
            chosen = own
        else:
            match = [a for a in accepted() if np.array_equal(a, g)]
            assert match, f"row {(b, h, qb)}: GPU selection {g.tolist()} != {own.tolist()} " \
                          f"and is not an acceptable near-tie alternative"
            chosen = match[0]
            alt += 1
        idx[b, h, qb, :len(chosen)] = chosen
        cnt[b, h, qb] = len(chosen)
    return idx, cnt, alt


def _gpu_route(case):
    p = case.p
    kf = ssa.route_features(case.kd, case.w.block_k, p, queries=False)
    qf = ssa.route_features(case.qd, case.w.block_q, p, queries=True)
    idx, cnt = ssa.route_cumulant(qf, kf, p)
    ssa.check_error()
    return qf, kf, idx, cnt


def _vech(m):
    d = m.shape[-1]
    iu = np.triu_indices(d)
    return m[..., iu[0], iu[1]]


@pytest.mark.parametrize("D,block", [(64, 16), (64, 64), (128, 64), (128, 128)])
def test_route_features_match_fp64_cumulants(D, block):
    case = Case(W("feat", B=2, Hq=2, Hkv=2, N=1024, D=D, beta=1.7, kind="clustered",
                  centres=8))
    p = case.p
    kf = ssa.route_features(case.kd, block, p, queries=False).cpu().numpy().astype(np.float64)
    qf = ssa.route_features(case.qd, block, p, queries=True).cpu().numpy().astype(np.float64)
    ssa.check_error()
    mu = O.block_summary(case.k64, block)
    cov = O.block_covariance(case.k64, block)
    np.testing.assert_allclose(kf[..., :D], mu, rtol=0, atol=1e-5)
    np.testing.assert_allclose(kf[..., D:], _vech(cov), rtol=0, atol=2e-5)
    qbar = O.block_summary(case.q64, block)
    m2 = O.block_second_moment(case.q64, block)
    w = np.where(np.eye(D, dtype=bool), 1.0, 2.0)
    np.testing.assert_allclose(qf[..., :D], qbar, rtol=0, atol=1e-5)
    np.testing.assert_allclose(qf[..., D:], _vech(0.85 * w * m2), rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_cumulant_route_matches_oracle(w):
    case = Case(w.with_(consensus=False))
    _, _, idx, cnt = _gpu_route(case)
    check_cumulant_rows(case, idx.cpu().numpy(), cnt.cpu().numpy(), case.all_rows())


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_cumulant_every_row(w):
    case = Case(w)
    op = case.op
    _, _, h_idx, h_cnt = _gpu_route(case.__class__(w.with_(consensus=False), case.u16))
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    rows = case.all_rows()
    r_idx, r_cnt, _ = check_cumulant_rows(case, h_idx.cpu().numpy(), h_cnt.cpu().numpy(), rows)
    if op.consensus:
        want_idx, want_cnt = O.route_consensus(r_idx, r_cnt, op)
        np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
        np.testing.assert_array_equal(cnt.cpu().numpy(), want_cnt)
        e_idx, e_cnt = O.expand_consensus(want_idx, want_cnt, op)
    else:
        np.testing.assert_array_equal(idx.cpu().numpy(), h_idx.cpu().numpy())
        e_idx, e_cnt = r_idx, r_cnt
    o_ref, l_ref = oracle_attend_rows(case, e_idx, e_cnt, rows)
    assert_close(gpu_rows(o, rows, op.block_q), o_ref, gpu_rows(lse, rows, op.block_q), l_ref,
                 what=w.name)


@pytest.mark.parametrize("cfg,beta,n", [(2, 0.5, 40), (3, 1.0, 24), (4, 1.0, 24)])
def test_forward_cumulant_full_size_sampled(cfg, beta, n):
    case = Case(CONFIGS[cfg].with_(beta=beta))
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    rows = case.sample_rows(n, seed=cfg)
    r_idx, r_cnt, _ = check_cumulant_rows(case, idx.cpu().numpy(), cnt.cpu().numpy(), rows)
    o_ref, l_ref = oracle_attend_rows(case, r_idx, r_cnt, rows)
    bq = case.op.block_q
    assert_close(gpu_rows(o, rows, bq), o_ref, gpu_rows(lse, rows, bq), l_ref, what=case.w.name)
    assert torch.isfinite(o).all()


def test_beta_moves_selections():
    w = W("move", Hq=2, Hkv=1, N=2048, top_k=6, window=128, kind="clustered", centres=16,
          beta=3.0)
    case = Case(w)
    _, _, i3, _ = _gpu_route(case)
    base = Case(w.with_(beta=0.0), case.u16)
    ks = ssa.block_summary(base.kd, 64, base.p)
    qs = ssa.block_summary(base.qd, 64, base.p)
    i0, _ = ssa.route(qs, ks, base.p)
    assert (i3.cpu() != i0.cpu()).any()
