"""Parity of two-level (fixed-beam tree) routing with the float64 oracle.

The super-block means are compared with fp64 means of the keys; the kept
super-blocks and the selections bit-exactly, except at the oracle's counted
near-ties (fp64 scores within 1e-4 relative, at either level), where the
GPU's pair must be one the oracle enumerates itself
(``acceptable_tree_selections``); outputs against the oracle's attend over
the oracle-side selection.  No expected value comes from the CUDA path.
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
    base = dict(B=1, Hq=2, Hkv=1, N=2048, D=64, block_k=64, block_q=64, top_k=4, window=128,
                causal=True, kind="clustered", centres=16, seed=37, tree_fanout=4, tree_beam=2)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    W("f4-beam2"),
    W("gqa7-f16-beam4", Hq=14, Hkv=2, N=8192, top_k=8, window=256, tree_fanout=16, tree_beam=4),
    # 44 blocks: five super-blocks of 8 and a 4-block tail that is always frontier
    W("ragged-tail", N=64 * 44, tree_fanout=8, tree_beam=3, kind="iid"),
    W("d128", D=128, N=1536, top_k=3, window=96, kind="iid"),
    W("bk16-k40", N=2048, block_k=16, block_q=16, top_k=40, window=40, tree_fanout=8,
      tree_beam=8),
    W("bk32-bq64", B=2, N=4096, block_k=32, block_q=64, top_k=12, window=70, tree_fanout=16,
      tree_beam=6),
    W("noncausal-image", Hq=2, Hkv=2, N=4096, block_k=16, block_q=16, top_k=8, window=0,
      causal=False, kind="image", tree_fanout=16, tree_beam=4),
    W("k64-beam64", N=64 * 160, top_k=64, window=64, tree_fanout=2, tree_beam=64),
    W("every-super-block", tree_fanout=4, tree_beam=64),      # the flat route
    W("fanout1", tree_fanout=1, tree_beam=6),
    W("window-only", top_k=0, window=200),
    W("consensus", Hq=4, Hkv=2, top_k=6, consensus=True),
]


class TreeOracle:
    """fp64 super-block summaries of one case and the row checks against them."""

    def __init__(self, case):
        self.case = case
        op = case.op
        self.ksum2 = O.tree_summary(case.k64, op.block_k, op.tree_fanout)

    def row(self, b, h, qb):
        case, op = self.case, self.case.op
        g = h // op.group
        return (case.qsum64[b, h, qb], case.ksum64[b, g], self.ksum2[b, g],
                len(O.admissible_blocks(qb, op)), op)

    def check(self, idx_g, cnt_g, rows, sup_g=None, supc_g=None):
        """Check the GPU's lists on ``rows``; return the oracle-side idx/cnt
        equal to the GPU's selections and the count of near-tie alternatives."""
        op = self.case.op
        idx = np.full((op.B, op.Hq, op.n_qblocks, op.top_k), -1, np.int32)
        cnt = np.zeros((op.B, op.Hq, op.n_qblocks), np.int32)
        alt = 0
        for b, h, qb in rows:
            args = self.row(b, h, qb)
            own_sup, own_sel, _, _ = O.route_tree_row(*args)
            n = int(cnt_g[b, h, qb])
            g_sel = idx_g[b, h, qb, :n]
            assert (idx_g[b, h, qb, n:] == -1).all(), f"row {(b, h, qb)}: bad padding"
            g_sup = None
            if sup_g is not None:
                m = int(supc_g[b, h, qb])
                g_sup = sup_g[b, h, qb, :m]
                assert (sup_g[b, h, qb, m:] == -1).all(), f"row {(b, h, qb)}: bad beam padding"
            same = np.array_equal(g_sel, own_sel) and (
                g_sup is None or np.array_equal(g_sup, own_sup))
            if same:
                chosen = own_sel
            else:
                acc = O.acceptable_tree_selections(*args)
                match = [sel for sup, sel in acc if np.array_equal(sel, g_sel) and (
                    g_sup is None or np.array_equal(sup, g_sup))]
                assert match, (f"row {(b, h, qb)}: GPU kept {None if g_sup is None else g_sup.tolist()}"
                               f" -> {g_sel.tolist()}; oracle {own_sup.tolist()} -> "
                               f"{own_sel.tolist()}, and no acceptable near-tie pair matches")
                chosen = match[0]
                alt += 1
            idx[b, h, qb, :len(chosen)] = chosen
            cnt[b, h, qb] = len(chosen)
        return idx, cnt, alt


def _gpu_tree(case):
    p = case.p
    ksum = ssa.block_summary(case.kd, case.w.block_k, p)
    qsum = ssa.block_summary(case.qd, case.w.block_q, p)
    ksum2 = ssa.tree_summary(ksum, p)
    sup, supc, idx, cnt = ssa.route_tree(qsum, ksum, ksum2, p)
    ssa.check_error()
    return ksum2, sup, supc, idx, cnt


@pytest.mark.parametrize("D,F", [(64, 4), (64, 16), (128, 8)])
def test_tree_summary_matches_fp64_means(D, F):
    case = Case(W("pool", B=2, Hq=2, Hkv=2, N=64 * 40, D=D, tree_fanout=F, tree_beam=1))
    ksum2 = _gpu_tree(case)[0].cpu().numpy().astype(np.float64)
    want = O.tree_summary(case.k64, 64, F)
    assert ksum2.shape == want.shape
    np.testing.assert_allclose(ksum2, want, rtol=0, atol=1e-5)


@pytest.mark.parametrize("w", [w for w in SMALL if not w.consensus], ids=lambda w: w.name)
def test_tree_route_matches_oracle(w):
    case = Case(w)
    _, sup, supc, idx, cnt = _gpu_tree(case)
    to = TreeOracle(case)
    to.check(idx.cpu().numpy(), cnt.cpu().numpy(), case.all_rows(), sup.cpu().numpy(),
             supc.cpu().numpy())


def test_every_super_block_kept_gives_the_flat_selection():
    case = Case(SMALL[8])
    _, _, _, idx, cnt = _gpu_tree(case)
    flat = Case(case.w.with_(tree_fanout=0, tree_beam=0), case.u16)
    ks = ssa.block_summary(flat.kd, 64, flat.p)
    qs = ssa.block_summary(flat.qd, 64, flat.p)
    i0, c0 = ssa.route(qs, ks, flat.p)
    # both are exact fp32 selections of the same scores up to summation
    # order: equal away from the oracle's counted near-ties
    r = O.route(flat.qsum64, flat.ksum64, flat.op)
    ties = O.near_tie_rows(r)
    same = (idx.cpu().numpy() == i0.cpu().numpy()).all(axis=-1)
    assert (same | ties).all()
    assert torch.equal(cnt.cpu(), c0.cpu())


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_tree_every_row(w):
    case = Case(w)
    op = case.op
    head = Case(w.with_(consensus=False), case.u16)
    _, sup, supc, h_idx, h_cnt = _gpu_tree(head)
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    rows = case.all_rows()
    r_idx, r_cnt, _ = TreeOracle(case).check(h_idx.cpu().numpy(), h_cnt.cpu().numpy(), rows,
                                             sup.cpu().numpy(), supc.cpu().numpy())
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


@pytest.mark.parametrize("cfg,F,beam,n", [(2, 16, 8, 40), (4, 16, 8, 32), (5, 16, 16, 24)])
def test_forward_tree_full_size_sampled(cfg, F, beam, n):
    case = Case(CONFIGS[cfg].with_(tree_fanout=F, tree_beam=beam))
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    rows = case.sample_rows(n, seed=cfg)
    r_idx, r_cnt, _ = TreeOracle(case).check(idx.cpu().numpy(), cnt.cpu().numpy(), rows)
    o_ref, l_ref = oracle_attend_rows(case, r_idx, r_cnt, rows)
    bq = case.op.block_q
    assert_close(gpu_rows(o, rows, bq), o_ref, gpu_rows(lse, rows, bq), l_ref, what=case.w.name)
    assert torch.isfinite(o).all()
