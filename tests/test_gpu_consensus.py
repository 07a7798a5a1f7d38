"""Parity of the GQA-shared (consensus) route and of the attend kernel's
packed tiles (two query heads of a KV group per CTA) with the float64 oracle.

The per-head lists are first checked against the oracle exactly as in
test_gpu_parity (bit-exact, or at a counted near-tie an alternative that the
oracle itself enumerates); the expected consensus is then the oracle's
``route_consensus`` of those oracle-side selections, and the expected output
the oracle's attend over the expanded group lists.  No expected value comes
from the CUDA path.
"""
import os

import numpy as np
import pytest
import torch

import oracle as O
from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, make_inputs
from parity_utils import Case, assert_close, check_route_rows, gpu_rows, oracle_attend_rows

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


@pytest.fixture(params=["pack2", "pack1"])
def pack(request):
    """Run a test with two heads per attend tile (the default for consensus
    lists) and with one (SSA_PACK=1)."""
    old = os.environ.get("SSA_PACK")
    if request.param == "pack1":
        os.environ["SSA_PACK"] = "1"
    else:
        os.environ.pop("SSA_PACK", None)
    yield request.param
    if old is None:
        os.environ.pop("SSA_PACK", None)
    else:
        os.environ["SSA_PACK"] = old


def W(name, **kw):
    base = dict(B=1, Hq=4, Hkv=2, N=1024, D=64, block_k=64, block_q=64, top_k=4, window=128,
                causal=True, kind="iid", seed=17, consensus=True)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    W("gqa2"),
    W("gqa7-clustered", Hq=14, Hkv=2, N=2048, top_k=8, window=256, kind="clustered",
      centres=16),
    W("gqa8-d128", B=2, Hq=8, Hkv=1, D=128, N=768, top_k=3, window=96),
    W("gqa3-bk16-ragged", Hq=3, Hkv=1, N=1040, block_k=16, block_q=16, top_k=5, window=40),
    W("gqa2-bq128", Hq=4, Hkv=2, N=1024, block_k=16, block_q=128, top_k=8, window=130),
    W("gqa2-bk128-bq32", Hq=2, Hkv=1, N=1024, block_k=128, block_q=32, top_k=2, window=50),
    W("gqa5-bk32", Hq=5, Hkv=1, N=768, block_k=32, block_q=64, top_k=6, window=70),
    W("gqa2-noncausal", Hq=4, Hkv=2, N=1024, block_k=16, block_q=16, top_k=8, window=0,
      causal=False, kind="image"),
    W("gqa4-k0", Hq=4, Hkv=1, N=640, top_k=0, window=100),
    W("groups-of-one", Hq=3, Hkv=3, N=640, top_k=3, window=64),
    W("gqa2-tiny", Hq=2, Hkv=1, N=64, block_k=16, block_q=16, top_k=2, window=20),
]


def _group_rows(case, groups):
    """Per-head rows (b, h, qb) of the given (b, kv, qb) groups."""
    g = case.op.group
    return [(b, h, qb) for b, kv, qb in groups for h in range(kv * g, (kv + 1) * g)]


def _all_groups(case):
    op = case.op
    return [(b, kv, qb) for b in range(op.B) for kv in range(op.Hkv)
            for qb in range(op.n_qblocks)]


def _sample_groups(case, n, seed):
    op = case.op
    rng = np.random.default_rng(seed)
    s = {(0, 0, 0), (op.B - 1, op.Hkv - 1, op.n_qblocks - 1)}
    while len(s) < min(n, op.B * op.Hkv * op.n_qblocks):
        s.add((int(rng.integers(op.B)), int(rng.integers(op.Hkv)),
               int(rng.integers(op.n_qblocks))))
    return sorted(s)


def _per_head_route(case):
    p = case.p
    ks = ssa.block_summary(case.kd, case.w.block_k, p)
    qs = ssa.block_summary(case.qd, case.w.block_q, p)
    idx, cnt = ssa.route(qs, ks, p)
    ssa.check_error()
    return idx, cnt


def _check_consensus(case, groups, idx_kv, cnt_kv, h_idx, h_cnt):
    """Compare GPU consensus lists on ``groups`` with the oracle's consensus
    of the oracle-side per-head selections; return the oracle's group lists."""
    r_idx, r_cnt, alt = check_route_rows(case, h_idx, h_cnt, _group_rows(case, groups))
    want_idx, want_cnt = O.route_consensus(r_idx, r_cnt, case.op, rows=groups)
    for b, kv, qb in groups:
        assert cnt_kv[b, kv, qb] == want_cnt[b, kv, qb], (b, kv, qb)
        np.testing.assert_array_equal(idx_kv[b, kv, qb], want_idx[b, kv, qb],
                                      err_msg=str((b, kv, qb)))
    return want_idx, want_cnt, alt


def _check_outputs(case, groups, o, lse, want_idx, want_cnt):
    rows = _group_rows(case, groups)
    e_idx, e_cnt = O.expand_consensus(want_idx, want_cnt, case.op)
    o_ref, l_ref = oracle_attend_rows(case, e_idx, e_cnt, rows)
    bq = case.op.block_q
    return assert_close(gpu_rows(o, rows, bq), o_ref, gpu_rows(lse, rows, bq), l_ref,
                        what=case.w.name)


# ------------------------------------------------------------------ the vote kernel
def _read_votes():
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


def test_consensus_kernel_on_hand_worked_votes():
    # the golden per-head lists are the kernel's input; the hand-derived
    # consensus is the expected output
    for k, sels, want in _read_votes():
        g = len(sels)
        p = ssa.make_params(1, g, 1, 64 * 64, 64, 64, 64, k, 64, True, consensus=True)
        idx = np.full((1, g, 64, k), -1, np.int32)
        cnt = np.zeros((1, g, 64), np.int32)
        for h, s in enumerate(sels):
            idx[0, h, 63, :len(s)] = s
            cnt[0, h, 63] = len(s)
        i_kv, c_kv = ssa.route_consensus(torch.from_numpy(idx).cuda(),
                                         torch.from_numpy(cnt).cuda(), p)
        ssa.check_error()
        i_kv, c_kv = i_kv.cpu().numpy(), c_kv.cpu().numpy()
        assert c_kv[0, 0, 63] == len(want)
        assert i_kv[0, 0, 63, :len(want)].tolist() == want
        assert (i_kv[0, 0, 63, len(want):] == -1).all()
        assert (c_kv[0, 0, :63] == 0).all()


def test_consensus_kernel_random_lists_and_bad_entries():
    rng = np.random.default_rng(8)
    g, k, nb, nqb = 7, 16, 512, 96
    p = ssa.make_params(2, g * 2, 2, nqb * 64, 64, 64, 64, k, 64, True, consensus=True)
    op = O.Params(2, g * 2, 2, nqb * 64, 64, 64, 64, k, 64, True, consensus=True)
    idx = np.full((2, 2 * g, nqb, k), -1, np.int32)
    cnt = np.zeros((2, 2 * g, nqb), np.int32)
    for b in range(2):
        for h in range(2 * g):
            for qb in range(nqb):
                n = int(rng.integers(0, k + 1))
                # a small pool makes shared votes and vote ties common
                pool = int(rng.integers(n, 3 * k + 1)) if n else 1
                s = np.sort(rng.choice(pool, size=n, replace=False))
                idx[b, h, qb, :n] = s
                cnt[b, h, qb] = n
    i_kv, c_kv = ssa.route_consensus(torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(), p)
    ssa.check_error()
    want_i, want_c = O.route_consensus(idx, cnt, op)
    np.testing.assert_array_equal(c_kv.cpu().numpy(), want_c)
    np.testing.assert_array_equal(i_kv.cpu().numpy(), want_i)
    # an out-of-range block and a bad count are reported (and skipped)
    bad_i, bad_c = idx.copy(), cnt.copy()
    bad_i[0, 0, 5, 0] = nb + 3
    bad_c[1, 3, 7] = k + 2
    ssa.route_consensus(torch.from_numpy(bad_i).cuda(), torch.from_numpy(bad_c).cuda(), p)
    with pytest.raises(ssa.SsaError) as e:
        ssa.check_error()
    assert e.value.status == 6
    ssa.check_error()


# ------------------------------------------------------------------ attend, packed tiles
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attend_consensus_with_oracle_lists(w, pack):
    case = Case(w)
    r = O.route(case.qsum64, case.ksum64, case.op)
    idx_kv, cnt_kv = O.route_consensus(r.idx, r.cnt, case.op)
    o, lse = ssa.attend(case.qd, case.kd, case.vd, torch.from_numpy(idx_kv).cuda(),
                        torch.from_numpy(cnt_kv).cuda(), case.p)
    ssa.check_error()
    _check_outputs(case, _all_groups(case), o, lse, idx_kv, cnt_kv)


# ------------------------------------------------------------------ whole path
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_forward_consensus_every_row(w, pack):
    case = Case(w)
    h_idx, h_cnt = _per_head_route(case)
    o, lse, idx_kv, cnt_kv = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    groups = _all_groups(case)
    want_idx, want_cnt, _ = _check_consensus(case, groups, idx_kv.cpu().numpy(),
                                             cnt_kv.cpu().numpy(), h_idx.cpu().numpy(),
                                             h_cnt.cpu().numpy())
    _check_outputs(case, groups, o, lse, want_idx, want_cnt)


@pytest.mark.parametrize("cfg,n", [(2, 24), (5, 6)])
def test_forward_consensus_full_size_sampled(cfg, n):
    case = Case(CONFIGS[cfg].with_(consensus=True))
    h_idx, h_cnt = _per_head_route(case)
    o, lse, idx_kv, cnt_kv = ssa.forward(case.qd, case.kd, case.vd, case.p)
    ssa.check_error()
    groups = _sample_groups(case, n, seed=cfg)
    want_idx, want_cnt, _ = _check_consensus(case, groups, idx_kv.cpu().numpy(),
                                             cnt_kv.cpu().numpy(), h_idx.cpu().numpy(),
                                             h_cnt.cpu().numpy())
    _check_outputs(case, groups, o, lse, want_idx, want_cnt)
    # properties of every group's list
    c = cnt_kv.cpu().numpy()
    qb = np.arange(case.op.n_qblocks)
    n_adm = np.minimum((qb * case.op.block_q) // case.op.block_k, case.op.n_kblocks)
    assert (c <= np.minimum(case.op.top_k, n_adm)[None, None, :]).all()
    assert (c[..., 1:] > 0).all()
    assert torch.isfinite(o).all()


def test_forward_consensus_is_deterministic_and_host_path_agrees():
    case = Case(SMALL[1])
    a = ssa.forward(case.qd, case.kd, case.vd, case.p)
    b = ssa.forward(case.qd, case.kd, case.vd, case.p)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    qh, kh, vh = (t.cpu().pin_memory() for t in (case.qd, case.kd, case.vd))
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    ssa.forward_host(qh, kh, vh, case.p, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, a[0].cpu())
