"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
check it against the float64 oracle.  No expected value comes from the CUDA
path: at a counted near-tie the oracle enumerates every acceptable selection
itself, and the GPU's selection must be one of them."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from content_routed_block_b200 import ssa
from content_routed_block_b200.workloads import Workload, make_inputs

MAX_ABS = 2e-2      # output tolerance vs the fp64 oracle for bf16 inputs
MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def to_dev(u16: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class Case:
    """Inputs of one workload on the host (fp64) and on the device (bf16)."""

    def __init__(self, w: Workload, inputs=None):
        self.w = w
        self.p = ssa.params_of(w)
        self.op = O.Params.of(w)
        x = inputs if inputs is not None else make_inputs(w)
        self.u16 = x
        self.q64, self.k64, self.v64 = (O.upcast_bf16(x[n]) for n in "qkv")
        self.qd, self.kd, self.vd = (to_dev(x[n]) for n in "qkv")
        self._qsum = None
        self._ksum = None

    @property
    def qsum64(self):
        if self._qsum is None:
            self._qsum = O.block_summary(self.q64, self.op.block_q)
        return self._qsum

    @property
    def ksum64(self):
        if self._ksum is None:
            self._ksum = O.block_summary(self.k64, self.op.block_k)
        return self._ksum

    def all_rows(self):
        return [(b, h, qb) for b in range(self.op.B) for h in range(self.op.Hq)
                for qb in range(self.op.n_qblocks)]

    def sample_rows(self, n: int, seed: int = 0):
        rng = np.random.default_rng(seed)
        op = self.op
        rows = {(0, 0, 0), (op.B - 1, op.Hq - 1, op.n_qblocks - 1), (0, op.Hq - 1, 1 % op.n_qblocks)}
        while len(rows) < min(n, op.B * op.Hq * op.n_qblocks):
            rows.add((int(rng.integers(op.B)), int(rng.integers(op.Hq)),
                      int(rng.integers(op.n_qblocks))))
        return sorted(rows)


def check_route_rows(case: Case, idx_g: np.ndarray, cnt_g: np.ndarray, rows):
    """Check the GPU's selections on ``rows``; return the oracle's idx/cnt
    arrays holding, for each row, the oracle selection equal to the GPU's (its
    own lexicographic one, or at a counted near-tie an enumerated alternative),
    and the number of near-tie rows where the GPU chose an alternative."""
    op = case.op
    idx = np.full((op.B, op.Hq, op.n_qblocks, op.top_k), -1, np.int32)
    cnt = np.zeros((op.B, op.Hq, op.n_qblocks), np.int32)
    alt = 0
    for b, h, qb in rows:
        cand = O.admissible_blocks(qb, op)
        mu = case.ksum64[b, h // op.group]
        qbar = case.qsum64[b, h, qb]
        own, _, _ = O.route_row(qbar, mu, cand, op.top_k)
        n = int(cnt_g[b, h, qb])
        g = idx_g[b, h, qb, :n]
        assert n == len(own), f"row {(b, h, qb)}: count {n} != {len(own)}"
        assert (idx_g[b, h, qb, n:] == -1).all(), f"row {(b, h, qb)}: bad padding"
        if np.array_equal(g, own):
            chosen = own
        else:
            accepted = O.acceptable_selections(qbar, mu, cand, op.top_k)
            match = [a for a in accepted if np.array_equal(a, g)]
            assert match, f"row {(b, h, qb)}: GPU selection {g.tolist()} != {own.tolist()} " \
                          f"and is not an acceptable near-tie alternative"
            chosen = match[0]
            alt += 1
        idx[b, h, qb, :len(chosen)] = chosen
        cnt[b, h, qb] = len(chosen)
    return idx, cnt, alt


def check_route_every_row(case: Case, idx_g: np.ndarray, cnt_g: np.ndarray):
    """Compare the GPU's lists with the oracle's on every row (flat
    mean-score route, ``O.route_flat_all``).  A row may differ only at a
    counted near-tie, and there the GPU's selection must be one the oracle
    enumerates (``O.acceptable_selections``).  Returns the oracle's idx/cnt
    with the GPU's accepted alternatives in place, the number of such rows,
    and the oracle's near-tie mask [B, Hq, NQB]."""
    op = case.op
    r = O.route_flat_all(case.qsum64, case.ksum64, op)
    near = O.near_tie_rows(r)
    assert (cnt_g == r.cnt).all(), "GPU counts differ from the oracle's"
    diff = (idx_g != r.idx).any(axis=-1) if op.top_k else np.zeros_like(near)
    idx = r.idx.copy()
    alt = 0
    for b, h, qb in zip(*np.nonzero(diff)):
        n = int(cnt_g[b, h, qb])
        g = idx_g[b, h, qb, :n]
        assert near[b, h, qb], (f"row {(b, h, qb)}: GPU selection {g.tolist()} != "
                                f"{r.idx[b, h, qb, :n].tolist()} outside a near-tie")
        accepted = O.acceptable_selections(case.qsum64[b, h, qb], case.ksum64[b, h // op.group],
                                           O.admissible_blocks(qb, op), op.top_k)
        assert any(np.array_equal(a, g) for a in accepted), \
            f"row {(b, h, qb)}: GPU selection {g.tolist()} is not an acceptable alternative"
        idx[b, h, qb, :n] = g
        alt += 1
    return idx, r.cnt, alt, near


def output_rows(case: Case, near: np.ndarray, seed: int = 0):
    """Query blocks whose outputs are compared at full size: one random block
    of every (b, head), the first and last blocks of every (b, head), and
    every near-tie row."""
    op = case.op
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(op.B):
        for h in range(op.Hq):
            rows.update({(b, h, 0), (b, h, op.n_qblocks - 1),
                         (b, h, int(rng.integers(op.n_qblocks)))})
    rows.update((int(b), int(h), int(q)) for b, h, q in zip(*np.nonzero(near)))
    return sorted(rows)


def oracle_attend_rows(case: Case, idx, cnt, rows):
    """fp64 oracle outputs for the query blocks ``rows`` -> ([n, Bq, D], [n, Bq])."""
    return O.attend_masked_dense(case.q64, case.k64, case.v64, idx, cnt, case.op, blocks=rows)


def gpu_rows(t: torch.Tensor, rows, bq: int) -> np.ndarray:
    """Gather query blocks ``rows`` of a [B, H, N, ...] GPU tensor to fp64."""
    out = []
    for b, h, qb in rows:
        out.append(t[b, h, qb * bq:(qb + 1) * bq].float().cpu().numpy().astype(np.float64))
    return np.stack(out)


def assert_close(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what=""):
    err = np.abs(o_gpu - o_ref)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    if lse_gpu is not None:
        le = np.abs(lse_gpu - lse_ref)
        assert le.max() <= LSE_ABS, f"{what}: lse max abs err {le.max():.3e}"
    return float(err.max()), float(err.mean())


def check_forward(case: Case, rows=None, with_route_all=True):
    """Run ssa_forward and check routing and outputs on ``rows`` (all rows
    when None).  Returns a small report dict."""
    p = case.p
    o, lse, idx, cnt = ssa.forward(case.qd, case.kd, case.vd, p)
    ssa.check_error()
    rows = case.all_rows() if rows is None else rows
    idx_g, cnt_g = idx.cpu().numpy(), cnt.cpu().numpy()
    r_idx, r_cnt, alt = check_route_rows(case, idx_g, cnt_g, rows)
    o_ref, l_ref = oracle_attend_rows(case, r_idx, r_cnt, rows)
    o_g = gpu_rows(o, rows, case.op.block_q)
    l_g = gpu_rows(lse, rows, case.op.block_q)
    mx, mean = assert_close(o_g, o_ref, l_g, l_ref, what=case.w.name)
    return {"max_abs": mx, "mean_abs": mean, "near_tie_alternatives": alt, "rows": len(rows),
            "o": o, "idx": idx_g, "cnt": cnt_g}
