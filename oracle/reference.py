"""Plain float64 CPU oracle for content-routed block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path (no kernels, headers, helpers, tables or pre-/post-processing);
the two meet only in the seeded input generator, which holds none of the
method's arithmetic.

What it computes, step by step, in the order the method states it
(jonsmirl/ssa README: the introduction, "Algorithm and complexity" and
"Mathematical status"; SingleZombie/LLSA README, "Minimum Usage" for the
non-causal variant):

1. Upcast bf16 Q, K, V to float64 (exact).
2. Query head h reads KV head h // (Hq / Hkv) (consecutive grouped-query
   attention, the "native grouped-query attention" of the SSA 10M run).
3. Block summaries: mu_c = mean of the Bk keys of key block c; the query
   block qb is summarised by qbar = mean of its Bq queries.  (SSA's routing
   score r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q is taken with beta = 0:
   mean pooling only.  Because the score is linear in q, scoring the mean
   query equals averaging the per-query scores over the block.)
4. Admissible key blocks of query block qb: causal -- the completed blocks
   that end at or before the block's first query, (c+1)*Bk <= qb*Bq, so no
   summary averages a future key; non-causal -- every key block.
5. Score s_c = <qbar, mu_c> (unscaled: a positive scale does not change the
   ranking).  With the second-cumulant weight beta != 0 (SSA's full score
   r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q), a query block scores by the
   mean of its queries' scores: s_c = <qbar, mu_c> + (beta/2) tr(Sigma_c Q2),
   Sigma_c the population covariance of block c's keys and Q2 the mean of
   q_i q_i^T over the block's queries (``block_scores``).
6. Selection: the first min(top_k, |A|) admissible blocks in the order
   (score descending, block index ascending) -- ties go to the lower index --
   stored ascending by block index, padded with -1, with their count.
6b. (Optional, ``Params.consensus``) GQA-shared consensus route: every query
   head of a KV group votes for the blocks of its own selection, and the
   group keeps the top_k blocks by (votes descending, block index ascending)
   -- one list per (b, KV head, query block) that all of the group's heads
   use ("Complete 10M transformer result": a cross-head consensus route
   carrying the highest-vote blocks).
6c. (Optional, ``Params.tree_fanout``) two-level fixed-beam routing: the
   blocks are grouped F at a time into super-blocks summarised by their key
   means; a query block keeps its best tree_beam complete admissible
   super-blocks (step 6's order) and selects its top_k blocks (step 6) among
   their children and the frontier blocks (``route_tree_row``).
7. Key set of query i as a SET: the keys of its query block's selected blocks
   united with the local causal window {j : i - W < j <= i} and cut at i
   (causal); only the selected blocks' keys (non-causal).  A key that is both
   routed and in the window counts once.
8. Exact softmax over that set: l_j = scale * <q_i, k_j>, scale = 1/sqrt(D)
   by default; o_i = sum_j softmax(l)_j v_j; lse_i = max l + log sum exp(l - max l)
   (natural log).  The dense N x N matrix is never needed: the masked-dense
   form builds one query block's rows at a time.

Two attend forms are provided and must agree: ``attend_masked_dense`` (a
[Bq, N] logit slab with -inf outside each row's set) and ``attend_gathered``
(each query's explicit key-index set).
"""
from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np

__all__ = [
    "Params", "upcast_bf16", "block_summary", "admissible_blocks", "route",
    "RouteResult", "key_set", "attend_masked_dense", "attend_gathered", "forward",
    "near_tie_rows", "acceptable_selections", "route_row",
    "consensus_row", "route_consensus", "expand_consensus",
    "block_covariance", "block_second_moment", "block_scores", "decode_step",
    "decode_attend", "tree_summary", "tree_candidates", "route_tree_row",
    "acceptable_tree_selections", "attend_backward", "route_flat_all",
    "attend_gathered_blocks",
]

NEAR_TIE_REL = 1e-4   # relative score gap under which two blocks count as tied


@dataclass(frozen=True)
class Params:
    """Method parameters (names follow the pages' notation)."""
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
    scale: float = 0.0          # 0 -> 1/sqrt(D)
    consensus: bool = False     # GQA-shared (consensus) routing, see route_consensus
    beta: float = 0.0           # weight of the second-cumulant score term, see block_scores
    tree_fanout: int = 0        # two-level routing: key blocks per super-block (0: flat)
    tree_beam: int = 0          # super-blocks kept at the upper level, see route_tree_row

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_kblocks(self) -> int:
        return self.N // self.block_k

    @property
    def n_qblocks(self) -> int:
        return self.N // self.block_q

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale > 0 else 1.0 / math.sqrt(self.D)

    @staticmethod
    def of(w) -> "Params":
        """Build from any object with the same field names (e.g. a workload)."""
        return Params(w.B, w.Hq, w.Hkv, w.N, w.D, w.block_k, w.block_q, w.top_k,
                      w.window, bool(w.causal), getattr(w, "scale", 0.0),
                      bool(getattr(w, "consensus", False)), float(getattr(w, "beta", 0.0)),
                      int(getattr(w, "tree_fanout", 0)), int(getattr(w, "tree_beam", 0)))


def upcast_bf16(u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64.  A bf16 value is a float32 whose low 16
    bits are zero, so the upcast is exact."""
    u32 = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# step 3: block summaries
# --------------------------------------------------------------------------
def block_summary(x: np.ndarray, block: int) -> np.ndarray:
    """Mean of every ``block`` consecutive rows of ``x[..., N, D]``.

    jonsmirl/ssa README, "Algorithm and complexity": mu_c is block c's mean
    key (the first cumulant of the second-cumulant routing score)."""
    n, d = x.shape[-2], x.shape[-1]
    if n % block:
        raise ValueError("sequence length must be a multiple of the block size")
    return x.reshape(*x.shape[:-2], n // block, block, d).mean(axis=-2)


# --------------------------------------------------------------------------
# step 4: admissible blocks
# --------------------------------------------------------------------------
def admissible_blocks(qb: int, p: Params) -> np.ndarray:
    """Key blocks query block ``qb`` may route to.

    Causal: only completed blocks that end at or before the query block's
    first token, (c + 1) * Bk <= qb * Bq -- a routed set is causal only once
    it is cut at each query's position (jonsmirl/ssa README, "Mathematical
    status" and "Known limitations"); taking whole past blocks keeps every
    summary free of future keys, and the current partial block is reached
    through the local window.  Non-causal: all key blocks (LLSA)."""
    if not p.causal:
        return np.arange(p.n_kblocks)
    last = (qb * p.block_q) // p.block_k          # blocks 0 .. last-1 are complete
    return np.arange(min(last, p.n_kblocks))


# --------------------------------------------------------------------------
# second-cumulant summaries (the beta term of the routing score)
# --------------------------------------------------------------------------
def block_covariance(x: np.ndarray, block: int) -> np.ndarray:
    """Second cumulant of every block of ``block`` rows of ``x[..., N, D]``:
    Sigma_c = (1/block) sum_t (x_t - mu_c)(x_t - mu_c)^T, the population
    covariance of the block's keys.  Returns [..., N/block, D, D].

    jonsmirl/ssa README, "Algorithm and complexity": the second-cumulant
    routing score r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q."""
    n, d = x.shape[-2], x.shape[-1]
    if n % block:
        raise ValueError("sequence length must be a multiple of the block size")
    xb = x.reshape(*x.shape[:-2], n // block, block, d)
    c = xb - xb.mean(axis=-2, keepdims=True)
    return np.einsum("...td,...te->...de", c, c) / block


def block_second_moment(x: np.ndarray, block: int) -> np.ndarray:
    """(1/block) sum_t x_t x_t^T for every block of ``block`` rows:
    [..., N/block, D, D].  Averaging q^T Sigma q over a query block's queries
    gives tr(Sigma Q2) with Q2 this moment."""
    n, d = x.shape[-2], x.shape[-1]
    if n % block:
        raise ValueError("sequence length must be a multiple of the block size")
    xb = x.reshape(*x.shape[:-2], n // block, block, d)
    return np.einsum("...td,...te->...de", xb, xb) / block


def block_scores(qbar, mu, cand, beta: float = 0.0, q2=None, sigma=None) -> np.ndarray:
    """Routing scores of the candidate blocks ``cand`` for one query block:
    s_c = <qbar, mu_c> + (beta/2) tr(Sigma_c Q2), the mean over the block's
    queries of SSA's r_c(q_i) = <q_i, mu_c> + (beta/2) q_i^T Sigma_c q_i
    (both terms are linear in q q^T).  With beta = 0 only the means enter."""
    s = mu[cand] @ qbar
    if beta != 0.0:
        s = s + 0.5 * beta * np.einsum("cde,de->c", sigma[cand], q2)
    return s


# --------------------------------------------------------------------------
# steps 5-6: scores and top-k
# --------------------------------------------------------------------------
@dataclass
class RouteResult:
    idx: np.ndarray        # int32 [B, Hq, NQB, top_k], ascending, -1 padded
    cnt: np.ndarray        # int32 [B, Hq, NQB]
    kth: np.ndarray        # float64 [B, Hq, NQB]: k-th best score (nan if none)
    next: np.ndarray       # float64 [B, Hq, NQB]: (k+1)-th best score (nan if none)
    sup_idx: np.ndarray = None   # tree form: int32 [B, Hq, NQB, tree_beam] kept super-blocks
    sup_cnt: np.ndarray = None   # tree form: int32 [B, Hq, NQB]


def route_row(qbar: np.ndarray, mu: np.ndarray, cand: np.ndarray, top_k: int,
              beta: float = 0.0, q2=None, sigma=None):
    """Select from candidate blocks ``cand`` for one query-block summary
    (scores from ``block_scores``; ``q2``/``sigma`` only when beta != 0).

    Returns (selected ascending, k-th score, (k+1)-th score)."""
    if len(cand) == 0 or top_k == 0:
        return np.zeros(0, dtype=np.int64), math.nan, math.nan
    s = block_scores(qbar, mu, cand, beta, q2, sigma)
    if not np.isfinite(s).all():
        raise ValueError("non-finite routing scores: the route is defined for finite inputs")
    # order: score descending, then block index ascending (lower index wins a tie)
    order = np.lexsort((cand, -s))
    take = min(top_k, len(cand))
    chosen = np.sort(cand[order[:take]])
    kth = s[order[take - 1]]
    nxt = s[order[take]] if take < len(cand) else math.nan
    return chosen, kth, nxt


def route(qsum: np.ndarray, ksum: np.ndarray, p: Params, rows=None, qm2=None,
          kcov=None, ksum2=None) -> RouteResult:
    """Top-k routing for every (b, query head, query block).

    ``qsum`` [B, Hq, NQB, D] and ``ksum`` [B, Hkv, NB, D] are block summaries
    (float64); with ``p.beta`` != 0 also ``qm2`` [B, Hq, NQB, D, D]
    (``block_second_moment`` of Q) and ``kcov`` [B, Hkv, NB, D, D]
    (``block_covariance`` of K); with ``p.tree_fanout`` > 0 (two-level form,
    ``route_tree_row``) also ``ksum2`` [B, Hkv, NS, D] (``tree_summary``).
    ``rows`` optionally restricts the work to a list of (b, h, qb) triples;
    the arrays keep their full shape and rows not listed stay at idx = -1,
    cnt = 0, scores nan."""
    nqb = p.n_qblocks
    idx = np.full((p.B, p.Hq, nqb, p.top_k), -1, dtype=np.int32)
    cnt = np.zeros((p.B, p.Hq, nqb), dtype=np.int32)
    kth = np.full((p.B, p.Hq, nqb), math.nan)
    nxt = np.full((p.B, p.Hq, nqb), math.nan)
    tree = p.tree_fanout > 0
    if tree:
        if p.beta != 0.0:
            raise ValueError("the two-level form scores by block means only (beta = 0)")
        if ksum2 is None:
            raise ValueError("the two-level form needs the super-block summaries ksum2")
        sup_idx = np.full((p.B, p.Hq, nqb, p.tree_beam), -1, dtype=np.int32)
        sup_cnt = np.zeros((p.B, p.Hq, nqb), dtype=np.int32)
    todo = rows if rows is not None else [
        (b, h, qb) for b in range(p.B) for h in range(p.Hq) for qb in range(nqb)]
    for b, h, qb in todo:
        mu = ksum[b, h // p.group]
        if tree:
            sup, sel, a, c = route_tree_row(qsum[b, h, qb], mu, ksum2[b, h // p.group],
                                            len(admissible_blocks(qb, p)), p)
            sup_idx[b, h, qb, :len(sup)] = sup
            sup_cnt[b, h, qb] = len(sup)
        else:
            extra = {}
            if p.beta != 0.0:
                extra = dict(beta=p.beta, q2=qm2[b, h, qb], sigma=kcov[b, h // p.group])
            sel, a, c = route_row(qsum[b, h, qb], mu, admissible_blocks(qb, p), p.top_k, **extra)
        idx[b, h, qb, :len(sel)] = sel
        cnt[b, h, qb] = len(sel)
        kth[b, h, qb], nxt[b, h, qb] = a, c
    if tree:
        return RouteResult(idx, cnt, kth, nxt, sup_idx, sup_cnt)
    return RouteResult(idx, cnt, kth, nxt)


def route_flat_all(qsum: np.ndarray, ksum: np.ndarray, p: Params, heads=None,
                   chunk: int = 1024) -> RouteResult:
    """Steps 5-6 for every query block at once: the flat mean-score route
    (beta = 0, no two-level form) of ``route``, written with whole-array
    operations so that it finishes at a million tokens.

    Same steps, same order: the scores of a (b, head) are one float64 product
    qsum @ ksum^T (``chunk`` query blocks at a time), the columns a query
    block may not route to (step 4) are excluded, and each row keeps the
    first min(top_k, |A|) admissible blocks in the order (score descending,
    block index ascending).  Selecting that prefix needs no sort: with s_k the
    row's k-th largest score, it is every block scoring above s_k plus the
    lowest-indexed blocks scoring exactly s_k until k are taken.  ``heads``
    optionally restricts the work to a list of (b, h) pairs (the other rows
    stay at idx = -1, cnt = 0, scores nan).  Returns the same RouteResult as
    ``route``."""
    if p.beta != 0.0 or p.tree_fanout > 0:
        raise ValueError("route_flat_all is the flat mean-score route (beta = 0, no tree)")
    nqb, nb, k = p.n_qblocks, p.n_kblocks, p.top_k
    idx = np.full((p.B, p.Hq, nqb, k), -1, dtype=np.int32)
    cnt = np.zeros((p.B, p.Hq, nqb), dtype=np.int32)
    kth = np.full((p.B, p.Hq, nqb), math.nan)
    nxt = np.full((p.B, p.Hq, nqb), math.nan)
    if k == 0:
        return RouteResult(idx, cnt, kth, nxt)
    if not (np.isfinite(qsum).all() and np.isfinite(ksum).all()):
        raise ValueError("non-finite summaries: the route is defined for finite inputs only")
    qb_all = np.arange(nqb)
    if p.causal:
        n_adm_all = np.minimum((qb_all * p.block_q) // p.block_k, nb)    # step 4
    else:
        n_adm_all = np.full(nqb, nb)
    todo = heads if heads is not None else [(b, h) for b in range(p.B) for h in range(p.Hq)]
    for b, h in todo:
        mu = ksum[b, h // p.group]
        for r0 in range(0, nqb, chunk):
            rows = qb_all[r0:r0 + chunk]
            n_adm = n_adm_all[rows]
            ncol = int(n_adm.max())
            if ncol == 0:
                continue
            s = qsum[b, h, rows] @ mu[:ncol].T                            # step 5
            col = np.arange(ncol)
            valid = col[None, :] < n_adm[:, None]
            sm = np.where(valid, s, -np.inf)
            take = np.minimum(k, n_adm)
            # k-th and (k+1)-th largest admissible score of each row
            # (descending order = ascending order of the negated scores)
            neg = -sm
            kk = min(k, ncol)
            kths = [kk - 1] + ([kk] if kk < ncol else [])
            part = np.partition(neg, kths, axis=1)
            s_k = -part[:, kk - 1]
            s_k1 = -part[:, kk] if kk < ncol else np.full(len(rows), -np.inf)
            # rows with fewer admissible blocks than k take all of them: their
            # last taken score is the row's smallest admissible score
            short = n_adm <= k
            if short.any():
                smallest = np.where(valid, s, np.inf).min(axis=1)
                s_k = np.where(short, smallest, s_k)
                s_k1 = np.where(short, -np.inf, s_k1)
            above = valid & (sm > s_k[:, None])
            tied = valid & (sm == s_k[:, None])
            need = take - above.sum(axis=1)
            chosen = above | (tied & (np.cumsum(tied, axis=1) <= need[:, None]))   # step 6
            # write each row's chosen blocks ascending (np.nonzero walks rows in
            # order and each row's columns ascending)
            rr, cc = np.nonzero(chosen)
            counts = chosen.sum(axis=1)
            pos = np.arange(len(rr)) - (np.cumsum(counts) - counts)[rr]
            idx[b, h, rows[rr], pos] = cc
            cnt[b, h, rows] = counts
            has = take > 0
            kth[b, h, rows[has]] = s_k[has]
            full = has & ~short
            nxt[b, h, rows[full]] = s_k1[full]
    return RouteResult(idx, cnt, kth, nxt)


def near_tie_rows(r: RouteResult, rel: float = NEAR_TIE_REL) -> np.ndarray:
    """Rows whose k-th and (k+1)-th scores differ by less than ``rel`` of the
    larger magnitude: at such a row either choice is an acceptable top-k."""
    a, c = r.kth, r.next
    with np.errstate(invalid="ignore"):
        gap = np.abs(a - c)
        tol = rel * np.maximum(np.abs(a), np.abs(c))
        return np.isfinite(gap) & (gap <= tol)


def acceptable_selections(qbar: np.ndarray, mu: np.ndarray, cand: np.ndarray, top_k: int,
                          rel: float = NEAR_TIE_REL, limit: int = 256, beta: float = 0.0,
                          q2=None, sigma=None) -> list:
    """Every selection that the near-tie rule accepts, ascending.

    Scores are fp64.  Let s_k be the k-th best score.  Blocks whose score is
    within ``rel`` (relative) of s_k form the tie band; blocks above the band
    are always selected and the remaining slots may be filled by any blocks of
    the band.  With no near-tie the list holds exactly the ``route_row``
    selection.  At most ``limit`` selections are listed."""
    import itertools
    if len(cand) == 0 or top_k == 0:
        return [np.zeros(0, dtype=np.int64)]
    s = block_scores(qbar, mu, cand, beta, q2, sigma)
    order = np.lexsort((cand, -s))
    take = min(top_k, len(cand))
    sk = s[order[take - 1]]
    band = np.abs(s - sk) <= rel * np.maximum(np.abs(s), abs(sk))
    sure = cand[(s > sk) & ~band]
    pool = cand[band]
    need = take - len(sure)
    out = []
    for combo in itertools.combinations(pool.tolist(), need):
        out.append(np.sort(np.concatenate([sure, np.array(combo, dtype=sure.dtype)])))
        if len(out) >= limit:
            break
    return out


# --------------------------------------------------------------------------
# steps 5-6, two-level form (optional): fixed-beam tree routing
# --------------------------------------------------------------------------
# jonsmirl/ssa README, "Algorithm and complexity": a hierarchical router with
# a fixed block size and a fixed budget approaches linear routing work on
# benign geometry, where a flat router scans every block; the measured 10M
# tree uses fanout 16.  "Mathematical status": fixed-beam routing is not an
# exact selector (its retrieval quality is an empirical matter).  Here the
# tree has two levels: super-block S covers the F key blocks S*F .. S*F+F-1
# and is summarised by the mean of its F*Bk keys; a query block scores the
# super-blocks like blocks (step 5), keeps the best tree_beam of them
# (step 6's order), and then selects its top_k blocks (step 6) among the
# children of the kept super-blocks plus the frontier -- the admissible
# blocks of the one super-block that is not yet completely admissible.  With
# every super-block kept this is the flat selection.
def tree_summary(k: np.ndarray, block_k: int, fanout: int) -> np.ndarray:
    """Super-block summaries of ``k[..., N, D]``: the mean of the F*Bk keys
    of every complete super-block (N // (F*Bk) of them), [..., NS, D]."""
    span = fanout * block_k
    ns = k.shape[-2] // span
    return block_summary(k[..., :ns * span, :], span)


def tree_candidates(sup, n_adm: int, fanout: int) -> np.ndarray:
    """Blocks scored at the lower level: the ``fanout`` children of every
    kept super-block ``sup``, then the frontier blocks (admissible blocks
    0 .. n_adm-1 past the last complete admissible super-block)."""
    ns = n_adm // fanout
    kids = (np.asarray(sup, dtype=np.int64)[:, None] * fanout
            + np.arange(fanout, dtype=np.int64)[None, :]).ravel()
    return np.concatenate([kids, np.arange(ns * fanout, n_adm, dtype=np.int64)])


def route_tree_row(qbar: np.ndarray, mu: np.ndarray, mu2: np.ndarray, n_adm: int, p: Params):
    """Two-level selection for one query-block summary.  The admissible key
    blocks are 0 .. n_adm-1 (step 4); the complete admissible super-blocks
    are 0 .. n_adm // F - 1.  Returns (kept super-blocks ascending, selected
    blocks ascending, k-th score, (k+1)-th score) -- the scores of the lower
    level, among its candidates."""
    F = p.tree_fanout
    sup, _, _ = route_row(qbar, mu2, np.arange(n_adm // F, dtype=np.int64), p.tree_beam)
    sel, kth, nxt = route_row(qbar, mu, tree_candidates(sup, n_adm, F), p.top_k)
    return sup, sel, kth, nxt


def acceptable_tree_selections(qbar: np.ndarray, mu: np.ndarray, mu2: np.ndarray, n_adm: int,
                               p: Params, rel: float = NEAR_TIE_REL, limit: int = 256) -> list:
    """Every (kept super-blocks, selected blocks) pair that the near-tie rule
    accepts at both levels: any super-block set ``acceptable_selections``
    accepts at the upper level, each followed by any selection it accepts
    among that set's candidates.  At most ``limit`` pairs."""
    F = p.tree_fanout
    out = []
    for sup in acceptable_selections(qbar, mu2, np.arange(n_adm // F, dtype=np.int64),
                                     p.tree_beam, rel, limit):
        for sel in acceptable_selections(qbar, mu, tree_candidates(sup, n_adm, F), p.top_k,
                                         rel, limit):
            out.append((sup, sel))
            if len(out) >= limit:
                return out
    return out


# --------------------------------------------------------------------------
# step 6b (optional): GQA-shared consensus route
# --------------------------------------------------------------------------
def consensus_row(head_selections, top_k: int) -> np.ndarray:
    """One selection shared by the query heads of a KV group.

    jonsmirl/ssa README, "Complete 10M transformer result": the first layer
    forms one route across heads by consensus and carries the blocks with
    the most votes forward; "Mathematical status": a highest-count reservoir
    keeps the items that the per-head selectors voted for most often.  Here
    every query head of the group votes once for each block of its own top-k
    selection (step 6).  The shared selection is the first
    min(top_k, #blocks with a vote) blocks in the order (votes descending,
    block index ascending) -- the method's lower-index tie rule -- stored
    ascending by block index."""
    votes = {}
    for sel in head_selections:
        for c in np.asarray(sel, dtype=np.int64).tolist():
            votes[c] = votes.get(c, 0) + 1
    ranked = sorted(votes, key=lambda c: (-votes[c], c))
    return np.array(sorted(ranked[:top_k]), dtype=np.int64)


def route_consensus(idx: np.ndarray, cnt: np.ndarray, p: Params, rows=None):
    """Consensus lists for every (b, KV head, query block) from the per-head
    lists ``idx`` [B, Hq, NQB, top_k] / ``cnt`` [B, Hq, NQB] of step 6.

    Returns (idx_kv int32 [B, Hkv, NQB, top_k] ascending and -1 padded,
    cnt_kv int32 [B, Hkv, NQB]).  ``rows`` optionally lists (b, kv, qb)
    triples; other rows stay empty.  The group of KV head kv is query heads
    kv*g .. kv*g + g - 1 (step 2)."""
    g = p.group
    idx_kv = np.full((p.B, p.Hkv, p.n_qblocks, p.top_k), -1, dtype=np.int32)
    cnt_kv = np.zeros((p.B, p.Hkv, p.n_qblocks), dtype=np.int32)
    todo = rows if rows is not None else [
        (b, kv, qb) for b in range(p.B) for kv in range(p.Hkv) for qb in range(p.n_qblocks)]
    for b, kv, qb in todo:
        heads = [idx[b, h, qb, :cnt[b, h, qb]] for h in range(kv * g, (kv + 1) * g)]
        sel = consensus_row(heads, p.top_k)
        idx_kv[b, kv, qb, :len(sel)] = sel
        cnt_kv[b, kv, qb] = len(sel)
    return idx_kv, cnt_kv


def expand_consensus(idx_kv: np.ndarray, cnt_kv: np.ndarray, p: Params):
    """Per-query-head view of consensus lists: query head h uses the list of
    its KV head h // g.  The result feeds the attend forms unchanged."""
    heads = np.arange(p.Hq) // p.group
    return idx_kv[:, heads].copy(), cnt_kv[:, heads].copy()


# --------------------------------------------------------------------------
# step 7: key sets
# --------------------------------------------------------------------------
def key_set(i: int, sel_blocks: np.ndarray, p: Params) -> np.ndarray:
    """Sorted key positions query ``i`` attends to (a set: no duplicates)."""
    routed = (np.asarray(sel_blocks, dtype=np.int64)[:, None] * p.block_k
              + np.arange(p.block_k)[None, :]).ravel()
    if not p.causal:
        return np.unique(routed)
    window = np.arange(max(0, i - p.window + 1), i + 1)
    s = np.union1d(routed, window)
    return s[s <= i]


# --------------------------------------------------------------------------
# step 8: exact softmax over each query's set
# --------------------------------------------------------------------------
def _softmax_read(logits: np.ndarray, vals: np.ndarray):
    m = logits.max(axis=-1, keepdims=True)
    w = np.exp(logits - m)
    z = w.sum(axis=-1, keepdims=True)
    return (w @ vals) / z, (m + np.log(z))[..., 0]


def attend_masked_dense(q, k, v, idx, cnt, p: Params, blocks=None):
    """Masked-dense form: for each query block, a [Bq, N] logit slab with -inf
    outside each row's key set.

    ``q`` [B, Hq, N, D], ``k``/``v`` [B, Hkv, N, *] float64.  ``blocks``
    optionally restricts the work to a list of (b, h, qb) triples; the
    returned arrays are then [len(blocks), Bq, Dv] and [len(blocks), Bq].
    Otherwise returns O [B, Hq, N, Dv] and LSE [B, Hq, N]."""
    scale = p.softmax_scale
    dv = v.shape[-1]
    todo = blocks if blocks is not None else [
        (b, h, qb) for b in range(p.B) for h in range(p.Hq) for qb in range(p.n_qblocks)]
    o_out = np.zeros((len(todo), p.block_q, dv))
    l_out = np.zeros((len(todo), p.block_q))
    jpos = np.arange(p.N)
    jblk = jpos // p.block_k
    for t, (b, h, qb) in enumerate(todo):
        g = h // p.group
        rows = np.arange(qb * p.block_q, (qb + 1) * p.block_q)
        routed = np.zeros(p.n_kblocks, dtype=bool)
        routed[idx[b, h, qb, :cnt[b, h, qb]]] = True
        allow = np.broadcast_to(routed[jblk][None, :], (len(rows), p.N)).copy()
        if p.causal:
            allow |= jpos[None, :] > rows[:, None] - p.window
            allow &= jpos[None, :] <= rows[:, None]
        logits = (q[b, h, rows] @ k[b, g].T) * scale
        logits = np.where(allow, logits, -np.inf)
        o_out[t], l_out[t] = _softmax_read(logits, v[b, g])
    if blocks is not None:
        return o_out, l_out
    o = o_out.reshape(p.B, p.Hq, p.N, dv)
    lse = l_out.reshape(p.B, p.Hq, p.N)
    return o, lse


def attend_backward(q, k, v, do, idx, cnt, p: Params, blocks=None):
    """Gradients of step 8 with the selection held fixed: the routed lists are
    a discrete choice and carry no gradient; within a row's key set the read
    is ordinary softmax attention (jonsmirl/ssa README, introduction).

    For query i with key set S_i, logits l_ij = scale <q_i, k_j>, weights
    P_ij = softmax_j(l_i), read o_i = sum_j P_ij v_j and an upstream gradient
    g_i = dL/do_i:
        dL/dv_j += P_ij g_i
        dP_ij    = <g_i, v_j>
        dl_ij    = P_ij (dP_ij - sum_m P_im dP_im)      (softmax derivative)
        dL/dq_i  = scale sum_j dl_ij k_j
        dL/dk_j += scale dl_ij q_i
    Query head h reads KV head h // g, so a KV head's gradients sum over its
    group.  ``do`` [B, Hq, N, D] float64.  Returns (dq [B, Hq, N, D], dk, dv
    [B, Hkv, N, D]).  ``blocks`` optionally restricts the sum to the listed
    (b, h, qb) query blocks: dq is then filled on their rows only and dk/dv
    hold only their contributions."""
    scale = p.softmax_scale
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    todo = blocks if blocks is not None else [
        (b, h, qb) for b in range(p.B) for h in range(p.Hq) for qb in range(p.n_qblocks)]
    jpos = np.arange(p.N)
    jblk = jpos // p.block_k
    for b, h, qb in todo:
        g = h // p.group
        rows = np.arange(qb * p.block_q, (qb + 1) * p.block_q)
        routed = np.zeros(p.n_kblocks, dtype=bool)
        routed[idx[b, h, qb, :cnt[b, h, qb]]] = True
        allow = np.broadcast_to(routed[jblk][None, :], (len(rows), p.N)).copy()
        if p.causal:
            allow |= jpos[None, :] > rows[:, None] - p.window
            allow &= jpos[None, :] <= rows[:, None]
        logits = np.where(allow, (q[b, h, rows] @ k[b, g].T) * scale, -np.inf)
        m = logits.max(axis=-1, keepdims=True)
        w = np.exp(logits - m)
        P = w / w.sum(axis=-1, keepdims=True)                  # [Bq, N], 0 off the key sets
        gi = do[b, h, rows]
        dP = gi @ v[b, g].T
        dl = P * (dP - (P * dP).sum(axis=-1, keepdims=True))
        dq[b, h, rows] = scale * (dl @ k[b, g])
        dk[b, g] += scale * (dl.T @ q[b, h, rows])
        dvv[b, g] += P.T @ gi
    return dq, dk, dvv


def attend_gathered(q, k, v, idx, cnt, p: Params, queries=None):
    """Gathered form: each query's explicit key set, then softmax over it.

    ``queries`` optionally lists (b, h, i) triples; the result is then
    ([len, Dv], [len]).  Otherwise returns O [B, Hq, N, Dv], LSE [B, Hq, N]."""
    scale = p.softmax_scale
    dv = v.shape[-1]
    todo = queries if queries is not None else [
        (b, h, i) for b in range(p.B) for h in range(p.Hq) for i in range(p.N)]
    o_out = np.zeros((len(todo), dv))
    l_out = np.zeros(len(todo))
    for t, (b, h, i) in enumerate(todo):
        g = h // p.group
        qb = i // p.block_q
        s = key_set(i, idx[b, h, qb, :cnt[b, h, qb]], p)
        logits = (k[b, g, s] @ q[b, h, i]) * scale
        o1, l1 = _softmax_read(logits[None, :], v[b, g, s])
        o_out[t], l_out[t] = o1[0], l1[0]
    if queries is not None:
        return o_out, l_out
    return o_out.reshape(p.B, p.Hq, p.N, dv), l_out.reshape(p.B, p.Hq, p.N)


def attend_gathered_blocks(q, k, v, idx, cnt, p: Params, blocks):
    """Gathered form, one query block at a time: for each listed (b, h, qb)
    the logits are taken only over the keys any of the block's queries can
    see -- the selected blocks' keys and, causal, the window span
    [qb*Bq - W + 1, (qb+1)*Bq - 1] -- and each row keeps exactly its own key
    set (step 7, the same mask as ``attend_masked_dense``); softmax as in
    ``_softmax_read``.  Keys outside every
    row's set would only add exp(-inf) = 0 terms, so this is step 8 on the
    columns where it can be non-zero, which makes sampled rows of a
    million-token sequence cheap.  Returns ([len(blocks), Bq, Dv],
    [len(blocks), Bq])."""
    scale = p.softmax_scale
    dv = v.shape[-1]
    o_out = np.zeros((len(blocks), p.block_q, dv))
    l_out = np.zeros((len(blocks), p.block_q))
    for t, (b, h, qb) in enumerate(blocks):
        g = h // p.group
        sel = np.asarray(idx[b, h, qb, :cnt[b, h, qb]], dtype=np.int64)
        rows = np.arange(qb * p.block_q, (qb + 1) * p.block_q)
        cols = (sel[:, None] * p.block_k + np.arange(p.block_k)[None, :]).ravel()
        if p.causal:
            cols = np.union1d(cols, np.arange(max(0, rows[0] - p.window + 1), rows[-1] + 1))
        else:
            cols = np.unique(cols)
        # step 7 on these columns, as in the masked-dense form: a routed key,
        # or (causal) a window key i - W < j, and never a key after i
        routed = np.isin(cols, (sel[:, None] * p.block_k + np.arange(p.block_k)[None, :]).ravel())
        allow = np.broadcast_to(routed[None, :], (len(rows), len(cols))).copy()
        if p.causal:
            allow |= cols[None, :] > rows[:, None] - p.window
            allow &= cols[None, :] <= rows[:, None]
        logits = np.where(allow, (q[b, h, rows] @ k[b, g, cols].T) * scale, -np.inf)
        o_out[t], l_out[t] = _softmax_read(logits, v[b, g, cols])
    return o_out, l_out


# --------------------------------------------------------------------------
# decode: one new query per head against the cached keys
# --------------------------------------------------------------------------
def decode_step(q, k, v, n_ctx: int, p: Params):
    """One decode step.  ``q`` [B, Hq, D] is the query at position
    i = n_ctx - 1 (its own key and value are already the cache's row i);
    ``k``/``v`` [B, Hkv, >= n_ctx, D] float64 caches.

    The query is its own query block (Bq = 1): it scores the completed key
    blocks (c+1)*Bk <= i by <q, mu_c> (step 5), keeps the top_k ordered by
    (score descending, block index ascending) (step 6), and reads exact
    softmax over the routed blocks' keys united with the window
    i - W < j <= i, cut at i (steps 7-8) -- the method's steps for one query.
    Causal only.  Returns (o [B, Hq, Dv], lse [B, Hq], idx [B, Hq, top_k]
    ascending and -1 padded, cnt [B, Hq])."""
    if not p.causal:
        raise ValueError("decode is causal")
    i = n_ctx - 1
    nb = i // p.block_k                       # admissible: c < i // Bk
    mu = block_summary(k[:, :, :nb * p.block_k], p.block_k) if nb else None
    scale = p.softmax_scale
    o = np.zeros((p.B, p.Hq, v.shape[-1]))
    lse = np.zeros((p.B, p.Hq))
    idx = np.full((p.B, p.Hq, p.top_k), -1, dtype=np.int32)
    cnt = np.zeros((p.B, p.Hq), dtype=np.int32)
    for b in range(p.B):
        for h in range(p.Hq):
            g = h // p.group
            if nb:
                sel, _, _ = route_row(q[b, h], mu[b, g], np.arange(nb), p.top_k)
            else:
                sel = np.zeros(0, dtype=np.int64)
            idx[b, h, :len(sel)] = sel
            cnt[b, h] = len(sel)
            o[b, h], lse[b, h] = decode_attend(q[b, h], k[b, g], v[b, g], i, sel, p)
    return o, lse, idx, cnt


def decode_attend(q, k, v, i: int, sel, p: Params):
    """The read of one decode query: exact softmax of ``q`` [D] over the keys
    of the selected blocks ``sel`` united with the window i - W < j <= i
    (``key_set``), against one head's caches ``k``/``v`` [>= i+1, D].
    Returns (o [Dv], lse)."""
    ks = key_set(i, np.asarray(sel, dtype=np.int64), p)
    logits = (k[ks] @ q) * p.softmax_scale
    o1, l1 = _softmax_read(logits[None, :], v[ks])
    return o1[0], l1[0]


def forward(q, k, v, p: Params, form: str = "dense"):
    """Whole path: summaries -> routing -> attend.  Inputs float64 arrays
    (use ``upcast_bf16`` on bf16 bit patterns).  Returns a dict with
    ``o``, ``lse``, ``idx``, ``cnt``, ``route`` (RouteResult: the per-head
    selections), ``qsum``, ``ksum``.  With ``p.consensus`` the per-head
    selections are reduced to one list per (b, KV head, query block)
    (``route_consensus``), which ``idx``/``cnt`` then hold, and every query
    head of a group attends over its group's list."""
    ksum = block_summary(k, p.block_k)
    qsum = block_summary(q, p.block_q)
    ksum2 = None
    if p.beta != 0.0:
        r = route(qsum, ksum, p, qm2=block_second_moment(q, p.block_q),
                  kcov=block_covariance(k, p.block_k))
    elif p.tree_fanout > 0:
        ksum2 = tree_summary(k, p.block_k, p.tree_fanout)
        r = route(qsum, ksum, p, ksum2=ksum2)
    else:
        r = route(qsum, ksum, p)
    attend = attend_masked_dense if form == "dense" else attend_gathered
    if p.consensus:
        idx, cnt = route_consensus(r.idx, r.cnt, p)
        o, lse = attend(q, k, v, *expand_consensus(idx, cnt, p), p)
    else:
        idx, cnt = r.idx, r.cnt
        o, lse = attend(q, k, v, idx, cnt, p)
    return {"o": o, "lse": lse, "idx": idx, "cnt": cnt, "route": r,
            "qsum": qsum, "ksum": ksum, "ksum2": ksum2}
