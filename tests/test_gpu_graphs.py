"""The library's calls inside CUDA graphs: the forward and a decode step are
captured once and replayed, with new inputs written in place before each
replay; every replay must match the eager call on the same inputs bit for
bit (the kernels are deterministic).  Nothing in the path synchronises or
allocates on the device, which is what capture requires."""
import numpy as np
import pytest
import torch

from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, make_inputs
from parity_utils import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ssa.lib()
    torch.cuda.init()
    ssa.check_error()


def _inputs(w, seed):
    x = make_inputs(w.with_(seed=seed))
    return [to_dev(x[n]) for n in "qkv"]


@pytest.mark.parametrize("kw", [dict(), dict(consensus=True), dict(beta=0.5),
                                dict(tree_fanout=4, tree_beam=2)],
                         ids=["per-head", "consensus", "second-cumulant", "two-level"])
def test_forward_replays_in_a_cuda_graph(kw):
    w = Workload("graph", B=1, Hq=4, Hkv=2, N=2048, D=64, block_k=64, block_q=64, top_k=6,
                 window=128, causal=True, kind="clustered", centres=16, seed=3, **kw)
    p = ssa.params_of(w)
    q, k, v = _inputs(w, 3)
    LH = w.Hkv if w.consensus else w.Hq
    ws = torch.empty(ssa.workspace_size(p), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, w.Hq, w.N), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, LH, w.N // 64, w.top_k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, LH, w.N // 64), dtype=torch.int32, device="cuda")

    def call():
        ssa.forward(q, k, v, p, workspace=ws, out=o, lse_out=lse, idx_out=idx, cnt_out=cnt)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for seed in (4, 5):
        q2, k2, v2 = _inputs(w, seed)
        q.copy_(q2), k.copy_(k2), v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, lse, idx, cnt)]
        want = ssa.forward(q2, k2, v2, p)
        ssa.check_error()
        for a, b in zip(got, want):
            assert torch.equal(a, b)


def test_decode_step_replays_in_a_cuda_graph():
    w = CONFIGS[2].with_(N=8192)
    p = ssa.params_of(w)
    q_all, k, v = _inputs(w, 1)
    ksum = ssa.block_summary(k, w.block_k, p)
    ws = torch.empty(ssa.decode_workspace_size(p), dtype=torch.uint8, device="cuda")
    n_ctx = 8000
    q = q_all[:, :, n_ctx - 1].contiguous()
    o = torch.empty((1, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")

    def call():
        ssa.decode(q, k, v, n_ctx, ksum, p, workspace=ws, out=o)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for pos in (n_ctx - 1, 17):
        q.copy_(q_all[:, :, pos])
        g.replay()
        torch.cuda.synchronize()
        got = o.clone()
        want, _, _, _ = ssa.decode(q.clone(), k, v, n_ctx, ksum, p)
        ssa.check_error()
        assert torch.equal(got, want)
