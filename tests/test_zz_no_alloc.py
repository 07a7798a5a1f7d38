"""ssa_forward_static: the whole path without a caller workspace.

Some callers cannot allocate device memory when they call in (a framework's
launch callback or plugin where cudaMalloc is forbidden, or code with no
allocator at hand).  ssa_forward_static serves them from a fixed scratch array
inside the library.  This file is collected last on purpose, so that a run that
stops at its first failure has already run every other test; it also passes on
its own in a fresh process.
"""
import ctypes

import pytest
import torch

from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, Workload, make_inputs
from parity_utils import to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


def W(name, **kw):
    base = dict(B=1, Hq=4, Hkv=2, N=2048, D=64, block_k=64, block_q=64, top_k=6, window=128,
                causal=True, kind="clustered", centres=16, seed=21)
    base.update(kw)
    return Workload(name, **base)


# every path that keeps state in the scratch: plain causal and non-causal
# routing, the consensus lists, the second-cumulant features and score
# matrix, and the two-level route's super-block summaries and kept lists
CASES = [
    CONFIGS[1],
    CONFIGS[4],
    W("consensus", Hq=6, Hkv=2, consensus=True),
    W("beta", N=1024, beta=0.75, kind="iid"),
    W("tree", N=4096, tree_fanout=4, tree_beam=3),
]

# a different shape and different values, run first so that the scratch holds
# its bytes when the case under test starts
FILLER = W("filler", B=2, Hq=16, Hkv=16, N=16384, block_k=16, block_q=16, top_k=12, window=0,
           causal=False, kind="iid", seed=5)


@pytest.fixture(scope="module")
def L():
    build.build()
    L = ssa.lib()
    fn = L.ssa_forward_static
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.POINTER(ssa.Params), vp, vp, vp, vp, vp, vp, vp, vp]
    return L


def _inputs(w):
    x = make_inputs(w)
    return tuple(to_dev(x[n]) for n in "qkv")


def _static_call(L, p, q, k, v):
    o = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq, p.N), dtype=torch.float32, device=q.device)
    idx = torch.empty((p.B, p.list_heads, p.n_qblocks, p.top_k), dtype=torch.int32,
                      device=q.device)
    cnt = torch.empty((p.B, p.list_heads, p.n_qblocks), dtype=torch.int32, device=q.device)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    status = L.ssa_forward_static(ctypes.byref(p), P(q), P(k), P(v), P(o), P(lse), P(idx), P(cnt),
                                  st)
    assert status == 0, L.ssa_last_error_message().decode()
    ssa.check_error()
    return o, lse, idx, cnt


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_static_scratch_matches_workspace_path_twice(L, w):
    p = ssa.params_of(w)
    assert ssa.workspace_size(p) <= SCRATCH_BYTES
    pf = ssa.params_of(FILLER)
    assert ssa.workspace_size(pf) <= SCRATCH_BYTES
    _static_call(L, pf, *_inputs(FILLER))        # leaves other bytes in the scratch
    q, k, v = _inputs(w)
    ref = ssa.forward(q, k, v, p)
    ssa.check_error()
    for _ in range(2):                           # two calls in a row share the scratch
        got = _static_call(L, p, q, k, v)
        # the same kernels on the same inputs: bit-identical results
        for name, a, b in zip(("o", "lse", "idx", "cnt"), got, ref):
            assert torch.equal(a, b), f"{w.name}: {name} differs from the workspace path"


def test_static_scratch_rejects_oversized_shapes(L):
    # a shape whose scratch exceeds 32 MiB; its tensors are real and sized
    # for the shape, so even a call that got past the size check could only
    # touch memory it owns
    p = ssa.make_params(1, 64, 64, 65536, 64, 64, 64, 16, 128, True)
    assert ssa.workspace_size(p) > SCRATCH_BYTES
    q, k, v, o = (torch.zeros((1, 64, 65536, 64), dtype=torch.bfloat16, device="cuda")
                  for _ in range(4))
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = L.ssa_forward_static(ctypes.byref(p), P(q), P(k), P(v), P(o), None, None, None, st)
    assert status == 3
    assert "scratch" in L.ssa_last_error_message().decode()
    torch.cuda.synchronize()
    ssa.check_error()
