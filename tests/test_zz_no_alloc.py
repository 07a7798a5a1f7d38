"""ssa_forward_static: the whole path without a caller workspace.

Some callers cannot allocate device memory when they call in (a framework's
launch callback or plugin where cudaMalloc is forbidden, or code with no
allocator at hand).  ssa_forward_static serves them from a fixed scratch array
inside the library.  This file is collected last on purpose, so that a run that
stops at its first failure has already run every other test; it also passes on
its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from content_routed_block_b200 import build, ssa
from content_routed_block_b200.workloads import CONFIGS, make_inputs
from parity_utils import MAX_ABS, MEAN_ABS, to_dev

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20


@pytest.fixture(scope="module")
def L():
    build.build()
    L = ssa.lib()
    fn = L.ssa_forward_static
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.POINTER(ssa.Params), vp, vp, vp, vp, vp, vp, vp, vp]
    return L


def _static_call(L, p, q, k, v):
    o = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq, p.N), dtype=torch.float32, device=q.device)
    idx = torch.empty((p.B, p.Hq, p.n_qblocks, p.top_k), dtype=torch.int32, device=q.device)
    cnt = torch.empty((p.B, p.Hq, p.n_qblocks), dtype=torch.int32, device=q.device)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    status = L.ssa_forward_static(ctypes.byref(p), P(q), P(k), P(v), P(o), P(lse), P(idx), P(cnt),
                                  st)
    assert status == 0, L.ssa_last_error_message().decode()
    ssa.check_error()
    return o, lse, idx, cnt


@pytest.mark.parametrize("cfg", [1, 4])
def test_static_scratch_matches_workspace_path_twice(L, cfg):
    w = CONFIGS[cfg]
    p = ssa.params_of(w)
    assert ssa.workspace_size(p) <= SCRATCH_BYTES
    x = make_inputs(w)
    q, k, v = (to_dev(x[n]) for n in "qkv")
    o_ref, lse_ref, idx_ref, cnt_ref = ssa.forward(q, k, v, p)
    ssa.check_error()
    for _ in range(2):                       # two calls in a row share the scratch
        o, lse, idx, cnt = _static_call(L, p, q, k, v)
        assert torch.equal(idx, idx_ref) and torch.equal(cnt, cnt_ref)
        err = (o.float() - o_ref.float()).abs()
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
        assert (lse - lse_ref).abs().max().item() <= 2e-3


def test_static_scratch_rejects_oversized_shapes(L):
    p = ssa.params_of(CONFIGS[5])
    assert ssa.workspace_size(p) > SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    status = L.ssa_forward_static(ctypes.byref(p), fake, fake, fake, fake, None, None, None, None)
    assert status == 3
    assert "32" in L.ssa_last_error_message().decode() or "scratch" in L.ssa_last_error_message().decode()
