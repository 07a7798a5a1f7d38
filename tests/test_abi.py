"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects invalid arguments synchronously, before any launch."""
import ctypes

import pytest

from content_routed_block_b200 import build, ssa


@pytest.fixture(scope="module")
def L():
    build.build()
    return ssa.lib()


def test_every_declared_function_is_exported(L):
    names = ssa.declared_functions()
    assert {"ssa_block_summary", "ssa_route", "ssa_attend", "ssa_forward",
            "ssa_workspace_size", "ssa_check_error"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert L.ssa_version() == 2
    for s in range(7):
        assert L.ssa_status_string(s).decode() not in ("", "unknown status")
    assert L.ssa_status_string(99).decode() == "unknown status"


def _p(**kw):
    base = dict(B=1, Hq=14, Hkv=2, N=32768, D=64, block_k=64, block_q=64, top_k=16,
                window=512, causal=True)
    base.update(kw)
    return ssa.make_params(**base)


def test_workspace_layout(L):
    p = _p()
    ks = 1 * 2 * 512 * 64 * 4
    qs = 1 * 14 * 512 * 64 * 4
    ix = 1 * 14 * 512 * 16 * 4
    cn = 1 * 14 * 512 * 4
    a = lambda x: (x + 255) // 256 * 256
    assert ssa.workspace_size(p) == a(ks) + a(qs) + a(ix) + a(cn)


def test_workspace_layout_with_the_routers_key_image(L, monkeypatch):
    # the tensor-core router's pre-split key summaries (tiles of 128 key
    # blocks: bf16 hi and lo parts of 128 x D each, and 128 fp32 norms) sit at
    # the end of the forward's workspace when that form routes the problem
    # (>= 2^25 admissible pairs over all heads) and form ssa_route's scratch
    monkeypatch.delenv("SSA_ROUTER", raising=False)
    a = lambda x: (x + 255) // 256 * 256
    p = _p(N=1 << 20, window=1024)                      # 16,384 blocks, 14 heads
    nb = 16384
    ks, qs = 2 * nb * 64 * 4, 14 * nb * 64 * 4
    ix, cn = 14 * nb * 16 * 4, 14 * nb * 4
    tiles = 2 * (nb // 128)
    img = a(tiles * 2 * 128 * 64 * 2) + a(tiles * 128 * 4)
    assert ssa.route_workspace_size(p) == img
    assert ssa.workspace_size(p) == a(ks) + a(qs) + a(ix) + a(cn) + img
    assert ssa.route_workspace_size(_p()) == 0          # 32K tokens: the fp32 form
    monkeypatch.setenv("SSA_ROUTER", "fp32")
    assert ssa.route_workspace_size(p) == 0
    monkeypatch.setenv("SSA_ROUTER", "tc")
    t = 2 * 4                                           # 512 blocks: four tiles per head
    assert ssa.route_workspace_size(_p()) == a(t * 2 * 128 * 64 * 2) + a(t * 128 * 4)
    # a ragged last tile: 200 blocks are two tiles
    q = _p(N=200 * 64, Hq=2, Hkv=1)
    assert ssa.route_workspace_size(q) == a(2 * 2 * 128 * 64 * 2) + a(2 * 128 * 4)


def test_route_with_workspace_rejects_bad_arguments_before_launch(L, monkeypatch):
    monkeypatch.setenv("SSA_ROUTER", "tc")
    p = _p()
    good = ctypes.c_void_p(1 << 20)
    need = ssa.route_workspace_size(p)
    f = L.ssa_route_with_workspace
    assert f(ctypes.byref(p), good, good, good, good, None, 0, None) == 3        # no scratch
    assert f(ctypes.byref(p), good, good, good, good, good, need - 1, None) == 3  # too small
    odd = ctypes.c_void_p((1 << 20) + 16)
    assert f(ctypes.byref(p), good, good, good, good, odd, need, None) == 1      # unaligned
    assert f(ctypes.byref(p), None, good, good, good, good, need, None) == 1     # no qsum


def test_workspace_layout_with_consensus(L):
    p = _p(consensus=True)
    ks = 1 * 2 * 512 * 64 * 4
    qs = 1 * 14 * 512 * 64 * 4
    ix = 1 * 14 * 512 * 16 * 4
    cn = 1 * 14 * 512 * 4
    a = lambda x: (x + 255) // 256 * 256
    assert ssa.workspace_size(p) == a(ks) + a(qs) + a(ix) + a(cn) + a(ix // 7) + a(cn // 7)


def test_consensus_entry_point_rejects_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    f = L.ssa_route_consensus
    p = _p()
    assert f(ctypes.byref(p), good, None, good, good, None) == 1
    assert f(ctypes.byref(p), good, good, good, None, None) == 1
    assert f(ctypes.byref(p), odd, good, good, good, None) == 1
    big = _p(Hq=16, Hkv=1, top_k=33)
    assert f(ctypes.byref(big), good, good, good, good, None) == 2
    flag = _p()
    flag.consensus = 2                   # the flag is 0 or 1
    assert L.ssa_workspace_size(ctypes.byref(flag)) == 0
    assert f(ctypes.byref(flag), good, good, good, good, None) == 1


@pytest.mark.parametrize("kw,status", [
    (dict(D=96), 2), (dict(D=32), 2), (dict(Hq=3, Hkv=2), 1), (dict(N=1000), 2),
    (dict(top_k=65), 2), (dict(top_k=-1), 2), (dict(block_k=48), 2), (dict(block_k=256), 2),
    (dict(block_q=8), 2), (dict(window=0), 1), (dict(causal=False), 1),
    (dict(causal=False, window=0, top_k=0), 1), (dict(window=-3), 1), (dict(B=0), 1),
    (dict(scale=float("nan")), 1), (dict(scale=-1.0), 1), (dict(wait_timeout_us=-5), 1),
    (dict(N=16 * 2 ** 23, block_k=16, block_q=16, B=1, Hq=1, Hkv=1), 2),
    (dict(window=200000, block_k=16, block_q=16), 2),
    (dict(consensus=True, Hq=16, Hkv=1, top_k=33), 2), (dict(beta=float("inf")), 1),
])
def test_invalid_params_are_rejected_before_launch(L, kw, status):
    p = _p(**kw)
    assert L.ssa_workspace_size(ctypes.byref(p)) == 0
    fake = ctypes.c_void_p(1 << 20)
    st = L.ssa_forward(ctypes.byref(p), fake, fake, fake, fake, None, None, None, fake,
                       1 << 40, None)
    assert st == status, L.ssa_last_error_message()
    assert L.ssa_last_error_message().decode()


def test_bad_pointers_and_workspace_are_rejected_before_launch(L):
    p = _p()
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    ws = ssa.workspace_size(p)
    f = L.ssa_forward
    assert f(ctypes.byref(p), None, good, good, good, None, None, None, good, ws, None) == 1
    assert f(ctypes.byref(p), odd, good, good, good, None, None, None, good, ws, None) == 1
    assert f(ctypes.byref(p), good, good, good, good, None, None, None, good, ws - 1, None) == 3
    assert f(ctypes.byref(p), good, good, good, good, None, None, None, None, ws, None) == 3
    assert f(ctypes.byref(p), good, good, good, good, None, None, None,
             ctypes.c_void_p((1 << 20) + 16), ws, None) == 1
    assert L.ssa_attend(ctypes.byref(p), good, good, good, None, good, good, None, None) == 1
    assert L.ssa_route(ctypes.byref(p), good, good, good, None, None) == 1
    assert L.ssa_block_summary(ctypes.byref(p), good, 14, 48, good, None) == 1
    assert L.ssa_block_summary(ctypes.byref(p), odd, 14, 64, good, None) == 1
    assert L.ssa_probe_wait_timeout(0, None) == 1
    assert L.ssa_forward(None, good, good, good, good, None, None, None, good, ws, None) == 1


def test_binding_rejects_wrong_tensors():
    import torch
    p = _p(N=1024, Hq=2, Hkv=2, top_k=4, window=128)
    q = torch.zeros(1, 2, 1024, 64, dtype=torch.bfloat16)   # CPU tensor: refused by the binding
    with pytest.raises(ValueError):
        ssa.forward(q, q, q, p)


def test_workspace_layout_with_second_cumulant(L):
    p = _p(beta=0.5)
    a = lambda x: (x + 255) // 256 * 256
    ks, qs = 2 * 512 * 64 * 4, 14 * 512 * 64 * 4
    ix, cn = 14 * 512 * 16 * 4, 14 * 512 * 4
    F = 64 + 64 * 65 // 2
    qf, kf, sc = 14 * 512 * F * 4, 2 * 512 * F * 4, 14 * 512 * 512 * 4
    assert ssa.workspace_size(p) == a(ks) + a(qs) + a(ix) + a(cn) + a(qf) + a(kf) + a(sc)


def test_second_cumulant_entry_points_reject_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    p = _p(beta=1.0)
    # the mean-only router refuses a nonzero beta
    assert L.ssa_route(ctypes.byref(p), good, good, good, good, None) == 1
    f = L.ssa_route_features
    assert f(ctypes.byref(p), good, 14, 64, 2, good, None) == 1      # queries flag
    assert f(ctypes.byref(p), good, 14, 256, 1, good, None) == 1     # block too large
    assert f(ctypes.byref(p), None, 14, 64, 1, good, None) == 1
    g = L.ssa_route_cumulant
    assert g(ctypes.byref(p), good, good, None, good, good, None) == 1
    assert g(ctypes.byref(p), good, good, good, None, good, None) == 1


def test_decode_entry_point_rejects_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    p = _p()
    ws = L.ssa_decode_workspace_size(ctypes.byref(p))
    assert ws > 0
    f = L.ssa_decode
    args = lambda n, w=good, wb=ws: (ctypes.byref(p), good, good, good, n, good, good, None, None,
                                     None, w, wb, None)
    assert f(*args(0)) == 1                       # n_ctx below 1
    assert f(*args(32769)) == 1                   # n_ctx above the capacity
    assert f(*args(100, wb=ws - 1)) == 3          # workspace too small
    assert f(*args(100, w=ctypes.c_void_p((1 << 20) + 16))) == 1
    for kw, status in ((dict(causal=False, window=0), 1), (dict(consensus=True), 2),
                       (dict(beta=0.5), 2)):
        bad = _p(**kw)
        assert L.ssa_decode_workspace_size(ctypes.byref(bad)) == 0
        assert f(ctypes.byref(bad), good, good, good, 100, good, good, None, None, None, good,
                 ws, None) == status


def test_workspace_layout_with_tree_routing(L):
    p = _p(tree_fanout=16, tree_beam=8)
    a = lambda x: (x + 255) // 256 * 256
    ks, qs = 2 * 512 * 64 * 4, 14 * 512 * 64 * 4
    ix, cn = 14 * 512 * 16 * 4, 14 * 512 * 4
    k2, s2 = 2 * 32 * 64 * 4, 14 * 512 * 8 * 4
    assert ssa.workspace_size(p) == a(ks) + a(qs) + a(ix) + a(cn) + a(k2) + a(s2) + a(cn)


@pytest.mark.parametrize("kw,status", [
    (dict(tree_fanout=3, tree_beam=4), 2),          # not a power of two
    (dict(tree_fanout=512, tree_beam=4), 2),        # above 256
    (dict(N=1024, tree_fanout=32, tree_beam=4), 2),  # more than N/Bk = 16 blocks
    (dict(tree_fanout=16, tree_beam=0), 2), (dict(tree_fanout=16, tree_beam=65), 2),
    (dict(tree_fanout=16, tree_beam=4, beta=0.5), 2),
    (dict(tree_beam=4), 1),                         # a beam without a tree
])
def test_invalid_tree_params_are_rejected_before_launch(L, kw, status):
    p = _p(**kw)
    assert L.ssa_workspace_size(ctypes.byref(p)) == 0
    fake = ctypes.c_void_p(1 << 20)
    assert L.ssa_forward(ctypes.byref(p), fake, fake, fake, fake, None, None, None, fake,
                         1 << 40, None) == status


def test_tree_entry_points_reject_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    flat = _p()
    p = _p(tree_fanout=16, tree_beam=4)
    assert L.ssa_tree_summary(ctypes.byref(flat), good, good, None) == 1     # no tree
    assert L.ssa_tree_summary(ctypes.byref(p), None, good, None) == 1
    assert L.ssa_tree_summary(ctypes.byref(p), good, odd, None) == 1
    f = L.ssa_route_tree
    assert f(ctypes.byref(flat), good, good, good, good, good, good, good, None) == 1
    assert f(ctypes.byref(p), good, good, None, good, good, good, good, None) == 1
    assert f(ctypes.byref(p), good, good, good, good, None, good, good, None) == 1
    assert f(ctypes.byref(p), good, good, good, odd, good, good, good, None) == 1
    # decode keeps the flat block list
    assert L.ssa_decode_workspace_size(ctypes.byref(p)) == 0


def test_backward_entry_point_rejects_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 4)
    p = _p()
    ws = L.ssa_backward_workspace_size(ctypes.byref(p))
    # two fp32 per query row (delta, lse * log2 e), one bit per (head, 128-key tile,
    # 64-query chunk): 14 heads x 256 tiles x 16 words of 32 chunks, then
    # each query head's share of dk and dv (fp32 [14, 32768, 64] each)
    assert ws == 2 * ((1 * 14 * 32768 * 4 + 255) // 256 * 256) + 14 * 256 * 16 * 4 + \
        2 * 14 * 32768 * 64 * 4
    f = L.ssa_attend_backward

    def call(**over):
        args = dict(q=good, k=good, v=good, o=good, lse=good, d_o=good, idx=good, cnt=good,
                    dq=good, dk=good, dv=good, ws=good, wsb=ws)
        args.update(over)
        return f(ctypes.byref(p), args["q"], args["k"], args["v"], args["o"], args["lse"],
                 args["d_o"], args["idx"], args["cnt"], args["dq"], args["dk"], args["dv"],
                 args["ws"], args["wsb"], None)

    for name in ("q", "o", "lse", "d_o", "cnt", "dq", "dk", "dv", "idx"):
        assert call(**{name: None}) == 1, name
    assert call(dk=odd) == 1
    assert call(wsb=ws - 1) == 3
    assert call(ws=None) == 3
    assert call(ws=ctypes.c_void_p((1 << 20) + 16)) == 1
    bad = _p(D=96)
    assert L.ssa_backward_workspace_size(ctypes.byref(bad)) == 0
    assert f(ctypes.byref(bad), good, good, good, good, good, good, good, good, good, good, good,
             good, ws, None) == 2


def test_binding_checks_backward_and_tree_tensors_before_calling():
    import torch
    p = _p(N=1024, Hq=2, Hkv=1, top_k=4, window=128)
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)          # CPU: refused  # noqa: E731
    q, k = bf(1, 2, 1024, 64), bf(1, 1, 1024, 64)
    lse = torch.zeros(1, 2, 1024)
    idx = torch.zeros(1, 2, 16, 4, dtype=torch.int32)
    cnt = torch.zeros(1, 2, 16, dtype=torch.int32)
    with pytest.raises(ValueError):
        ssa.backward(q, k, k, q, lse, q, idx, cnt, p)                # host tensors
    t = _p(N=1024, Hq=2, Hkv=1, top_k=4, window=128, tree_fanout=4, tree_beam=2)
    ksum = torch.zeros(1, 1, 16, 64)
    with pytest.raises(ValueError):
        ssa.tree_summary(ksum, t)
    with pytest.raises(ValueError):
        ssa.route_tree(torch.zeros(1, 2, 16, 64), ksum, torch.zeros(1, 1, 3, 64), t)


def test_static_forward_rejects_oversized_shapes_before_any_cuda_call(L):
    # the scratch size check comes first: no pointer is looked at and no CUDA
    # call is made, so NULL pointers are never dereferenced or launched on
    fn = L.ssa_forward_static
    vp = ctypes.c_void_p
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.POINTER(ssa.Params), vp, vp, vp, vp, vp, vp, vp, vp]
    p = _p(N=1 << 20, window=1024)
    assert ssa.workspace_size(p) > (32 << 20)
    assert fn(ctypes.byref(p), None, None, None, None, None, None, None, None) == 3
    assert "scratch" in L.ssa_last_error_message().decode()
    bad = _p(D=96)
    assert fn(ctypes.byref(bad), None, None, None, None, None, None, None, None) == 2


def test_ex2_probe_rejects_bad_arguments_before_launch(L):
    good = ctypes.c_void_p(1 << 20)
    assert L.ssa_probe_ex2_rate(0, 10, good, None) == 1
    assert L.ssa_probe_ex2_rate(10, 0, good, None) == 1
    assert L.ssa_probe_ex2_rate(10, 10, None, None) == 1
