"""Thin Python binding of libssa.so (ctypes, argument marshalling only).

Every step of the path runs in the library's CUDA kernels; this module only
checks tensor shapes / dtypes / devices, allocates outputs with PyTorch and
passes raw pointers plus the current CUDA stream.  There is no fallback: if
libssa.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "Params", "SsaError", "lib", "make_params", "params_of", "workspace_size", "block_summary",
    "route", "route_workspace_size", "route_consensus", "route_features", "route_cumulant",
    "tree_summary", "route_tree",
    "attend", "forward",
    "forward_host", "backward", "decode", "decode_workspace_size", "check_error",
    "probe_wait_timeout", "probe_ex2_rate",
    "declared_functions", "LIB_PATH", "HEADER_PATH",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssa.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "ssa.h")

SSA_OK = 0


class SsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"ssa status {status}: {message}")
        self.status = status
        self.message = message


class Params(ctypes.Structure):
    """Mirror of ``ssa_params`` in include/ssa.h."""
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
        ("N", ctypes.c_int32), ("D", ctypes.c_int32), ("block_k", ctypes.c_int32),
        ("block_q", ctypes.c_int32), ("top_k", ctypes.c_int32), ("window", ctypes.c_int32),
        ("causal", ctypes.c_int32), ("scale", ctypes.c_float),
        ("wait_timeout_us", ctypes.c_int32), ("consensus", ctypes.c_int32),
        ("beta", ctypes.c_float), ("tree_fanout", ctypes.c_int32), ("tree_beam", ctypes.c_int32),
    ]

    @property
    def n_kblocks(self) -> int:
        return self.N // self.block_k

    @property
    def n_qblocks(self) -> int:
        return self.N // self.block_q

    @property
    def list_heads(self) -> int:
        """Heads the attended lists span: Hkv with consensus routing, else Hq."""
        return self.Hkv if self.consensus else self.Hq


def make_params(B, Hq, Hkv, N, D, block_k, block_q, top_k, window, causal, scale=0.0,
                wait_timeout_us=0, consensus=False, beta=0.0, tree_fanout=0,
                tree_beam=0) -> Params:
    return Params(B, Hq, Hkv, N, D, block_k, block_q, top_k, window, int(bool(causal)),
                  float(scale), wait_timeout_us, int(bool(consensus)), float(beta),
                  int(tree_fanout), int(tree_beam))


def params_of(w, **over) -> Params:
    """Params from any object with the workload field names."""
    f = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, D=w.D, block_k=w.block_k, block_q=w.block_q,
             top_k=w.top_k, window=w.window, causal=w.causal, scale=getattr(w, "scale", 0.0),
             consensus=getattr(w, "consensus", False), beta=getattr(w, "beta", 0.0),
             tree_fanout=getattr(w, "tree_fanout", 0), tree_beam=getattr(w, "tree_beam", 0))
    f.update(over)
    return make_params(**f)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libssa.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m content_routed_block_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Params)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "ssa_workspace_size": (sz, [P]),
        "ssa_block_summary": (i32, [P, vp, i32, i32, vp, vp]),
        "ssa_route": (i32, [P, vp, vp, vp, vp, vp]),
        "ssa_route_workspace_size": (sz, [P]),
        "ssa_route_with_workspace": (i32, [P, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_route_consensus": (i32, [P, vp, vp, vp, vp, vp]),
        "ssa_tree_summary": (i32, [P, vp, vp, vp]),
        "ssa_route_tree": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "ssa_route_features": (i32, [P, vp, i32, i32, i32, vp, vp]),
        "ssa_route_cumulant": (i32, [P, vp, vp, vp, vp, vp, vp]),
        "ssa_attend": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp]),
        "ssa_forward": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_backward_workspace_size": (sz, [P]),
        "ssa_attend_backward": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_decode_workspace_size": (sz, [P]),
        "ssa_decode": (i32, [P, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_check_error": (i32, [vp]),
        "ssa_probe_wait_timeout": (i32, [i32, vp]),
        "ssa_probe_ex2_rate": (i32, [i32, i32, vp, vp]),
        "ssa_status_string": (ctypes.c_char_p, [i32]),
        "ssa_last_error_message": (ctypes.c_char_p, []),
        "ssa_version": (i32, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def declared_functions() -> list[str]:
    """Entry points declared in include/ssa.h."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssa_[a-z_]+)\s*\(", src)))


def _check(status: int):
    if status != SSA_OK:
        L = lib()
        raise SsaError(status, f"{L.ssa_status_string(status).decode()}: "
                               f"{L.ssa_last_error_message().decode()}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def workspace_size(p: Params) -> int:
    return int(lib().ssa_workspace_size(ctypes.byref(p)))


def block_summary(x: torch.Tensor, block: int, p: Params) -> torch.Tensor:
    """fp32 [B, H, N/block, D] means of every ``block`` rows of bf16 x [B, H, N, D]."""
    H = x.shape[1]
    _need(x, torch.bfloat16, (p.B, H, p.N, p.D), "x")
    out = torch.empty((p.B, H, p.N // block, p.D), dtype=torch.float32, device=x.device)
    _check(lib().ssa_block_summary(ctypes.byref(p), _ptr(x), H, block, _ptr(out), _stream()))
    return out


def route_workspace_size(p: Params) -> int:
    return int(lib().ssa_route_workspace_size(ctypes.byref(p)))


def route(qsum: torch.Tensor, ksum: torch.Tensor, p: Params, workspace: torch.Tensor | None = None,
          in_kernel_split: bool = False):
    """(idx int32 [B, Hq, NQB, top_k], cnt int32 [B, Hq, NQB]).  Routes through
    ssa_route_with_workspace (scratch from ``workspace`` or a fresh buffer);
    ``in_kernel_split`` calls ssa_route, which needs no scratch."""
    _need(qsum, torch.float32, (p.B, p.Hq, p.n_qblocks, p.D), "qsum")
    _need(ksum, torch.float32, (p.B, p.Hkv, p.n_kblocks, p.D), "ksum")
    dev = qsum.device
    idx = torch.empty((p.B, p.Hq, p.n_qblocks, p.top_k), dtype=torch.int32, device=dev)
    cnt = torch.empty((p.B, p.Hq, p.n_qblocks), dtype=torch.int32, device=dev)
    if in_kernel_split:
        _check(lib().ssa_route(ctypes.byref(p), _ptr(qsum), _ptr(ksum),
                               _ptr(idx) if p.top_k else None, _ptr(cnt), _stream()))
        return idx, cnt
    ws = route_workspace_size(p)
    if ws and (workspace is None or workspace.numel() < ws):
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    _check(lib().ssa_route_with_workspace(
        ctypes.byref(p), _ptr(qsum), _ptr(ksum), _ptr(idx) if p.top_k else None, _ptr(cnt),
        _ptr(workspace) if ws else None, ws, _stream()))
    return idx, cnt


def tree_summary(ksum: torch.Tensor, p: Params) -> torch.Tensor:
    """Super-block means fp32 [B, Hkv, (N/Bk) // tree_fanout, D] from block means."""
    _need(ksum, torch.float32, (p.B, p.Hkv, p.n_kblocks, p.D), "ksum")
    ns = p.n_kblocks // max(p.tree_fanout, 1)
    out = torch.empty((p.B, p.Hkv, ns, p.D), dtype=torch.float32, device=ksum.device)
    _check(lib().ssa_tree_summary(ctypes.byref(p), _ptr(ksum), _ptr(out), _stream()))
    return out


def route_tree(qsum: torch.Tensor, ksum: torch.Tensor, ksum2: torch.Tensor, p: Params):
    """Two-level routing: (sup_idx int32 [B, Hq, NQB, tree_beam], sup_cnt int32
    [B, Hq, NQB], idx int32 [B, Hq, NQB, top_k], cnt int32 [B, Hq, NQB])."""
    _need(qsum, torch.float32, (p.B, p.Hq, p.n_qblocks, p.D), "qsum")
    _need(ksum, torch.float32, (p.B, p.Hkv, p.n_kblocks, p.D), "ksum")
    _need(ksum2, torch.float32, (p.B, p.Hkv, p.n_kblocks // max(p.tree_fanout, 1), p.D), "ksum2")
    dev = qsum.device
    sup_idx = torch.empty((p.B, p.Hq, p.n_qblocks, p.tree_beam), dtype=torch.int32, device=dev)
    sup_cnt = torch.empty((p.B, p.Hq, p.n_qblocks), dtype=torch.int32, device=dev)
    idx = torch.empty((p.B, p.Hq, p.n_qblocks, p.top_k), dtype=torch.int32, device=dev)
    cnt = torch.empty((p.B, p.Hq, p.n_qblocks), dtype=torch.int32, device=dev)
    _check(lib().ssa_route_tree(ctypes.byref(p), _ptr(qsum), _ptr(ksum), _ptr(ksum2),
                                _ptr(sup_idx), _ptr(sup_cnt), _ptr(idx) if p.top_k else None,
                                _ptr(cnt), _stream()))
    return sup_idx, sup_cnt, idx, cnt


def route_consensus(idx: torch.Tensor, cnt: torch.Tensor, p: Params):
    """Per-group consensus lists from per-head lists:
    (idx_kv int32 [B, Hkv, NQB, top_k], cnt_kv int32 [B, Hkv, NQB])."""
    _need(idx, torch.int32, (p.B, p.Hq, p.n_qblocks, p.top_k), "idx")
    _need(cnt, torch.int32, (p.B, p.Hq, p.n_qblocks), "cnt")
    dev = cnt.device
    idx_kv = torch.empty((p.B, p.Hkv, p.n_qblocks, p.top_k), dtype=torch.int32, device=dev)
    cnt_kv = torch.empty((p.B, p.Hkv, p.n_qblocks), dtype=torch.int32, device=dev)
    _check(lib().ssa_route_consensus(ctypes.byref(p), _ptr(idx) if p.top_k else None, _ptr(cnt),
                                     _ptr(idx_kv) if p.top_k else None, _ptr(cnt_kv), _stream()))
    return idx_kv, cnt_kv


def route_features(x: torch.Tensor, block: int, p: Params, queries: bool) -> torch.Tensor:
    """Second-cumulant routing features, fp32 [B, H, N/block, D + D(D+1)/2]:
    [mean | vech(covariance)] of key blocks, or [mean | (beta/2) w . vech(second
    moment)] of query blocks."""
    H = x.shape[1]
    _need(x, torch.bfloat16, (p.B, H, p.N, p.D), "x")
    F = p.D + p.D * (p.D + 1) // 2
    out = torch.empty((p.B, H, p.N // block, F), dtype=torch.float32, device=x.device)
    _check(lib().ssa_route_features(ctypes.byref(p), _ptr(x), H, block, int(bool(queries)),
                                    _ptr(out), _stream()))
    return out


def route_cumulant(qfeat: torch.Tensor, kfeat: torch.Tensor, p: Params):
    """Routing on the second-cumulant score: (idx, cnt) as ``route``."""
    F = p.D + p.D * (p.D + 1) // 2
    _need(qfeat, torch.float32, (p.B, p.Hq, p.n_qblocks, F), "qfeat")
    _need(kfeat, torch.float32, (p.B, p.Hkv, p.n_kblocks, F), "kfeat")
    dev = qfeat.device
    scores = torch.empty((p.B, p.Hq, p.n_qblocks, p.n_kblocks), dtype=torch.float32, device=dev)
    idx = torch.empty((p.B, p.Hq, p.n_qblocks, p.top_k), dtype=torch.int32, device=dev)
    cnt = torch.empty((p.B, p.Hq, p.n_qblocks), dtype=torch.int32, device=dev)
    _check(lib().ssa_route_cumulant(ctypes.byref(p), _ptr(qfeat), _ptr(kfeat), _ptr(scores),
                                    _ptr(idx) if p.top_k else None, _ptr(cnt), _stream()))
    return idx, cnt


def attend(q, k, v, idx, cnt, p: Params, with_lse: bool = True):
    """(o bf16 [B, Hq, N, D], lse fp32 [B, Hq, N] or None).  idx/cnt span Hq
    heads, or Hkv groups with ``p.consensus``."""
    _need(q, torch.bfloat16, (p.B, p.Hq, p.N, p.D), "q")
    _need(k, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "k")
    _need(v, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "v")
    _need(idx, torch.int32, (p.B, p.list_heads, p.n_qblocks, p.top_k), "idx")
    _need(cnt, torch.int32, (p.B, p.list_heads, p.n_qblocks), "cnt")
    o = torch.empty_like(q)
    lse = torch.empty((p.B, p.Hq, p.N), dtype=torch.float32, device=q.device) if with_lse else None
    _check(lib().ssa_attend(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                            _ptr(idx) if p.top_k else None, _ptr(cnt), _ptr(o), _ptr(lse),
                            _stream()))
    return o, lse


def forward(q, k, v, p: Params, workspace: torch.Tensor | None = None, with_lse: bool = True,
            out: torch.Tensor | None = None, lse_out: torch.Tensor | None = None,
            idx_out: torch.Tensor | None = None, cnt_out: torch.Tensor | None = None):
    """Whole path in one library call.  Returns (o, lse, idx, cnt); idx/cnt are
    the lists attend used (per KV group with ``p.consensus``), in the caller's
    ``idx_out``/``cnt_out`` if given, else in fresh tensors."""
    _need(q, torch.bfloat16, (p.B, p.Hq, p.N, p.D), "q")
    _need(k, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "k")
    _need(v, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "v")
    dev = q.device
    ws = workspace_size(p)
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
    o = out if out is not None else torch.empty_like(q)
    lse = lse_out if lse_out is not None else (
        torch.empty((p.B, p.Hq, p.N), dtype=torch.float32, device=dev) if with_lse else None)
    idx = idx_out if idx_out is not None else torch.empty(
        (p.B, p.list_heads, p.n_qblocks, max(p.top_k, 0)), dtype=torch.int32, device=dev)
    cnt = cnt_out if cnt_out is not None else torch.empty(
        (p.B, p.list_heads, p.n_qblocks), dtype=torch.int32, device=dev)
    _need(idx, torch.int32, (p.B, p.list_heads, p.n_qblocks, max(p.top_k, 0)), "idx_out")
    _need(cnt, torch.int32, (p.B, p.list_heads, p.n_qblocks), "cnt_out")
    _check(lib().ssa_forward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                             _ptr(idx) if p.top_k else None, _ptr(cnt), _ptr(workspace),
                             workspace.numel(), _stream()))
    return o, lse, idx, cnt


def _forward_raw(p: Params, q: int, k: int, v: int, o: int, lse, idx, cnt, ws: torch.Tensor,
                 stream) -> None:
    """ssa_forward on raw device addresses (sub-problems of larger tensors)."""
    vp = ctypes.c_void_p
    _check(lib().ssa_forward(ctypes.byref(p), vp(q), vp(k), vp(v), vp(o), lse, idx, cnt,
                             vp(ws.data_ptr()), ws.numel(), vp(stream.cuda_stream)))


def forward_host(q_host, k_host, v_host, p: Params, o_host: torch.Tensor,
                 device: torch.device | str = "cuda", dev_bufs: dict | None = None):
    """End-to-end call from host memory: pinned bf16 Q, K, V in, O out.

    Every (batch, query head) is an independent problem given its KV head, so
    the call streams it: the K/V of a group and the Q of each head go to the
    device on one copy stream, each head's forward (one ``ssa_forward`` on the
    head's slice, B = Hq = Hkv = 1) runs on the compute stream as soon as its
    inputs have landed, and its O returns on a second copy stream while later
    heads are still arriving or computing.  With consensus routing the heads
    of a group depend on one another, so the unit is the (batch, KV head)
    group (Hq = g, Hkv = 1).  ``dev_bufs`` may hold
    preallocated device tensors and streams to reuse between calls.  The call
    returns once all work is queued; the caller's current stream waits for it.
    """
    d = dev_bufs if dev_bufs is not None else {}
    dev = torch.device(device)
    for name, src in (("q", q_host), ("k", k_host), ("v", v_host)):
        if name not in d:
            d[name] = torch.empty(src.shape, dtype=src.dtype, device=dev)
    if "o" not in d:
        d["o"] = torch.empty(q_host.shape, dtype=torch.bfloat16, device=dev)
    grp = p.Hq // p.Hkv
    unit = grp if p.consensus else 1          # query heads per sub-problem
    sub = make_params(1, unit, 1, p.N, p.D, p.block_k, p.block_q, p.top_k, p.window, p.causal,
                      p.scale, p.wait_timeout_us, p.consensus, p.beta, p.tree_fanout, p.tree_beam)
    if "ws" not in d:
        d["ws"] = torch.empty(workspace_size(sub), dtype=torch.uint8, device=dev)
    if "streams" not in d:
        d["streams"] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    s_in, s_out = d["streams"]
    compute = torch.cuda.current_stream(dev)
    s_in.wait_stream(compute)       # buffers may still be read by earlier work
    s_out.wait_stream(compute)
    q, k, v, o = d["q"], d["k"], d["v"], d["o"]
    row = p.N * p.D * 2             # bytes of one head
    for b in range(p.B):
        for g in range(p.Hkv):
            with torch.cuda.stream(s_in):
                k[b, g].copy_(k_host[b, g], non_blocking=True)
                v[b, g].copy_(v_host[b, g], non_blocking=True)
            for h in range(g * grp, (g + 1) * grp, unit):
                hs = slice(h, h + unit)
                with torch.cuda.stream(s_in):
                    q[b, hs].copy_(q_host[b, hs], non_blocking=True)
                    ready = torch.cuda.Event()
                    ready.record(s_in)
                compute.wait_event(ready)
                _forward_raw(sub, q.data_ptr() + (b * p.Hq + h) * row,
                             k.data_ptr() + (b * p.Hkv + g) * row,
                             v.data_ptr() + (b * p.Hkv + g) * row,
                             o.data_ptr() + (b * p.Hq + h) * row, None, None, None, d["ws"],
                             compute)
                done = torch.cuda.Event()
                done.record(compute)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    o_host[b, hs].copy_(o[b, hs], non_blocking=True)
    compute.wait_stream(s_out)
    compute.wait_stream(s_in)
    return o_host


def backward(q, k, v, o, lse, d_o, idx, cnt, p: Params, workspace: torch.Tensor | None = None,
             out=None):
    """Gradients of the read with the lists held fixed: (dq fp32 [B, Hq, N, D],
    dk fp32 [B, Hkv, N, D], dv fp32 [B, Hkv, N, D]).  ``o``/``lse``/``idx``/
    ``cnt`` are the forward's outputs; ``out`` may hold preallocated (dq, dk, dv)."""
    for t, name in ((q, "q"), (o, "o"), (d_o, "d_o")):
        _need(t, torch.bfloat16, (p.B, p.Hq, p.N, p.D), name)
    _need(k, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "k")
    _need(v, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "v")
    _need(lse, torch.float32, (p.B, p.Hq, p.N), "lse")
    _need(idx, torch.int32, (p.B, p.list_heads, p.n_qblocks, max(p.top_k, 0)), "idx")
    _need(cnt, torch.int32, (p.B, p.list_heads, p.n_qblocks), "cnt")
    dev = q.device
    ws = lib().ssa_backward_workspace_size(ctypes.byref(p))
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    if out is None:
        out = (torch.empty((p.B, p.Hq, p.N, p.D), dtype=torch.float32, device=dev),
               torch.empty((p.B, p.Hkv, p.N, p.D), dtype=torch.float32, device=dev),
               torch.empty((p.B, p.Hkv, p.N, p.D), dtype=torch.float32, device=dev))
    dq, dk, dv = out
    _check(lib().ssa_attend_backward(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                     _ptr(lse), _ptr(d_o), _ptr(idx) if p.top_k else None,
                                     _ptr(cnt), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                     workspace.numel(), _stream()))
    return dq, dk, dv


def decode_workspace_size(p: Params) -> int:
    return int(lib().ssa_decode_workspace_size(ctypes.byref(p)))


def decode(q, k_cache, v_cache, n_ctx: int, ksum_cache, p: Params,
           workspace: torch.Tensor | None = None, with_lse: bool = True, out=None):
    """One decode step.  q bf16 [B, Hq, D] (the queries at position n_ctx-1);
    k_cache / v_cache bf16 [B, Hkv, N, D] with N = p.N the capacity;
    ksum_cache fp32 [B, Hkv, N/Bk, D], updated in place (the block that
    becomes admissible at this step).  Returns (o, lse, idx, cnt)."""
    _need(q, torch.bfloat16, (p.B, p.Hq, p.D), "q")
    _need(k_cache, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "k_cache")
    _need(v_cache, torch.bfloat16, (p.B, p.Hkv, p.N, p.D), "v_cache")
    _need(ksum_cache, torch.float32, (p.B, p.Hkv, p.n_kblocks, p.D), "ksum_cache")
    dev = q.device
    ws = decode_workspace_size(p)
    if workspace is None or workspace.numel() < ws:
        workspace = torch.empty(max(ws, 1), dtype=torch.uint8, device=dev)
    o = out if out is not None else torch.empty((p.B, p.Hq, p.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((p.B, p.Hq), dtype=torch.float32, device=dev) if with_lse else None
    idx = torch.empty((p.B, p.Hq, max(p.top_k, 1)), dtype=torch.int32, device=dev)
    cnt = torch.empty((p.B, p.Hq), dtype=torch.int32, device=dev)
    _check(lib().ssa_decode(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache), int(n_ctx),
                            _ptr(ksum_cache), _ptr(o), _ptr(lse), _ptr(idx) if p.top_k else None,
                            _ptr(cnt), _ptr(workspace), workspace.numel(), _stream()))
    return o, lse, idx[..., :p.top_k], cnt


def check_error(stream=None):
    """Synchronise the stream and raise if a kernel recorded a device error."""
    s = _stream() if stream is None else stream
    _check(lib().ssa_check_error(s))


def probe_wait_timeout(timeout_us: int):
    _check(lib().ssa_probe_wait_timeout(int(timeout_us), _stream()))


def probe_ex2_rate(n_ctas: int, iters: int, sink: torch.Tensor):
    """Launch the exponential-rate probe (``ssa_probe_ex2_rate``) on the
    current stream; the caller times it.  ``sink``: a device float32 tensor."""
    _need(sink, torch.float32, (1,), "sink")
    _check(lib().ssa_probe_ex2_rate(int(n_ctas), int(iters), _ptr(sink), _stream()))
