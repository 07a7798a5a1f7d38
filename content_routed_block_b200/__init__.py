"""Content-routed block-sparse exact attention on NVIDIA B200 (sm_100a).

Keys (and queries) are mean-pooled into blocks; each query block keeps its
top-k causally admissible key blocks (ties to the lower index), adds a local
causal window of W tokens, and attends with exact softmax over that union
only.  The work runs in three hand-written sm_100a kernels behind the C ABI
of ``libssa.so`` (declared in ``include/ssa.h``):

* ``ssa.block_summary`` -- vectorised mean pooling (K1)
* ``ssa.route``         -- fp32 block scores + warp top-k (K2)
* ``ssa.attend``        -- TMA block gather + tcgen05/TMEM attention (K3)
* ``ssa.forward``       -- the whole path in one call

``workloads`` draws the seeded synthetic inputs.  Import ``ssa`` for the
binding (it needs PyTorch and a built ``libssa.so``).
"""
__version__ = "0.1.0"
