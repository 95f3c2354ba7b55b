"""gated_deltanet_fwd_b200 -- the gated delta rule on B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA behind the C ABI of ``include/gdn.h``).
``gated_deltanet_fwd_b200.gdn`` is the thin ctypes binding with the same call names; importing
this package does not load the library, so ``gated_deltanet_fwd_b200.inputs`` works on any host.
"""
__all__ = ["gdn", "inputs"]
