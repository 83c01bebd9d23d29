"""Gated delta rule (the Gated DeltaNet sequence mixer) on NVIDIA B200.

The product is ``libgdn.so`` (C ABI in ``include/gdn.h``) with hand-written
sm_100a kernels; ``linear_attention_sequence_sm_b200.gdn`` is its Python
binding.  Import the binding explicitly (``from linear_attention_sequence_sm_b200
import gdn``); this package init loads nothing, so the seeded input generator
(``inputs``) can be used without the library.
"""

__all__ = ["gdn", "inputs", "build"]


def __getattr__(name):
    if name in ("chunk_forward", "decode_step", "workspace_size", "read_device_status", "launch_count"):
        from . import gdn
        return getattr(gdn, name)
    raise AttributeError(name)
