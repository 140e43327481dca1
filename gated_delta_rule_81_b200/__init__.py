"""B200-native gated-delta-rule token mixer.

The compute path is the C-ABI library ``libgdn.so`` (hand-written sm_100a CUDA);
``gated_delta_rule_81_b200.gdn`` is its thin ctypes binding.  Nothing is
imported eagerly, so the input generator can be used without a GPU.
"""

__all__ = ["gdn", "inputs"]
