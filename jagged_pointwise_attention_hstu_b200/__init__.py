"""Jagged HSTU layer forward for B200 (sm_100a).

The compute path is the C-ABI library ``libhstu.so`` built from ``csrc/``;
``jagged_pointwise_attention_hstu_b200.hstu`` is its thin ctypes binding.
``workloads`` draws the seeded synthetic inputs.
"""
