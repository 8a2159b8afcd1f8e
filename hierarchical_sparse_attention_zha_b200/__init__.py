"""ZHA decode hot path for B200 (sm_100a): tree-summarised KV-cache attention.

``hierarchical_sparse_attention_zha_b200.zha`` is the binding of the C-ABI
library ``libzha.so`` (build it with ``__graft_entry__.build()`` or
``python -m hierarchical_sparse_attention_zha_b200.build``); importing it raises
if the library is missing. ``workloads`` draws the seeded synthetic inputs.
"""
