"""CPU oracle of the ZHA decode hot path (fp64, numpy) -- TEST INFRASTRUCTURE.

This package exists only to check the CUDA library. Nothing on the product path
imports it: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
``cpu_baseline`` leg and ``--impl reference`` arm may import or run it. It shares
no code with ``hierarchical_sparse_attention_zha_b200`` (no kernels, headers,
helpers, tables or constants); the only common input is the seeded synthetic
data from ``hierarchical_sparse_attention_zha_b200.workloads``, which holds none
of the method's arithmetic.
"""

from .zha_oracle import (  # noqa: F401
    bf16_bits_to_f64,
    logsumexp,
    sdpa,
    chunk_log_mass,
    summarise_chunk,
    tangent_planes,
    node_score,
    combine_log_masses,
    merge_children,
    OracleTree,
    build_tree,
    rope_angles,
    rope_rotate,
    node_position,
    summarise_chunk_rope,
    merge_children_rope,
    build_tree_rope,
    top_p_prefix,
    top_k_prefix,
    RoutePolicy,
    depth_scaled_p,
    select_level,
    TopP,
    route,
    RouteTrace,
    leaf_token_set,
    attend,
    captured_mass,
    level_target_mass,
    level_estimate,
    level_kl,
    plane_usage,
)
