"""DeepSeekMoE layer forward on NVIDIA B200 (sm_100a).

The work runs in ``libmoe.so`` (hand-written CUDA behind the C ABI of
``include/moe.h``, built in-tree by ``build.py``). This package holds the thin
Python side:

* ``_lib``: ctypes binding of every C entry point, under the same names.
* ``layer.MoELayer``: device weights, packed W13, workspace; ``forward`` runs
  ``moe_layer_forward`` on torch's current stream, ``forward_host`` runs
  ``moe_layer_forward_host`` on pinned host buffers.
* ``synthetic``: seeded counter-based inputs of the benchmark workloads (no
  layer arithmetic).

There is no CPU fallback: calls fail with ``MoeError`` when the library or a
B200 is missing.
"""
