"""janus-b200: element-type-routed sparse MoE layer and edge-to-atom
aggregation as hand-written sm_100a CUDA kernels behind a C ABI (libjanus.so).

``element_routed_moe_b200.janus`` is the thin ctypes binding over the library;
``element_routed_moe_b200.synth`` draws seeded synthetic layer inputs.
"""
