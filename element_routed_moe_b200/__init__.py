"""janus-b200: element-type-routed sparse MoE layer and edge-to-atom
aggregation as hand-written sm_100a CUDA kernels behind a C ABI (libjanus.so).

``element_routed_moe_b200.janus``  the thin ctypes binding, one function per
                                   C entry point;
``element_routed_moe_b200.layer``  MoELayer: one layer pass (forward + input
                                   VJP) with preallocated buffers, and a
                                   pinned-host pipeline with overlapped copies;
``element_routed_moe_b200.ep``     ExpertParallelLayer: the same pass with the
                                   experts split over the ranks of a node;
``element_routed_moe_b200.synth``  seeded synthetic layer inputs.
"""
