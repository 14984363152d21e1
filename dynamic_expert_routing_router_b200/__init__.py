"""BEAM-masked MoE layer forward pass on B200 (sm_100a).

The CUDA library ``libbeam_moe.so`` (built from ``csrc/``) holds every step of
the layer.  ``dynamic_expert_routing_router_b200.abi`` is a thin ctypes binding
of its C entry points (argument marshalling only);
``dynamic_expert_routing_router_b200.inputs`` draws the seeded synthetic
workloads.  Import the submodule you need; importing the package itself loads
nothing.
"""
