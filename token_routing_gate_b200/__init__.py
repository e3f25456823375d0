"""B200-native MoE gating and routing: gate/top-k -> token-to-expert map -> expand -> reduce.

The work runs in hand-written CUDA kernels (sm_100a) inside ``libtk_route.so``, reached through
its C ABI (``include/tk_route.h``). ``token_routing_gate_b200.tk`` is the thin Python binding:
it passes torch tensors' device pointers and the current stream, nothing more.
"""
from . import workloads  # noqa: F401
