"""liblisa: the LISA attention-module forward pass as hand-written CUDA for B200 (sm_100a).

``lisa`` is the ctypes binding of the C ABI declared in ``include/lisa.h``;
``inputs`` draws the seeded synthetic workloads.
"""
__all__ = ["lisa", "inputs"]
