"""On-Demand Attention (ODA) decode hot path for NVIDIA B200 (sm_100a).

    oda      - Python binding of the C ABI in include/oda.h (one function per entry point)
    engine   - OdaDecoder: device state of a synthetic workload and the step call sequence
    build    - in-tree nvcc build of lib/liboda.so

Every compute step runs in liboda.so; importing ``oda`` without the built library raises.
"""
__all__ = ["oda", "engine", "build"]
