"""B200-native REANN energy+force hot path.

The compute path lives in the CUDA library ``libreann.so`` (built from
``csrc/``) and is reached through the thin ctypes binding in
:mod:`molecular_dynamics_b200.reann`.  Importing this package does not load
the library; :func:`molecular_dynamics_b200.reann.load` does, and fails
loudly when it is missing.
"""
__all__ = ["presets", "synth"]
