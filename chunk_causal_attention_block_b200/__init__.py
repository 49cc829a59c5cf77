"""Chunk-causal attention of one Wave Forcing wave round on B200 (sm_100a).

The product is the C-ABI library ``libwf.so`` (``include/wf.h``); ``wf`` is
its ctypes binding, ``rollout`` drives a streaming rollout through it, and
``synth`` draws the seeded synthetic inputs.  Importing the package loads
nothing; ``wf.lib()`` loads the library and fails loudly if it is missing.
"""
__all__ = ["wf", "rollout", "synth", "build"]
