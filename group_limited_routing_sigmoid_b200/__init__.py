"""Beam sparse MoE block (group-limited sigmoid routing) on B200.

The compute lives in ``libbeam_moe.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/beam_moe.h``); ``binding`` marshals arguments
to it with ctypes.  ``workloads`` draws the seeded synthetic inputs.
"""
