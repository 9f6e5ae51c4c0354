"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

Test and benchmark infrastructure only: this package holds no arithmetic of the
MoE layer. See ``synth.h`` for the per-element generator definition.
"""
