"""B200-native (sm_100a) attention forward for the MiMo-V2 text decoder.

Submodules:

* ``mimo_attn`` -- Python binding of the C-ABI library (``libmimo_attn.so``);
  argument marshalling only, every step runs in the CUDA kernels.
* ``synth`` -- seeded synthetic input generator.
* ``workloads`` -- the named layer-shaped workloads.

Importing the package loads nothing; ``mimo_attn`` loads the shared library
on first use and raises if it is missing.
"""
__all__ = ["mimo_attn", "synth", "workloads"]
