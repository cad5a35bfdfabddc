"""ss24: online 2:4 prune + compress + quantize + error energies on B200 (sm_100a).

The compute path is a C-ABI CUDA library (``libss24.so``, declared in
``include/ss24.h``); ``semi_structured_sparsity_online_b200.ss24`` is its thin
ctypes binding. ``synth`` draws the seeded synthetic operands. Importing the
package loads nothing; the binding loads the library on first use and raises
if it is missing.
"""
__all__ = ["ss24", "synth"]
