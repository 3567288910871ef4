"""BinaryAttention forward pass for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libbinattn.so`` built from ``csrc/``; this
package only marshals arguments to it.
"""
