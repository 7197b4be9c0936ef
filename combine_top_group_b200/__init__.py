"""B200-native MoE expert-parallel dispatch / combine with group-limited top-k.

The C-ABI library (libep.so, built from csrc/) does all of the path's work.
`combine_top_group_b200.ep` is its thin ctypes binding. Importing this
package does not load the library. Importing `.ep` does, and fails loudly
if the library is missing.
"""
__all__ = ["workloads"]
