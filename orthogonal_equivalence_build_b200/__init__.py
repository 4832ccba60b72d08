"""POET-X linear layer on B200: C-ABI library (lib/libpoetx.so) and its Python binding.

    from orthogonal_equivalence_build_b200 import poetx
"""
__all__ = ["poetx"]
