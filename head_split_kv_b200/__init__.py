"""B200-native head-split (retrieval / streaming) attention.

The compute path lives in the C-ABI library ``libduo.so`` built from
``csrc/``; ``head_split_kv_b200.duo`` is the thin ctypes binding over it.
Importing the package itself loads nothing, so the seeded input generators in
``head_split_kv_b200.synthetic`` work on machines without the library.
"""

__all__ = ["duo", "synthetic"]
