"""B200 (sm_100a) implementation of SparSTAR's per-scale dynamic block-sparse attention.

`sparstar` is the Python binding of the C-ABI library libsparstar.so (selection and
block-sparse attention kernels); `synth` draws seeded synthetic inputs. Importing the
package does not load the library; the first binding call does, and fails loudly if the
library was not built.
"""
__all__ = ["sparstar", "synth"]
