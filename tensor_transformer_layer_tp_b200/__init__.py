"""B200-native tensor-parallel transformer layer and vocab-parallel cross-entropy.

The compute path is the C-ABI library libtplayer.so (include/tplayer.h), built
in-tree from csrc/ for sm_100a.  ``binding`` marshals torch tensors into it;
``runner`` allocates the buffers a call needs with torch (device memory only).
"""
from . import binding  # noqa: F401

__all__ = ["binding"]
