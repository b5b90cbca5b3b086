"""libssd: the Mamba-2 SSD layer (chunked prefill + O(1) cached decode) for B200.

The compute path is the C-ABI shared library `libssd.so` built from `csrc/`; `ssd` is
its thin Python binding (argument marshalling only).  Importing the package does not
load the library; `selective_state_space_10_b200.ssd` does, and fails loudly if it is
missing.
"""
__all__ = ["inputs", "ssd"]
