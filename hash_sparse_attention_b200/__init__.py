"""HHR (Hierarchical Hash Retrieval) decode path for NVIDIA B200 (sm_100a).

The work is done by libhhr.so (C ABI in include/hhr.h); ``hhr`` holds the thin
ctypes binding and ``synth`` the seeded synthetic inputs.  Importing the
package does not load the library; the first call into ``hhr`` does, and
fails loudly if it has not been built.
"""

__all__ = ["hhr", "synth"]
