"""pkv: paged KV-cache decode kernels for B200 (sm_100a).

The compute path is the C-ABI library libpkv.so (hand-written CUDA). The
Python binding in `binding` only marshals arguments to it; importing this
package does not load the library, calling a kernel does (and fails loudly if
the library is missing).
"""
