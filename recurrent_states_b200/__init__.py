"""Taylor-series causal attention with n additive recurrent states on B200.

The compute path is the C-ABI library ``libtaylor_attn.so`` built from
``csrc/`` (hand-written CUDA for sm_100a).  ``taylor_attn`` is its thin
ctypes binding; ``synth`` holds the seeded input recipes.  Importing this
package does not load the library; the first call through the binding does,
and fails loudly if it has not been built."""
