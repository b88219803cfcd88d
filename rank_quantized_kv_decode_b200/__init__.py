"""B200-native low-rank, quantised KV-cache decode (STAR-KV-style latent cache).

The compute path is the CUDA library ``libstarkv.so`` (sm_100a) behind a C ABI; this
package is its thin Python binding.  Submodules load lazily so that ``synth`` (seeded
inputs) can be imported without a GPU or a built library.
"""
__all__ = ["synth"]
