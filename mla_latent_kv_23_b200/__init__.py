"""B200-native absorbed Multi-head Latent Attention (MLA) decode.

The compute path lives in ``libmla.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/mla.h``); ``mla_latent_kv_23_b200.mla`` is its
thin ctypes binding.  ``synth`` draws seeded synthetic inputs.  Importing the
package loads nothing; the binding loads the library on first use and raises
if it is missing.
"""
__all__ = ["synth"]
