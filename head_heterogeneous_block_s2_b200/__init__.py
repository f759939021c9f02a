"""HHST sparse attention (S2-Attention) for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libs2attn.so`` built from ``csrc/``;
``s2attn`` is its thin ctypes binding (argument marshalling only). ``synth``
makes the seeded synthetic inputs. Importing this package loads nothing; the
binding loads the library on first use and raises if it is missing.
"""

__all__ = ["s2attn", "synth"]
