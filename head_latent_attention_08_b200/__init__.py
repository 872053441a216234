"""Absorbed Multi-head Latent Attention decode for B200 (sm_100a).

The compute lives in the C-ABI library ``libmla_b200.so`` (hand-written CUDA). ``mla`` is its thin
Python binding; ``inputs`` draws the seeded synthetic workloads. Importing this package loads
nothing: the library is opened on first use of ``head_latent_attention_08_b200.mla`` and a missing
or unloadable library raises at that point.
"""

__all__ = ["mla", "inputs"]
