"""B200-native greedy-verified speculative MoE decode step (FastMTP draft + MoE verifier).

The compute path is the CUDA library ``libocrdec.so`` (C ABI in ``include/ocrdec.h``),
reached through :mod:`speculative_moe_decoding_b200.ocrdec`.  Importing the package
itself loads nothing native, so the seeded input generator (:mod:`.synth`) and the
metric helpers (:mod:`.metrics`) work on machines without a GPU.
"""
