"""B200 (sm_100a) Infini-attention layer forward.

``compressive_memory_segment_b200.binding`` loads the CUDA library
(``libinfini_attn.so``) and exposes its C ABI under the same names;
``compressive_memory_segment_b200.synth`` holds the seeded synthetic inputs.
Importing this package itself loads nothing.
"""
__all__ = ["binding", "synth"]
