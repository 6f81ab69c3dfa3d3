"""B200-native (sm_100a) fused causal self-attention at GPT-2 shapes.

The compute lives in libgpt2attn.so (C ABI in include/gpt2attn.h), and
``causal_self_attention_flashattention_b200.ops`` is its Python binding. This
package init imports nothing heavy, so the seeded-input module ``workload``
and the build script stay usable on a machine without the built library.
"""

__all__ = ["ops", "workload", "build"]
