"""Split-KV paged attention for single-token decode and speculative
verification over a fragment-addressed K/V cache, for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``liblse_attn.so`` (CUDA kernels for
sm_100a) behind the thin ctypes binding in :mod:`.binding`.  Importing the
package does not load the library; ``from verify_attention_paged_b200 import
binding`` does, and fails loudly when the library is missing.
"""

__all__ = ["binding", "workloads"]
