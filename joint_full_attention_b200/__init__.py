"""Joint full self-attention with 3D RoPE (HunyuanVideo-style DiT) for B200.

The product is the C-ABI library ``libhvattn.so`` (``include/hv_attn.h``);
``hvattn`` is its thin Python binding and ``workloads`` the seeded input
generator used by the tests and the benchmark.
"""

__all__ = ["hvattn", "workloads", "build"]
