"""host_streamed_nf4_b200 -- B200-native streamed NF4 LoRA layers.

The compute path lives in the C-ABI library ``libhsnf4.so`` (CUDA for
sm_100a); ``host_streamed_nf4_b200.hsnf4`` is its thin ctypes binding.  The
binding is imported lazily so that the CPU-only parts (``synth``) load
without a GPU.
"""
__all__ = ["synth", "hsnf4"]
