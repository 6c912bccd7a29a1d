"""SP-KV (Self-Pruned Key-Value attention) hot path for NVIDIA B200 (sm_100a).

The compute runs in ``libspkv.so`` (hand-written CUDA kernels behind a C ABI);
``spkv`` is the thin ctypes binding.  PyTorch provides device memory and streams.
"""
