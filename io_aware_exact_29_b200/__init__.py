"""B200-native exact attention (sm_100a): forward and KV-cache decode kernels.

The compute path is the C-ABI library ``libattn.so`` built from ``csrc/``;
``attn`` binds it with ctypes (argument marshalling only).
"""
