"""B200-native (sm_100a) VC-Attention-style FP8 attention for video DiTs.

The compute path lives in the C-ABI library ``libvca.so`` (hand-written CUDA for
sm_100a, declared in ``include/vca.h``); ``bit_attention_video_02_b200.vca`` is
its thin ctypes binding.  ``workloads`` holds the seeded synthetic inputs.
"""
