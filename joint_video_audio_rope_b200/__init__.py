"""B200-native (sm_100a) attention hot path of a dual-stream MMDiT joint
video/audio diffusion transformer: 3D RoPE with negative conditioning time
and 21/218 audio scaling, joint self-attention, bidirectional audio<->video
cross-attention, and a block-sparse mode (mean-pooled block scores, hybrid
top-k/top-p selection, attention over the selected blocks).

The compute lives in libmmdit.so (C ABI: include/mmdit.h); ``mmdit`` is its
ctypes binding and ``workloads`` the seeded synthetic inputs.
"""
__all__ = ["mmdit", "workloads", "build"]
