"""ltxattn: B200 (sm_100a) attention for the LTX-2 joint audio-video DiT block.

The compute lives in ``libltxattn.so`` (hand-written CUDA behind a C ABI, see
``include/ltxattn.h``); :mod:`joint_audio_video_flash_b200.ltxattn` is the thin
ctypes binding.  Importing this package loads nothing; the binding loads the
library on first use and raises if it is missing.
"""
__all__ = ["ltxattn", "synth", "workloads"]
