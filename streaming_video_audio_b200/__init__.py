"""B200-native chunk-streaming joint video+audio self-attention.

The hot path is the C-ABI library ``libsr.so`` (include/sr.h), built for
sm_100a by ``streaming_video_audio_b200.build``; ``capi`` is its ctypes
binding (argument marshalling only) and ``window.StreamingWindow`` holds the
persistent per-layer window buffers and runs the streaming step.  There is no
CPU or library fallback: every step runs in the library's kernels.
"""
__all__ = ["capi", "window", "build"]
