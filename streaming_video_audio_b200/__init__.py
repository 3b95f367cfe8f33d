"""B200-native chunk-streaming joint video+audio self-attention.

The hot path is the C-ABI library ``libsr.so`` (include/sr.h), built for
sm_100a by ``streaming_video_audio_b200.build``; ``capi`` is its ctypes
binding (argument marshalling only).  On top of it:

* ``window.StreamingWindow`` -- the persistent per-layer window buffers of a
  batch of sessions and the streaming step (KV append, RoPE, attention), the
  window slide after a chunk (tier re-pooling over frame rings), the prefix /
  moving-part split, CUDA-graph replay of the step;
* ``window.HostStepPipeline`` -- the step for callers holding host buffers,
  transfers overlapped with compute;
* ``ulysses.UlyssesAttention`` -- one session's chunk sharded over ranks with
  heads re-partitioned by all-to-all;
* ``vae_window.RingWindowAttention`` -- shifted-window attention with
  per-window KV rings (causal VAE decoder layer).

There is no CPU or library fallback: every step runs in the library's kernels.
"""
__all__ = ["capi", "window", "build", "ulysses", "vae_window"]
