"""TokenGate pruned-prefill hot path for NVIDIA B200 (sm_100a).

The kernels live in libtokengate.so (C ABI: include/tg.h), built in-tree by
learned_token_pruning_b200.build; `tokengate` is its thin ctypes binding and
`pipeline` strings the entry points into one gated prefill step.  `synth`
draws the seeded synthetic inputs.
"""
__all__ = ["build", "pipeline", "synth", "tokengate"]
