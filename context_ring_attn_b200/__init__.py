"""B200-native context-parallel ring attention: partial attention blocks,
LSE merge, load-balanced shard plans and split-KV decode behind a C ABI
(libcpattn.so, include/cp_attn.h).

Submodules:
  binding  -- ctypes wrappers with the C entry points' names
  ring     -- pass-KV / pass-Q schedules over virtual ranks on one GPU
  synth    -- seeded synthetic inputs (no attention arithmetic)
  build    -- nvcc build of libcpattn.so for sm_100a
"""
