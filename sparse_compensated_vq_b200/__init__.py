"""vqlin: a VQ + sparse-correction linear layer for NVIDIA B200 (sm_100a).

`sparse_compensated_vq_b200.vqlin` binds the C ABI of libvqlin.so (declared in
include/vqlin.h); importing it loads the compiled library and fails if it is
missing.  `sparse_compensated_vq_b200.synth` generates seeded inputs.
"""
__all__ = ["vqlin", "synth"]
