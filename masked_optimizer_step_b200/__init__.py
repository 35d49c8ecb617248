"""B200-native sparse training step of Sparse-First fine-tuning (masked optimizer step).

The hot path -- row masks, masked weight gradient, embedding-row gradient and the fused sparse
update -- runs as hand-written CUDA kernels for sm_100a behind a C ABI (include/sf.h). The
Python module `binding` marshals torch tensors into that ABI; `synth` draws seeded inputs.
"""
