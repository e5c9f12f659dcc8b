"""Prism dynamic block-sparse video self-attention for NVIDIA B200 (sm_100a).

The path (plan -> select -> sparse attention forward/backward) runs in
libprism.so, a C-ABI library of hand-written CUDA kernels; ``api`` is a thin
torch wrapper around it and ``synth`` draws seeded synthetic inputs.
"""
__all__ = ["api", "synth", "build"]
