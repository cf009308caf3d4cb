"""SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).

The C ABI (include/svdq.h) is implemented by the CUDA library libsvdq.so in
this directory; ``w4a4_diffusion_model_b200.svdq`` is its Python binding and
``w4a4_diffusion_model_b200.synth`` draws the seeded synthetic workloads.
Importing the package does not load the library; the first call does.
"""
__all__ = ["svdq", "synth", "build"]
