"""B200-native TwoTower denoiser refinement step: CUDA kernels for sm_100a behind a C ABI.

Importing the package does not load the CUDA library; the first call does, and fails loudly if
the library is missing (there is no CPU fallback). `synth` holds the seeded synthetic inputs.
"""
__all__ = ["binding", "api", "synth", "build"]
