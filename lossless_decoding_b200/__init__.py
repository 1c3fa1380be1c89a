"""B200 (sm_100a) hot path of one Psi-Spec decode step of a diffusion-augmented LLM.

The kernels live in libuno.so (C ABI in include/uno.h); ``api`` is its PyTorch
binding. Importing ``lossless_decoding_b200.api`` loads the library and fails
loudly when it has not been built. ``inputs`` (seeded synthetic inputs) needs
no GPU and no library.
"""

__all__ = ["api", "inputs", "build"]
