"""B200-native residual block-diffusion decoding: one denoising round over a block of
masked positions, repeated on the device until the block commits.

The compute lives in the CUDA library ``libdlm.so`` (C ABI, see include/dlm.h); this
package only marshals arguments to it (``dlm``) and draws seeded inputs (``gen``).
"""
