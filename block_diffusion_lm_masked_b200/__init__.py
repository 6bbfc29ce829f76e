"""B200-native block-diffusion denoising pass.

The product is the C-ABI library libdg.so (built from csrc/ for sm_100a); the
binding in `dg.py` marshals arguments to it.  Importing this package loads
nothing; `block_diffusion_lm_masked_b200.dg` loads the library and fails loudly
if it is missing.
"""
