"""CPU oracle of the block-diffusion denoising pass: test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm
may import this package.  It shares no code with the CUDA path.  `dg_oracle` binds
the C++ oracle (`dg_oracle.cpp`); `dg_oracle_np` is its numpy cross-check.
"""
