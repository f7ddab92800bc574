"""FlashBlock cached block-diffusion attention for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library libflashblock.so (include/flashblock.h);
``flashblock`` is its ctypes binding, ``schedule`` runs a block of denoising
steps through it, ``synth`` draws the seeded synthetic workloads.
"""
