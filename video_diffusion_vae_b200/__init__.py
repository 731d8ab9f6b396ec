"""B200-native Wan-style video-VAE decoder residual-block hot path.

The compute path is ``libwvae.so`` (hand-written CUDA for sm_100a behind the C
ABI in ``include/wvae.h``); :mod:`video_diffusion_vae_b200.binding` marshals
torch tensors into it.  Importing the package does not load the library; the
first binding call does, and fails loudly if it is missing.
"""
__all__ = ["binding", "synth"]
