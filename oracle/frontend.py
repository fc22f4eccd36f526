"""Pixel front-end of the patch-input model (oracle; test infrastructure).

The Flash-WAM setting (Flash-WAM close reading, 数据与训练流程 / 方法) feeds the
video stream with 128 x 128 RGB frames cut into 16 x 16 patches, each a
3 * 8 * 8 = 192-vector; a chunk of K = 4 frames is 1024 patch tokens.  The
pages give no VAE architecture or weights, so the front-end stated here is
the exact patchify and its inverse.

Reading taken: frames are channel-first [B, F, C, H, W]; token t of a
sample is (frame f, patch row py, patch column px) with t = f (H/p)(W/p) +
py (W/p) + px (frame-major, then raster order), and feature c p^2 + iy p + ix
holds pixel (c, py p + iy, px p + ix).
"""
from __future__ import annotations

import numpy as np


def patchify(frames: np.ndarray, p: int) -> np.ndarray:
    """[B, F, C, H, W] -> [B, F (H/p) (W/p), C p p]."""
    B, F, C, H, W = frames.shape
    if H % p or W % p:
        raise ValueError("frame size must be a multiple of the patch size")
    x = frames.reshape(B, F, C, H // p, p, W // p, p)
    x = x.transpose(0, 1, 3, 5, 2, 4, 6)
    return np.ascontiguousarray(x.reshape(B, F * (H // p) * (W // p), C * p * p))


def unpatchify(patches: np.ndarray, F: int, C: int, H: int, W: int, p: int) -> np.ndarray:
    """Inverse of patchify: [B, F (H/p) (W/p), C p p] -> [B, F, C, H, W]."""
    B = patches.shape[0]
    x = patches.reshape(B, F, H // p, W // p, C, p, p)
    x = x.transpose(0, 1, 4, 2, 5, 3, 6)
    return np.ascontiguousarray(x.reshape(B, F, C, H, W))
