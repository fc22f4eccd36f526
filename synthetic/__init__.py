"""Seeded synthetic inputs for the MoT world-action-model forward.

This module is the one piece of code that both the CPU oracle and the CUDA
library's callers (tests, bench) use: it draws the per-chunk inputs from a
seed and nothing else.  It holds none of the method's arithmetic -- no
noising, no time shift, no network.  Model parameters are NOT drawn here:
the CUDA library's ``wam_init`` and the oracle each generate them from the
seed with their own implementation of the counter-based generator.

Inputs of one chunk (shapes use the model's notation):

* ``video``  -- video tokens ``[B, L_vid, d_v]`` already embedded at the video
  width, N(0, 1); for the patch-input variant ``[B, L_vid, P_v]`` clean patch
  vectors x_0, N(0, 1).
* ``cond``   -- conditioning tokens ``[B, L_c, d_v]``, N(0, 1) (absent if L_c=0).
* ``noise``  -- the action chunk at t = 1, ``[B, L_a, P_a]``, N(0, 1).

For the joint one-step variant (patch input, consistency endpoints) the
chunk additionally carries

* ``video_eps`` ``[B, L_vid, P_v]`` and ``action_clean`` ``[B, L_a, P_a]``, N(0, 1),
* ``u_video``, ``u_action`` -- the unshifted noise levels, U(0, 1) scalars.

All arrays are float32, C-contiguous.  The generator is numpy's PCG64 seeded
with ``seed``; each array is drawn from its own child stream so adding an
array never changes the others.
"""
from __future__ import annotations

import numpy as np

__all__ = ["make_inputs", "child_rng"]

_STREAMS = {
    "video": 0,
    "cond": 1,
    "noise": 2,
    "video_eps": 3,
    "action_clean": 4,
    "u_video": 5,
    "u_action": 6,
}


def child_rng(seed: int, name: str) -> np.random.Generator:
    """Independent PCG64 stream for input ``name`` under ``seed``."""
    ss = np.random.SeedSequence([int(seed) & 0xFFFFFFFF, (int(seed) >> 32) & 0xFFFFFFFF, _STREAMS[name]])
    return np.random.Generator(np.random.PCG64(ss))


def _normal(seed: int, name: str, shape) -> np.ndarray:
    return child_rng(seed, name).standard_normal(size=shape, dtype=np.float64).astype(np.float32)


def make_inputs(seed: int, *, batch: int, l_cond: int, l_video: int, video_width: int,
                l_action: int, action_dim: int, patch_input: bool = False, action_clean: bool = False) -> dict:
    """Draw one chunk's inputs.

    ``video_width`` is d_v for embedded tokens or P_v when ``patch_input``.
    ``l_cond`` conditioning tokens have width ``video_width`` (only used when
    not ``patch_input``).  ``action_clean`` also draws a clean action chunk
    (always drawn with ``patch_input``); every array has its own stream, so
    asking for it changes none of the others.
    """
    out = {
        "video": _normal(seed, "video", (batch, l_video, video_width)),
        "noise": _normal(seed, "noise", (batch, l_action, action_dim)),
    }
    out["cond"] = (_normal(seed, "cond", (batch, l_cond, video_width))
                   if l_cond > 0 else np.zeros((batch, 0, video_width), np.float32))
    if patch_input or action_clean:
        out["action_clean"] = _normal(seed, "action_clean", (batch, l_action, action_dim))
    if patch_input:
        out["video_eps"] = _normal(seed, "video_eps", (batch, l_video, video_width))
        out["u_video"] = float(child_rng(seed, "u_video").uniform())
        out["u_action"] = float(child_rng(seed, "u_action").uniform())
    return out
