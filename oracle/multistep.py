"""Float64 multi-step-video chunk (oracle; test infrastructure).

The wavefront extended to a video expert that keeps several denoising steps
(RealtimeWAM summary page, 未来方向 (2): carry the block-dependency analysis of
the cross-expert wavefront over to video experts with many denoising steps, as
in LingBot-VA, for a video-action wavefront).  What the path computes:

* the video expert generates the chunk's patch latents by N_v Euler steps of
  flow matching (前置知识 "流匹配与速度场去噪": x_{s_{j-1}} = x_{s_j} -
  (s_j - s_{j-1}) v^v(x_{s_j}, s_j)), each step one full forward of the video
  expert at its noise level;
* the action expert's block i attends over the K/V of video block i -- the
  ones of the LAST video forward, the step whose output is the chunk's video
  (MoT, 前置知识 "Mixture-of-Transformers" / "KV 缓存");
* the action chunk is then integrated by S Euler steps as in the one-pass
  chunk (oracle.model.infer_chunk).

Readings taken where the pages are silent (each one argument or function):

* the video latents start from pure noise at level 1: x_1 = eps_v (the
  patch-vector chunk of the video generator), the grid is given by the caller
  (uniform j / N_v by default), and the video output map is the plain
  flow-matching velocity, as for the action expert;
* the action's K/V are those of the video forward at the last grid point
  above 0 (s_1), the forward whose Euler step produces x_0.
"""
from __future__ import annotations

import numpy as np

from .config import WamConfig
from .model import action_velocity, euler_step, f64, uniform_schedule, video_expert


def video_rollout(cfg: WamConfig, P: dict, x1: np.ndarray, sched_v) -> tuple:
    """N_v Euler steps of the video expert from x1 over sched_v
    ([s_{N_v}, ..., s_0], decreasing).  Returns (x_0, kv_last, passes) where
    kv_last[i] = (K^v_i, V^v_i) of the last forward and passes is the list of
    every forward's (input state, level, kv)."""
    if not cfg.video_has_output or cfg.video_patch_dim <= 0:
        raise ValueError("a multi-step video expert needs patch input and a video output")
    sched_v = f64(sched_v)
    x = f64(x1)
    passes = []
    kv = None
    for j in range(len(sched_v) - 1):
        kv, _, v = video_expert(cfg, P, x, None, float(sched_v[j]), run_last_rest=True)
        passes.append((x, float(sched_v[j]), kv))
        x = euler_step(x, v, sched_v[j], sched_v[j + 1])
    return x, kv, passes


def multistep_chunk(cfg: WamConfig, P: dict, inputs: dict, n_video: int = None, sched_v=None, S: int = None,
                    sched_a=None) -> dict:
    """One chunk with a multi-step video expert.  inputs: "video_eps" (the
    video latents at level 1, [B, L_vid, P_v]) and "noise" (the action chunk
    at t = 1).  Returns x_0, a_0 and v_eff = a_{t_S} - a_0."""
    if sched_v is None:
        sched_v = uniform_schedule(n_video if n_video is not None else 1)
    if sched_a is None:
        sched_a = uniform_schedule(S if S is not None else 1)
    sched_a = f64(sched_a)
    x0, kv, _ = video_rollout(cfg, P, inputs["video_eps"], sched_v)
    a = f64(inputs["noise"])
    a_start = a
    for j in range(len(sched_a) - 1):
        a = euler_step(a, action_velocity(cfg, P, a, sched_a[j], kv), sched_a[j], sched_a[j + 1])
    return {"video": x0, "a0": a, "v_eff": a_start - a}
