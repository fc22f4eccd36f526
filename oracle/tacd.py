"""Float64 statement of the TACD training targets (oracle; test infrastructure).

Teacher-Anchored Consistency Distillation, forward only: the quantities one
training step of the action expert's LoRA is supervised with, for synthetic
weights.  No optimiser, no EMA update.  Sources: RealtimeWAM summary page
(paper.rainbus.top), 前置知识 "一致性蒸馏 (Consistency Distillation, CD)" and
"流匹配与速度场去噪"; 核心方法 (the interval-average velocity and the error
bound); 方法步骤详情 (the training pipeline: noising, frozen video expert once,
K = 10 teacher rollout to 0, student and EMA endpoints, L_CD + lambda L_TA
with lambda = 0.2); 论文图表 (rollout-interval ablation: t -> 0 is the
default).

What the pages fix:

* a_t = (1 - t) a_0^data + t eps;
* the frozen video expert runs once on the observation; its per-block K/V
  z(o, l) serve the teacher, the student and the EMA target alike (only the
  action expert carries LoRA);
* the teacher integrates from a_t over [t, 0] in K Euler steps to a_0^T, and
  u_T(a_t, t) = (a_t - a_0^T) / t is the interval-average velocity;
* the endpoint map is f(a_t, t) = a_t - t v(a_t, t), for student and EMA;
* CD compares the student endpoint at (a_t, t) with the EMA target's
  endpoint at the teacher's one-step result a~_s;
* both losses are stated on the velocity prediction, L = L_CD + lambda L_TA.

Readings taken where the pages are silent (each one function or argument):

* the teacher's K steps are uniform on [t, 0]: t_k = t k / K;
* s, the point CD's teacher step lands on, is the first point of that same
  grid, s = t (K - 1) / K, so a~_s is the rollout's first state;
* "defined on the velocity prediction": each loss is the squared distance
  between the student velocity and the velocity that would carry a_t to the
  loss's endpoint in one step, u = (a_t - endpoint) / t; for L_TA that
  endpoint is a_0^T, for L_CD it is the EMA endpoint f^-(a~_s, s);
* E||.||^2: the squared L2 norm over one sample's chunk [L_a, P_a], averaged
  over the batch;
* one t for the whole batch (the pages write a single a_t).

Pins (tests/test_oracle_tacd.py): constant velocity (u = b, both losses 0,
exactly on a dyadic grid); K = 1 reduces both targets to the teacher's own
velocity at (a_t, t), for any weights; student = teacher and K = 1 gives
L_TA = 0; L_TA equals the 1/t^2-weighted endpoint error ||f - a_0^T||^2 / t^2
(核心方法); the error bound E||e_total||^2 <= 2 L_TA + 2 E||delta||^2 against
a fine rollout; the teacher's Euler error falls as 1/K.
"""
from __future__ import annotations

import numpy as np

from .config import WamConfig
from .model import action_velocity, endpoint, euler_step, f64, noise_to, video_expert

LAMBDA_TA = 0.2   # 方法步骤详情: L = L_CD + lambda L_TA, lambda = 0.2
TEACHER_STEPS = 10  # 方法步骤详情 / 论文图表: K = 10


def without_lora(P: dict) -> dict:
    """The frozen teacher: the base weights, no low-rank factors."""
    return {k: v for k, v in P.items() if not (k.endswith(".la") or k.endswith(".lb"))}


def teacher_grid(t: float, K: int, t_end: float = 0.0) -> np.ndarray:
    """[t_K, ..., t_0] uniform on [t, t_end]: t_k = t_end + (t - t_end) k / K."""
    return t_end + (t - t_end) * np.arange(K, -1, -1, dtype=np.float64) / K


def teacher_rollout(cfg: WamConfig, P_teacher: dict, a_t: np.ndarray, t: float, kv, K: int = TEACHER_STEPS):
    """K Euler steps of the teacher from (a_t, t) to 0; returns every state,
    [a_t, a_{t_{K-1}}, ..., a_0^T]."""
    grid = teacher_grid(t, K)
    states = [f64(a_t)]
    for k in range(K):
        v = action_velocity(cfg, P_teacher, states[-1], grid[k], kv)
        states.append(euler_step(states[-1], v, grid[k], grid[k + 1]))
    return states


def interval_velocity(a_t: np.ndarray, a_end: np.ndarray, t: float) -> np.ndarray:
    """u = (a_t - a_end) / t: the constant velocity that carries a_t to a_end over [t, 0]."""
    return (f64(a_t) - f64(a_end)) / t


def chunk_mean_sq(x: np.ndarray) -> float:
    """E||x||^2: squared L2 norm over each sample's [L_a, P_a], batch mean."""
    x = f64(x)
    return float(np.mean(np.sum(x.reshape(x.shape[0], -1) ** 2, axis=1)))


def tacd_targets(cfg: WamConfig, P_teacher: dict, P_student: dict, P_ema: dict, inputs: dict, t: float,
                 K: int = TEACHER_STEPS, lam: float = LAMBDA_TA) -> dict:
    """One TACD target forward.

    inputs: "video", "cond" (the observation tokens), "action_clean"
    (a_0^data, [B, L_a, P_a]) and "noise" (eps, same shape).  The video expert
    is evaluated once, with the teacher's (frozen, shared) video weights.

    Returns a dict with a_t, the teacher rollout end a0_T, u_ta, the CD step
    point s and state a_s, the student velocity and endpoint, the EMA
    endpoint, u_cd and the losses l_ta, l_cd, loss = l_cd + lam l_ta.
    """
    if not (0.0 < t <= 1.0) or K < 1:
        raise ValueError("need 0 < t <= 1 and K >= 1")
    kv, _, _ = video_expert(cfg, P_teacher, inputs["video"], inputs.get("cond"), 0.0)
    a_t = noise_to(inputs["action_clean"], inputs["noise"], t)
    states = teacher_rollout(cfg, P_teacher, a_t, t, kv, K)
    a0_T = states[-1]
    u_ta = interval_velocity(a_t, a0_T, t)
    s = teacher_grid(t, K)[1]
    a_s = states[1]
    v_student = action_velocity(cfg, P_student, a_t, t, kv)
    f_student = endpoint(a_t, v_student, t)
    v_ema = action_velocity(cfg, P_ema, a_s, s, kv)
    f_ema = endpoint(a_s, v_ema, s)
    u_cd = interval_velocity(a_t, f_ema, t)
    l_ta = chunk_mean_sq(v_student - u_ta)
    l_cd = chunk_mean_sq(v_student - u_cd)
    return {
        "a_t": a_t, "a0_T": a0_T, "u_ta": u_ta, "s": s, "a_s": a_s,
        "v_student": v_student, "f_student": f_student, "f_ema": f_ema, "u_cd": u_cd,
        "l_ta": l_ta, "l_cd": l_cd, "loss": l_cd + lam * l_ta,
    }
