"""Float64 forward of the MoT world-action model (oracle; test infrastructure).

Everything here is the plain definition, evaluated in float64 from the exact
parameter values (``oracle.params``): numpy matmul is the only library
primitive used.  No blocking, fusion or reordering beyond what the method
states.

What the method computes (RealtimeWAM summary page, 前置知识 "Mixture-of-
Transformers" and "KV 缓存"; 核心方法; 方法步骤详情):

* two Transformer experts of N DiT blocks each; block i of the action expert
  attends over the concatenation of the video expert's block-i keys/values
  and its own, [K^v_i; K^a_i] and [V^v_i; V^a_i]; video queries see video
  keys only, so the video expert runs once per chunk and publishes
  z = {(K^v_i, V^v_i)}_{i=1..N};
* each block splits into projection P_i (norm + QKV), attention Attn_i and
  the remainder R_i (out-projection + FFN);
* the action chunk is integrated by Euler flow matching,
  a_{t_{j-1}} = a_{t_j} - (t_j - t_{j-1}) v(a_{t_j}, t_j), and the endpoint
  map is f(a_t, t) = a_t - t v(a_t, t) (前置知识, "流匹配与速度场去噪").

Readings taken where the pages are silent (each a single function below):

* block layout: pre-norm DiT block with AdaLN modulation,
  h = rms(x)(1+sc1)+sh1; x += g1 * Attn-out; h2 = rms(x)(1+sc2)+sh2;
  x += g2 * FFN(h2); RMSNorm eps 1e-6, no gain inside the modulated norms;
* the fused "RMSNorm/RoPE" operator (方法步骤详情) is read as per-head
  QK-RMSNorm (unit-initialised gain) followed by rotate-half RoPE;
* timestep embedding: 256 sinusoidal features of 1000 t, two-layer SiLU MLP
  to c, one SiLU + linear map to 6d shared modulation, plus a per-block
  table T_i;
* GELU is the tanh form; attention is non-causal with scale 1/sqrt(Dh);
* positions: video-expert tokens 0..L_v-1 ([cond; video] order), action
  tokens L_v..L_v+L_a-1;
* the video expert runs at t_v = 0 (clean observation) unless the joint
  one-step variant gives it a noise level;
* the default Euler grid is uniform, t_j = j/S.
"""
from __future__ import annotations

import numpy as np

from .config import WamConfig

EPS = 1e-6
ROPE_BASE = 10000.0
TIME_FREQ_BASE = 10000.0
TIME_SCALE = 1000.0
TIME_FEATURES = 256


def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# elementwise pieces
# --------------------------------------------------------------------------

def rms_norm(x: np.ndarray, eps: float = EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) over the last axis (no gain)."""
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


def timestep_features(t: float) -> np.ndarray:
    """tau(t) = [cos(1000 t w_k), sin(1000 t w_k)], w_k = 10000^(-k/128), k < 128."""
    half = TIME_FEATURES // 2
    k = np.arange(half, dtype=np.float64)
    w = TIME_FREQ_BASE ** (-k / half)
    arg = TIME_SCALE * float(t) * w
    return np.concatenate([np.cos(arg), np.sin(arg)])


def rope(x: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """Rotate-half rotary embedding over the last axis.

    Channel j < Dh/2 is paired with j + Dh/2 and turned by the angle
    pos * 10000^(-2j/Dh).  ``x``: [..., L, Dh]; ``pos``: [L].
    """
    dh = x.shape[-1]
    half = dh // 2
    j = np.arange(half, dtype=np.float64)
    theta = f64(pos)[:, None] * ROPE_BASE ** (-2.0 * j / dh)[None, :]
    c, s = np.cos(theta), np.sin(theta)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def linear(x: np.ndarray, P: dict, name: str, lora_scale: float = 1.0) -> np.ndarray:
    """y = x W^T + b, plus the unmerged low-rank term s (x A^T) B^T when the
    parameter set carries LoRA factors ``name.la`` [r, in] / ``name.lb`` [out, r]."""
    y = x @ f64(P[name + ".w"]).T + f64(P[name + ".b"])
    if name + ".la" in P:
        y = y + lora_scale * ((x @ f64(P[name + ".la"]).T) @ f64(P[name + ".lb"]).T)
    return y


def split_heads(x: np.ndarray, n_heads: int) -> np.ndarray:
    """[B, L, H*Dh] -> [B, H, L, Dh]."""
    b, l, a = x.shape
    return x.reshape(b, l, n_heads, a // n_heads).transpose(0, 2, 1, 3)


def merge_heads(x: np.ndarray) -> np.ndarray:
    """[B, H, L, Dh] -> [B, L, H*Dh]."""
    b, h, l, d = x.shape
    return x.transpose(0, 2, 1, 3).reshape(b, l, h * d)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, head_group: int = 8) -> np.ndarray:
    """softmax(q k^T / sqrt(Dh)) v per (sample, head); the row maximum is
    subtracted before exponentiation.  q: [B,H,Lq,Dh], k/v: [B,H,Lk,Dh]."""
    scale = 1.0 / np.sqrt(q.shape[-1])
    out = np.empty(q.shape[:-1] + (v.shape[-1],), np.float64)
    for b in range(q.shape[0]):
        for h0 in range(0, q.shape[1], head_group):
            hs = slice(h0, h0 + head_group)
            s = (q[b, hs] @ k[b, hs].transpose(0, 2, 1)) * scale
            s = np.exp(s - s.max(axis=-1, keepdims=True))
            out[b, hs] = (s / s.sum(axis=-1, keepdims=True)) @ v[b, hs]
    return out


# --------------------------------------------------------------------------
# expert pieces
# --------------------------------------------------------------------------

def modulation(cfg: WamConfig, P: dict, expert: str, t: float) -> np.ndarray:
    """Shared AdaLN vector m(t) in R^{6d}:
    c = W_t2 SiLU(W_t1 tau(t) + b_t1) + b_t2;  m = W_m SiLU(c) + b_m."""
    p = expert + "."
    tau = timestep_features(t)
    c = linear(silu(linear(tau, P, p + "t1")), P, p + "t2")
    return linear(silu(c), P, p + "mod")


def block_modulation(m: np.ndarray, T_i: np.ndarray):
    """(sh1, sc1, g1, sh2, sc2, g2) = split6(m) + T_i (T_i is [6, d])."""
    mm = m.reshape(6, -1) + f64(T_i)
    return tuple(mm[r] for r in range(6))


def modulate(x: np.ndarray, shift: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """rms(x) (1 + scale) + shift."""
    return rms_norm(x) * (1.0 + scale) + shift


def project_qkv(cfg: WamConfig, P: dict, b: str, h: np.ndarray, pos: np.ndarray,
                lora_scale: float):
    """P_i: merged QKV projection, per-head QK-RMSNorm with gains, RoPE on q and k.
    Returns q, k, v as [B, H, L, Dh] (k after norm and RoPE, v raw)."""
    A = cfg.attn_dim
    H = cfg.n_heads
    qkv = linear(h, P, b + "qkv", lora_scale)
    q = split_heads(qkv[..., :A], H)
    k = split_heads(qkv[..., A:2 * A], H)
    v = split_heads(qkv[..., 2 * A:], H)
    gq = f64(P[b + "qn.g"]).reshape(H, 1, -1)
    gk = f64(P[b + "kn.g"]).reshape(H, 1, -1)
    q = rope(rms_norm(q) * gq, pos)
    k = rope(rms_norm(k) * gk, pos)
    return q, k, v


def block_rest(cfg: WamConfig, P: dict, b: str, x: np.ndarray, o: np.ndarray,
               mods, lora_scale: float) -> np.ndarray:
    """R_i: x += g1 (o W_o^T + b_o); x += g2 FFN(rms(x)(1+sc2)+sh2)."""
    _, _, g1, sh2, sc2, g2 = mods
    x = x + g1 * linear(merge_heads(o), P, b + "o", lora_scale)
    h2 = modulate(x, sh2, sc2)
    f = linear(gelu_tanh(linear(h2, P, b + "ffn1", lora_scale)), P, b + "ffn2", lora_scale)
    return x + g2 * f


def video_expert(cfg: WamConfig, P: dict, video: np.ndarray, cond, t_v: float,
                 run_last_rest=None):
    """Video expert, run once per chunk.

    Returns (kv, x, out): kv[i] = (K^v_i, V^v_i) as [B, H, L_v, Dh]; x the final
    residual stream; out the video velocity v^v (joint variant) or None.

    The last block's attention and remainder only matter for the video output;
    with ``run_last_rest`` False they are skipped (the action expert never
    reads them) -- by default they run exactly when the model has a video output.
    """
    if run_last_rest is None:
        run_last_rest = cfg.video_has_output
    if cfg.video_patch_dim > 0:
        x = linear(f64(video), P, "video.in")
    else:
        parts = [f64(cond)] if cfg.l_cond > 0 else []
        x = np.concatenate(parts + [f64(video)], axis=1)
    pos = np.arange(x.shape[1], dtype=np.float64)
    m = modulation(cfg, P, "video", t_v)
    kv = []
    for i in range(cfg.n_blocks):
        b = f"video.blk{i}."
        mods = block_modulation(m, P[b + "T"])
        h = modulate(x, mods[0], mods[1])
        q, k, v = project_qkv(cfg, P, b, h, pos, 1.0)
        kv.append((k, v))
        if i == cfg.n_blocks - 1 and not run_last_rest:
            break
        o = attention(q, k, v)
        x = block_rest(cfg, P, b, x, o, mods, 1.0)
    out = None
    if run_last_rest and cfg.video_has_output:
        out = linear(rms_norm(x) * f64(P["video.fn.g"]), P, "video.out")
    return kv, x, out


def action_velocity(cfg: WamConfig, P: dict, a: np.ndarray, t: float, kv, hook=None) -> np.ndarray:
    """v_theta(a_t, t): the action expert over the joint keys/values.

    Block i's action queries attend over [K^v_i; K^a_i], [V^v_i; V^a_i].
    ``hook(i, kv)`` (optional) is called right after block i's attention has
    consumed kv[i]; it may replace later entries of kv (invariant tests).
    """
    x = linear(f64(a), P, "action.in")
    l_v = kv[0][0].shape[2]
    pos = l_v + np.arange(x.shape[1], dtype=np.float64)
    m = modulation(cfg, P, "action", t)
    s = cfg.lora_scale
    for i in range(cfg.n_blocks):
        b = f"action.blk{i}."
        mods = block_modulation(m, P[b + "T"])
        h = modulate(x, mods[0], mods[1])
        q, k, v = project_qkv(cfg, P, b, h, pos, s)
        kj = np.concatenate([kv[i][0], k], axis=2)
        vj = np.concatenate([kv[i][1], v], axis=2)
        o = attention(q, kj, vj)
        if hook is not None:
            hook(i, kv)
        x = block_rest(cfg, P, b, x, o, mods, s)
    return linear(rms_norm(x) * f64(P["action.fn.g"]), P, "action.out")


# --------------------------------------------------------------------------
# samplers
# --------------------------------------------------------------------------

def uniform_schedule(S: int) -> np.ndarray:
    """[t_S, ..., t_0] with t_j = j/S (t_S = 1, t_0 = 0)."""
    return np.arange(S, -1, -1, dtype=np.float64) / S


def euler_step(a: np.ndarray, v: np.ndarray, t_from: float, t_to: float) -> np.ndarray:
    """a_{t_{j-1}} = a_{t_j} - (t_j - t_{j-1}) v."""
    return a - (t_from - t_to) * v


def endpoint(a: np.ndarray, v: np.ndarray, t: float) -> np.ndarray:
    """f(a_t, t) = a_t - t v."""
    return a - t * v


def infer_chunk(cfg: WamConfig, P: dict, inputs: dict, S=None, t_sched=None, t_video: float = 0.0):
    """One chunk: video expert once, then S Euler steps of the action expert.

    Returns (a_0, v_eff) where v_eff = a_{t_S} - a_0 is the total displacement.
    """
    if t_sched is None:
        t_sched = uniform_schedule(S if S is not None else cfg.default_steps)
    t_sched = f64(t_sched)
    kv, _, _ = video_expert(cfg, P, inputs["video"], inputs.get("cond"), t_video)
    a = f64(inputs["noise"])
    a_start = a
    for j in range(len(t_sched) - 1):
        v = action_velocity(cfg, P, a, t_sched[j], kv)
        a = euler_step(a, v, t_sched[j], t_sched[j + 1])
    return a, a_start - a


# --------------------------------------------------------------------------
# joint one-step variant: SNR shift, noising, consistency endpoints
# (Flash-WAM close reading: 概念 "SNR shift", 方法 "动作流"/"视频流",
#  数据与训练流程 hyper-parameters s_v = 5, s_a = 1, sigma_d = 0.5)
# --------------------------------------------------------------------------

def snr_shift(u: float, s: float) -> float:
    """sigma = s u / (1 + (s - 1) u)."""
    return s * u / (1.0 + (s - 1.0) * u)


def noise_to(x0: np.ndarray, eps: np.ndarray, sigma: float) -> np.ndarray:
    """x_sigma = (1 - sigma) x_0 + sigma eps (the flow-matching interpolation)."""
    return (1.0 - sigma) * f64(x0) + sigma * f64(eps)


def lcm_coefficients(sigma: float, sigma_d: float = 0.5):
    """c_skip = sd^2 / (s^2 + sd^2), c_out = s sd / sqrt(s^2 + sd^2)."""
    c_skip = sigma_d ** 2 / (sigma ** 2 + sigma_d ** 2)
    c_out = sigma * sigma_d / np.sqrt(sigma ** 2 + sigma_d ** 2)
    return c_skip, c_out


def video_endpoint(x_sigma: np.ndarray, v: np.ndarray, sigma: float, sigma_d: float = 0.5) -> np.ndarray:
    """f^v = c_skip x_sigma + c_out (x_sigma - sigma v)."""
    c_skip, c_out = lcm_coefficients(sigma, sigma_d)
    return c_skip * x_sigma + c_out * (x_sigma - sigma * v)


def joint_one_step(cfg: WamConfig, P: dict, inputs: dict, s_video: float = 5.0,
                   s_action: float = 1.0, sigma_d: float = 0.5):
    """One video denoise step and one action step (1v/1a).

    Returns dict(f_action, f_video, sigma_video, sigma_action)."""
    sv = snr_shift(inputs["u_video"], s_video)
    sa = snr_shift(inputs["u_action"], s_action)
    x_sigma = noise_to(inputs["video"], inputs["video_eps"], sv)
    a_sigma = noise_to(inputs["action_clean"], inputs["noise"], sa)
    kv, _, v_vid = video_expert(cfg, P, x_sigma, None, sv)
    v_act = action_velocity(cfg, P, a_sigma, sa, kv)
    return {
        "f_action": endpoint(a_sigma, v_act, sa),
        "f_video": video_endpoint(x_sigma, v_vid, sv, sigma_d),
        "sigma_video": sv,
        "sigma_action": sa,
    }
