"""Shared helpers of the GPU parity tests: oracle config from a library
config, seeded chunk inputs, device round trips and the parity metric."""
from __future__ import annotations

import numpy as np

import synthetic
from oracle import model as M
from oracle import params as PR
from oracle.config import WamConfig as OCfg

TOL = {0: 1e-4, 1: 1e-2}   # fp32 debug path / bf16 path (relative L2)

# A bf16 model small enough for the oracle to run in about a second, with
# ragged sizes: L_v = 64 + 200 = 264 video-expert tokens per sample (not a
# multiple of the 128-row GEMM tile or the 64-key attention tile), 4 heads of
# 64 channels (A = 256, whole 128-feature QKV tiles), batch 2.
MID_BF16 = dict(n_blocks=3, d_video=256, d_action=128, n_heads=4, head_dim=64, ffn_video=512, ffn_action=256,
                l_cond=64, l_video=200, l_action=32, action_dim=30, video_patch_dim=0, batch=2, lora_rank=0,
                lora_scale=1.0, video_has_output=0, dtype=1)


def ocfg(c) -> OCfg:
    return OCfg(n_blocks=c.n_blocks, d_video=c.d_video, d_action=c.d_action, n_heads=c.n_heads,
                head_dim=c.head_dim, ffn_video=c.ffn_video, ffn_action=c.ffn_action, l_cond=c.l_cond,
                l_video=c.l_video, l_action=c.l_action, action_dim=c.action_dim,
                video_patch_dim=c.video_patch_dim, batch=c.batch, lora_rank=c.lora_rank,
                lora_scale=float(c.lora_scale), video_has_output=bool(c.video_has_output),
                dtype="bf16" if c.dtype == 1 else "fp32")


def inputs(c, seed: int) -> dict:
    return synthetic.make_inputs(seed, batch=c.batch, l_cond=c.l_cond, l_video=c.l_video,
                                 video_width=c.video_patch_dim or c.d_video, l_action=c.l_action,
                                 action_dim=c.action_dim, patch_input=c.video_patch_dim > 0)


def rel_l2(x, ref) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def f32_sched(S: int, t_sched=None) -> np.ndarray:
    """The schedule as the library sees it (fp32 values), in float64 for the oracle."""
    t = M.uniform_schedule(S) if t_sched is None else np.asarray(t_sched, np.float64)
    return t.astype(np.float32).astype(np.float64)


def run_chunk(wam, inp, S=1, t_sched=None, mode=1, use_graph=True):
    import torch
    dev = torch.device("cuda", 0)
    video = torch.from_numpy(inp["video"]).to(dev)
    cond = torch.from_numpy(inp["cond"]).to(dev) if inp["cond"].shape[1] > 0 else None
    noise = torch.from_numpy(inp["noise"]).to(dev)
    out = torch.empty_like(noise)
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    wam.infer_chunk(video, cond, noise, out, S=S, t_sched=t_sched, mode=mode, use_graph=use_graph,
                    stream_video=sv, stream_action=sa)
    sv.synchronize()
    wam.check_device_status()
    return out.cpu().numpy()


def oracle_chunk(c, seed, inp, S=1, t_sched=None, P=None):
    oc = ocfg(c)
    if P is None:
        P = PR.generate_params(oc, seed)
    return M.infer_chunk(oc, P, inp, t_sched=f32_sched(S, t_sched))


def check_parity(a0, inp, ref_a0, ref_veff, dtype):
    veff = inp["noise"].astype(np.float64) - a0
    e_a0, e_v = rel_l2(a0, ref_a0), rel_l2(veff, ref_veff)
    tol = TOL[dtype]
    assert e_a0 <= tol and e_v <= tol, f"rel L2 a0={e_a0:.3e} v_eff={e_v:.3e} (tol {tol})"
    return e_a0, e_v
