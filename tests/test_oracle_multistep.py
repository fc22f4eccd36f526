"""Pins of the multi-step-video oracle (oracle/multistep.py), CPU only:
closed forms and reductions to the one-pass definitions."""
import numpy as np
import pytest

from oracle import model as M
from oracle import multistep as MS
from oracle import params as PR
from oracle.config import preset
import synthetic


def _cfg(**kw):
    return preset(5).with_(n_blocks=2, d_video=64, d_action=64, n_heads=4, head_dim=16, ffn_video=128,
                           ffn_action=128, l_video=32, l_action=8, video_patch_dim=24, lora_rank=0, dtype="fp32",
                           **kw)


def _inputs(cfg, seed):
    return synthetic.make_inputs(seed, batch=cfg.batch, l_cond=0, l_video=cfg.l_video,
                                 video_width=cfg.video_patch_dim, l_action=cfg.l_action,
                                 action_dim=cfg.action_dim, patch_input=True)


@pytest.mark.parametrize("nv,S", [(1, 1), (4, 2), (8, 8)])
def test_constant_velocities_closed_form(nv, S):
    """Every parameter zero except the two output biases (0.5 video, 0.25
    action): both velocities are constant, so x_0 = x_1 - 0.5 and
    a_0 = a_1 - 0.25, exactly on dyadic grids."""
    cfg = _cfg()
    P = {k: np.zeros_like(v) for k, v in PR.generate_params(cfg, 0).items()}
    P["video.out.b"] = np.full(cfg.video_patch_dim, 0.5, np.float32)
    P["action.out.b"] = np.full(cfg.action_dim, 0.25, np.float32)
    inp = _inputs(cfg, 1)
    r = MS.multistep_chunk(cfg, P, inp, n_video=nv, S=S)
    np.testing.assert_array_equal(r["video"], inp["video_eps"].astype(np.float64) - 0.5)
    np.testing.assert_array_equal(r["a0"], inp["noise"].astype(np.float64) - 0.25)


def test_one_video_step_is_one_forward_at_level_one():
    """N_v = 1: x_0 = x_1 - v^v(x_1, 1) (the endpoint map at level 1), and the
    action expert uses that forward's K/V: the one-pass chunk."""
    cfg = _cfg()
    P = PR.generate_params(cfg, 3)
    inp = _inputs(cfg, 3)
    r = MS.multistep_chunk(cfg, P, inp, n_video=1, S=2)
    x1 = inp["video_eps"].astype(np.float64)
    kv, _, v = M.video_expert(cfg, P, x1, None, 1.0, run_last_rest=True)
    np.testing.assert_array_equal(r["video"], M.endpoint(x1, v, 1.0))
    a = inp["noise"].astype(np.float64)
    for t0, t1 in ((1.0, 0.5), (0.5, 0.0)):
        a = M.euler_step(a, M.action_velocity(cfg, P, a, t0, kv), t0, t1)
    np.testing.assert_array_equal(r["a0"], a)


def test_action_reads_the_last_video_forward():
    """N_v = 3 written out step by step: the video state follows three Euler
    steps, and the action result equals the one computed on the K/V of the
    third forward -- and differs from the one on the first forward's K/V
    (negative control: the K/V do change between denoising steps)."""
    cfg = _cfg()
    P = PR.generate_params(cfg, 4)
    inp = _inputs(cfg, 4)
    grid = np.array([1.0, 0.75, 0.25, 0.0])
    r = MS.multistep_chunk(cfg, P, inp, sched_v=grid, S=1)
    x = inp["video_eps"].astype(np.float64)
    kvs = []
    for j in range(3):
        kv, _, v = M.video_expert(cfg, P, x, None, grid[j], run_last_rest=True)
        kvs.append(kv)
        x = x - (grid[j] - grid[j + 1]) * v
    np.testing.assert_array_equal(r["video"], x)
    a1 = inp["noise"].astype(np.float64)
    want = a1 - M.action_velocity(cfg, P, a1, 1.0, kvs[2])
    np.testing.assert_array_equal(r["a0"], want)
    first = a1 - M.action_velocity(cfg, P, a1, 1.0, kvs[0])
    assert np.abs(first - want).max() > 1e-6


def test_rollout_rejects_a_model_without_video_output():
    cfg = preset(1)
    with pytest.raises(ValueError):
        MS.video_rollout(cfg, PR.generate_params(cfg, 0), np.zeros((1, 64, 64)), [1.0, 0.0])
