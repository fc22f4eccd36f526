"""Pins of the TACD target oracle (oracle/tacd.py) against facts outside it.

Closed forms (constant velocity), reductions (one teacher step), the pages'
own identities (L_TA is the 1/t^2-weighted endpoint error; the bound on the
student's endpoint error) and the first-order convergence of the teacher's
Euler rollout.  A wrong sign or scale in u, the EMA evaluated at the wrong
point or time, or the student and teacher weights swapped fails one of them.
"""
import numpy as np
import pytest

import synthetic
from oracle import model as M
from oracle import params as PR
from oracle import tacd as T
from oracle.config import preset


def _cfg():
    return preset(1).with_(batch=2, lora_rank=8)


def _inputs(cfg, seed):
    return synthetic.make_inputs(seed, batch=cfg.batch, l_cond=cfg.l_cond, l_video=cfg.l_video,
                                 video_width=cfg.d_video, l_action=cfg.l_action, action_dim=cfg.action_dim,
                                 action_clean=True)


def _kv(cfg, P, inp):
    kv, _, _ = M.video_expert(cfg, P, inp["video"], inp["cond"], 0.0)
    return kv


def test_clean_action_draw_leaves_other_inputs_unchanged():
    cfg = _cfg()
    a = _inputs(cfg, 4)
    b = synthetic.make_inputs(4, batch=cfg.batch, l_cond=cfg.l_cond, l_video=cfg.l_video, video_width=cfg.d_video,
                              l_action=cfg.l_action, action_dim=cfg.action_dim)
    assert set(a) - set(b) == {"action_clean"}
    for k in b:
        np.testing.assert_array_equal(a[k], b[k])


def test_constant_velocity_targets_are_exact():
    """All weights zero except the action output bias b = 0.5, so v = b for
    every network, input and time.  The teacher then lands on a_t - t b, so
    u_TA = b; the CD target is f^-(a~_s, s) = a_t - (t - s) b - s b = a_t - t b,
    so u_CD = b too, and both losses vanish.  Inputs on a 2^-10 grid and
    t = 1/2, K = 8 keep every step exact."""
    cfg = _cfg()
    P = {k: np.zeros_like(v) for k, v in PR.generate_params(cfg, 0).items()}
    P["action.out.b"] = np.full(cfg.action_dim, 0.5, np.float32)
    inp = _inputs(cfg, 1)
    for k in ("action_clean", "noise"):
        inp[k] = (np.round(inp[k] * 1024) / 1024).astype(np.float32)
    r = T.tacd_targets(cfg, T.without_lora(P), P, P, inp, t=0.5, K=8)
    np.testing.assert_array_equal(r["a_t"], 0.5 * inp["action_clean"].astype(np.float64) + 0.5 * inp["noise"])
    np.testing.assert_array_equal(r["a0_T"], r["a_t"] - 0.25)
    np.testing.assert_array_equal(r["u_ta"], 0.5)
    assert r["s"] == 7 / 16
    np.testing.assert_array_equal(r["a_s"], r["a_t"] - 1 / 32)
    np.testing.assert_array_equal(r["f_ema"], r["a_t"] - 0.25)
    np.testing.assert_array_equal(r["u_cd"], 0.5)
    assert r["l_ta"] == 0.0 and r["l_cd"] == 0.0 and r["loss"] == 0.0


def test_noising_end_points():
    cfg = _cfg()
    P = PR.generate_params(cfg, 2)
    inp = _inputs(cfg, 2)
    r = T.tacd_targets(cfg, T.without_lora(P), P, P, inp, t=1.0, K=2)
    np.testing.assert_array_equal(r["a_t"], inp["noise"].astype(np.float64))
    with pytest.raises(ValueError):
        T.tacd_targets(cfg, P, P, P, inp, t=0.0)


def test_one_teacher_step_reduces_to_teacher_velocity():
    """K = 1: a_0^T = a_t - t v_T(a_t, t), so u_TA = v_T(a_t, t); and s = 0,
    where the endpoint map is the identity, so f^-(a~_0, 0) = a_0^T and
    u_CD = u_TA whatever the EMA weights are.  L_TA is then the squared gap
    between the student's and the teacher's velocity at (a_t, t)."""
    cfg = _cfg()
    P = PR.generate_params(cfg, 5)
    P_ema = PR.generate_params(cfg, 6)
    Pt = T.without_lora(P)
    inp = _inputs(cfg, 5)
    t = 0.6
    r = T.tacd_targets(cfg, Pt, P, P_ema, inp, t=t, K=1)
    kv = _kv(cfg, Pt, inp)
    a_t = M.noise_to(inp["action_clean"], inp["noise"], t)
    v_T = M.action_velocity(cfg, Pt, a_t, t, kv)
    v_S = M.action_velocity(cfg, P, a_t, t, kv)
    assert r["s"] == 0.0
    np.testing.assert_allclose(r["u_ta"], v_T, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(r["u_cd"], r["u_ta"])
    np.testing.assert_array_equal(r["v_student"], v_S)
    gap = np.sum((v_S - v_T).reshape(cfg.batch, -1) ** 2, axis=1).mean()
    assert r["l_ta"] == pytest.approx(gap, rel=1e-10)
    assert r["l_ta"] > 1e-6          # the LoRA factors move the student off the teacher
    # a student equal to the teacher has nothing left to learn at K = 1
    r0 = T.tacd_targets(cfg, Pt, Pt, P_ema, inp, t=t, K=1)
    assert r0["l_ta"] < 1e-24 and r0["l_cd"] < 1e-24


def test_teacher_rollout_is_the_euler_sampler_on_t_to_0():
    """The teacher's K steps are the chunk sampler run from a_t on the grid
    t k / K (the sampler is pinned on its own in test_oracle.py)."""
    cfg = _cfg()
    P = T.without_lora(PR.generate_params(cfg, 7))
    inp = _inputs(cfg, 7)
    t, K = 0.75, 10
    a_t = M.noise_to(inp["action_clean"], inp["noise"], t)
    states = T.teacher_rollout(cfg, P, a_t, t, _kv(cfg, P, inp), K)
    a0, _ = M.infer_chunk(cfg, P, dict(inp, noise=a_t), t_sched=t * np.arange(K, -1, -1) / K)
    np.testing.assert_array_equal(states[-1], a0)
    assert len(states) == K + 1
    np.testing.assert_allclose(T.teacher_grid(t, K)[[0, 1, -1]], [t, t * 0.9, 0.0], rtol=0, atol=1e-16)


def test_ta_loss_is_endpoint_error_weighted_by_inverse_t_squared():
    """核心方法: supervising the velocity with u_TA is endpoint supervision
    weighted by 1/t^2, since f_theta - a_0^T = -t (v_theta - u_TA)."""
    cfg = _cfg()
    P = PR.generate_params(cfg, 8)
    inp = _inputs(cfg, 8)
    for t in (0.3, 0.9):
        r = T.tacd_targets(cfg, T.without_lora(P), P, P, inp, t=t, K=10)
        endpoint_err = np.sum((r["f_student"] - r["a0_T"]).reshape(cfg.batch, -1) ** 2, axis=1).mean()
        assert r["l_ta"] == pytest.approx(endpoint_err / t ** 2, rel=1e-9)
        # the same identity for CD, against the EMA endpoint
        cd_err = np.sum((r["f_student"] - r["f_ema"]).reshape(cfg.batch, -1) ** 2, axis=1).mean()
        assert r["l_cd"] == pytest.approx(cd_err / t ** 2, rel=1e-9)
        assert r["loss"] == pytest.approx(r["l_cd"] + 0.2 * r["l_ta"], rel=1e-15)


def _fine_endpoint(cfg, P, inp, t, K=640):
    kv = _kv(cfg, P, inp)
    a_t = M.noise_to(inp["action_clean"], inp["noise"], t)
    return a_t, kv, T.teacher_rollout(cfg, P, a_t, t, kv, K)[-1]


def test_teacher_error_falls_as_one_over_k_and_bounds_the_student():
    """Euler is first order: against a 640-step rollout the endpoint error
    halves when K doubles (so E||delta||^2 is O(K^-2), as 核心方法 states).
    With a_0 taken as that fine endpoint, the pages' bound
    E||e_total||^2 <= 2 L_TA + 2 E||delta||^2 holds for the student."""
    cfg = _cfg()
    P = PR.generate_params(cfg, 9)
    Pt = T.without_lora(P)
    inp = _inputs(cfg, 9)
    t = 0.7
    a_t, kv, a0 = _fine_endpoint(cfg, Pt, inp, t)
    err = {K: np.linalg.norm(T.teacher_rollout(cfg, Pt, a_t, t, kv, K)[-1] - a0) for K in (10, 20)}
    assert 1.85 < err[10] / err[20] < 2.15
    r = T.tacd_targets(cfg, Pt, P, P, inp, t=t, K=10)
    e_total = np.sum((r["f_student"] - a0).reshape(cfg.batch, -1) ** 2, axis=1).mean()
    delta = np.sum((r["a0_T"] - a0).reshape(cfg.batch, -1) ** 2, axis=1).mean()
    assert e_total <= 2 * r["l_ta"] + 2 * delta
    assert delta < 1e-2 * e_total    # the teacher's own error is small next to the student's
