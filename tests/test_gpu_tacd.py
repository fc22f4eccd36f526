"""The TACD target forward on the GPU, composed from the chunk entry point,
against the oracle's tacd_targets (oracle/tacd.py).

The heavy parts run in the library: the frozen teacher's K = 10 Euler rollout
from a_t over [t, 0] (a non-uniform schedule starting below 1), the teacher's
one step to s, and the student's endpoints at (a_t, t) and at (a~_s, s) (the
EMA target equals the student before any update).  Teacher and student share
the video expert's weights: the video parameters come first in the generation
order, so a model with and without LoRA draws them identically from the same
seed.  The noising a_t and the loss reductions are done here, on the host.

Every compared quantity is a velocity, so a_t passing through unchanged cannot
hide an error: u_TA = (a_t - a_0^T)/t, the teacher's velocity (a_t - a~_s)/(t - s),
the student's v = (a_t - f)/t and u_CD = (a_t - f^-)/t.  Tolerance: rel. L2
1e-4 (fp32 path) and 1e-2 (bf16 path); L_TA within 5x that (it is a squared
distance between velocities that differ by more than their norm here).
t = 5/8 with K = 10 puts every grid point on a multiple of 1/16, exact in fp32.
"""
import numpy as np
import pytest

import mot_dit_b200 as W
import synthetic
from oracle import model as M
from oracle import params as PR
from oracle import tacd as T
from wam_testlib import MID_BF16, TOL, ocfg, rel_l2, run_chunk

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_tacd_targets_through_the_chunk_entry_point(dtype):
    if dtype == "fp32":
        c = W.preset(1).replace(lora_rank=64, lora_scale=0.5)
    else:
        c = W.WamConfig(**MID_BF16).replace(lora_rank=128, lora_scale=1.0, n_blocks=2)
    c_teacher = c.replace(lora_rank=0)
    seed, t, K = 23, 0.625, 10
    inp = synthetic.make_inputs(seed, batch=c.batch, l_cond=c.l_cond, l_video=c.l_video, video_width=c.d_video,
                                l_action=c.l_action, action_dim=c.action_dim, action_clean=True)
    # on a 2^-12 grid, a_t = (3/8) a_0 + (5/8) eps is exact in fp32, so the
    # library and the oracle start from the same a_t
    for k in ("action_clean", "noise"):
        inp[k] = (np.round(inp[k] * 4096) / 4096).astype(np.float32)
    oc = ocfg(c)
    P_student = PR.generate_params(oc, seed)
    P_teacher = PR.generate_params(ocfg(c_teacher), seed)
    for k in P_teacher:
        if k.startswith("video."):
            assert np.array_equal(P_teacher[k], P_student[k]), k
    ref = T.tacd_targets(oc, P_teacher, P_student, P_student, inp, t=t, K=K)

    teacher = W.Wam(c_teacher, seed=seed)
    student = W.Wam(c, seed=seed)
    a_t = M.noise_to(inp["action_clean"], inp["noise"], t).astype(np.float32)
    assert np.array_equal(a_t.astype(np.float64), ref["a_t"])
    grid = T.teacher_grid(t, K)
    s = float(grid[1])
    assert s == ref["s"] == 0.5625
    a0_T = run_chunk(teacher, dict(inp, noise=a_t), S=K, t_sched=grid)
    a_s = run_chunk(teacher, dict(inp, noise=a_t), S=1, t_sched=[t, s])
    f_student = run_chunk(student, dict(inp, noise=a_t), S=1, t_sched=[t, 0.0])
    f_ema = run_chunk(student, dict(inp, noise=a_s), S=1, t_sched=[s, 0.0])
    teacher.close()
    student.close()

    at = a_t.astype(np.float64)
    got = {
        "u_ta": T.interval_velocity(at, a0_T, t),
        "v_teacher": (at - a_s) / (t - s),
        "v_student": (at - f_student) / t,
        "u_cd": T.interval_velocity(at, f_ema, t),
    }
    want = {
        "u_ta": ref["u_ta"],
        "v_teacher": (ref["a_t"] - ref["a_s"]) / (t - s),
        "v_student": ref["v_student"],
        "u_cd": ref["u_cd"],
    }
    tol = TOL[c.dtype]
    for k in got:
        assert np.isfinite(got[k]).all(), k
        e = rel_l2(got[k], want[k])
        assert e <= tol, f"{k}: rel L2 {e:.3e} (tol {tol})"
    l_ta = T.chunk_mean_sq(got["v_student"] - got["u_ta"])
    assert abs(l_ta - ref["l_ta"]) <= 5 * tol * ref["l_ta"], (l_ta, ref["l_ta"])
