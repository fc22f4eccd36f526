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


def _ema_params(c, seed, P_student):
    """The EMA target's parameters: the student's, with LoRA factors drawn
    from another seed (an EMA that has drifted from the student)."""
    other = PR.generate_params(ocfg(c), seed + 1)
    return {k: (other[k] if k.endswith((".la", ".lb")) else v) for k, v in P_student.items()}


@pytest.mark.parametrize("dtype,K", [("fp32", 10), ("fp32", 1), ("bf16", 10)])
def test_tacd_targets_entry_point(dtype, K):
    """wam_tacd_targets: video once, the teacher (base weights) K steps over
    [t, 0], the student and a distinct EMA LoRA over the shared K/V, device-side
    noising, targets and the deterministic loss reduction -- against the
    oracle's tacd_targets (rel. L2 1e-4 fp32 / 1e-2 bf16 on u_TA, v_student,
    u_CD; the losses within 5x that, relative)."""
    if dtype == "fp32":
        c = W.preset(1).replace(lora_rank=64, lora_scale=0.5)
    else:
        c = W.WamConfig(**MID_BF16).replace(lora_rank=128, lora_scale=1.0, n_blocks=2)
    seed, t = 31, 0.625
    inp = synthetic.make_inputs(seed, batch=c.batch, l_cond=c.l_cond, l_video=c.l_video, video_width=c.d_video,
                                l_action=c.l_action, action_dim=c.action_dim, action_clean=True)
    for k in ("action_clean", "noise"):   # a_t exact in fp32 on this grid (see above)
        inp[k] = (np.round(inp[k] * 4096) / 4096).astype(np.float32)
    oc = ocfg(c)
    P_student = PR.generate_params(oc, seed)
    P_ema = _ema_params(c, seed, P_student)
    ref = T.tacd_targets(oc, T.without_lora(P_student), P_student, P_ema, inp, t=t, K=K)

    student = W.Wam(c, seed=seed)
    ema = W.Wam(c, seed=seed)
    names = [n for n, _, _ in PR.param_specs(oc)]
    ema.import_params(np.concatenate([np.asarray(P_ema[n], np.float32).ravel() for n in names]))
    dev = torch.device("cuda", 0)
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(dev) for k in ("video", "action_clean", "noise")}
    cond = torch.from_numpy(inp["cond"]).to(dev) if c.l_cond else None
    outs = {k: torch.full_like(d["noise"], float("nan")) for k in ("u_ta", "v_student", "u_cd", "a_t", "a0_T")}
    losses = torch.full((3,), float("nan"), device=dev)
    s = torch.cuda.Stream()
    student.tacd_targets(ema, d["video"], cond, d["action_clean"], d["noise"], t, K, 0.2, outs["u_ta"],
                         outs["v_student"], outs["u_cd"], losses, a_t=outs["a_t"], a0_teacher=outs["a0_T"], stream=s)
    s.synchronize()
    student.check_device_status()
    got = {k: v.cpu().numpy().astype(np.float64) for k, v in outs.items()}
    l = losses.cpu().numpy().astype(np.float64)
    student.close()
    ema.close()
    assert np.array_equal(got["a_t"], ref["a_t"])
    tol = TOL[c.dtype]
    for k, want in (("u_ta", ref["u_ta"]), ("v_student", ref["v_student"]), ("u_cd", ref["u_cd"])):
        assert np.isfinite(got[k]).all(), k
        e = rel_l2(got[k], want)
        assert e <= tol, f"{k}: rel L2 {e:.3e} (tol {tol})"
    assert rel_l2(got["a0_T"], ref["a0_T"]) <= tol
    for i, key in enumerate(("l_ta", "l_cd")):
        assert abs(l[i] - ref[key]) <= 5 * tol * ref[key], (key, l[i], ref[key])
    assert abs(l[2] - (l[1] + 0.2 * l[0])) <= 1e-6 * l[2]
    if K == 1:   # s = 0: the EMA endpoint is the teacher's one-step state, so u_CD = u_TA
        np.testing.assert_array_equal(got["u_cd"], got["u_ta"])
