"""Parity at the benchmark sizes, in the launch configuration bench.py times
(CEWP schedule replayed from a CUDA graph, bf16, seed 0):

* the Fast-WAM-shaped one-step chunk (28 blocks, 1536/768, 64+1024 video
  tokens, 32 action tokens): a_0 and v_eff within rel. L2 1e-2 of the oracle;
* the same model with the 10-step uniform teacher schedule;
* the batch-8 throughput shape (2048 video tokens per sample): batch
  elements 0 and 7, each computed by the oracle as an independent chunk;
* the Flash-WAM-like joint 1v/1a step (30 blocks at 1536, 1024 patch tokens
  of 192, 16 action tokens, rank-128 LoRA on the action expert): the action
  and video endpoints within rel. L2 1e-2.

The oracle's parameters for these three (identical architecture) are
generated once per session.
"""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle import params as PR
from wam_testlib import check_parity, f32_sched, inputs, ocfg, rel_l2, run_chunk

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def oracle_params():
    return PR.generate_params(ocfg(W.preset(2)), 0)


def test_fastwam_shaped_one_step(oracle_params):
    c = W.preset(2)
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 0)
    a0 = run_chunk(wam, inp, S=1, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=1, mode=W.SEQUENTIAL, use_graph=True)
    assert np.array_equal(a0, seq)
    ref_a0, ref_veff = M.infer_chunk(ocfg(c), oracle_params, inp, t_sched=f32_sched(1))
    e = check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    print("config-2 rel L2 (a0, v_eff):", e)


def test_teacher_ten_steps(oracle_params):
    c = W.preset(3)
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 1)
    a0 = run_chunk(wam, inp, S=10, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=10, mode=W.SEQUENTIAL, use_graph=True)
    assert np.array_equal(a0, seq)
    ref_a0, ref_veff = M.infer_chunk(ocfg(c), oracle_params, inp, t_sched=f32_sched(10))
    e = check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    print("config-3 rel L2 (a0, v_eff):", e)


def test_batch8_sampled_elements(oracle_params):
    c = W.preset(4)
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 2)
    a0 = run_chunk(wam, inp, S=1, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=1, mode=W.SEQUENTIAL, use_graph=True)
    assert np.array_equal(a0, seq)   # the wavefront reordering is exact at this shape too
    oc1 = ocfg(c).with_(batch=1)
    for b in (0, 7):
        one = {k: (v[b:b + 1] if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
        ref_a0, ref_veff = M.infer_chunk(oc1, oracle_params, one, t_sched=f32_sched(1))
        e = check_parity(a0[b:b + 1], one, ref_a0, ref_veff, c.dtype)
        print(f"config-4 sample {b} rel L2 (a0, v_eff):", e)


def test_flash_wam_joint_config5():
    c = W.preset(5)
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 3)
    dev = torch.device("cuda", 0)
    t = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(dev)
         for k in ("video", "video_eps", "action_clean", "noise")}
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for mode in (W.CEWP, W.SEQUENTIAL):
        v_out = torch.full_like(t["video"], float("nan"))
        a_out = torch.full_like(t["noise"], float("nan"))
        wam.joint_one_step(t["video"], t["video_eps"], t["action_clean"], t["noise"], inp["u_video"],
                           inp["u_action"], v_out, a_out, mode=mode, use_graph=True, stream_video=sv,
                           stream_action=sa)
        sv.synchronize()
        outs.append((v_out.cpu().numpy(), a_out.cpu().numpy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    oc = ocfg(c)
    ref = M.joint_one_step(oc, PR.generate_params(oc, 0), inp)
    ea, ev = rel_l2(outs[0][1], ref["f_action"]), rel_l2(outs[0][0], ref["f_video"])
    print("config-5 rel L2 (f_action, f_video):", ea, ev)
    assert ea < 1e-2 and ev < 1e-2
