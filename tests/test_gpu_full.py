"""Parity at the benchmark sizes, in the launch configuration bench.py times
(CEWP schedule replayed from a CUDA graph, bf16, seed 0):

* the Fast-WAM-shaped one-step chunk (28 blocks, 1536/768, 64+1024 video
  tokens, 32 action tokens): a_0 and v_eff within rel. L2 1e-2 of the oracle;
* the same model with the 10-step uniform teacher schedule;
* the batch-8 throughput shape (2048 video tokens per sample): batch
  elements 0 and 7, each computed by the oracle as an independent chunk.

The oracle's parameters for these three (identical architecture) are
generated once per session.
"""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle import params as PR
from wam_testlib import check_parity, f32_sched, inputs, ocfg, run_chunk

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
    oc1 = ocfg(c).with_(batch=1)
    for b in (0, 7):
        one = {k: (v[b:b + 1] if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
        ref_a0, ref_veff = M.infer_chunk(oc1, oracle_params, one, t_sched=f32_sched(1))
        e = check_parity(a0[b:b + 1], one, ref_a0, ref_veff, c.dtype)
        print(f"config-4 sample {b} rel L2 (a0, v_eff):", e)
