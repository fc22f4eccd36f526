"""The chunk with a multi-step video expert (wam_infer_chunk_multistep)
against the oracle (oracle/multistep.py), through the C ABI: the video
latents after N_v Euler steps and the action chunk over the last video
forward's K/V, fp32 (rel. L2 <= 1e-4) and bf16 (<= 1e-2) on the video result,
a_0 and v_eff; CEWP == sequential and graph == eager bitwise."""
import numpy as np
import pytest

import mot_dit_b200 as W
import synthetic
from oracle import model as M
from oracle import multistep as MS
from oracle import params as PR
from wam_testlib import TOL, ocfg, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FP32 = dict(n_blocks=2, d_video=64, d_action=64, n_heads=4, head_dim=16, ffn_video=128, ffn_action=128, l_cond=0,
            l_video=32, l_action=8, action_dim=30, video_patch_dim=24, batch=1, lora_rank=0, lora_scale=1.0,
            video_has_output=1, dtype=0)
BF16 = dict(FP32, d_video=256, d_action=128, head_dim=64, ffn_video=512, ffn_action=256, l_video=128, l_action=16,
            video_patch_dim=64, dtype=1)


def _run(wam, c, inp, nv, S, mode, graph):
    dev = torch.device("cuda", 0)
    eps = torch.from_numpy(np.ascontiguousarray(inp["video_eps"])).to(dev)
    noise = torch.from_numpy(inp["noise"]).to(dev)
    vout = torch.full_like(eps, float("nan"))
    aout = torch.full_like(noise, float("nan"))
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    wam.infer_chunk_multistep(eps, noise, vout, aout, n_video=nv, S=S, mode=mode, use_graph=graph, stream_video=sv,
                              stream_action=sa)
    sv.synchronize()
    wam.check_device_status()
    return vout.cpu().numpy(), aout.cpu().numpy()


@pytest.mark.parametrize("shape", ["fp32", "bf16"])
@pytest.mark.parametrize("nv,S", [(1, 1), (3, 2)])
def test_multistep_video_chunk(shape, nv, S):
    c = W.WamConfig(**(FP32 if shape == "fp32" else BF16))
    seed = 41 + nv
    wam = W.Wam(c, seed=seed)
    inp = synthetic.make_inputs(seed, batch=c.batch, l_cond=0, l_video=c.l_video, video_width=c.video_patch_dim,
                                l_action=c.l_action, action_dim=c.action_dim, patch_input=True)
    v1, a1 = _run(wam, c, inp, nv, S, W.CEWP, True)
    v2, a2 = _run(wam, c, inp, nv, S, W.SEQUENTIAL, True)
    v3, a3 = _run(wam, c, inp, nv, S, W.CEWP, False)
    wam.close()
    assert np.array_equal(v1, v2) and np.array_equal(a1, a2)
    assert np.array_equal(v1, v3) and np.array_equal(a1, a3)
    f32 = lambda n: M.uniform_schedule(n).astype(np.float32).astype(np.float64)
    oc = ocfg(c)
    ref = MS.multistep_chunk(oc, PR.generate_params(oc, seed), inp, sched_v=f32(nv), sched_a=f32(S))
    tol = TOL[c.dtype]
    e_v = rel_l2(v1, ref["video"])
    e_a = rel_l2(a1, ref["a0"])
    e_d = rel_l2(inp["noise"].astype(np.float64) - a1, ref["v_eff"])
    # the video displacement x_1 - x_0 too (x_1 passes through)
    e_dv = rel_l2(inp["video_eps"].astype(np.float64) - v1, inp["video_eps"].astype(np.float64) - ref["video"])
    assert max(e_v, e_a, e_d, e_dv) <= tol, (e_v, e_a, e_d, e_dv)


def test_multistep_rejects_models_without_video_output():
    c = W.preset(1)
    wam = W.Wam(c, seed=0)
    with pytest.raises(W.WamError) as e:
        wam.infer_chunk_multistep(0x1000, 0x1000, 0x1000, 0x1000, n_video=2)
    assert e.value.status == 2
    wam.close()
