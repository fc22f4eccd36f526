"""Unmerged LoRA on the action expert and the joint one-step (1v/1a) variant
on the GPU, through the C ABI, against the oracle.

LoRA runs as one GEMM over the concatenated reduction [x | s x A^T] . [W | B]^T
(the down-projection u = s x A^T is a small GEMM writing the r extra input
columns).  The fp32 path is held to rel. L2 <= 1e-4, the bf16 path to 1e-2."""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle import params as PR
from wam_testlib import MID_BF16, check_parity, inputs, ocfg, oracle_chunk, rel_l2, run_chunk

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("dtype,rank,scale", [("fp32", 64, 0.5), ("bf16", 128, 1.0), ("bf16", 64, 4.0)])
def test_lora_chunk_parity(dtype, rank, scale):
    if dtype == "fp32":
        c = W.preset(1).replace(lora_rank=rank, lora_scale=scale)
    else:
        c = W.WamConfig(**MID_BF16).replace(lora_rank=rank, lora_scale=scale, n_blocks=2)
    wam = W.Wam(c, seed=21)
    inp = inputs(c, 21)
    a0 = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=2, mode=W.SEQUENTIAL, use_graph=False)
    assert np.array_equal(a0, seq)
    ref_a0, ref_veff = oracle_chunk(c, 21, inp, S=2)
    check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    # the LoRA term is resolved: the velocity is much closer to the model with
    # LoRA than to the same model without it
    P = PR.generate_params(ocfg(c), 21)
    for k in list(P):
        if k.endswith(".lb"):
            P[k] = np.zeros_like(P[k])
    _, base_veff = oracle_chunk(c, 21, inp, S=2, P=P)
    veff = inp["noise"].astype(np.float64) - a0
    assert rel_l2(veff, ref_veff) < 0.5 * rel_l2(veff, base_veff)
    wam.close()


def _joint_cfg(dtype):
    if dtype == "fp32":
        return W.preset(5).replace(n_blocks=2, d_video=64, d_action=64, n_heads=4, head_dim=16, ffn_video=128,
                                   ffn_action=128, l_video=32, l_action=8, video_patch_dim=24, lora_rank=64,
                                   dtype=0)
    return W.preset(5).replace(n_blocks=2, d_video=256, d_action=256, n_heads=4, head_dim=64, ffn_video=512,
                               ffn_action=512, l_video=128, l_action=16, video_patch_dim=192, lora_rank=128)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_joint_one_step_parity(dtype):
    """Flash-WAM-style 1v/1a step: SNR-shifted noising of both streams on the
    device, the video expert with patch in-projection and the f^v endpoint,
    the action expert (with LoRA) and the action endpoint."""
    c = _joint_cfg(dtype)
    wam = W.Wam(c, seed=31)
    inp = inputs(c, 31)
    t = {k: torch.from_numpy(np.ascontiguousarray(inp[k])).to(DEV)
         for k in ("video", "video_eps", "action_clean", "noise")}
    v_out = torch.full_like(t["video"], float("nan"))
    a_out = torch.full_like(t["noise"], float("nan"))
    outs = []
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    for mode, graph in ((W.CEWP, True), (W.SEQUENTIAL, False)):
        wam.joint_one_step(t["video"], t["video_eps"], t["action_clean"], t["noise"], inp["u_video"], inp["u_action"],
                           v_out, a_out, mode=mode, use_graph=graph, stream_video=sv, stream_action=sa)
        sv.synchronize()
        torch.cuda.synchronize()
        outs.append((v_out.cpu().numpy().copy(), a_out.cpu().numpy().copy()))
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
    oc = ocfg(c)
    P = PR.generate_params(oc, 31)
    ref = M.joint_one_step(oc, P, inp)
    tol = 1e-4 if dtype == "fp32" else 1e-2
    assert np.isfinite(outs[0][0]).all() and np.isfinite(outs[0][1]).all()
    assert rel_l2(outs[0][1], ref["f_action"]) < tol
    assert rel_l2(outs[0][0], ref["f_video"]) < tol
    wam.close()
