"""The persistent action-block path (one launch per action block: attention,
out-projection, FFN and the next block's QKV separated by grid barriers)
against the oracle, through the C ABI.

It serves bf16 models without LoRA whose chunk has at most 32 action tokens
(the Fast-WAM-shaped configs).  Checked here on small models with ragged
sizes: parity with the oracle (rel. L2 <= 1e-2 on a_0 and v_eff), CEWP ==
sequential and graph == eager bitwise, independence of the grid size (the
launches that run beside the video expert take fewer CTAs; the work units and
the reduction order are fixed by the shapes), and agreement with the
per-operation kernels (WAM_ACTION_BLOCKS=0) within the same tolerance.
"""
import numpy as np
import pytest

import mot_dit_b200 as W
from wam_testlib import check_parity, inputs, oracle_chunk, rel_l2, run_chunk

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# L_v = 64 + 200 = 264 video-expert tokens (ragged against the 128-key split),
# 4 heads, d_a = 128, F_a = 256: every phase has a ragged unit layout.
SMALL = dict(n_blocks=3, d_video=256, d_action=128, n_heads=4, head_dim=64, ffn_video=512, ffn_action=256,
             l_cond=64, l_video=200, l_action=32, action_dim=30, video_patch_dim=0, batch=1, lora_rank=0,
             lora_scale=1.0, video_has_output=0, dtype=1)


def _wam(monkeypatch, seed, ctas=None, blocks=True, **kw):
    monkeypatch.setenv("WAM_ACTION_BLOCKS", "1" if blocks else "0")   # (the path is opt-in)
    if ctas is not None:
        monkeypatch.setenv("WAM_ACTION_BLOCK_CTAS", str(ctas))
    else:
        monkeypatch.delenv("WAM_ACTION_BLOCK_CTAS", raising=False)
    c = W.WamConfig(**{**SMALL, **kw})
    return c, W.Wam(c, seed=seed)


@pytest.mark.parametrize("shape", [dict(), dict(l_action=16), dict(batch=2, l_action=16),
                                   dict(d_action=768, ffn_action=3072, n_heads=24, l_cond=0, l_video=100)])
@pytest.mark.parametrize("S", [1, 3])
def test_action_blocks_parity_and_schedules(monkeypatch, shape, S):
    c, wam = _wam(monkeypatch, 11, **shape)
    inp = inputs(c, 11)
    cewp = run_chunk(wam, inp, S=S, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=S, mode=W.SEQUENTIAL, use_graph=True)
    eager = run_chunk(wam, inp, S=S, mode=W.CEWP, use_graph=False)
    assert np.array_equal(cewp, seq)
    assert np.array_equal(cewp, eager)
    ref_a0, ref_veff = oracle_chunk(c, 11, inp, S=S)
    check_parity(cewp, inp, ref_a0, ref_veff, c.dtype)
    wam.close()


def test_action_blocks_grid_size_does_not_change_the_result(monkeypatch):
    """The CEWP first step runs its launches on a smaller grid (the SMs the
    video GEMMs leave free); the work units and the split-reduction order do
    not depend on it, so any grid gives the same bits."""
    outs = []
    for ctas in (None, 8, 23, 64):
        c, wam = _wam(monkeypatch, 12, ctas=ctas)
        inp = inputs(c, 12)
        outs.append(run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True))
        outs.append(run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=False))
        wam.close()
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_action_blocks_match_the_per_operation_kernels(monkeypatch):
    c, wam = _wam(monkeypatch, 13)
    inp = inputs(c, 13)
    a_blocks = run_chunk(wam, inp, S=2)
    wam.close()
    c, wam = _wam(monkeypatch, 13, blocks=False)
    a_ops = run_chunk(wam, inp, S=2)
    wam.close()
    v_blocks, v_ops = inp["noise"] - a_blocks, inp["noise"] - a_ops
    assert rel_l2(v_blocks, v_ops) <= 1e-2
    ref_a0, ref_veff = oracle_chunk(c, 13, inp, S=2)
    check_parity(a_blocks, inp, ref_a0, ref_veff, c.dtype)
    check_parity(a_ops, inp, ref_a0, ref_veff, c.dtype)


def test_action_blocks_replays_are_stable(monkeypatch):
    """Fifty graph replays of the same chunk: the grid barriers, the per-tile
    counters and the attention counters reset themselves every launch."""
    c, wam = _wam(monkeypatch, 14)
    inp = inputs(c, 14)
    dev = torch.device("cuda", 0)
    video = torch.from_numpy(inp["video"]).to(dev)
    cond = torch.from_numpy(inp["cond"]).to(dev)
    noise = torch.from_numpy(inp["noise"]).to(dev)
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(50):
        out = torch.empty_like(noise)
        wam.infer_chunk(video, cond, noise, out, S=2, mode=W.CEWP, use_graph=True, stream_video=sv,
                        stream_action=sa)
        outs.append(out)
    sv.synchronize()
    wam.check_device_status()
    first = outs[0].cpu().numpy()
    for o in outs[1:]:
        assert np.array_equal(o.cpu().numpy(), first)
    wam.close()


def test_eager_action_steps_on_the_block_path(monkeypatch):
    """wam_video_forward then wam_action_step on another stream: the action
    launches wait on the per-block events and give the chunk's bits."""
    c, wam = _wam(monkeypatch, 15)
    inp = inputs(c, 15)
    ref = run_chunk(wam, inp, S=1, mode=W.CEWP, use_graph=True)
    dev = torch.device("cuda", 0)
    video = torch.from_numpy(inp["video"]).to(dev)
    cond = torch.from_numpy(inp["cond"]).to(dev)
    a = torch.from_numpy(inp["noise"]).to(dev)
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    wam.video_forward(video, cond, 0.0, stream=sv)
    wam.action_step(a, 1.0, 0.0, stream=sa)
    sa.synchronize()
    sv.synchronize()
    wam.check_device_status()
    assert np.array_equal(a.cpu().numpy(), ref)
    wam.close()
