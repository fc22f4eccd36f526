"""The wavefront trace (wam_trace_chunk): timing events at every block
boundary of both streams of a graph-replayed CEWP chunk.  Checks the
structure of the records and the ordering the schedule guarantees: action
block i's attention starts only after video block i's K/V are published
(RealtimeWAM summary page, 方法步骤详情: P^a_i -> wait(e_i) -> Attn^a_i), and
both streams advance block by block."""
import numpy as np
import pytest

import mot_dit_b200 as W
from wam_testlib import MID_BF16, inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("batch,blocks", [(1, "0"), (1, "1"), (2, "0")])
def test_trace_records_the_wavefront(monkeypatch, batch, blocks):
    monkeypatch.setenv("WAM_ACTION_BLOCKS", blocks)   # per-operation kernels / persistent action blocks
    c = W.WamConfig(**MID_BF16).replace(batch=batch)
    wam = W.Wam(c, seed=3)
    inp = inputs(c, 3)
    dev = torch.device("cuda", 0)
    video, cond, noise = (torch.from_numpy(inp[k]).to(dev) for k in ("video", "cond", "noise"))
    out = torch.empty_like(noise)
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    rec = wam.trace_chunk(video, cond, noise, out, S=2, mode=W.CEWP, stream_video=sv, stream_action=sa)
    wam.check_device_status()
    N = c.n_blocks
    by = {}
    for kind, b, j, t in rec:
        by.setdefault(kind, []).append((b, j, t))
    assert len(by["start"]) == 1 and len(by["end"]) == 1 and by["start"][0][2] == 0.0
    assert [b for b, _, _ in by["video_kv"]] == list(range(N))
    assert [b for b, _, _ in by["video_end"]] == list(range(N - 1))   # the last block stops after its K/V
    for kind in ("action_attn", "action_end"):
        assert [(b, j) for b, j, _ in by[kind]] == [(b, j) for j in range(2) for b in range(N)]
    kv = {b: t for b, _, t in by["video_kv"]}
    for b, j, t in by["action_attn"]:
        if j == 0:
            assert t >= kv[b], (b, t, kv[b])   # Attn^a_i waits for e_i
    for kind in ("video_kv", "action_attn", "action_end"):
        ts = [t for _, _, t in by[kind]]
        assert all(x <= y for x, y in zip(ts, ts[1:])), kind
    t_end = by["end"][0][2]
    assert all(t <= t_end for _, _, t in by["action_end"])
    # the traced chunk computes the same result as the graph
    ref = torch.empty_like(noise)
    wam.infer_chunk(video, cond, noise, ref, S=2, mode=W.CEWP, stream_video=sv, stream_action=sa)
    sv.synchronize()
    assert torch.equal(out, ref)
    wam.close()
