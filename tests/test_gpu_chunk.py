"""End-to-end parity of the chunk on the GPU, through the C ABI, against the
oracle: seeded parameters, the fp32 debug path (rel. L2 <= 1e-4), the bf16
path (rel. L2 <= 1e-2) on a_0 and v_eff = a_1 - a_0, CEWP == sequential
bitwise, graph == eager bitwise, the per-block K/V publish, the closed-form
constant-velocity case and the eager video/action API (also under stream
delays)."""
import time

import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle import params as PR
from wam_testlib import MID_BF16, check_parity, f32_sched, inputs, ocfg, oracle_chunk, rel_l2, run_chunk

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _mid():
    return W.WamConfig(**MID_BF16)


@pytest.mark.parametrize("cfg", ["tiny", "mid", "tiny_lora", "mid_lora"])
def test_seeded_params_match_oracle_generator(cfg):
    """Every parameter the library generated on the device (LoRA factors
    included: B lives inside its layer's weight matrix) equals the oracle's."""
    c = W.preset(1) if cfg.startswith("tiny") else _mid()
    if cfg.endswith("lora"):
        c = c.replace(lora_rank=64)
    wam = W.Wam(c, seed=1234)
    flat = wam.export_params()
    P = PR.generate_params(ocfg(c), 1234)
    ref = np.concatenate([P[n].ravel() for n, _, _ in PR.param_specs(ocfg(c))])
    assert flat.shape == ref.shape
    diff = flat != ref
    # device and host libm may differ by one ulp in log/cos: allow a rare
    # one-ulp (fp32) difference, nothing else
    if diff.any():
        assert diff.mean() < 1e-5
        ulp = np.abs(flat[diff].view(np.int32).astype(np.int64) - ref[diff].view(np.int32).astype(np.int64))
        assert ulp.max() <= (1 << 16 if c.dtype == 1 else 1)
    wam.close()


@pytest.mark.parametrize("S,mode,graph", [(1, W.CEWP, True), (1, W.SEQUENTIAL, False), (3, W.CEWP, False),
                                          (3, W.SEQUENTIAL, True)])
def test_tiny_fp32_parity(S, mode, graph):
    c = W.preset(1)
    wam = W.Wam(c, seed=5)
    inp = inputs(c, 5)
    a0 = run_chunk(wam, inp, S=S, mode=mode, use_graph=graph)
    ref_a0, ref_veff = oracle_chunk(c, 5, inp, S=S)
    check_parity(a0, inp, ref_a0, ref_veff, c.dtype)


@pytest.mark.parametrize("batch", [1, 2])
def test_fused_action_norm(monkeypatch, batch):
    """Opt-in fused action norm (WAM_FUSE_NORM=1): the QKV / FFN-up / final
    out-proj GEMMs normalise the token rows themselves (32- and 64-token
    tiles); parity with the oracle, and CEWP == sequential bitwise."""
    monkeypatch.setenv("WAM_FUSE_NORM", "1")
    c = _mid().replace(batch=batch)
    wam = W.Wam(c, seed=13)
    inp = inputs(c, 13)
    a0 = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    seq = run_chunk(wam, inp, S=2, mode=W.SEQUENTIAL, use_graph=False)
    assert np.array_equal(a0, seq)
    ref_a0, ref_veff = oracle_chunk(c, 13, inp, S=2)
    check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    wam.close()


@pytest.mark.parametrize("batch", [1, 2])
def test_video_cta_pairs(monkeypatch, batch):
    """Opt-in CTA-pair video GEMMs (WAM_VIDEO_PAIR=1: 2-SM MMAs, M = 256 over
    two SMs): parity with the oracle, CEWP == sequential and graph == eager
    bitwise."""
    monkeypatch.setenv("WAM_VIDEO_PAIR", "1")
    c = _mid().replace(batch=batch)
    wam = W.Wam(c, seed=17)
    inp = inputs(c, 17)
    a0 = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    for mode, graph in ((W.SEQUENTIAL, True), (W.CEWP, False)):
        assert np.array_equal(a0, run_chunk(wam, inp, S=2, mode=mode, use_graph=graph))
    ref_a0, ref_veff = oracle_chunk(c, 17, inp, S=2)
    check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    wam.close()


@pytest.mark.parametrize("batch", [1, 2])
def test_video_cluster_split(monkeypatch, batch):
    """The video FFN-down on 256-wide tiles split between the two CTAs of a
    cluster (finished in column halves, the partials crossing in shared
    memory): the grid is set to twice its tile count so the rule picks it at
    this size.  Bitwise equal to the same partition reduced through global
    memory, at parity with the oracle, CEWP == sequential."""
    # FFN width 3072: FFN-down's k-range is deep enough (48 k-blocks) for the split
    c = _mid().replace(batch=batch, ffn_video=3072)
    ctas = str(2 * ((c.batch * (c.l_cond + c.l_video) + 127) // 128) * (c.d_video // 256))
    inp = inputs(c, 23)
    monkeypatch.setenv("WAM_VIDEO_GEMM_CTAS", ctas)
    for k in ("WAM_VIDEO_CSPLIT", "WAM_VIDEO_OPROJ_BN", "WAM_VIDEO_FFN2_BN"):
        monkeypatch.delenv(k, raising=False)
    wam = W.Wam(c, seed=23)
    got = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    for mode, graph in ((W.SEQUENTIAL, True), (W.CEWP, False)):
        assert np.array_equal(run_chunk(wam, inp, S=2, mode=mode, use_graph=graph), got)
    wam.close()
    monkeypatch.setenv("WAM_VIDEO_CSPLIT", "0")
    monkeypatch.setenv("WAM_VIDEO_FFN2_BN", "256")
    wam = W.Wam(c, seed=23)
    assert np.array_equal(run_chunk(wam, inp, S=2), got)
    wam.close()
    ref_a0, ref_veff = oracle_chunk(c, 23, inp, S=2)
    check_parity(got, inp, ref_a0, ref_veff, c.dtype)


@pytest.mark.parametrize("batch,shape", [
    (1, dict(n_heads=8, ffn_action=1536)),
    (2, dict(n_heads=8, ffn_action=1536)),
    (1, dict(d_action=256, n_heads=16, ffn_action=3072)),
])
def test_action_cluster_reduce(monkeypatch, batch, shape):
    """Action GEMMs split over clusters, the pieces summed in shared memory:
    out-projection and FFN-down (the first shape: 2 and 8 CTAs per
    128-feature tile over 8 and 24 k-blocks; at batch 2 on 64-token tiles),
    and the wide QKV / FFN-up (the last shape: 24 feature tiles each, 4 CTAs
    per tile; the QK-norm / RoPE and GELU epilogues).  Bitwise equal to the
    same splits summed through global partials, CEWP == sequential, at parity
    with the oracle."""
    c = _mid().replace(batch=batch, **shape)
    monkeypatch.delenv("WAM_ACTION_WIDE_SPLITS", raising=False)
    monkeypatch.setenv("WAM_ACTION_QKV_SPLITS", "4")  # the QKV epilogue on clusters too
    inp = inputs(c, 29)
    monkeypatch.delenv("WAM_ACTION_CRED", raising=False)
    wam = W.Wam(c, seed=29)
    got = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    for mode, graph in ((W.SEQUENTIAL, True), (W.CEWP, False)):
        assert np.array_equal(run_chunk(wam, inp, S=2, mode=mode, use_graph=graph), got)
    wam.close()
    monkeypatch.setenv("WAM_ACTION_CRED", "0")
    wam = W.Wam(c, seed=29)
    assert np.array_equal(run_chunk(wam, inp, S=2), got)
    wam.close()
    ref_a0, ref_veff = oracle_chunk(c, 29, inp, S=2)
    check_parity(got, inp, ref_a0, ref_veff, c.dtype)


def test_video_qkv_192_wide(monkeypatch):
    """Six heads (attention width 384): the video QKV runs on 192-wide tiles
    (18 whole tiles against 15 at 256 wide), the QK-norm / RoPE epilogue
    takes three heads a tile.  Parity with the oracle, CEWP == sequential,
    and the 256-wide form agrees to rounding."""
    c = _mid().replace(batch=1, n_heads=6)
    inp = inputs(c, 29)
    monkeypatch.delenv("WAM_VIDEO_QKV_BN", raising=False)
    wam = W.Wam(c, seed=29)
    got = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    assert np.array_equal(run_chunk(wam, inp, S=2, mode=W.SEQUENTIAL, use_graph=False), got)
    wam.close()
    ref_a0, ref_veff = oracle_chunk(c, 29, inp, S=2)
    check_parity(got, inp, ref_a0, ref_veff, c.dtype)
    monkeypatch.setenv("WAM_VIDEO_QKV_BN", "256")
    wam = W.Wam(c, seed=29)
    other = run_chunk(wam, inp, S=2)
    wam.close()
    assert rel_l2(inp["noise"] - got, inp["noise"] - other) < 1e-3


@pytest.mark.parametrize("pair", ["0", "1"])
def test_video_fused_norm(monkeypatch, pair):
    """Opt-in fused video norm (WAM_VIDEO_FUSED_NORM=1): the QKV / FFN-up
    GEMMs write their own A operand from x_v in a prologue (the rows shared out
    through a counter).  It rounds like the norm kernel, so the chunk is
    bitwise the unfused one; CEWP == sequential, graph == eager, and fifty
    replays (the counters reset themselves every launch)."""
    monkeypatch.setenv("WAM_VIDEO_PAIR", pair)
    c = _mid().replace(batch=2)
    inp = inputs(c, 19)
    monkeypatch.setenv("WAM_VIDEO_FUSED_NORM", "0")
    wam = W.Wam(c, seed=19)
    ref = run_chunk(wam, inp, S=2)
    wam.close()
    monkeypatch.setenv("WAM_VIDEO_FUSED_NORM", "1")
    wam = W.Wam(c, seed=19)
    got = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    assert np.array_equal(got, ref)
    for mode, graph in ((W.SEQUENTIAL, True), (W.CEWP, False)):
        assert np.array_equal(run_chunk(wam, inp, S=2, mode=mode, use_graph=graph), ref)
    for _ in range(50):
        assert np.array_equal(run_chunk(wam, inp, S=2), ref)
    wam.check_device_status()
    wam.close()


def test_mid_bf16_parity_and_kv_publish():
    c = _mid()
    wam = W.Wam(c, seed=11)
    inp = inputs(c, 11)
    a0 = run_chunk(wam, inp, S=1)
    oc = ocfg(c)
    P = PR.generate_params(oc, 11)
    ref_a0, ref_veff = M.infer_chunk(oc, P, inp, t_sched=f32_sched(1))
    check_parity(a0, inp, ref_a0, ref_veff, c.dtype)
    # the K/V every video block publishes (rows [0, L_v) of the cache) and the
    # action expert's own K/V of the last step (rows [L_v, L_v + L_a))
    kv, _, _ = M.video_expert(oc, P, inp["video"], inp["cond"], 0.0)
    for i in range(c.n_blocks):
        k = wam.read_kv(i, 0)
        v = wam.read_kv(i, 1)
        assert rel_l2(k[:, :, :oc.l_v], kv[i][0]) < 1e-2, i
        assert rel_l2(v[:, :, :oc.l_v], kv[i][1]) < 1e-2, i
        assert np.abs(k[:, :, oc.l_v:]).sum() > 0


@pytest.mark.parametrize("cfg", ["tiny", "mid"])
def test_cewp_equals_sequential_bitwise(cfg):
    c = W.preset(1) if cfg == "tiny" else _mid()
    wam = W.Wam(c, seed=3)
    for seed in (0, 1, 2, 3, 4):
        inp = inputs(c, seed)
        outs = [run_chunk(wam, inp, S=S, mode=m, use_graph=g)
                for S in (1, 3) for m, g in ((W.CEWP, True), (W.SEQUENTIAL, True), (W.CEWP, False),
                                              (W.SEQUENTIAL, False))]
        for S_idx in (0, 1):
            group = outs[4 * S_idx: 4 * S_idx + 4]
            for o in group[1:]:
                assert np.array_equal(o, group[0])
    # repeated graph launches stay bitwise stable
    inp = inputs(c, 9)
    first = run_chunk(wam, inp, S=1)
    for _ in range(100):
        assert np.array_equal(run_chunk(wam, inp, S=1), first)
    wam.close()


@pytest.mark.parametrize("delay", ["video", "action", "host"])
def test_eager_chunks_under_stream_delays(delay):
    """Two back-to-back chunks through the eager API, with one stream held
    back by a sleep kernel (or the host pausing between enqueues).  Action
    attention i waits for video block i's K/V, and the next chunk's video
    block i waits until the last action attention i has read the cache, so
    the order comes from events, not timing: both chunks equal the pipelined
    graph bitwise.  A missing consumed-K/V wait shows under the action delay
    (chunk 1's video would overwrite K/V that chunk 0 has not read yet)."""
    c = _mid()
    wam = W.Wam(c, seed=17)
    ins = [inputs(c, 40 + k) for k in range(2)]
    refs = [run_chunk(wam, inp, S=2) for inp in ins]
    dev = torch.device("cuda", 0)
    vids = [(torch.from_numpy(inp["video"]).to(dev), torch.from_numpy(inp["cond"]).to(dev)) for inp in ins]
    acts = [torch.from_numpy(inp["noise"]).to(dev) for inp in ins]
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    spin = 20_000_000   # clock cycles (about 10 ms): longer than a whole chunk of this model
    for k in range(2):
        if delay == "video":
            with torch.cuda.stream(sv):
                torch.cuda._sleep(spin)
        wam.video_forward(*vids[k], 0.0, stream=sv)
        if delay == "host":
            time.sleep(0.01)
        if delay == "action":
            with torch.cuda.stream(sa):
                torch.cuda._sleep(spin)
        wam.action_step(acts[k], 1.0, 0.5, stream=sa)
        wam.action_step(acts[k], 0.5, 0.0, stream=sa)
    sa.synchronize()
    sv.synchronize()
    wam.check_device_status()
    for k in range(2):
        assert np.array_equal(acts[k].cpu().numpy(), refs[k]), k
    wam.close()


@pytest.mark.parametrize("cfg,S", [("tiny", 1), ("tiny", 8), ("mid", 1), ("mid", 8)])
def test_constant_velocity_closed_form(cfg, S):
    """All parameters zero except the action output bias b = 0.5: v = b for any
    input, so a_0 = a_1 - 0.5 exactly (dyadic grid)."""
    c = W.preset(1) if cfg == "tiny" else _mid()
    wam = W.Wam(c, seed=0)
    names = [n for n, _, _ in PR.param_specs(ocfg(c))]
    sizes = [int(np.prod(s)) for _, s, _ in PR.param_specs(ocfg(c))]
    flat = np.zeros(sum(sizes), np.float32)
    at = 0
    for n, sz in zip(names, sizes):
        if n == "action.out.b":
            flat[at:at + sz] = 0.5
        at += sz
    wam.import_params(flat)
    inp = inputs(c, 4)
    a0 = run_chunk(wam, inp, S=S)
    # the state is fp32: each Euler step subtracts 0.5/S = 2^-k and rounds once,
    # which is exact except where a negative value crosses a power of two
    want = inp["noise"].copy()
    for _ in range(S):
        want = want - np.float32(0.5 / S)
    np.testing.assert_array_equal(a0, want)
    assert np.abs(a0.astype(np.float64) - (inp["noise"].astype(np.float64) - 0.5)).max() <= S * 2.0 ** -22 * 4


def test_eager_video_and_action_steps_match_chunk():
    c = _mid()
    wam = W.Wam(c, seed=21)
    inp = inputs(c, 21)
    ref = run_chunk(wam, inp, S=2, mode=W.CEWP, use_graph=True)
    dev = torch.device("cuda", 0)
    video = torch.from_numpy(inp["video"]).to(dev)
    cond = torch.from_numpy(inp["cond"]).to(dev)
    a = torch.from_numpy(inp["noise"]).to(dev)
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    wam.video_forward(video, cond, 0.0, stream=sv)
    wam.action_step(a, 1.0, 0.5, stream=sa)
    wam.action_step(a, 0.5, 0.0, stream=sa)
    sa.synchronize()
    sv.synchronize()
    wam.check_device_status()
    assert np.array_equal(a.cpu().numpy(), ref)


def test_host_buffer_entry_point_matches_device_one():
    c = _mid()
    wam = W.Wam(c, seed=8)
    inp = inputs(c, 8)
    ref = run_chunk(wam, inp, S=1)
    out = np.zeros_like(inp["noise"])
    sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
    wam.infer_chunk_host(inp["video"], inp["cond"], inp["noise"], out, S=1, stream_video=sv, stream_action=sa)
    assert np.array_equal(out, ref)


def test_argument_errors_enqueue_nothing():
    c = _mid()
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 0)
    dev = torch.device("cuda", 0)
    video = torch.from_numpy(inp["video"]).to(dev)
    noise = torch.from_numpy(inp["noise"]).to(dev)
    out = torch.empty_like(noise)
    with pytest.raises(W.WamError) as e:
        wam.infer_chunk(video, None, noise, out, S=1)           # missing conditioning tokens
    assert e.value.status == 1
    cond = torch.from_numpy(inp["cond"]).to(dev)
    for S, t in ((0, None), (65, None), (2, [1.0, 0.7, 0.8]), (1, [1.5, 0.0])):
        with pytest.raises(W.WamError):
            wam.infer_chunk(video, cond, noise, out, S=S, t_sched=t)
    sv = torch.cuda.Stream()
    with pytest.raises(W.WamError):   # CEWP with one stream
        wam.infer_chunk(video, cond, noise, out, S=1, mode=W.CEWP, stream_video=sv, stream_action=sv)
    fresh = W.Wam(c, seed=0)
    with pytest.raises(W.WamError) as e:
        fresh.action_step(out, 1.0, 0.0)
    assert e.value.status == 6
    wam.check_device_status()


def test_device_memory_limit_reports_oom(monkeypatch):
    """A context whose allocations would pass WAM_DEVICE_MEMORY_LIMIT fails
    with WAM_ERR_OOM before calling cudaMalloc, leaves *out NULL and releases
    what it had allocated; the same config builds and runs without the limit."""
    import ctypes as C
    c = _mid()
    monkeypatch.setenv("WAM_DEVICE_MEMORY_LIMIT", str(1 << 20))   # far below the model's weights
    h = C.c_void_p()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert W.lib().wam_init(C.byref(c), 0, C.byref(h)) == 3 and not h.value
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] >= free0 - (64 << 20)   # nothing left behind
    monkeypatch.delenv("WAM_DEVICE_MEMORY_LIMIT")
    wam = W.Wam(c, seed=0)
    inp = inputs(c, 0)
    a0 = run_chunk(wam, inp, S=1)
    assert np.isfinite(a0).all()
    wam.close()


def test_bounded_wait_timeout_is_reported_and_the_next_call_is_clean(monkeypatch):
    """Failure detection without a GPU fault: the test hook makes the last
    piece of every split GEMM tile wait for one partial tile more than exists
    (a count nothing raises) with a 20 ms limit.  The kernels give up, wind
    down and return; wam_check_device_status reports WAM_ERR_TIMEOUT and
    resets the tickets; with the hook off the next chunk equals the reference
    bitwise and the status is clean.  (The video GEMMs run stream-K here, so
    their tiles are split over several CTAs.)"""
    monkeypatch.setenv("WAM_VIDEO_SPLIT_FREE", "0")
    c = _mid()
    wam = W.Wam(c, seed=9)
    inp = inputs(c, 9)
    ref = run_chunk(wam, inp, S=1)
    assert W.lib().wam_test_peer_wait(1, 20_000_000) == 0
    try:
        dev = torch.device("cuda", 0)
        video, cond, noise = (torch.from_numpy(inp[k]).to(dev) for k in ("video", "cond", "noise"))
        out = torch.empty_like(noise)
        sv, sa = torch.cuda.Stream(), torch.cuda.Stream()
        wam.infer_chunk(video, cond, noise, out, S=1, mode=W.CEWP, use_graph=False, stream_video=sv,
                        stream_action=sa)
        sv.synchronize()
        with pytest.raises(W.WamError) as e:
            wam.check_device_status()
        assert e.value.status == 5
    finally:
        assert W.lib().wam_test_peer_wait(0, 0) == 0
    again = run_chunk(wam, inp, S=1)   # run_chunk checks the status itself
    assert np.array_equal(again, ref)
    wam.close()
