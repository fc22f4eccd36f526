"""Pins of the CPU oracle against facts outside itself (no GPU needed).

Each test checks an oracle function against a closed form, a special case,
an independent library routine (torch fp64 CPU ops) or a published value,
chosen so that a dropped term, a wrong sign or index or a transposed operand
in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import synthetic
from oracle import model as M
from oracle import params as PR
from oracle.config import preset

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _tiny(**kw):
    return preset(1).with_(**kw)


def _zero_params(cfg, seed=0):
    P = PR.generate_params(cfg, seed)
    return {k: np.zeros_like(v) for k, v in P.items()}


# --------------------------------------------------------------------------
# generator
# --------------------------------------------------------------------------

def test_splitmix64_published_sequence():
    vals = [int(l, 16) for l in open(os.path.join(GOLD, "splitmix64_state0.txt"))
            if l.strip() and not l.startswith("#")]
    states = np.array([(k * int(PR.G)) % 2 ** 64 for k in range(4)], dtype=np.uint64)
    assert [int(v) for v in PR.splitmix64(states)] == vals


def test_generator_random_access_and_stats():
    a = PR.normal_block(7, 3, 0, 200000)
    b = PR.normal_block(7, 3, 1000, 500)
    np.testing.assert_array_equal(a[1000:1500], b)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    # fourth moment of a standard normal is 3
    assert abs(np.mean(a ** 4) - 3.0) < 0.05
    c = PR.normal_block(7, 4, 0, 200000)
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.01
    d = PR.normal_block(8, 3, 0, 200000)
    assert abs(np.corrcoef(a, d)[0, 1]) < 0.01


def test_bf16_rounding_matches_torch():
    x = (np.random.default_rng(0).standard_normal(100000) * 0.02).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0]  # ties both ways
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(PR.round_bf16(x), ref)


def test_param_specs_shapes_and_gains():
    cfg = preset(2)
    specs = PR.param_specs(cfg)
    names = [s[0] for s in specs]
    assert len(names) == len(set(names))
    d = dict((s[0], s) for s in specs)
    assert d["video.blk0.qkv.w"][1] == (3 * 1536, 1536)
    assert d["action.blk27.qkv.w"][1] == (3 * 1536, 768)
    assert d["action.blk3.o.w"][1] == (768, 1536)
    assert d["action.out.w"][1] == (30, 768)
    assert d["action.fn.g"][2] is None and d["video.blk5.qn.g"][2] is None
    P = PR.generate_params(preset(1), 3)
    assert np.all(P["action.fn.g"] == 1.0)
    s = np.concatenate([P[k].ravel() for k, _, sd in PR.param_specs(preset(1)) if sd is not None])
    assert abs(s.std() - 0.02) < 0.001
    P5 = PR.param_specs(preset(5))
    assert any(n == "action.blk0.qkv.la" for n, _, _ in P5)
    assert not any(n.startswith("video.") and ".la" in n for n, _, _ in P5)


# --------------------------------------------------------------------------
# elementwise definitions
# --------------------------------------------------------------------------

def test_rms_norm_pins():
    x = np.random.default_rng(1).standard_normal((5, 64)) * 3.0
    y = M.rms_norm(x)
    np.testing.assert_allclose(np.mean(y * y, -1), 1.0 / (1.0 + 1e-6 / np.mean(x * x, -1)), rtol=1e-12)
    np.testing.assert_array_equal(M.rms_norm(np.zeros((2, 8))), 0.0)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), eps=1e-6).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_gelu_silu_against_torch():
    x = np.linspace(-8, 8, 1001)
    t = torch.from_numpy(x)
    np.testing.assert_allclose(M.gelu_tanh(x), torch.nn.functional.gelu(t, approximate="tanh").numpy(),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(M.silu(x), torch.nn.functional.silu(t).numpy(), rtol=1e-12, atol=1e-15)
    assert M.gelu_tanh(np.array(0.0)) == 0.0


def test_timestep_features_closed_form():
    tau0 = M.timestep_features(0.0)
    np.testing.assert_array_equal(tau0, np.r_[np.ones(128), np.zeros(128)])
    t = math.pi / 2000.0   # 1000 t w_0 = pi/2
    tau = M.timestep_features(t)
    assert abs(tau[0]) < 1e-12 and abs(tau[128] - 1.0) < 1e-12
    # w_64 = 10000^(-1/2) = 0.01: feature 64 is cos(10 t)
    assert abs(tau[64] - math.cos(10.0 * t)) < 1e-12


def test_rope_is_a_rotation_by_plus_theta():
    rng = np.random.default_rng(2)
    dh = 16
    x = rng.standard_normal((3, 7, dh))
    pos = np.arange(7.0) * 13.0
    y = M.rope(x, pos)
    np.testing.assert_allclose(M.rope(x, np.zeros(7)), x, rtol=0, atol=0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    # complex form: (x_j + i x_{j+dh/2}) * exp(i pos 10000^(-2j/dh))
    z = x[..., : dh // 2] + 1j * x[..., dh // 2:]
    th = pos[:, None] * 10000.0 ** (-2.0 * np.arange(dh // 2) / dh)
    w = z * np.exp(1j * th)
    np.testing.assert_allclose(y, np.concatenate([w.real, w.imag], -1), rtol=1e-12, atol=1e-12)
    # relative position: <R(m) q, R(n) k> depends on m - n only
    q, k = rng.standard_normal((1, dh)), rng.standard_normal((1, dh))
    d1 = (M.rope(q, np.array([5.0])) * M.rope(k, np.array([2.0]))).sum()
    d2 = (M.rope(q, np.array([105.0])) * M.rope(k, np.array([102.0]))).sum()
    assert abs(d1 - d2) < 1e-10


def test_linear_and_lora_against_torch_and_merged():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 6, 32))
    P = {"l.w": rng.standard_normal((24, 32)), "l.b": rng.standard_normal(24)}
    ref = torch.nn.functional.linear(torch.from_numpy(x), torch.from_numpy(P["l.w"]),
                                     torch.from_numpy(P["l.b"])).numpy()
    np.testing.assert_allclose(M.linear(x, P, "l"), ref, rtol=1e-12, atol=1e-12)
    P["l.la"] = rng.standard_normal((8, 32))
    P["l.lb"] = np.zeros((24, 8))
    np.testing.assert_allclose(M.linear(x, P, "l"), ref, rtol=1e-12, atol=1e-12)   # B = 0: base model
    P["l.lb"] = rng.standard_normal((24, 8))
    merged = {"l.w": P["l.w"] + 0.5 * P["l.lb"] @ P["l.la"], "l.b": P["l.b"]}
    np.testing.assert_allclose(M.linear(x, P, "l", 0.5), M.linear(x, merged, "l"), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def test_attention_against_torch_sdpa_and_special_cases():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((2, 3, 9, 16))
    k = rng.standard_normal((2, 3, 13, 16))
    v = rng.standard_normal((2, 3, 13, 16))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(M.attention(q, k, v), ref, rtol=1e-12, atol=1e-13)
    # one key: softmax = 1, output = V
    np.testing.assert_allclose(M.attention(q, k[:, :, :1], v[:, :, :1]),
                               np.broadcast_to(v[:, :, :1], q.shape), rtol=1e-13)
    # equal keys: output = mean of V
    ke = np.broadcast_to(k[:, :, :1], k.shape)
    np.testing.assert_allclose(M.attention(q, ke, v),
                               np.broadcast_to(v.mean(2, keepdims=True), q.shape), rtol=1e-12)
    # large logits do not overflow
    assert np.isfinite(M.attention(q * 1e3, k * 1e3, v)).all()


def test_joint_attention_equals_masked_full_sequence():
    """Concatenated-KV MoT attention vs one masked attention over [video; action]."""
    rng = np.random.default_rng(5)
    B, H, Lv, La, Dh = 2, 2, 11, 4, 8
    qv, kv_, vv = (rng.standard_normal((B, H, Lv, Dh)) for _ in range(3))
    qa, ka, va = (rng.standard_normal((B, H, La, Dh)) for _ in range(3))
    ov = M.attention(qv, kv_, vv)
    oa = M.attention(qa, np.concatenate([kv_, ka], 2), np.concatenate([vv, va], 2))
    q = torch.from_numpy(np.concatenate([qv, qa], 2))
    k = torch.from_numpy(np.concatenate([kv_, ka], 2))
    v = torch.from_numpy(np.concatenate([vv, va], 2))
    allowed = torch.ones(Lv + La, Lv + La, dtype=torch.bool)
    allowed[:Lv, Lv:] = False            # video queries do not see action keys
    full = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed).numpy()
    np.testing.assert_allclose(ov, full[:, :, :Lv], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(oa, full[:, :, Lv:], rtol=1e-12, atol=1e-13)


def _naive_attention_row(q, keys, vals):
    """softmax(q . k / sqrt(Dh)) V for one query, in plain Python loops."""
    scale = 1.0 / math.sqrt(len(q))
    scores = [sum(qi * ki for qi, ki in zip(q, k)) * scale for k in keys]
    m = max(scores)
    w = [math.exp(x - m) for x in scores]
    z = sum(w)
    return [sum(wj * v[c] for wj, v in zip(w, vals)) / z for c in range(len(vals[0]))]


def test_joint_attention_against_naive_loops():
    """The O(n^2) definition, loop by loop, on a tiny shape: video queries over
    video keys only, action queries over [video; action] keys."""
    rng = np.random.default_rng(15)
    H, Lv, La, Dh = 2, 5, 3, 4
    qv, kv_, vv = (rng.standard_normal((1, H, Lv, Dh)) for _ in range(3))
    qa, ka, va = (rng.standard_normal((1, H, La, Dh)) for _ in range(3))
    ov = M.attention(qv, kv_, vv)
    oa = M.attention(qa, np.concatenate([kv_, ka], 2), np.concatenate([vv, va], 2))
    for h in range(H):
        keys_v, vals_v = kv_[0, h].tolist(), vv[0, h].tolist()
        for i in range(Lv):
            want = _naive_attention_row(qv[0, h, i].tolist(), keys_v, vals_v)
            np.testing.assert_allclose(ov[0, h, i], want, rtol=1e-12, atol=1e-14)
        keys_j, vals_j = keys_v + ka[0, h].tolist(), vals_v + va[0, h].tolist()
        for i in range(La):
            want = _naive_attention_row(qa[0, h, i].tolist(), keys_j, vals_j)
            np.testing.assert_allclose(oa[0, h, i], want, rtol=1e-12, atol=1e-14)


def test_mot_block_equals_joint_sequence_formulation():
    """One MoT block of the action expert written as a single masked attention
    over the joint token sequence (per-token expert weights, positions 0..L_v+L_a-1)."""
    cfg = _tiny(n_blocks=1)
    P = {k: v.astype(np.float64) for k, v in PR.generate_params(cfg, 11).items()}
    rng = np.random.default_rng(6)
    x_v = rng.standard_normal((1, cfg.l_v, cfg.d_video))
    a = rng.standard_normal((1, cfg.l_action, cfg.action_dim))
    t = 0.37
    kv, _, _ = M.video_expert(cfg, P, x_v, None, 0.0)
    got = M.action_velocity(cfg, P, a, t, kv)

    # joint formulation, reusing only projection / remainder / head helpers
    mv = M.block_modulation(M.modulation(cfg, P, "video", 0.0), P["video.blk0.T"])
    ma = M.block_modulation(M.modulation(cfg, P, "action", t), P["action.blk0.T"])
    xa = M.linear(a, P, "action.in")
    Lv, La = cfg.l_v, cfg.l_action
    pos = np.arange(Lv + La, dtype=np.float64)
    qv, kvv, vv = M.project_qkv(cfg, P, "video.blk0.", M.modulate(x_v, mv[0], mv[1]), pos[:Lv], 1.0)
    qa, ka, va = M.project_qkv(cfg, P, "action.blk0.", M.modulate(xa, ma[0], ma[1]), pos[Lv:], 1.0)
    allowed = torch.ones(Lv + La, Lv + La, dtype=torch.bool)
    allowed[:Lv, Lv:] = False
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(np.concatenate([qv, qa], 2)), torch.from_numpy(np.concatenate([kvv, ka], 2)),
        torch.from_numpy(np.concatenate([vv, va], 2)), attn_mask=allowed).numpy()
    xa = M.block_rest(cfg, P, "action.blk0.", xa, o[:, :, Lv:], ma, 1.0)
    want = M.linear(M.rms_norm(xa) * P["action.fn.g"], P, "action.out")
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# samplers and closed forms
# --------------------------------------------------------------------------

def _inputs(cfg, seed=0):
    return synthetic.make_inputs(seed, batch=cfg.batch, l_cond=cfg.l_cond, l_video=cfg.l_video,
                                 video_width=cfg.video_patch_dim or cfg.d_video,
                                 l_action=cfg.l_action, action_dim=cfg.action_dim,
                                 patch_input=cfg.video_patch_dim > 0)


@pytest.mark.parametrize("S", [1, 3, 8])
def test_euler_closed_form_constant_velocity(S):
    """All parameters zero except the output bias b: v = b, so a_0 = a_1 - b
    (rms(0) = 0 and every gate is 0).  Exact for dyadic b and grids."""
    cfg = _tiny()
    P = _zero_params(cfg)
    P["action.out.b"] = np.full(cfg.action_dim, 0.5, np.float32)
    inp = _inputs(cfg, 1)
    a0, veff = M.infer_chunk(cfg, P, inp, S=S)
    want = inp["noise"].astype(np.float64) - 0.5
    if S in (1, 8):
        np.testing.assert_array_equal(a0, want)
        np.testing.assert_array_equal(veff, 0.5)
    else:
        np.testing.assert_allclose(a0, want, rtol=0, atol=4e-16 * S)


def test_euler_steps_compose():
    cfg = _tiny()
    P = PR.generate_params(cfg, 2)
    inp = _inputs(cfg, 2)
    sched = np.array([1.0, 0.6, 0.0])
    a0, veff = M.infer_chunk(cfg, P, inp, t_sched=sched)
    kv, _, _ = M.video_expert(cfg, P, inp["video"], inp["cond"], 0.0)
    a = inp["noise"].astype(np.float64)
    a = a - 0.4 * M.action_velocity(cfg, P, a, 1.0, kv)
    a = a - 0.6 * M.action_velocity(cfg, P, a, 0.6, kv)
    np.testing.assert_array_equal(a0, a)
    np.testing.assert_allclose(veff, inp["noise"] - a, rtol=0, atol=1e-15)
    # S = 1 from t = 1: the Euler step is the endpoint map f = a_1 - 1 * v
    a1, _ = M.infer_chunk(cfg, P, inp, S=1)
    v = M.action_velocity(cfg, P, inp["noise"].astype(np.float64), 1.0, kv)
    np.testing.assert_array_equal(a1, M.endpoint(inp["noise"].astype(np.float64), v, 1.0))


def test_modulation_bias_path_and_gates():
    """With every matrix zero: m = b_m, and each block adds g1*b_o + g2*b_2 to x."""
    cfg = _tiny(n_blocks=1)
    P = _zero_params(cfg)
    rng = np.random.default_rng(7)
    d = cfg.d_action
    for k in ("action.mod.b", "action.blk0.T", "action.in.b", "action.blk0.o.b", "action.blk0.ffn2.b",
              "action.blk0.ffn1.b", "action.out.b"):
        P[k] = rng.standard_normal(P[k].shape).astype(np.float32)
    P["action.fn.g"] = np.ones(d, np.float32)
    np.testing.assert_array_equal(M.modulation(cfg, P, "action", 0.3), P["action.mod.b"].astype(np.float64))
    mods = M.block_modulation(M.modulation(cfg, P, "action", 0.3), P["action.blk0.T"])
    x = P["action.in.b"].astype(np.float64) + mods[2] * P["action.blk0.o.b"] + mods[5] * P["action.blk0.ffn2.b"]
    want = M.rms_norm(x) @ np.zeros((d, cfg.action_dim)) + P["action.out.b"]
    kv = [(np.zeros((1, cfg.n_heads, 3, cfg.head_dim)),) * 2]
    a = np.zeros((1, cfg.l_action, cfg.action_dim))
    np.testing.assert_allclose(M.action_velocity(cfg, P, a, 0.3, kv), np.broadcast_to(want, a.shape), rtol=1e-14)
    # the residual itself before the output map
    xs = []
    M_block_rest = M.block_rest

    def spy(cfg_, P_, b_, x_, o_, mods_, s_):
        r = M_block_rest(cfg_, P_, b_, x_, o_, mods_, s_)
        xs.append(r)
        return r
    M.block_rest = spy
    try:
        M.action_velocity(cfg, P, a, 0.3, kv)
    finally:
        M.block_rest = M_block_rest
    np.testing.assert_allclose(xs[0][0, 0], x, rtol=1e-14)


# --------------------------------------------------------------------------
# block-dependency invariants (the premise of the wavefront pipeline)
# --------------------------------------------------------------------------

def test_dropping_last_video_remainder_leaves_action_unchanged():
    cfg = _tiny(n_blocks=3)
    P = PR.generate_params(cfg, 8)
    inp = _inputs(cfg, 8)
    kv_a, _, _ = M.video_expert(cfg, P, inp["video"], inp["cond"], 0.0, run_last_rest=True)
    kv_b, _, _ = M.video_expert(cfg, P, inp["video"], inp["cond"], 0.0, run_last_rest=False)
    a = inp["noise"]
    va = M.action_velocity(cfg, P, a, 1.0, kv_a)
    vb = M.action_velocity(cfg, P, a, 1.0, kv_b)
    np.testing.assert_array_equal(va, vb)


@pytest.mark.parametrize("j", [0, 1])
def test_kv_perturbed_after_consumption_is_harmless(j):
    cfg = _tiny(n_blocks=3)
    P = PR.generate_params(cfg, 9)
    inp = _inputs(cfg, 9)
    kv, _, _ = M.video_expert(cfg, P, inp["video"], inp["cond"], 0.0)
    base = M.action_velocity(cfg, P, inp["noise"], 1.0, list(kv))

    def after(i, kvl):
        if i == j:
            kvl[j] = (kvl[j][0] + 1.0, kvl[j][1] - 1.0)
    np.testing.assert_array_equal(M.action_velocity(cfg, P, inp["noise"], 1.0, list(kv), hook=after), base)

    def before(i, kvl):   # negative control: perturb block j+1 before it is read
        if i == j:
            kvl[j + 1] = (kvl[j + 1][0] + 1.0, kvl[j + 1][1] - 1.0)
    assert np.abs(M.action_velocity(cfg, P, inp["noise"], 1.0, list(kv), hook=before) - base).max() > 1e-6


# --------------------------------------------------------------------------
# joint one-step variant
# --------------------------------------------------------------------------

def test_snr_shift_pins():
    g = json.load(open(os.path.join(GOLD, "closed_forms.json")))
    for r in g["snr_shift"]:
        assert M.snr_shift(r["u"], r["s"]) == pytest.approx(r["sigma"], rel=1e-15)
    u = np.linspace(0, 1, 101)
    for s in (1.0, 5.0):
        sig = M.snr_shift(u, s)
        assert sig[0] == 0.0 and sig[-1] == 1.0
        assert np.all(np.diff(sig) > 0)
        np.testing.assert_allclose(sig / (s - (s - 1.0) * sig), u, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(M.snr_shift(u, 1.0), u, rtol=0, atol=0)


def test_lcm_coefficients_and_b_lcm():
    g = json.load(open(os.path.join(GOLD, "closed_forms.json")))
    for r in g["lcm"]:
        cs, co = M.lcm_coefficients(r["sigma"], r["sigma_d"])
        assert cs == pytest.approx(r["c_skip"], rel=1e-15) and co == pytest.approx(r["c_out"], abs=1e-16)
    # f^v written as a(sigma) x + b(sigma) v has b = -sigma c_out = b_LCM, a = c_skip + c_out
    rng = np.random.default_rng(10)
    x, v = rng.standard_normal(50), rng.standard_normal(50)
    for sig in (1e-3, 0.1, 0.5, 0.9):
        cs, co = M.lcm_coefficients(sig, 0.5)
        b_lcm = -sig ** 2 * 0.5 / math.sqrt(sig ** 2 + 0.25)
        np.testing.assert_allclose(M.video_endpoint(x, v, sig), (cs + co) * x + b_lcm * v, rtol=1e-13, atol=1e-15)
    # Proposition 1: |b_LCM| is O(sigma^2) near 0
    assert abs(-1e-4 * 0.5 / math.sqrt(1e-4 + 0.25)) < 2 * (1e-2) ** 2


def test_joint_one_step_composition():
    cfg = preset(5).with_(n_blocks=2, d_video=64, d_action=64, n_heads=4, head_dim=16, ffn_video=128,
                          ffn_action=128, l_video=32, l_action=8, video_patch_dim=24, lora_rank=4,
                          dtype="fp32")
    P = PR.generate_params(cfg, 12)
    inp = _inputs(cfg, 12)
    r = M.joint_one_step(cfg, P, inp)
    sa = M.snr_shift(inp["u_action"], 1.0)
    assert r["sigma_action"] == sa and r["sigma_video"] == M.snr_shift(inp["u_video"], 5.0)
    a_s = (1 - sa) * inp["action_clean"].astype(np.float64) + sa * inp["noise"].astype(np.float64)
    xs = (1 - r["sigma_video"]) * inp["video"].astype(np.float64) + r["sigma_video"] * inp["video_eps"].astype(np.float64)
    kv, _, vv = M.video_expert(cfg, P, xs, None, r["sigma_video"])
    va = M.action_velocity(cfg, P, a_s, sa, kv)
    np.testing.assert_allclose(r["f_action"], a_s - sa * va, rtol=1e-13, atol=1e-15)
    assert vv is not None and r["f_video"].shape == xs.shape
    # LoRA active: zeroing B changes the action output, zeroing A's effect equals base
    P0 = dict(P)
    for k in list(P0):
        if k.endswith(".lb"):
            P0[k] = np.zeros_like(P0[k])
    r0 = M.joint_one_step(cfg, P0, inp)
    assert np.abs(r0["f_action"] - r["f_action"]).max() > 1e-8
    np.testing.assert_array_equal(r0["f_video"], r["f_video"])   # LoRA is on the action expert only


# --------------------------------------------------------------------------
# P_i's QK-norm + RoPE, the timestep MLP and the FFN: closed forms with
# hand-chosen weights (summary page, 方法步骤详情: the fused "RMSNorm/RoPE"
# operator and the merged QKV projection; the AdaLN timestep modulation and
# the GELU FFN of the shared block definition)
# --------------------------------------------------------------------------

def test_project_qkv_per_head_norm_then_rope_closed_form():
    """Two heads of two channels, every weight zero, so q/k/v are the bias.
    Head 0's q = (3, 4) with gain (1, 0), head 1's q = (-2, 0) with gain (1, 1),
    one token at position pi/2 (RoPE turns channel pair (0, 1) by pi/2).

    Per-head RMS: head 0 has mean square 12.5, head 1 has 2.  Norm, then
    gain, then a quarter turn (x, y) -> (-y, x):
      head 0: (3, 4)/sqrt(12.5+eps) -> gain -> (3r0, 0) -> (0, 3r0)
      head 1: (-2, 0)/sqrt(2+eps)   -> gain -> (-2r1, 0) -> (0, -2r1).
    RoPE first would give head 0 (-4r0, 0); a norm over both heads (mean
    square 7.25) gives other magnitudes; v is the raw projection."""
    cfg = _tiny(n_heads=2, head_dim=2)
    P = _zero_params(cfg)
    b = "video.blk0."
    q_vals = [3.0, 4.0, -2.0, 0.0]
    k_vals = [0.0, 5.0, 1.0, 1.0]
    v_vals = [0.25, -0.5, 1.5, -2.0]
    P[b + "qkv.b"] = np.array(q_vals + k_vals + v_vals, np.float32)
    P[b + "qn.g"] = np.array([1.0, 0.0, 1.0, 1.0], np.float32)
    P[b + "kn.g"] = np.array([2.0, 1.0, 1.0, 1.0], np.float32)
    h = np.zeros((1, 1, cfg.d_video))
    q, k, v = M.project_qkv(cfg, P, b, h, np.array([math.pi / 2]), 1.0)
    r0, r1 = 1.0 / math.sqrt(12.5 + 1e-6), 1.0 / math.sqrt(2.0 + 1e-6)
    np.testing.assert_allclose(q[0, 0, 0], [0.0, 3.0 * r0], atol=1e-15)
    np.testing.assert_allclose(q[0, 1, 0], [0.0, -2.0 * r1], atol=1e-15)
    # k head 0 = (0, 5): mean square 12.5, gain (2, 1) -> (0, 5 r0) -> (-5 r0, 0);
    # k head 1 = (1, 1): mean square 1 -> (1, 1)/sqrt(1+eps) -> (-1, 1)/sqrt(1+eps)
    rk = 1.0 / math.sqrt(1.0 + 1e-6)
    np.testing.assert_allclose(k[0, 0, 0], [-5.0 * r0, 0.0], atol=1e-15)
    np.testing.assert_allclose(k[0, 1, 0], [-rk, rk], atol=1e-15)
    np.testing.assert_array_equal(v[0, :, 0].ravel(), v_vals)


def test_project_qkv_norm_is_per_head_and_per_token():
    """Unit gains at position 0 (RoPE = identity): every (token, head) slice
    of q and k has mean square ms/(ms+eps) of its own pre-norm mean square ms;
    scaling one head's rows of W_qkv by 10 changes no other head's q or k."""
    cfg = _tiny()
    P = {k: v.astype(np.float64) for k, v in PR.generate_params(cfg, 21).items()}
    b = "video.blk0."
    rng = np.random.default_rng(22)
    h = rng.standard_normal((2, 5, cfg.d_video))
    pos = np.zeros(5)
    q, k, v = M.project_qkv(cfg, P, b, h, pos, 1.0)
    A, H, Dh = cfg.attn_dim, cfg.n_heads, cfg.head_dim
    raw = h @ P[b + "qkv.w"].T + P[b + "qkv.b"]
    for sec, got in ((0, q), (1, k)):
        pre = raw[..., sec * A:(sec + 1) * A].reshape(2, 5, H, Dh).transpose(0, 2, 1, 3)
        ms = np.mean(pre ** 2, -1)
        np.testing.assert_allclose(np.mean(got ** 2, -1), ms / (ms + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(v, raw[..., 2 * A:].reshape(2, 5, H, Dh).transpose(0, 2, 1, 3), rtol=1e-13)
    # head 2's q and k rows (weights and bias) scaled by 10
    P2 = dict(P)
    w, bb = P[b + "qkv.w"].copy(), P[b + "qkv.b"].copy()
    for sec in (0, 1):
        rows = slice(sec * A + 2 * Dh, sec * A + 3 * Dh)
        w[rows] *= 10.0
        bb[rows] *= 10.0
    P2[b + "qkv.w"], P2[b + "qkv.b"] = w, bb
    q2, k2, _ = M.project_qkv(cfg, P2, b, h, pos, 1.0)
    for hh in range(H):
        # head 2 itself moves only through eps (relative change about eps / ms, ms ~ 0.03 here)
        tol = 2e-3 if hh == 2 else 0.0
        np.testing.assert_allclose(q2[:, hh], q[:, hh], rtol=tol, atol=0)
        np.testing.assert_allclose(k2[:, hh], k[:, hh], rtol=tol, atol=0)


def test_modulation_mlp_closed_form():
    """tau(t) -> c = W_t2 SiLU(W_t1 tau + b_t1) + b_t2 -> m = W_m SiLU(c) + b_m
    with selection weights.  At t = pi/2000 feature 128 (sin(1000 t w_0)) is 1
    and feature 0 (cos) is 0.  W_t1 picks 2 x feature 128 plus bias 0.5 into
    unit 0; W_t2 = I with bias -1; W_m copies unit 0 into outputs 0 and 7,
    with bias 0.25 on output 7.  So
      c_0 = silu(2.5) - 1,  m_0 = silu(c_0),  m_7 = silu(c_0) + 0.25,
    and every other output is 0.  A SiLU dropped, doubled or moved changes m_0."""
    cfg = _tiny(n_blocks=1)
    P = _zero_params(cfg)
    d = cfg.d_action
    P["action.t1.w"][0, 128] = 2.0
    P["action.t1.b"][0] = 0.5
    P["action.t2.w"] = np.eye(d, dtype=np.float32)
    P["action.t2.b"][0] = -1.0
    P["action.mod.w"][0, 0] = 1.0
    P["action.mod.w"][7, 0] = 1.0
    P["action.mod.b"][7] = 0.25
    m = M.modulation(cfg, P, "action", math.pi / 2000.0)

    def silu(z):
        return z / (1.0 + math.exp(-z))
    c0 = silu(2.5) - 1.0
    want = np.zeros(6 * d)
    want[0] = silu(c0)
    want[7] = silu(c0) + 0.25
    np.testing.assert_allclose(m, want, rtol=1e-13, atol=1e-13)
    # a dropped SiLU before the modulation map would give c_0 itself
    assert abs(m[0] - c0) > 0.2


def test_block_rest_ffn_activation_between_the_two_layers():
    """R_i with selection weights and (1 + sc2) = 0, so h2 = sh2 exactly.
    sh2_0 = -0.75 reaches hidden unit 0 through ffn1 (w = e_0 e_0^T, no bias);
    ffn2 copies hidden unit 0 into output 3 and adds b2.  The out-projection is
    zero apart from its bias, so x += g1 b_o + g2 (GELU_tanh(-0.75) e_3 + b2).
    GELU_tanh comes from torch; SiLU (-0.256), the identity (-0.75) or GELU
    after ffn2 would all give other values."""
    cfg = _tiny(n_blocks=1)
    P = _zero_params(cfg)
    d, F = cfg.d_action, cfg.ffn_action
    b = "action.blk0."
    rng = np.random.default_rng(23)
    P[b + "o.b"] = rng.standard_normal(d).astype(np.float32)
    P[b + "ffn1.w"][0, 0] = 1.0
    P[b + "ffn2.w"][3, 0] = 1.0
    P[b + "ffn2.b"] = rng.standard_normal(d).astype(np.float32)
    sh1, sc1, g1 = (rng.standard_normal(d) for _ in range(3))
    sh2 = np.zeros(d)
    sh2[0] = -0.75
    sc2 = -np.ones(d)
    g2 = rng.standard_normal(d)
    x = rng.standard_normal((1, 2, d))
    o = np.zeros((1, cfg.n_heads, 2, cfg.head_dim))
    got = M.block_rest(cfg, P, b, x, o, (sh1, sc1, g1, sh2, sc2, g2), 1.0)
    gelu = float(torch.nn.functional.gelu(torch.tensor(-0.75, dtype=torch.float64), approximate="tanh"))
    f = P[b + "ffn2.b"].astype(np.float64).copy()
    f[3] += gelu
    want = x + g1 * P[b + "o.b"] + g2 * f
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)
    assert abs(gelu - (-0.75 / (1 + math.exp(0.75)))) > 0.05 and abs(gelu + 0.75) > 0.5
