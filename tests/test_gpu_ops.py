"""Single-kernel parity on the GPU, through the C ABI: the tcgen05 GEMM (both
orientations, split-K), the fp32 SIMT GEMM, and the attention kernels (video
single pass, action split-KV, fp32) against the oracle's definitions."""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle.params import round_bf16
from wam_testlib import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV).to(torch.bfloat16)


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(DEV)


# Normal orientation: `splits` = persistent CTAs (0: one per SM); the
# k-blocks of all tiles are divided evenly between them (stream-K).
@pytest.mark.parametrize("M_,N,K,swap,splits", [
    (200, 384, 256, False, 1),     # ragged M tail, 2 x 3 tiles, one CTA walks all
    (200, 384, 256, False, 0),     # 24 k-blocks on 24 CTAs: every tile in 4 pieces
    (1088, 256, 128, False, 0),    # 8.5 row tiles
    (1088, 1536, 1536, False, 7),  # 7 CTAs: pieces of uneven length
    (1088, 1536, 1536, False, 0),  # out-projection shape on all SMs
    (32, 300, 512, True, 1),       # few tokens, ragged feature tail
    (32, 300, 512, True, 4),       # split-K, fixed-order reduction
    (16, 30, 768, True, 3),        # action out-projection shape
    (256, 128, 192, True, 1),      # 256-token column tile
])
def test_linear_bf16(M_, N, K, swap, splits):
    rng = np.random.default_rng(M_ + N + K)
    x = round_bf16(rng.standard_normal((M_, K)).astype(np.float32))
    w = round_bf16((0.05 * rng.standard_normal((N, K))).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    out = torch.full((M_, N), float("nan"), device=DEV)
    W.op_linear(W.BF16, _bf16(x), _bf16(w), _f32(b), out, M_, N, K, swap=swap, splits=splits)
    torch.cuda.synchronize()
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) < 2e-6


# Cluster forms of the 256-wide video tiles: mode 1, CTA pairs sharing each
# M = 256 tensor-core MMA (each CTA its own 128 rows of X and half of the 256
# rows of W); mode 2, single-CTA tiles in clusters of two, a tile split
# between the two CTAs of a cluster finished in column halves.  `ctas` =
# persistent CTAs.
@pytest.mark.parametrize("M_,N,K,ctas", [
    (1088, 1536, 6144, 108),  # FFN-down shape: 5 pair rows (the last pair's rank 1 past M) / 54 tiles split in two
    (1088, 4608, 1536, 90),   # QKV shape: two whole tiles per pair
    (1088, 1536, 1536, 0),    # out-projection shape on all SMs
    (200, 512, 256, 2),       # one pair walks every tile; M ends inside rank 1's rows
    (64, 256, 64, 0),         # one k-block in all; rank 1 has no valid row
    (300, 768, 512, 14),      # 7 pairs: pieces of uneven length, split tiles across clusters
    (1088, 1536, 1536, 108),  # out-projection shape, every tile split between the CTAs of one cluster
])
def test_linear_cluster_forms(M_, N, K, ctas):
    rng = np.random.default_rng(M_ + N + K + ctas)
    x = round_bf16(rng.standard_normal((M_, K)).astype(np.float32))
    w = round_bf16((0.05 * rng.standard_normal((N, K))).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    outs = []
    for mode in (1, 2, 0):
        out = torch.full((M_, N), float("nan"), device=DEV)
        W.op_linear_tiled(_bf16(x), _bf16(w), _f32(b), out, M_, N, K, bn=256, mode=mode, ctas=ctas)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.isfinite(got).all()
        # fp32 accumulation of K bf16 products against the exact sum
        assert rel_l2(got, ref) < 4e-6
        outs.append(got)
    # the three forms split k differently: agreement to rounding
    assert rel_l2(outs[0], outs[2]) < 4e-6
    # the cluster split and the global split-tile reduction add the same
    # pieces on the same stream-K split: the same bits
    assert np.array_equal(outs[1], outs[2])


@pytest.mark.parametrize("M_,N,K,ctas", [
    (1088, 4608, 1536, 108),  # the video QKV shape on 192-wide tiles: two whole tiles per CTA
    (200, 384, 256, 3),       # ragged rows, uneven stream-K pieces
    (300, 576, 512, 0),       # all SMs: split tiles
])
def test_linear_192_wide(M_, N, K, ctas):
    rng = np.random.default_rng(M_ + N + K)
    x = round_bf16(rng.standard_normal((M_, K)).astype(np.float32))
    w = round_bf16((0.05 * rng.standard_normal((N, K))).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    out = torch.full((M_, N), float("nan"), device=DEV)
    W.op_linear_tiled(_bf16(x), _bf16(w), _f32(b), out, M_, N, K, bn=192, mode=0, ctas=ctas)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) < 4e-6


# Swapped orientation (the action expert's 32-token GEMMs): each 128-feature
# tile split over a cluster of `ctas` CTAs, one equal k-range each, the pieces
# summed in shared memory (mode 3), against the exact sum and bitwise against
# the global split-tile reduction on the same split (op_linear, swap).
@pytest.mark.parametrize("M_,N,K,ctas", [
    (32, 768, 1536, 8),   # action out-projection shape: 6 tiles x 8 CTAs, 3 k-blocks each
    (32, 768, 3072, 8),   # action FFN-down shape: 6 k-blocks each
    (20, 300, 512, 4),    # ragged tokens and features: 3 tiles, 8-column shares
    (64, 256, 1024, 8),   # 64 tokens: a 64-wide token tile, 8-column shares
    (7, 130, 128, 2),     # one k-block per CTA, a second tile of 2 rows
])
def test_linear_swapped_cluster_reduce(M_, N, K, ctas):
    rng = np.random.default_rng(M_ * 7 + N + K + ctas)
    x = round_bf16(rng.standard_normal((M_, K)).astype(np.float32))
    w = round_bf16((0.05 * rng.standard_normal((N, K))).astype(np.float32))
    b = rng.standard_normal(N).astype(np.float32)
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    got_cr = torch.full((M_, N), float("nan"), device=DEV)
    W.op_linear_tiled(_bf16(x), _bf16(w), _f32(b), got_cr, M_, N, K, mode=3, ctas=ctas)
    got_tk = torch.full((M_, N), float("nan"), device=DEV)
    W.op_linear(W.BF16, _bf16(x), _bf16(w), _f32(b), got_tk, M_, N, K, swap=True, splits=ctas)
    torch.cuda.synchronize()
    a, t = got_cr.cpu().numpy(), got_tk.cpu().numpy()
    assert np.isfinite(a).all()
    assert rel_l2(a, ref) < 4e-6
    # the same pieces added in the same (k) order: the same bits
    assert np.array_equal(a, t)


def test_linear_swapped_cluster_reduce_rejects_bad_shapes():
    x = torch.zeros((32, 1536), device=DEV, dtype=torch.bfloat16)
    w = torch.zeros((768, 1536), device=DEV, dtype=torch.bfloat16)
    b = torch.zeros(768, device=DEV)
    out = torch.zeros((32, 768), device=DEV)
    for ctas in (1, 9, 5):  # outside 2..8, or not dividing the 24 k-blocks
        with pytest.raises(W.WamError):
            W.op_linear_tiled(x, w, b, out, 32, 768, 1536, mode=3, ctas=ctas)


def test_linear_cluster_forms_repeatable():
    """The same launch three times gives the same bits (fixed split points and
    fixed-order partial sums, whatever the timing of the clusters)."""
    M_, N, K = 1088, 1536, 6144
    rng = np.random.default_rng(5)
    x = _bf16(round_bf16(rng.standard_normal((M_, K)).astype(np.float32)))
    w = _bf16(round_bf16((0.05 * rng.standard_normal((N, K))).astype(np.float32)))
    b = _f32(rng.standard_normal(N).astype(np.float32))
    for mode in (1, 2):
        outs = []
        for _ in range(3):
            out = torch.empty((M_, N), device=DEV)
            W.op_linear_tiled(x, w, b, out, M_, N, K, bn=256, mode=mode, ctas=108)
            outs.append(out)
        torch.cuda.synchronize()
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


# Joint action attention: (sample, head) split over a cluster of CTAs.
@pytest.mark.parametrize("B,H,Lq,Lk,Lc,splits,ready", [
    (1, 24, 32, 1120, 1120, 0, 1088),  # the Fast-WAM-shaped action attention (4 splits), video rows early
    (1, 4, 32, 1120, 1120, 8, 0),      # 8 splits of 140 keys (ragged tiles)
    (2, 3, 16, 300, 310, 2, 256),      # 16 queries, a key list shorter than the cache
    (1, 2, 64, 200, 256, 4, 0),        # 64 queries, 50-key splits (one partial tile each)
    (3, 2, 7, 70, 70, 1, 70),          # one CTA per (sample, head): no merge
])
def test_attention_joint(B, H, Lq, Lk, Lc, splits, ready):
    q, k, v = _attn_case(B, H, 64, Lq, Lk, Lc, Lq + Lk + splits)
    q, k, v = (round_bf16(a) for a in (q, k, v))
    outs = []
    for rd in (ready, 0):
        out = torch.full((B * Lq, H * 64), float("nan"), device=DEV, dtype=torch.bfloat16)
        W.op_attention_joint(_bf16(q), _bf16(k), _bf16(v), out, B, H, Lq, Lk, Lc, ready=rd, splits=splits)
        torch.cuda.synchronize()
        outs.append(out.float().cpu().numpy())
    # reading the early rows before the wait changes only when they load
    assert np.array_equal(outs[0], outs[1])
    got = outs[0]
    q64, k64, v64 = q.astype(np.float64), k[:, :, :Lk].astype(np.float64), v[:, :, :Lk].astype(np.float64)
    ref = M.merge_heads(M.attention(q64, k64, v64)).reshape(B * Lq, H * 64)
    ref_absv = M.merge_heads(M.attention(q64, k64, np.abs(v64))).reshape(B * Lq, H * 64)
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) < 1e-2
    assert_elementwise(got, ref, ref_absv)


def test_linear_f32():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((70, 48)).astype(np.float32)
    w = rng.standard_normal((50, 48)).astype(np.float32)
    b = rng.standard_normal(50).astype(np.float32)
    out = torch.zeros(70, 50, device=DEV)
    W.op_linear(W.FP32, _f32(x), _f32(w), _f32(b), out, 70, 50, 48)
    torch.cuda.synchronize()
    ref = x.astype(np.float64) @ w.astype(np.float64).T + b
    assert rel_l2(out.cpu().numpy(), ref) < 1e-6


def _attn_case(B, H, Dh, Lq, Lk, Lc, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Lq, Dh)).astype(np.float32)
    k = rng.standard_normal((B, H, Lc, Dh)).astype(np.float32)
    v = rng.standard_normal((B, H, Lc, Dh)).astype(np.float32)
    return q, k, v


@pytest.mark.parametrize("B,H,Lq,Lk,Lc,splits", [
    (2, 3, 100, 100, 130, 1),      # video: ragged queries and keys
    (1, 2, 1088, 1088, 1120, 1),   # full video length
    (1, 4, 32, 1120, 1120, 9),     # action: joint keys, split-KV
    (2, 2, 16, 300, 310, 3),       # action, 16 queries, ragged split
])
def test_attention_bf16(B, H, Lq, Lk, Lc, splits):
    q, k, v = _attn_case(B, H, 64, Lq, Lk, Lc, Lq + Lk)
    q, k, v = (round_bf16(a) for a in (q, k, v))
    out = torch.full((B * Lq, H * 64), float("nan"), device=DEV, dtype=torch.bfloat16)
    W.op_attention(W.BF16, _bf16(q), _bf16(k), _bf16(v), out, B, H, 64, Lq, Lk, Lc, splits=splits)
    torch.cuda.synchronize()
    q64, k64, v64 = q.astype(np.float64), k[:, :, :Lk].astype(np.float64), v[:, :, :Lk].astype(np.float64)
    ref = M.merge_heads(M.attention(q64, k64, v64)).reshape(B * Lq, H * 64)
    ref_absv = M.merge_heads(M.attention(q64, k64, np.abs(v64))).reshape(B * Lq, H * 64)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) < 1e-2
    assert_elementwise(got, ref, ref_absv)


def assert_elementwise(got, ref, ref_absv):
    """Every output element within 2^-8 (|o| + sum_k p_k |v_k| / l), where
    ref_absv is the oracle's attention over |V| (sum_k p_k |v_k| / l).  The
    kernel rounds the output to bf16 (at most 2^-9 |o|) and each probability
    p_k of the PV product to bf16 (at most 2^-9 p_k each, so at most
    2^-9 sum_k p_k |v_k| / l in all); the bound is twice that worst case.  A
    wrong key row, head or split, or a stale partial, is far outside it."""
    ref = np.asarray(ref, np.float64)
    bound = 2.0 ** -8 * (np.abs(ref) + np.asarray(ref_absv, np.float64))
    err = np.abs(np.asarray(got, np.float64) - ref)
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} elements out of bound, worst excess {float((err - bound).max()):.3e}"


def test_video_attention_repeatable_at_full_load():
    """The tcgen05 kernel's hand-offs (S / P / O through TMEM and shared
    memory) are ordered by barriers, not by timing: at the 8 x 2112-token
    shape (every SM busy, 17 key tiles per row) repeated launches agree
    bitwise, and every head of every sample matches the oracle."""
    B, H, L = 8, 24, 2112
    q, k, v = _attn_case(B, H, 64, L, L, L, 4242)
    q, k, v = (round_bf16(a) for a in (q, k, v))
    tq, tk, tv = _bf16(q), _bf16(k), _bf16(v)
    outs = []
    for _ in range(6):
        out = torch.full((B * L, H * 64), float("nan"), device=DEV, dtype=torch.bfloat16)
        W.op_attention(W.BF16, tq, tk, tv, out, B, H, 64, L, L, L, splits=1)
        outs.append(out)
    torch.cuda.synchronize()
    first = outs[0].float().cpu().numpy()
    for o in outs[1:]:
        assert np.array_equal(first, o.float().cpu().numpy())
    got = first.reshape(B, L, H, 64)
    for b in range(B):   # every (sample, head) against the oracle
        q64, k64, v64 = (x[b:b + 1].astype(np.float64) for x in (q, k, v))
        ref = M.attention(q64, k64, v64)[0]
        ref_absv = M.attention(q64, k64, np.abs(v64))[0]
        for h in range(H):
            assert rel_l2(got[b, :, h], ref[h]) < 1e-2, (b, h)
            assert_elementwise(got[b, :, h], ref[h], ref_absv[h])


def test_attention_f32():
    B, H, Dh, Lq, Lk, Lc = 1, 4, 16, 80, 80, 96
    q, k, v = _attn_case(B, H, Dh, Lq, Lk, Lc, 7)
    out = torch.zeros(B * Lq, H * Dh, device=DEV)
    W.op_attention(W.FP32, _f32(q), _f32(k), _f32(v), out, B, H, Dh, Lq, Lk, Lc)
    torch.cuda.synchronize()
    ref = M.merge_heads(M.attention(q.astype(np.float64), k[:, :, :Lk].astype(np.float64),
                                    v[:, :, :Lk].astype(np.float64))).reshape(B * Lq, H * Dh)
    assert rel_l2(out.cpu().numpy(), ref) < 1e-5


@pytest.mark.parametrize("dtype,rows,d,mode", [(W.BF16, 1088, 1536, "mod"), (W.BF16, 32, 768, "mod"),
                                             (W.BF16, 37, 768, "gain"), (W.FP32, 80, 64, "mod")])
def test_norm_modulation(dtype, rows, d, mode):
    """rms(x)(1 + scale) + shift (block prologue) and rms(x) * gain (final norm)."""
    rng = np.random.default_rng(rows + d)
    x = (3.0 * rng.standard_normal((rows, d))).astype(np.float32)
    sc, sh, g = (rng.standard_normal(d).astype(np.float32) * 0.1 for _ in range(3))
    tdt = torch.bfloat16 if dtype == W.BF16 else torch.float32
    h = torch.full((rows, d), float("nan"), device=DEV, dtype=tdt)
    if mode == "mod":
        W.op_norm_mod(dtype, _f32(x), h, rows, d, scale=_f32(sc), shift=_f32(sh))
        ref = M.modulate(x.astype(np.float64), sh.astype(np.float64), sc.astype(np.float64))
    else:
        W.op_norm_mod(dtype, _f32(x), h, rows, d, gain=_f32(g))
        ref = M.rms_norm(x.astype(np.float64)) * g
    torch.cuda.synchronize()
    got = h.float().cpu().numpy()
    assert rel_l2(got, ref) < (4e-3 if dtype == W.BF16 else 1e-6)
