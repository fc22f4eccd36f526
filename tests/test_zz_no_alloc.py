"""The allocation-free split-KV attention entry point, through the C ABI.

Callers that cannot let the library allocate device memory while they run
(a control loop that must not call cudaMalloc after start-up, a process whose
device memory belongs to another allocator) use wam_op_attention_noalloc; its
scratch is a fixed array inside the library.  Its output must match the
allocating entry point, wam_op_attention, on two calls in a row (the second
call finds the first call's scratch contents), and a call beyond its scratch
limit must be refused.  This file runs last so that a failure here does not
hide the other tests.
"""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import model as M
from oracle.params import round_bf16
from wam_testlib import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(B, H, Lq, Lc, seed):
    rng = np.random.default_rng(seed)
    mk = lambda *s: torch.from_numpy(round_bf16(rng.standard_normal(s).astype(np.float32))).to(DEV).to(torch.bfloat16)
    return mk(B, H, Lq, 64), mk(B, H, Lc, 64), mk(B, H, Lc, 64)


def test_noalloc_attention_matches_allocating_entry_point_twice():
    """Two calls in a row.  The second has fewer (sample, head, split) slots
    than the first (24 against 216), so partials the first call left in the
    shared scratch would show up if the second read any of them.  Both entry
    points run the same kernel with the same split rule and a fixed-order
    combine: their outputs are bitwise equal, and both match the oracle."""
    cases = [(1, 24, 32, 1120, 1120, 9, 0), (2, 4, 16, 300, 310, 3, 1)]
    for B, H, Lq, Lk, Lc, splits, seed in cases:
        q, k, v = _case(B, H, Lq, Lc, seed)
        ref = torch.full((B * Lq, H * 64), float("nan"), device=DEV, dtype=torch.bfloat16)
        got = torch.full_like(ref, float("nan"))
        W.op_attention(W.BF16, q, k, v, ref, B, H, 64, Lq, Lk, Lc, splits=splits)
        W.op_attention_noalloc(q, k, v, got, B, H, Lq, Lk, Lc, splits)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
        g = got.float().cpu().numpy()
        assert np.isfinite(g).all()
        f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
        want = M.merge_heads(M.attention(f64(q), f64(k)[:, :, :Lk], f64(v)[:, :, :Lk])).reshape(B * Lq, H * 64)
        assert rel_l2(g, want) <= 1e-2


def test_noalloc_attention_refuses_beyond_its_scratch():
    q, k, v = _case(8, 64, 64, 128, 2)
    out = torch.zeros(8 * 64, 64 * 64, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(W.WamError) as e:   # 8*64*2 splits * 4224 floats > 2^21
        W.op_attention_noalloc(q, k, v, out, 8, 64, 64, 128, 128, 2)
    assert e.value.status == 2
    torch.cuda.synchronize()
