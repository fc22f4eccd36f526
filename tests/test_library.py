"""The C-ABI library on a host without a GPU: it loads, exports every entry
point include/wam.h declares, its presets match the oracle's shapes, and its
host-side argument checks reject bad input before touching a device."""
import ctypes as C
import os
import re

import pytest

import mot_dit_b200 as W
from oracle.config import PRESETS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "wam.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wam_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = W.lib()
    names = _declared()
    assert "wam_infer_chunk" in names and "wam_init" in names and len(names) >= 15
    for n in names:
        assert hasattr(L, n), n


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5])
def test_presets_match_oracle_shapes(k):
    c = W.preset(k)
    o = PRESETS[k]
    for f in ("n_blocks", "d_video", "d_action", "n_heads", "head_dim", "ffn_video", "ffn_action", "l_cond",
              "l_video", "l_action", "action_dim", "video_patch_dim", "batch", "lora_rank"):
        assert getattr(c, f) == getattr(o, f), f
    assert bool(c.video_has_output) == o.video_has_output
    assert c.dtype == (W.BF16 if o.dtype == "bf16" else W.FP32)


def test_unknown_preset_rejected():
    with pytest.raises(W.WamError):
        W.preset(9)


@pytest.mark.parametrize("bad", [
    dict(n_blocks=0), dict(head_dim=48, dtype=W.BF16), dict(head_dim=15), dict(l_action=0),
    dict(video_has_output=1), dict(d_video=100, dtype=W.BF16), dict(dtype=7), dict(batch=0),
    dict(d_video=2048, dtype=W.BF16), dict(d_action=1600),
])
def test_init_rejects_bad_config_without_device(bad):
    base = W.preset(2) if bad.get("dtype") == W.BF16 else W.preset(1)
    cfg = base.replace(**bad)
    h = C.c_void_p()
    st = W.lib().wam_init(C.byref(cfg), 0, C.byref(h))
    assert st == 1 and not h.value


def test_init_without_a_device_fails_cleanly():
    """A valid config on a host with no GPU: WAM_ERR_CUDA, *out left NULL,
    and the half-built context released (a second call behaves the same)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    cfg = W.preset(1)
    for _ in range(2):
        h = C.c_void_p()
        assert W.lib().wam_init(C.byref(cfg), 0, C.byref(h)) == 4 and not h.value


def test_status_strings():
    L = W.lib()
    assert L.wam_status_str(0) == b"ok"
    assert L.wam_status_str(5) == b"device wait timed out"
    assert L.wam_last_error(None) == b""


# ---------------------------------------------------------------- binding
def _shell(k):
    """A Wam object with preset k's shapes and no device context: the
    binding's buffer checks run, and a call that gets past them reaches the
    library with a NULL context (WAM_ERR_INVALID_ARG, nothing enqueued)."""
    w = W.Wam.__new__(W.Wam)
    w.cfg = W.preset(k)
    w._lib = W.lib()
    w._h = None
    return w


def test_binding_io_sizes_follow_the_config():
    assert _shell(2).io_sizes() == (1024 * 1536, 64 * 1536, 32 * 30)
    assert _shell(4).io_sizes() == (8 * 2048 * 1536, 8 * 64 * 1536, 8 * 32 * 30)
    assert _shell(5).io_sizes() == (1024 * 192, 0, 16 * 30)


def test_binding_rejects_buffers_the_library_would_misread():
    import numpy as np
    import torch
    w = _shell(1)
    nv, nc, na = w.io_sizes()
    video, noise = torch.zeros(nv), torch.zeros(na)
    with pytest.raises(W.WamError, match="device buffer") as e:      # host memory for a device entry point
        w.infer_chunk(video, None, noise, torch.zeros(na))
    assert e.value.status == 1
    with pytest.raises(W.WamError, match="device buffer"):
        w.action_step(noise, 1.0, 0.0)
    hv, hn, ho = (np.zeros(n, np.float32) for n in (nv, na, na))
    with pytest.raises(W.WamError, match="out: need"):                # wrong size
        w.infer_chunk_host(hv, None, hn, np.zeros(na + 1, np.float32))
    with pytest.raises(W.WamError, match="noise: need"):              # wrong dtype
        w.infer_chunk_host(hv, None, hn.astype(np.float64), ho)
    with pytest.raises(W.WamError, match="video: need"):              # not contiguous
        w.infer_chunk_host(torch.zeros(nv, 2)[:, 0], None, hn, ho)
    with pytest.raises(W.WamError, match="t_sched has 2 values"):
        w.infer_chunk_host(hv, None, hn, ho, S=2, t_sched=[1.0, 0.0])
    # well-formed host buffers pass the checks and reach the library
    with pytest.raises(W.WamError) as e:
        w.infer_chunk_host(hv, None, hn, ho, S=2, t_sched=[1.0, 0.5, 0.0])
    assert e.value.status == 1 and "need" not in str(e.value)


def test_header_compiles_as_c_and_links_from_c():
    """include/wam.h is a C header: a C99 program (tests/c_abi/abi_check.c)
    compiles with -pedantic -Werror, links against the library and gets the
    documented argument errors without a device."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(W.library_path())
    W.lib()  # raises if the library has not been built
    out_dir = os.path.join(lib_dir, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-L", lib_dir, "-lmotdit",
           f"-Wl,-rpath,{lib_dir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr


def test_noalloc_attention_refusals_without_a_device():
    """wam_op_attention_noalloc checks its arguments and its scratch limits
    before any CUDA call, so every refusal path runs on a host without a GPU
    (the pointers are dummies that are never dereferenced)."""
    L = W.lib()
    p = C.c_void_p(0x1000)

    def call(B=1, H=24, Lq=32, Lk=1120, Lc=1120, splits=9, ptrs=(p, p, p, p)):
        return L.wam_op_attention_noalloc(*ptrs, B, H, Lq, Lk, Lc, splits, None)
    assert call(splits=1) == 1                 # split-KV needs at least two splits
    assert call(Lq=65) == 1                    # at most 64 queries per (sample, head)
    assert call(Lq=0) == 1 and call(Lk=0) == 1 and call(B=0) == 1 and call(H=0) == 1
    assert call(Lk=1121) == 1                  # keys beyond the cache rows
    assert call(ptrs=(None, p, p, p)) == 1 and call(ptrs=(p, p, p, None)) == 1
    assert call(Lk=64 * 33, Lc=64 * 33, splits=33) == 2     # 33 non-empty splits: more than the combine holds
    assert call(B=8, H=64, Lq=64, Lk=128, Lc=128, splits=2) == 2   # 8*64*2 slots * 4224 floats > 2^21
    # more (sample, head) pairs than the 1024 tickets: the partials' limit
    # (at least two splits of 4224 floats each) already refuses beyond 248 pairs
    assert call(B=1025, H=1, Lq=1, Lk=128, Lc=128, splits=2) == 2
    assert call(B=248, H=1, Lq=1, Lk=128, Lc=128, splits=2, ptrs=(None, p, p, p)) == 1


def test_linear_tiled_refusals_without_a_device():
    """wam_op_linear_tiled refuses bad shapes and values before any CUDA call,
    for the swapped cluster form (mode 3) among them: every path below runs on
    a host without a GPU (the pointers are dummies that are never
    dereferenced)."""
    L = W.lib()
    p = C.c_void_p(0x1000)

    def call(M=32, N=768, K=1536, bn=128, mode=3, ctas=8, ptrs=(p, p, p, p)):
        return L.wam_op_linear_tiled(*ptrs, M, N, K, bn, mode, ctas, None)
    assert call(mode=4) == 1 and call(mode=-1) == 1      # no such form
    assert call(ctas=-1) == 1
    assert call(ptrs=(None, p, p, p)) == 1 and call(ptrs=(p, p, None, p)) == 1
    assert call(M=0) == 1 and call(N=0) == 1 and call(K=0) == 1
    assert call(mode=2, ctas=7) == 1                     # clusters of two: an even grid
    # mode 3: 2..8 CTAs per tile, dividing the k-blocks and the token tile's 4-column slices
    assert call(ctas=1) == 1 and call(ctas=9) == 1 and call(ctas=0) == 1
    assert call(ctas=5) == 1                             # 24 k-blocks
    assert call(K=1600, ctas=2) == 1                     # K/64 = 25: not a multiple of 2
    assert call(M=65) == 1                               # at most 64 tokens
    assert call(M=20, K=3 * 64 * 4, ctas=3) == 1         # 32 columns: 8 slices do not split in 3
