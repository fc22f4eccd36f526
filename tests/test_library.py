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
])
def test_init_rejects_bad_config_without_device(bad):
    base = W.preset(2) if bad.get("dtype") == W.BF16 else W.preset(1)
    cfg = base.replace(**bad)
    h = C.c_void_p()
    st = W.lib().wam_init(C.byref(cfg), 0, C.byref(h))
    assert st == 1 and not h.value


def test_status_strings():
    L = W.lib()
    assert L.wam_status_str(0) == b"ok"
    assert L.wam_status_str(5) == b"device wait timed out"
    assert L.wam_last_error(None) == b""
