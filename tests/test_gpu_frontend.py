"""The pixel front-end (wam_patchify) against the oracle's patchify: an exact
rearrangement, so bitwise; the Flash-WAM frame size and a ragged one; and the
inverse."""
import numpy as np
import pytest

import mot_dit_b200 as W
from oracle import frontend as FE

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,F,C,H,Wd,p", [(1, 4, 3, 128, 128, 8), (2, 3, 3, 16, 24, 8), (1, 1, 2, 12, 20, 4)])
def test_patchify_is_the_oracle_rearrangement(B, F, C, H, Wd, p):
    rng = np.random.default_rng(B + F + H)
    frames = rng.standard_normal((B, F, C, H, Wd)).astype(np.float32)
    want = FE.patchify(frames, p)
    dev = torch.device("cuda", 0)
    tf = torch.from_numpy(frames).to(dev)
    tp = torch.full(want.shape, float("nan"), device=dev)
    W.patchify(tf, tp, B, F, C, H, Wd, p)
    back = torch.full_like(tf, float("nan"))
    W.patchify(back, tp, B, F, C, H, Wd, p, inverse=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(tp.cpu().numpy(), want)
    np.testing.assert_array_equal(back.cpu().numpy(), frames)
