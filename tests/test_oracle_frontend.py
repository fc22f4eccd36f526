"""Pins of the pixel front-end oracle (oracle/frontend.py): the token and
feature index of individual pixels written out by hand, the shape of the
Flash-WAM setting, and the round trip."""
import numpy as np
import pytest

from oracle import frontend as FE


def test_patchify_index_closed_form():
    B, F, C, H, W, p = 2, 3, 3, 16, 24, 8
    frames = np.arange(B * F * C * H * W, dtype=np.float64).reshape(B, F, C, H, W)
    x = FE.patchify(frames, p)
    assert x.shape == (B, F * 2 * 3, C * 64)
    # pixel (b=1, f=2, c=1, y=13, x=18): patch row 1, column 2, offsets (5, 2)
    # -> token 2*6 + 1*3 + 2 = 17, feature 1*64 + 5*8 + 2 = 106
    assert x[1, 17, 106] == frames[1, 2, 1, 13, 18]
    # pixel (0, 0, 2, 7, 23) -> token 0*6 + 0*3 + 2 = 2, feature 2*64 + 7*8 + 7 = 191
    assert x[0, 2, 191] == frames[0, 0, 2, 7, 23]
    assert x[0, 0, 0] == frames[0, 0, 0, 0, 0]


def test_flash_wam_shape_and_round_trip():
    rng = np.random.default_rng(0)
    frames = rng.standard_normal((1, 4, 3, 128, 128)).astype(np.float32)
    x = FE.patchify(frames, 8)
    assert x.shape == (1, 1024, 192)   # 4 frames x 16 x 16 patches of 3 x 8 x 8
    np.testing.assert_array_equal(FE.unpatchify(x, 4, 3, 128, 128, 8), frames)
    # a permutation: every pixel appears once
    np.testing.assert_array_equal(np.sort(x.ravel()), np.sort(frames.ravel()))


def test_patchify_rejects_ragged_frames():
    with pytest.raises(ValueError):
        FE.patchify(np.zeros((1, 1, 3, 12, 16)), 8)
