"""Token coordinates without integer division, as the prologue kernels take
them: n / d = umulhi(n, m) with m = ceil(2^32 / d), exact while
n * (m d - 2^32) < 2^32 (the host checks that bound for every video token and
otherwise lets the kernels divide).  Checked exhaustively over the video
tokens of every workload's grid, and on a grid where the bound fails."""
import numpy as np
import pytest

from int4_quantized_attention_b200 import synth


def magic(d):
    return -(-(1 << 32) // d)      # ceil(2^32 / d)


def bound_ok(d, n_video):
    m = magic(d)
    return d == 1 or n_video * (m * d - (1 << 32)) < (1 << 32)


def umulhi_div(n, d):
    if d == 1:
        return n
    return (n.astype(np.uint64) * np.uint64(magic(d))) >> np.uint64(32)


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_coordinates_of_every_video_token(name):
    cfg = synth.CONFIGS[name]
    nv = cfg.F * cfg.Hh * cfg.W
    if nv == 0:
        return
    n = np.arange(nv, dtype=np.uint64)
    for d in (cfg.W, cfg.Hh * cfg.W):
        assert bound_ok(d, nv)
        assert np.array_equal(umulhi_div(n, d), n // np.uint64(d))
    f = umulhi_div(n, cfg.Hh * cfg.W)
    nw = umulhi_div(n, cfg.W)
    h = nw - f * np.uint64(cfg.Hh)
    w = n - nw * np.uint64(cfg.W)
    assert np.array_equal(f, n // np.uint64(cfg.Hh * cfg.W))
    assert np.array_equal(h, (n // np.uint64(cfg.W)) % np.uint64(cfg.Hh))
    assert np.array_equal(w, n % np.uint64(cfg.W))


def test_bound_detects_where_the_multiplier_fails():
    # 2^32 mod (2^16 + 1) = 1, so m d - 2^32 = 2^16: the bound holds only for
    # fewer than 2^16 tokens, and past 2^16 the shortcut gives wrong quotients
    d = (1 << 16) + 1
    assert bound_ok(d, (1 << 16) - 1) and not bound_ok(d, 1 << 18)
    n = np.arange((1 << 16) - 1, dtype=np.uint64)
    assert np.array_equal(umulhi_div(n, d), n // np.uint64(d))
    n = np.arange(1 << 18, dtype=np.uint64)
    assert not np.array_equal(umulhi_div(n, d), n // np.uint64(d))
