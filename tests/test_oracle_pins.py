"""Pins for the CPU oracle: each test checks it against something other than
itself -- a constant the pages print (tests/golden), a closed form, an
invariant, or a library routine (numpy matmul / softmax) -- chosen so that a
plausible slip (dropped term, wrong sign or index, transposed operand) fails.
"""
import json
import math
import os

import numpy as np
import pytest

from int4_quantized_attention_b200 import synth
from int4_quantized_attention_b200.schedule import Schedule

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_cfg(**kw):
    base = synth.Config("t", 1, 1, 2, 3, 4, 0, (44, 42, 42), "none", "normal", 1)
    return base.replace(**kw)


def cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


# ---------------------------------------------------------------- constants

def test_p_map_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "p_map.json")))
    for P, code in g["endpoints"]:
        assert oracle_mod.p_code(P) == code
    lo, hi = g["code_range"]
    # P = k / scale maps exactly onto code k + zero_point (k = 0..15)
    for kk in range(16):
        assert oracle_mod.p_code(np.float32(kk) / np.float32(g["scale"])) == kk + g["zero_point"]
    grid = np.linspace(0.0, 1.0, 20001, dtype=np.float32)
    codes = np.array([oracle_mod.p_code(float(x)) for x in grid])
    assert codes.min() == lo and codes.max() == hi
    assert np.all(np.diff(codes) >= 0)
    # quantisation error of the affine map is at most half a step: 1/30
    assert np.max(np.abs((codes - g["zero_point"]) / g["scale"] - grid)) <= 1.0 / 30 + 1e-7


def test_p_map_symmetric_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "p_map_symmetric.json")))
    for P, code in g["endpoints"]:
        assert oracle_mod.p_code_sym(P) == code
    lo, hi = g["code_range"]
    for kk in range(8):
        assert oracle_mod.p_code_sym(np.float32(kk) / np.float32(g["scale"])) == kk + g["zero_point"]
    grid = np.linspace(0.0, 1.0, 20001, dtype=np.float32)
    codes = np.array([oracle_mod.p_code_sym(float(x)) for x in grid])
    assert codes.min() == lo and codes.max() == hi
    assert np.all(np.diff(codes) >= 0)
    # half a step of the symmetric map is 1/14: twice the range-optimised 1/30
    assert np.max(np.abs(codes / g["scale"] - grid)) <= 1.0 / 14 + 1e-7
    # round half to even at the step midpoints, like the range-optimised map
    assert oracle_mod.p_code_sym(0.5 / 7) == 0 and oracle_mod.p_code_sym(1.5 / 7) == 2


def test_p_weight_matches_the_p_map(oracle_mod):
    """The quantised path decides w = rne(levels 2^x) from the exponent in log2
    units (P = 2^x): it must agree with the golden P maps, code = w - 8
    (range-optimised, 15 levels) or w (symmetric, 7 levels), at the endpoints,
    at every exact level, and wherever levels * P is not within float
    rounding of a half-integer; it is monotone, and the one exact tie,
    x = -1 (15 / 2 = 7.5), rounds half to even."""
    g = json.load(open(os.path.join(GOLDEN, "p_map.json")))
    gs = json.load(open(os.path.join(GOLDEN, "p_map_symmetric.json")))
    for golden, levels, zp in ((g, 15, 8), (gs, 7, 0)):
        for P, code in golden["endpoints"]:
            x = -math.inf if P == 0.0 else math.log2(P)
            assert oracle_mod.p_weight(x, levels) - zp == code
        for kk in range(1, levels + 1):
            assert oracle_mod.p_weight(float(np.float32(math.log2(kk / levels))), levels) == kk
    assert oracle_mod.p_weight(-1.0, 15) == 8 and oracle_mod.p_weight(-1.0, 7) == 4   # 7.5 -> 8, 3.5 -> 4
    xs = np.linspace(-8.0, 0.0, 40001, dtype=np.float32)
    w = np.array([oracle_mod.p_weight(float(x), 15) for x in xs])
    assert np.all(np.diff(w) >= 0) and w[0] == 0 and w[-1] == 15
    exact = 15.0 * np.exp2(xs.astype(np.float64))
    away = np.abs(exact - np.floor(exact) - 0.5) > 1e-5
    codes = np.array([oracle_mod.p_code(float(np.exp2(np.float64(x)))) for x in xs])
    assert np.array_equal(w[away], codes[away] + 8)
    assert np.max(np.abs(w / 15.0 - np.exp2(xs.astype(np.float64)))) <= 1.0 / 30 + 1e-12
    # at every rounding boundary, float by float: w steps up exactly at the
    # first fp32 x with levels * 2^x >= k + 1/2 (extended precision here)
    ld = np.longdouble
    for levels in (15, 7):
        for k in range(levels):
            edge = np.log2(ld(2 * k + 1) / ld(2 * levels))
            x = np.float32(edge)
            for _ in range(3):
                x = np.nextafter(x, np.float32(-np.inf))
            for _ in range(7):
                want = k + 1 if ld(x) >= edge else k
                assert oracle_mod.p_weight(float(x), levels) == want, (levels, k, float(x))
                x = np.nextafter(x, np.float32(np.inf))


def test_ambiguous_weights_are_those_near_a_boundary(oracle_mod):
    """orc_p_weight_amb: the same weight as orc_p_weight, flagged ambiguous
    exactly where levels * 2^x lies within 2^-20 (relative) of a half-integer:
    the floats next to every rounding boundary are, exact levels and the
    zero region are not."""
    ld = np.longdouble
    rel = 2.0 ** -20
    for levels in (15, 7):
        for k in range(levels):
            edge = np.log2(ld(2 * k + 1) / ld(2 * levels))
            x = np.float32(edge)
            for _ in range(2):
                x = np.nextafter(x, np.float32(-np.inf))
            for _ in range(5):
                w, amb = oracle_mod.p_weight_amb(float(x), levels)
                assert w == oracle_mod.p_weight(float(x), levels)
                v = levels * np.exp2(ld(x))
                assert amb == bool(abs(v - (k + ld(0.5))) <= v * ld(rel)), (levels, k, float(x))
                assert amb                              # the two floats either side are that close
                x = np.nextafter(x, np.float32(np.inf))
        for kk in range(1, levels + 1):                 # exact levels: half a unit from any boundary
            assert not oracle_mod.p_weight_amb(float(np.float32(math.log2(kk / levels))), levels)[1]
        assert not oracle_mod.p_weight_amb(-30.0, levels)[1]


def test_flipping_an_ambiguous_key(oracle_mod):
    """A key whose exponent is exactly -1 (15 / 2 = 7.5, the one exact tie) is
    ambiguous; the oracle's row rounds it to 8 (half to even), the flipped row
    to 7, and both equal the closed form sum w v / sum w on one tile."""
    cfg = small_cfg(F=2, Hh=8, W=8, rot="none")                        # N = 128: one tile
    qc = np.zeros((128, 128), np.int8)
    qc[:, 0] = 1
    kc = np.zeros((128, 128), np.int8)
    kc[5, 0] = 7                                 # the row max, S = 7
    kc[9, 0] = -1                                # S = -1
    # scales: c = fl(fl(s_Q K) s_K) = 1/8 exactly with s_Q = 1 and this s_K
    # (K = fl(log2 e) / fl(sqrt 128)), so x = (S - 7) / 8: -1 for key 9
    ks = np.full(2, np.float32(0.9802581071853638), np.float32)
    qz = dict(qc=qc, qs=np.ones(2, np.float32), kc=kc, ks=ks)
    rng = np.random.default_rng(16)
    vc = rng.integers(-7, 8, (128, 128)).astype(np.int8)
    qz.update(vc=vc, sv=np.ones(128, np.float32),
              colsum=vc.astype(np.int32).reshape(2, 64, 128).sum(axis=1).astype(np.int32))
    (o, o64), cnt, keys = oracle_mod.attention_rows(cfg, qz, rows=np.array([0]), want64=True, ambiguous=True)
    assert cnt[0] == 1 and keys[0, 0] == 9
    S = kc[:, 0].astype(np.float64)
    w = np.rint(15 * np.exp2((S - 7) / 8))
    assert w[9] == 8 and w[5] == 15
    ref = (w @ vc.astype(np.float64)) / w.sum()
    assert np.allclose(o64[0], ref, rtol=1e-12, atol=1e-12)
    w2 = w.copy()
    w2[9] = 7
    ref2 = (w2 @ vc.astype(np.float64)) / w2.sum()
    got2 = oracle_mod.attention_row_flipped(cfg, qz, 0, [9])
    assert np.allclose(got2, ref2, rtol=1e-12, atol=1e-12)
    assert not np.allclose(got2, ref, rtol=1e-6)
    _, P, mask = oracle_mod.attention_row_debug(cfg, qz, 0, 0, with_ambiguous=True)
    assert mask[9] and mask.sum() == 1 and P[9] == 0


def test_schedule_golden():
    g = json.load(open(os.path.join(GOLDEN, "schedule.json")))
    for c in g["cases"]:
        s = Schedule(c["steps"], c["blocks"], c["first_steps"], c["last_steps"],
                     c["first_blocks"], c["last_blocks"])
        assert round(100 * s.int4_fraction) == c["int4_percent"]


# ---------------------------------------------------------------- 3D RoPE

def test_token_positions(oracle_mod):
    cfg = small_cfg(F=3, Hh=4, W=5, n_text=2)
    assert oracle_mod.token_pos(cfg, 0) == (0, 0, 0)
    assert oracle_mod.token_pos(cfg, 1) == (0, 0, 1)
    assert oracle_mod.token_pos(cfg, 5) == (0, 1, 0)
    assert oracle_mod.token_pos(cfg, 20) == (1, 0, 0)
    assert oracle_mod.token_pos(cfg, 3 * 4 * 5 - 1) == (2, 3, 4)
    assert oracle_mod.token_pos(cfg, 60) == (0, 0, 0)      # text tokens: no RoPE
    assert oracle_mod.token_pos(cfg, 61) == (0, 0, 0)


def test_rope_frequencies(oracle_mod):
    cfg = small_cfg()
    for s, ds in enumerate(cfg.split):
        assert oracle_mod.rope_angle(cfg, s, 0, 3) == 0.0
        assert oracle_mod.rope_angle(cfg, s, 7, 0) == pytest.approx(7.0, rel=1e-15)
        # geometric progression with ratio theta^(-2/d_s) from pair to pair
        ratio = cfg.theta ** (-2.0 / ds)
        for j in range(ds // 2 - 1):
            a0 = oracle_mod.rope_angle(cfg, s, 5, j)
            a1 = oracle_mod.rope_angle(cfg, s, 5, j + 1)
            assert a1 / a0 == pytest.approx(ratio, rel=1e-12)
        # linear in position
        assert oracle_mod.rope_angle(cfg, s, 6, 2) == pytest.approx(
            2 * oracle_mod.rope_angle(cfg, s, 3, 2), rel=1e-14)


def unit(d, i):
    x = np.zeros((d,), np.float16)
    x[i] = 1.0
    return x


def test_rope_identity_at_origin(oracle_mod):
    cfg = small_cfg(n_text=1)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((cfg.N, 128)).astype(np.float16)
    z = oracle_mod.rotate_head(cfg, x, rot="none")
    # token 0 sits at (0,0,0), the text token too: RoPE is the identity, bit-exact
    assert np.array_equal(z[0], x[0].astype(np.float32))
    assert np.array_equal(z[-1], x[-1].astype(np.float32))


def test_rope_rotates_pairs_counterclockwise(oracle_mod):
    cfg = small_cfg(F=5, Hh=6, W=7)
    n = 4 * 42 + 3 * 7 + 5          # (f, h, w) = (4, 3, 5)
    assert oracle_mod.token_pos(cfg, n) == (4, 3, 5)
    offs = [0, 44, 86]
    for s, pos in zip(range(3), (4, 3, 5)):
        for j in (0, 1, cfg.split[s] // 2 - 1):
            a = oracle_mod.rope_angle(cfg, s, pos, j)
            i0 = offs[s] + 2 * j
            x = np.zeros((cfg.N, 128), np.float16)
            x[n] = unit(128, i0)
            z = oracle_mod.rotate_head(cfg, x, rot="none")[n]
            assert z[i0] == pytest.approx(math.cos(a), abs=1e-6)
            assert z[i0 + 1] == pytest.approx(math.sin(a), abs=1e-6)
            x[n] = unit(128, i0 + 1)
            z = oracle_mod.rotate_head(cfg, x, rot="none")[n]
            assert z[i0] == pytest.approx(-math.sin(a), abs=1e-6)
            assert z[i0 + 1] == pytest.approx(math.cos(a), abs=1e-6)
            assert np.count_nonzero(z) <= 2


@pytest.mark.parametrize("rot", ["none", "interleaved", "half", "full"])
def test_rope_relative_position(oracle_mod, rot):
    """q(p+D).k(p'+D) == q(p).k(p'): only the offset along each axis matters."""
    cfg = small_cfg(F=4, Hh=5, W=6, rot=rot)
    rng = np.random.default_rng(1)
    qv = rng.standard_normal(128).astype(np.float16)
    kv = rng.standard_normal(128).astype(np.float16)
    x = np.zeros((cfg.N, 128), np.float16)
    x[:] = qv
    zq = oracle_mod.rotate_head(cfg, x).astype(np.float64)
    x[:] = kv
    zk = oracle_mod.rotate_head(cfg, x).astype(np.float64)

    def tok(f, h, w):
        return (f * cfg.Hh + h) * cfg.W + w

    base = zq[tok(0, 1, 2)] @ zk[tok(1, 0, 0)]
    shifted = zq[tok(2, 4, 5)] @ zk[tok(3, 3, 3)]
    scale = np.linalg.norm(qv.astype(np.float64)) * np.linalg.norm(kv.astype(np.float64))
    assert abs(base - shifted) <= 2e-6 * scale
    other = zq[tok(0, 1, 2)] @ zk[tok(2, 0, 0)]          # a different offset differs
    assert abs(base - other) > 1e-3 * scale


# ---------------------------------------------------------------- rotation

def test_interleaved_is_h2_on_adjacent_pairs(oracle_mod):
    cfg = small_cfg(rot="interleaved")
    r = 1.0 / math.sqrt(2.0)
    for i0 in (0, 2, 42, 44, 86, 126):
        x = np.zeros((cfg.N, 128), np.float16)
        x[0] = unit(128, i0)                       # token 0: RoPE is the identity
        z = oracle_mod.rotate_head(cfg, x)[0]
        assert z[i0] == pytest.approx(r, abs=1e-7) and z[i0 + 1] == pytest.approx(r, abs=1e-7)
        x[0] = unit(128, i0 + 1)
        z = oracle_mod.rotate_head(cfg, x)[0]
        assert z[i0] == pytest.approx(r, abs=1e-7) and z[i0 + 1] == pytest.approx(-r, abs=1e-7)
        assert np.count_nonzero(z) == 2


def test_half_pairs_opposite_half_segments(oracle_mod):
    cfg = small_cfg(rot="half", split=(44, 42, 42))
    r = 1.0 / math.sqrt(2.0)
    for off, ds in ((0, 44), (44, 42), (86, 42)):
        h = ds // 2
        for i in (0, 1, h - 1):
            x = np.zeros((cfg.N, 128), np.float16)
            x[0] = unit(128, off + i)
            z = oracle_mod.rotate_head(cfg, x)[0]
            nz = np.nonzero(z)[0].tolist()
            assert nz == [off + i, off + i + h]
            assert z[off + i] == pytest.approx(r, abs=1e-7)
            assert z[off + i + h] == pytest.approx(r, abs=1e-7)
            x[0] = unit(128, off + i + h)
            z = oracle_mod.rotate_head(cfg, x)[0]
            assert z[off + i] == pytest.approx(r, abs=1e-7)
            assert z[off + i + h] == pytest.approx(-r, abs=1e-7)


@pytest.mark.parametrize("rot", ["interleaved", "half", "full"])
@pytest.mark.parametrize("split", [(44, 42, 42), (16, 56, 56)])
def test_rotation_is_orthogonal(oracle_mod, rot, split):
    """QR.(KR)^T == QK^T and |xR| == |x| (the paper's orthogonality argument)."""
    cfg = small_cfg(F=3, Hh=4, W=5, n_text=3, split=split)
    rng = np.random.default_rng(2)
    q = (rng.standard_normal((cfg.N, 128)) * 3).astype(np.float16)
    k = (rng.standard_normal((cfg.N, 128)) * 3).astype(np.float16)
    yq = oracle_mod.rotate_head(cfg, q, rot="none").astype(np.float64)
    yk = oracle_mod.rotate_head(cfg, k, rot="none").astype(np.float64)
    zq = oracle_mod.rotate_head(cfg.replace(rot=rot), q).astype(np.float64)
    zk = oracle_mod.rotate_head(cfg.replace(rot=rot), k).astype(np.float64)
    ref = yq @ yk.T
    assert np.max(np.abs(zq @ zk.T - ref)) <= 1e-5 * np.max(np.abs(ref))
    assert np.allclose(np.linalg.norm(zq, axis=1), np.linalg.norm(yq, axis=1), rtol=1e-6)
    # it really rotates: the coordinates change
    assert np.max(np.abs(zq - yq)) > 0.1


def test_full_rotation_is_the_normalised_hadamard(oracle_mod):
    """Full rotation == RoPE output times H/sqrt(128), H the Sylvester
    Hadamard matrix (scipy), in float64, to fp32 rounding."""
    from scipy.linalg import hadamard
    cfg = small_cfg(F=2, Hh=3, W=4, n_text=2)
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((cfg.N, 128)) * 2).astype(np.float16)
    y = oracle_mod.rotate_head(cfg, x, rot="none").astype(np.float64)
    z = oracle_mod.rotate_head(cfg.replace(rot="full"), x).astype(np.float64)
    ref = y @ (hadamard(128).astype(np.float64) / math.sqrt(128))
    assert np.max(np.abs(z - ref)) <= 4e-6 * np.max(np.abs(ref))
    # a single channel spreads evenly over all 128 outputs
    e = np.zeros((1, 128), np.float16)
    e[0, 5] = 1
    zz = oracle_mod.rotate_head(small_cfg(F=0, Hh=0, W=0, n_text=1, rot="full"), e)
    assert np.allclose(np.abs(zz), 1 / math.sqrt(128), rtol=1e-6)


def _block_diag(blocks, split, mode):
    """The d x d matrix (column-vector convention z = M y) of the pair blocks."""
    M = np.zeros((128, 128))
    o = 0
    for seg in split:
        h = seg // 2
        for j in range(h):
            p = o // 2 + j
            r = np.array(blocks[4 * p:4 * p + 4]).reshape(2, 2)
            a, b = (o + 2 * j, o + 2 * j + 1) if mode == "blocks_interleaved" else (o + j, o + j + h)
            M[np.ix_([a, b], [a, b])] = r
        o += seg
    return M


@pytest.mark.parametrize("mode", ["blocks_interleaved", "blocks_half"])
@pytest.mark.parametrize("split", [(44, 42, 42), (16, 56, 56)])
def test_learned_blocks_are_the_block_diagonal_matrix(oracle_mod, mode, split):
    """Caller blocks: z = B (RoPE y) with B block-diagonal over the pairs of the
    mode (numpy, float64) to fp32 rounding; QK^T and norms preserved; with the
    exact H2 blocks the modes reproduce Interleaved / Half to fp32 rounding."""
    blocks = synth.random_pair_blocks(31)
    cfg = small_cfg(F=2, Hh=3, W=4, n_text=2, split=split, rot=mode, blocks=blocks)
    rng = np.random.default_rng(4)
    q = (rng.standard_normal((cfg.N, 128)) * 2).astype(np.float16)
    k = (rng.standard_normal((cfg.N, 128)) * 2).astype(np.float16)
    y = oracle_mod.rotate_head(cfg, q, rot="none").astype(np.float64)
    yk = oracle_mod.rotate_head(cfg, k, rot="none").astype(np.float64)
    z = oracle_mod.rotate_head(cfg, q).astype(np.float64)
    zk = oracle_mod.rotate_head(cfg, k).astype(np.float64)
    ref = y @ _block_diag(blocks, split, mode).T
    assert np.max(np.abs(z - ref)) <= 2e-6 * np.max(np.abs(ref))
    qk = y @ yk.T
    assert np.max(np.abs(z @ zk.T - qk)) <= 1e-5 * np.max(np.abs(qk))
    h2 = tuple([math.sqrt(0.5), math.sqrt(0.5), math.sqrt(0.5), -math.sqrt(0.5)] * 64)
    std = "interleaved" if mode == "blocks_interleaved" else "half"
    zh = oracle_mod.rotate_head(cfg.replace(blocks=h2), q).astype(np.float64)
    zs = oracle_mod.rotate_head(cfg.replace(rot=std, blocks=None), q).astype(np.float64)
    assert np.max(np.abs(zh - zs)) <= 2e-6 * np.max(np.abs(zs))


# ---------------------------------------------------------------- quantisers

@pytest.mark.parametrize("rot", ["interleaved", "half", "full"])
def test_qk_quantiser_properties(oracle_mod, rot):
    cfg = small_cfg(F=2, Hh=10, W=10, n_text=16, rot=rot)     # N = 216: ragged 64-blocks
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((cfg.N, 128)) * rng.lognormal(0, 1, 128)).astype(np.float16)
    x[64:128] = 0                                              # an all-zero block
    codes, scales = oracle_mod.quantize_qk_head(cfg, x)
    z = oracle_mod.rotate_head(cfg, x)
    N, Np = cfg.N, oracle_mod.n_pad(cfg)
    assert codes.shape == (Np, 128) and scales.shape == (Np // 64,)
    assert np.all(codes[N:] == 0) and np.all(scales[(N + 63) // 64:] == 0)
    assert scales[1] == 0 and np.all(codes[64:128] == 0)
    for g in range((N + 63) // 64):
        blk = z[64 * g:min(64 * g + 64, N)]
        amax = np.abs(blk).max()
        assert scales[g] == np.float32(amax) / np.float32(7)
        if amax == 0:
            continue
        c = codes[64 * g:64 * g + len(blk)].astype(np.float64)
        assert np.abs(c).max() == 7
        assert np.all(np.abs(c * scales[g] - blk) <= 0.5 * scales[g] * (1 + 1e-6))
        # rounding to nearest: no other code is closer
        assert np.all(np.abs(c * scales[g] - blk) <= np.abs((c + 1) * scales[g] - blk) + 1e-6 * scales[g])
        assert np.all(np.abs(c * scales[g] - blk) <= np.abs((c - 1) * scales[g] - blk) + 1e-6 * scales[g])


def test_qk_blocks_are_independent(oracle_mod):
    cfg = small_cfg(F=2, Hh=8, W=16, rot="half")               # N = 256
    rng = np.random.default_rng(4)
    x = rng.standard_normal((cfg.N, 128)).astype(np.float16)
    c0, s0 = oracle_mod.quantize_qk_head(cfg, x)
    x[130, 5] = 100.0                                          # token 130 is in block 2
    c1, s1 = oracle_mod.quantize_qk_head(cfg, x)
    changed = np.nonzero(s0 != s1)[0].tolist()
    assert changed == [2]
    assert np.array_equal(c0[:128], c1[:128]) and np.array_equal(c0[192:], c1[192:])


def test_v_quantiser_properties(oracle_mod):
    cfg = small_cfg(F=3, Hh=7, W=9)                            # N = 189
    rng = np.random.default_rng(5)
    v = (rng.standard_normal((cfg.N, 128)) * rng.lognormal(0, 1, 128)).astype(np.float16)
    v[:, 7] = 0
    codes, sv, colsum = oracle_mod.quantize_v_head(cfg, v)
    N, Np = cfg.N, oracle_mod.n_pad(cfg)
    vf = v.astype(np.float32)
    assert np.array_equal(sv, np.abs(vf).max(axis=0) / np.float32(7))
    assert sv[7] == 0 and np.all(codes[:, 7] == 0)
    c = codes[:N].astype(np.float64)
    nz = sv > 0
    assert np.all(np.abs(c[:, nz]).max(axis=0) == 7)
    assert np.all(np.abs(c * sv - vf) <= 0.5 * sv * (1 + 1e-6) + 1e-30)
    assert np.all(codes[N:] == 0)
    ref = codes.astype(np.int64).reshape(Np // 64, 64, 128).sum(axis=1)
    assert np.array_equal(colsum.astype(np.int64), ref)


# ---------------------------------------------------------------- attention

def random_qz(oracle_mod, cfg, seed, qscale=1.0):
    rng = np.random.default_rng(seed)
    q = (rng.standard_normal((cfg.N, 128)) * qscale).astype(np.float16)
    k = (rng.standard_normal((cfg.N, 128)) * qscale).astype(np.float16)
    v = rng.standard_normal((cfg.N, 128)).astype(np.float16)
    return q, k, v, oracle_mod.quantize_head(cfg, q, k, v)


def dequant_logits(cfg, qz):
    N = cfg.N
    S = qz["qc"][:N].astype(np.int64) @ qz["kc"][:N].astype(np.int64).T
    sq = np.repeat(qz["qs"], 64)[:N].astype(np.float64)
    sk = np.repeat(qz["ks"], 64)[:N].astype(np.float64)
    return S, S * sq[:, None] * sk[None, :] / math.sqrt(128)


@pytest.mark.parametrize("tile", [64, 128, 192, 10_000])
def test_online_loop_equals_two_pass_softmax(oracle_mod, tile):
    """With P left unquantised, the tiled online softmax equals plain softmax
    attention over the dequantised logits and V, for any tile width."""
    cfg = small_cfg(F=2, Hh=10, W=10, n_text=16, rot="interleaved")   # N = 216
    _, _, _, qz = random_qz(oracle_mod, cfg, 6, qscale=2.0)
    _, s = dequant_logits(cfg, qz)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = p @ (qz["vc"][:cfg.N].astype(np.float64) * qz["sv"].astype(np.float64))
    _, o64 = oracle_mod.attention_rows(cfg, qz, tile=tile, quant_p=False, want64=True)
    assert np.max(np.abs(o64 - ref)) <= 1e-5 * np.abs(ref).max()


def test_S_is_the_integer_product(oracle_mod):
    cfg = small_cfg(F=2, Hh=10, W=10, n_text=16, rot="half")          # 2 tiles, ragged
    _, _, _, qz = random_qz(oracle_mod, cfg, 7)
    S, _ = dequant_logits(cfg, qz)
    for i in (0, 63, 64, 200, cfg.N - 1):
        for j in (0, 1):
            Sd, Pd = oracle_mod.attention_row_debug(cfg, qz, i, j)
            n1 = min(128 * j + 128, cfg.N)
            assert np.array_equal(Sd[:n1 - 128 * j], S[i, 128 * j:n1])
            assert np.all(Pd[n1 - 128 * j:] == -128)
            assert Pd[:n1 - 128 * j].min() >= -8 and Pd[:n1 - 128 * j].max() <= 7


def test_zero_point_identity_single_tile(oracle_mod):
    """Within one tile: PV with the colsum correction equals sum (code+8) v."""
    cfg = small_cfg(F=2, Hh=8, W=8, rot="interleaved")                 # N = 128: one tile
    _, _, _, qz = random_qz(oracle_mod, cfg, 8, qscale=1.5)
    _, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
    for i in (0, 17, 127):
        _, P = oracle_mod.attention_row_debug(cfg, qz, i, 0)
        w = P.astype(np.int64) + 8
        ref = (w @ qz["vc"][:128].astype(np.int64)) * qz["sv"].astype(np.float64) / w.sum()
        assert np.allclose(o64[i], ref, rtol=1e-12, atol=1e-12)
        assert w.max() == 15                               # the row max always gets P = 1


def test_symmetric_p_single_tile_and_error_bound(oracle_mod):
    """Symmetric P map: within one tile O = sum code * v / sum code (no
    zero-point term), the row max gets code 7, and every code is within half
    a step (1/14) of exp(s - m) (numpy, float64)."""
    cfg = small_cfg(F=2, Hh=8, W=8, rot="interleaved", p_mode="symmetric")   # N = 128: one tile
    _, _, _, qz = random_qz(oracle_mod, cfg, 8, qscale=1.5)
    _, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
    _, s = dequant_logits(cfg, qz)
    for i in (0, 17, 127):
        _, P = oracle_mod.attention_row_debug(cfg, qz, i, 0)
        w = P.astype(np.int64)
        assert w.min() >= 0 and w.max() == 7
        ref = (w @ qz["vc"][:128].astype(np.int64)) * qz["sv"].astype(np.float64) / w.sum()
        assert np.allclose(o64[i], ref, rtol=1e-12, atol=1e-12)
        assert np.max(np.abs(w / 7.0 - np.exp(s[i, :128] - s[i, :128].max()))) <= 1 / 14 + 1e-6
    # the two maps differ on the same inputs (the range-optimised one is finer)
    o_range = oracle_mod.attention_rows(cfg.replace(p_mode="range"), qz)
    o_sym = oracle_mod.attention_rows(cfg, qz)
    assert not np.array_equal(o_range, o_sym)


def test_v_hadamard_quantiser_and_inverse(oracle_mod):
    """v_rot = 1: V is quantised as V H / sqrt(128) (scipy's Hadamard, float64,
    to fp32 rounding; codes within half a step of it) and the output row is
    taken back through H: exact-P attention on the rotated V equals attention
    on the dequantised rotated V times H, and both paths approximate
    unquantised attention."""
    from scipy.linalg import hadamard
    H = hadamard(128).astype(np.float64) / math.sqrt(128)
    cfg = small_cfg(F=2, Hh=6, W=10, n_text=7, rot="half", v_rot=1)        # N = 127
    rng = np.random.default_rng(21)
    q = (rng.standard_normal((cfg.N, 128)) * 0.8).astype(np.float16)
    k = (rng.standard_normal((cfg.N, 128)) * 0.8).astype(np.float16)
    v = rng.standard_normal((cfg.N, 128)).astype(np.float16)
    v[:, 3] *= 8                                         # an outlier channel
    vr = v.astype(np.float64) @ H
    vc, sv, colsum = oracle_mod.quantize_v_head(cfg, v)
    assert np.allclose(sv, np.abs(vr).max(axis=0) / 7, rtol=2e-6)
    deq = vc[:cfg.N].astype(np.float64) * sv.astype(np.float64)
    assert np.all(np.abs(deq - vr) <= sv.astype(np.float64) / 2 * (1 + 1e-5) + 1e-6)
    qz = oracle_mod.quantize_head(cfg, q, k, v)
    _, o_exactp = oracle_mod.attention_rows(cfg, qz, quant_p=False, want64=True)
    S, s = dequant_logits(cfg, qz)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = ((p / p.sum(axis=1, keepdims=True)) @ deq) @ H.T
    assert np.allclose(o_exactp, ref, rtol=1e-6, atol=1e-7)   # fp32 logits in the oracle
    exact = oracle_mod.exact_attention_rows(cfg, q, k, v)
    _, o_rot = oracle_mod.attention_rows(cfg, qz, want64=True)
    qz0 = oracle_mod.quantize_head(cfg.replace(v_rot=0), q, k, v)
    _, o_plain = oracle_mod.attention_rows(cfg.replace(v_rot=0), qz0, want64=True)
    # both approximate unquantised attention (INT4 Q, K, P and V on random
    # data); without the inverse transform the cosine would be near 0
    assert cos(o_rot, exact) > 0.95 and cos(o_plain, exact) > 0.95
    assert not np.allclose(o_rot, o_plain, rtol=1e-9, atol=1e-9)


def test_uniform_logits_give_the_mean(oracle_mod):
    """All keys equal -> P = 1 -> code 7 -> O = mean of the dequantised V."""
    cfg = small_cfg(F=3, Hh=8, W=8, rot="none")                        # N = 192
    rng = np.random.default_rng(9)
    qz = dict(qc=np.zeros((256, 128), np.int8), qs=np.ones(4, np.float32),
              kc=np.zeros((256, 128), np.int8), ks=np.ones(4, np.float32))
    qz["qc"][:192] = rng.integers(-7, 8, (192, 128))
    qz["kc"][:192] = np.tile(rng.integers(-7, 8, (1, 128)), (192, 1))
    vc = np.zeros((256, 128), np.int8)
    vc[:192] = rng.integers(-7, 8, (192, 128))
    qz.update(vc=vc, sv=rng.uniform(0.1, 1, 128).astype(np.float32),
              colsum=vc.astype(np.int32).reshape(4, 64, 128).sum(axis=1).astype(np.int32))
    _, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
    ref = vc[:192].astype(np.float64).mean(axis=0) * qz["sv"]
    assert np.allclose(o64, ref[None, :], rtol=1e-12, atol=1e-12)


def test_running_max_rescale_closed_form(oracle_mod):
    """Tile 0 logits 0, tile 1 logits delta: tile 0 codes are taken against its
    own running max (P = 1), then rescaled by exp(-delta) at tile 1."""
    cfg = small_cfg(F=4, Hh=8, W=8, rot="none")                        # N = 256
    rng = np.random.default_rng(10)
    qc = np.zeros((256, 128), np.int8)
    qc[:, 0] = 1
    kc = np.zeros((256, 128), np.int8)
    kc[128:, 0] = 3                                            # S = 0 (tile 0), 3 (tile 1)
    sq = np.float32(0.5)
    qz = dict(qc=qc, qs=np.full(4, sq, np.float32), kc=kc, ks=np.ones(4, np.float32))
    vc = rng.integers(-7, 8, (256, 128)).astype(np.int8)
    qz.update(vc=vc, sv=np.ones(128, np.float32),
              colsum=vc.astype(np.int32).reshape(4, 64, 128).sum(axis=1).astype(np.int32))
    delta = float(np.float32(np.float32(3.0) * sq) * np.float32(1 / math.sqrt(128)))
    a = math.exp(-delta)
    s0 = vc[:128].astype(np.float64).sum(axis=0)
    s1 = vc[128:].astype(np.float64).sum(axis=0)
    ref = (15 * a * s0 + 15 * s1) / (15 * 128 * a + 15 * 128)
    _, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
    assert np.allclose(o64, ref[None, :], rtol=1e-6)
    # a global-max reading would have quantised tile 0 against delta instead
    c0 = oracle_mod.p_code(float(a)) + 8
    wrong = (c0 * s0 + 15 * s1) / (c0 * 128 + 15 * 128)
    assert np.max(np.abs(wrong - ref)) > 1e-3


def test_dominant_key_selects_its_value(oracle_mod):
    """A key whose logit leads the rest by more than ln 30 takes all weight:
    exactly when it sits in the first tile (every later key is quantised to
    code -8 against it), and up to exp(-gap) when it arrives in a later tile
    (earlier tiles were quantised against their own running max and are only
    rescaled, not dropped)."""
    cfg = small_cfg(F=3, Hh=8, W=8, rot="none")                        # N = 192
    rng = np.random.default_rng(11)
    for star, rtol in ((50, 1e-12), (150, 1e-6)):
        qc = np.zeros((256, 128), np.int8)
        qc[:192, :] = 7
        kc = np.zeros((256, 128), np.int8)
        kc[:192] = rng.integers(-1, 2, (192, 128))
        kc[star] = 7       # S = 6272 vs |S| <= 896: logit gap 5376*0.04/sqrt(128) = 19 > ln 30
        qz = dict(qc=qc, qs=np.full(4, 0.2, np.float32), kc=kc, ks=np.full(4, 0.2, np.float32))
        vc = np.zeros((256, 128), np.int8)
        vc[:192] = rng.integers(-7, 8, (192, 128))
        qz.update(vc=vc, sv=rng.uniform(0.1, 1, 128).astype(np.float32),
                  colsum=vc.astype(np.int32).reshape(4, 64, 128).sum(axis=1).astype(np.int32))
        _, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
        ref = vc[star].astype(np.float64) * qz["sv"]
        assert np.allclose(o64, ref[None, :], rtol=rtol, atol=rtol)
        if star > 128:
            assert not np.allclose(o64, ref[None, :], rtol=1e-12, atol=1e-12)


def test_convex_combination_and_p_error_bound(oracle_mod):
    """Every output row is a convex combination of dequantised V rows, and
    every P code is within half a step (1/30) of exp(s - m_j), m_j being the
    running max over tiles 0..j of the dequantised logits (numpy, float64)."""
    cfg = small_cfg(F=4, Hh=10, W=12, n_text=20, rot="half")          # N = 500, 4 tiles
    _, _, _, qz = random_qz(oracle_mod, cfg, 12, qscale=1.0)
    o, o64 = oracle_mod.attention_rows(cfg, qz, want64=True)
    bound = 7 * qz["sv"].astype(np.float64)
    assert np.all(np.abs(o64) <= bound[None, :] * (1 + 1e-12))
    # fp16 output is the RNE rounding of the float64 value
    assert np.array_equal(o, o64.astype(np.float16))
    _, s = dequant_logits(cfg, qz)
    N = cfg.N
    for i in (0, 99, 257, N - 1):
        m = -np.inf
        for j in range((N + 127) // 128):
            n0, n1 = 128 * j, min(128 * j + 128, N)
            m = max(m, s[i, n0:n1].max())
            _, Pc = oracle_mod.attention_row_debug(cfg, qz, i, j)
            Phat = (Pc[:n1 - n0].astype(np.float64) + 8) / 15
            assert np.max(np.abs(Phat - np.exp(s[i, n0:n1] - m))) <= 1 / 30 + 1e-6


def test_softmax_attention_matches_numpy(oracle_mod):
    cfg = small_cfg(F=2, Hh=5, W=7)                                    # N = 70
    rng = np.random.default_rng(13)
    q, k, v = (rng.standard_normal((cfg.N, 128)) for _ in range(3))
    s = q @ k.T / math.sqrt(128)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ v
    out = oracle_mod.softmax_attention_rows(cfg, q, k, v)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_fp16_rope_is_rounded_rope(oracle_mod):
    cfg = small_cfg(F=2, Hh=5, W=7, n_text=4)
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((cfg.N, 128)) * 4).astype(np.float16)
    y = oracle_mod.rope_fp16_head(cfg, x)
    z = oracle_mod.rotate_head(cfg, x, rot="none")
    assert np.array_equal(y, z.astype(np.float16))
