"""Host-only checks of the C ABI: the library builds and loads, exports every
function the header declares, validates arguments before touching the GPU,
and builds RoPE/rotation tables identical to the oracle's."""
import ctypes
import os
import re

import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "rotate_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_function(lib):
    names = header_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"
    assert set(names) == set(api._SIGNATURES), "binding and header disagree"


def test_library_is_sm100a(lib):
    # the build flags target sm_100a only
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.NVCC_FLAGS)


def prob(**kw):
    return api.problem(synth.CONFIGS["tiny"].replace(**kw))


def test_validation_codes(lib):
    assert api.validate(prob()) == api.RA_OK
    assert api.validate(prob(d=64)) == api.RA_ERR_UNSUPPORTED
    assert api.validate(prob(split=(44, 42, 40))) == api.RA_ERR_INVALID_ARG   # sum != d
    assert api.validate(prob(split=(43, 43, 42))) == api.RA_ERR_INVALID_ARG   # odd
    assert api.validate(prob(F=0, Hh=0, W=0, n_text=0)) == api.RA_ERR_INVALID_ARG   # N = 0
    assert api.validate(prob(H=0)) == api.RA_ERR_INVALID_ARG
    assert api.validate(prob(p_mode="symmetric")) == api.RA_OK
    bad = prob()
    bad.p_mode = 2                                                           # unknown P map
    assert api.validate(bad) == api.RA_ERR_INVALID_ARG
    blocks = synth.random_pair_blocks(1)
    assert api.validate(prob(rot="blocks_half", blocks=blocks)) == api.RA_OK
    assert api.validate(prob(rot="blocks_interleaved")) == api.RA_ERR_INVALID_ARG     # no blocks
    skew = tuple(b * 1.01 for b in blocks)                                   # not orthogonal
    assert api.validate(prob(rot="blocks_half", blocks=skew)) == api.RA_ERR_INVALID_ARG


def test_longest_sequence_bound(lib):
    # the int32 P.V accumulator (offset 0x4B400000 plus up to 112 * 15 * N)
    # admits N <= 2^19 tokens
    assert 0x4B400000 + 112 * 15 * (1 << 19) < 2 ** 31
    assert 0x4B400000 + 112 * 15 * ((1 << 19) + 4096) >= 2 ** 31   # the bound is within 1 % of tight
    assert api.validate(prob(F=1, Hh=1, W=1 << 19, n_text=0)) == api.RA_OK
    assert api.validate(prob(F=1, Hh=1, W=(1 << 19) - 5, n_text=5)) == api.RA_OK
    assert api.validate(prob(F=1, Hh=1, W=1 << 19, n_text=1)) == api.RA_ERR_UNSUPPORTED
    assert api.validate(prob(F=8, Hh=256, W=257, n_text=0)) == api.RA_ERR_UNSUPPORTED
    assert b"at most 524288" in lib.ra_last_error_detail()
    assert api.validate(prob(theta=0.0)) == api.RA_ERR_INVALID_ARG
    p = prob()
    p.rot = 7
    assert api.validate(p) == api.RA_ERR_INVALID_ARG
    assert api.validate(prob(F=0, Hh=0, W=0, n_text=5)) == api.RA_OK          # text only
    assert api.validate(prob(F=2, Hh=0, W=3, n_text=5)) == api.RA_ERR_INVALID_ARG
    api.validate(prob(split=(44, 42, 40)))
    assert b"split" in lib.ra_last_error_detail()


def test_sizes(lib):
    for name, cfg in synth.CONFIGS.items():
        p = api.problem(cfg)
        assert api.seq_len(p) == cfg.N
        assert api.seq_pad(p) == (cfg.N + 127) // 128 * 128
        Np, BH = api.seq_pad(p), cfg.B * cfg.H
        min_qkv = 3 * BH * Np * 64 + 2 * BH * (Np // 64) * 4 + BH * 128 * 4 + BH * (Np // 64) * 128 * 4
        assert api.qkv4_bytes(p) >= min_qkv
        assert api.workspace_bytes(p, True) >= api.workspace_bytes(p, False) + 3 * BH * Np * 128 * 2
        # the INT4 path holds the INT8 operand images of Q, K and V^T
        assert api.workspace_bytes(p, False) >= 3 * BH * Np * 128


def test_each_call_checks_its_own_workspace_size(lib):
    """The prologue needs only header, tables and V amax; the INT4 attention
    also needs the operand images: a workspace between the two sizes serves
    the first and is refused (RA_ERR_WORKSPACE) by the second, before any
    launch."""
    cfg = synth.CONFIGS["tiny"]
    p = api.problem(cfg)
    full = api.workspace_bytes(p, False)
    Np, BH = api.seq_pad(p), cfg.B * cfg.H
    mid = full - 3 * BH * Np * 128                      # room for everything but the images
    q = api.Qkv4()
    assert lib.ra_qkv4_bind(ctypes.byref(p), 256, 1 << 30, ctypes.byref(q)) == api.RA_OK
    st = lib.ra_int4_attention_fwd(ctypes.byref(p), ctypes.byref(q), 256, 256, mid, None)
    assert st == api.RA_ERR_WORKSPACE
    assert b"needs" in lib.ra_last_error_detail()
    st = lib.ra_fp16_attention_fwd(ctypes.byref(p), 256, 256, 256, 256, 256, full, None)
    assert st == api.RA_ERR_WORKSPACE                   # the FP16 path needs its images too


def test_calls_reject_bad_arguments_without_a_gpu(lib):
    p = prob()
    q = api.Qkv4()
    ws = ctypes.c_void_p(None)
    st = lib.ra_rotate_quantize_qkv(ctypes.byref(p), None, None, None, ctypes.byref(q), ws, 0, None)
    assert st == api.RA_ERR_INVALID_ARG
    st = lib.ra_int4_attention_fwd(ctypes.byref(p), ctypes.byref(q), None, ws, 0, None)
    assert st == api.RA_ERR_INVALID_ARG
    st = lib.ra_fp16_attention_fwd(ctypes.byref(p), 16, 16, 16, 16, 32, 10, None)
    assert st == api.RA_ERR_WORKSPACE                 # undersized workspace
    st = lib.ra_fp16_attention_fwd(ctypes.byref(p), 17, 16, 16, 16, 32, 1 << 40, None)
    assert st == api.RA_ERR_INVALID_ARG               # misaligned q
    st = lib.ra_prepare(ctypes.byref(p), 32, 16, None)
    assert st == api.RA_ERR_WORKSPACE
    bad = prob(d=96)
    st = lib.ra_int4_attention_fwd(ctypes.byref(bad), ctypes.byref(q), 16, 32, 1 << 40, None)
    assert st == api.RA_ERR_UNSUPPORTED
    buf = api.Qkv4()
    st = lib.ra_qkv4_bind(ctypes.byref(p), 256, 10, ctypes.byref(buf))
    assert st == api.RA_ERR_INVALID_ARG
    st = lib.ra_qkv4_bind(ctypes.byref(p), 512, 1 << 30, ctypes.byref(buf))
    assert st == api.RA_OK and buf.q4 == 512 and buf.k4 > buf.q4
    st = lib.ra_debug_int4_tile(ctypes.byref(p), ctypes.byref(buf), 0, 5, 0, 16, 16, 32, 1 << 40, None)
    assert st == api.RA_ERR_INVALID_ARG               # q tile out of range (N_pad/128 = 2)
    for s in range(7):
        assert api.status_string(s)


def test_host_entry_plan_and_argument_checks(lib):
    """ra_int4_attention_host: the staging buffer holds three slots, each with
    q, k, v, o, the quantised tensors and a workspace for the largest chunk;
    bad arguments are refused before any CUDA call."""
    cfg = synth.CONFIGS["wan"]
    p = api.problem(cfg)
    head = cfg.N * 128 * 2

    def a256(x):
        return (x + 255) // 256 * 256

    for per in (1, 5, 7, 40):
        chunk = api.problem(cfg.replace(H=per))
        slot = a256(api.workspace_bytes(chunk, False)) + a256(api.qkv4_bytes(chunk)) + a256(4 * per * head)
        assert api.host_staging_bytes(p, per) == 3 * slot
    assert api.host_staging_bytes(p, 0) == api.host_staging_bytes(p, 5)     # default: ramp up to BH / 8 heads
    assert api.host_staging_bytes(p, 400) == api.host_staging_bytes(p, 40)  # capped at B*H
    assert api.host_staging_bytes(p, -1) == 0
    # B = 2 flattens to B*H heads
    p2 = api.problem(cfg.replace(B=2, H=4))
    assert api.host_staging_bytes(p2, 0) == api.host_staging_bytes(api.problem(cfg.replace(H=8)), 1)
    need = api.host_staging_bytes(p, 0)
    st = lib.ra_int4_attention_host(ctypes.byref(p), 16, 16, 16, 16, -1, 256, need, None)
    assert st == api.RA_ERR_INVALID_ARG
    st = lib.ra_int4_attention_host(ctypes.byref(p), 16, None, 16, 16, 0, 256, need, None)
    assert st == api.RA_ERR_INVALID_ARG
    st = lib.ra_int4_attention_host(ctypes.byref(p), 16, 16, 16, 16, 0, 272, need, None)
    assert st == api.RA_ERR_INVALID_ARG               # staging not 256-byte aligned
    st = lib.ra_int4_attention_host(ctypes.byref(p), 16, 16, 16, 16, 0, 256, need - 1, None)
    assert st == api.RA_ERR_WORKSPACE
    assert b"needs" in lib.ra_last_error_detail()
    bad = api.problem(cfg.replace(d=64))
    st = lib.ra_int4_attention_host(ctypes.byref(bad), 16, 16, 16, 16, 0, 256, 1 << 40, None)
    assert st == api.RA_ERR_UNSUPPORTED


@pytest.mark.parametrize("BH", [1, 2, 3, 5, 8, 9, 16, 24, 33, 40, 41, 47, 64, 100, 333, 999])
def test_host_chunk_schedule(lib, BH):
    """The default schedule covers the B*H heads in order, never exceeds
    ceil(B*H/8) heads a chunk, starts and (when there is room for both ramps)
    ends with one head, and grows by at most 4/3 (+1) per step; an explicit
    size gives equal chunks and a remainder."""
    p = api.problem(synth.CONFIGS["tiny"].replace(B=1, H=BH))
    per = -(-BH // 8)
    c = api.host_chunks(p, 0)
    assert sum(c) == BH and min(c) >= 1 and max(c) <= per and c[0] == 1
    for a, b in zip(c, c[1:]):   # growth the copy-in can hide behind the previous chunk's kernels
        assert b <= max(a + 1, 4 * a // 3)
    if BH >= 8:
        assert c[-1] == 1        # room for the down ramp: the last copy back is of one head
    assert api.host_chunks(p, 7) == [7] * (BH // 7) + ([BH % 7] if BH % 7 else [])
    assert api.host_chunks(p, 10 ** 6) == [BH]
    assert lib.ra_host_chunks(ctypes.byref(p), -1, None, 0) == -1
    # the staging size follows the largest chunk
    assert api.host_staging_bytes(p, 0) == api.host_staging_bytes(p, max(c))


def test_host_chunk_schedule_wan_and_hunyuan(lib):
    assert api.host_chunks(api.problem(synth.CONFIGS["wan"])) == [1, 1, 2, 2, 3, 3, 4, 4, 5, 5, 4, 3, 2, 1]
    assert api.host_chunks(api.problem(synth.CONFIGS["hunyuan"])) == [1, 1, 2, 2, 3, 3, 3, 3, 3, 2, 1]


@pytest.mark.parametrize("name", ["tiny", "half", "wan", "hunyuan"])
def test_tables_bit_exact_against_oracle(lib, oracle_mod, name):
    cfg = synth.CONFIGS[name]
    tab = api.build_tables_host(api.problem(cfg))
    npos = (cfg.F, cfg.Hh, cfg.W)
    k = 0
    rng = np.random.default_rng(0)
    for s in range(3):
        half = cfg.split[s] // 2
        q = (half + 3) // 4      # a position's block: 4 q slots, pair j at (j % 4) q + j // 4
        used = np.zeros(4 * q, bool)
        used[[(j % 4) * q + j // 4 for j in range(half)]] = True
        assert used.sum() == half                      # distinct slots
        blocks = tab[k:k + npos[s] * 4 * q].reshape(npos[s], 4 * q, 4)
        assert not blocks[:, ~used].any()              # the other slots are zero
        # every entry for small grids, a sample for the large ones
        cells = [(pos, j) for pos in range(npos[s]) for j in range(half)]
        if len(cells) > 400:
            idx = rng.choice(len(cells), 400, replace=False)
            cells = [cells[i] for i in idx] + [(npos[s] - 1, half - 1)]
        for pos, j in cells:
            ref = np.array(oracle_mod.rope_coef(cfg, s, pos, j), np.float32)
            got = tab[k + pos * 4 * q + (j % 4) * q + j // 4]
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), (name, s, pos, j)
        k += npos[s] * 4 * q
    assert k + 64 == len(tab)                 # then the 64 pair-block entries (zero here)
    assert not tab[k:].any()


def test_host_chunk_schedule_every_head_count(lib):
    """The default schedule's invariants for every B*H up to 2000: it covers
    the heads, stays within ceil(B*H/8) heads a chunk, starts with one head
    (and ends with one when there are at least 8), and grows by at most 4/3
    (+1) per step."""
    for BH in range(1, 2001):
        p = api.problem(synth.CONFIGS["tiny"].replace(B=1, H=BH))
        per = -(-BH // 8)
        c = api.host_chunks(p, 0)
        assert sum(c) == BH and min(c) >= 1 and max(c) <= per and c[0] == 1, BH
        assert all(b <= max(a + 1, 4 * a // 3) for a, b in zip(c, c[1:])), (BH, c)
        assert BH < 8 or c[-1] == 1, (BH, c)
