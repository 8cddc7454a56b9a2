"""ra_rotate_quantize_qkv_noalloc against ra_rotate_quantize_qkv.

The no-alloc variant exists for callers that can pass the library their own
input and output tensors but cannot give it any other device memory -- an
engine plugin whose enqueue step must not allocate (an allocation may
synchronise the device or fail in the middle of a run), or a program whose
device memory is planned up front.  Its scratch lives in a fixed device array
inside the library.  It runs the same kernels, so its outputs must equal the
workspace entry point's bit for bit (the prologue's parity bar), on
consecutive calls that reuse the array for different problems.

Collected last on purpose (file name), so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

FIELDS = ("q4", "k4", "v4t", "sq", "sk", "sv", "vsum")


def field_bytes(cfg):
    BH = cfg.B * cfg.H
    Np = (cfg.N + 127) // 128 * 128
    packed = BH * Np * 64
    nblk = Np // 64
    return dict(q4=packed, k4=packed, v4t=packed, sq=4 * BH * nblk, sk=4 * BH * nblk, sv=4 * BH * 128,
                vsum=4 * BH * nblk * 128)


def snapshot(buf, qkv4, cfg):
    """The defined bytes of every quantised output, read back to the host."""
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    base = buf.data_ptr()
    sizes = field_bytes(cfg)
    return {f: host[getattr(qkv4, f) - base:getattr(qkv4, f) - base + sizes[f]].copy() for f in FIELDS}


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.lib()
    return torch.device("cuda:0")


def test_noalloc_matches_workspace_entry_point(dev):
    # two consecutive calls on different problems share the one fixed array
    for name in ("half", "tiny"):
        cfg = synth.CONFIGS[name]
        q, k, v = (torch.from_numpy(t).to(dev) for t in synth.make_qkv(cfg))
        ref = api.RotateAttention(cfg, dev, fp16_path=False)
        ref.rotate_quantize(q, k, v)
        o_ref = ref.int4_attention()
        ref.check()
        want = snapshot(ref.qkv4_buf, ref.qkv4, cfg)

        p = api.problem(cfg)
        buf = torch.full((api.qkv4_bytes(p),), 0x5A, dtype=torch.uint8, device=dev)
        qkv4 = api.qkv4_bind(p, buf)
        api.rotate_quantize_qkv_noalloc(p, q, k, v, qkv4)
        api.noalloc_check_device_error()            # the scratch's error word is clear
        got = snapshot(buf, qkv4, cfg)
        for f in FIELDS:
            assert np.array_equal(got[f], want[f]), (name, f)

        # and the attention on its outputs is the same, bit for bit
        o = torch.empty_like(o_ref)
        api.int4_attention_fwd(p, qkv4, o, ref.workspace)
        ref.check()
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16)), name


def test_noalloc_on_a_side_stream(dev):
    # the same call enqueued on a non-default stream: same bytes, clear error word
    cfg = synth.CONFIGS["tiny"]
    q, k, v = (torch.from_numpy(t).to(dev) for t in synth.make_qkv(cfg))
    ref = api.RotateAttention(cfg, dev, fp16_path=False)
    ref.rotate_quantize(q, k, v)
    ref.check()
    want = snapshot(ref.qkv4_buf, ref.qkv4, cfg)
    p = api.problem(cfg)
    buf = torch.full((api.qkv4_bytes(p),), 0xA5, dtype=torch.uint8, device=dev)
    qkv4 = api.qkv4_bind(p, buf)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.rotate_quantize_qkv_noalloc(p, q, k, v, qkv4, stream=side)
        api.noalloc_check_device_error(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    got = snapshot(buf, qkv4, cfg)
    for f in FIELDS:
        assert np.array_equal(got[f], want[f]), f


def test_noalloc_rejects_problems_beyond_its_scratch(dev):
    lib = api.lib()
    # 600 heads need 600 * 512 bytes of V-amax scratch alone: over 256 KiB
    big = api.problem(synth.CONFIGS["tiny"].replace(H=600))
    q = api.Qkv4(*(256 for _ in FIELDS))
    st = lib.ra_rotate_quantize_qkv_noalloc(ctypes.byref(big), 256, 256, 256, ctypes.byref(q), None)
    assert st == api.RA_ERR_WORKSPACE
    assert b"RA_NOALLOC_SCRATCH_BYTES" in lib.ra_last_error_detail()
