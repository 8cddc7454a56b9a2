"""Padding and scratch poisoned with 0x77 before a run (the substitute for a
memory checker, which is not available here): the INT4 path must give the
same output, bit for bit, as on zero-filled buffers, and the prologue must
write every padded token of the quantised tensors (code 0, scale 0 for a
block of padding only), so no kernel ever reads bytes it did not define."""
import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

POISON = 0x77


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.lib()
    return torch.device("cuda:0")


def run(cfg, dev, q, k, v, fill):
    p = api.problem(cfg)
    ws = torch.full((api.workspace_bytes(p, True),), fill, dtype=torch.uint8, device=dev)
    buf = torch.full((api.qkv4_bytes(p),), fill, dtype=torch.uint8, device=dev)
    qkv4 = api.qkv4_bind(p, buf)
    api.prepare(p, ws)
    o = torch.full(q.shape, float("nan"), dtype=torch.float16, device=dev)
    api.rotate_quantize_qkv(p, q, k, v, qkv4, ws)
    api.int4_attention_fwd(p, qkv4, o, ws)
    o16 = torch.full(q.shape, float("nan"), dtype=torch.float16, device=dev)
    api.fp16_attention_fwd(p, q, k, v, o16, ws)
    api.check_device_error(ws)
    return o, o16, buf, qkv4


# ragged cases: N mod 128 in {66, 2, 90, 80}; text tokens; batch 2
CASES = {
    "ragged_text": synth.Config("ragged_text", 1, 3, 3, 7, 9, 5, (44, 42, 42), "interleaved", "lognormal1", 11),
    "text_only": synth.Config("text_only", 1, 1, 0, 0, 0, 130, (44, 42, 42), "half", "outlier8", 14),
    "norot_b2": synth.Config("norot_b2", 2, 2, 2, 5, 9, 0, (44, 42, 42), "none", "lognormal1", 13),
    "vrot_tail80": synth.Config("vrot_tail80", 1, 2, 2, 8, 13, 0, (16, 56, 56), "full", "lognormal1.5", 23,
                                v_rot=1),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_poisoned_buffers_change_nothing(dev, name):
    cfg = CASES[name]
    q, k, v = (torch.from_numpy(t).to(dev) for t in synth.make_qkv(cfg))
    o0, f0, _, _ = run(cfg, dev, q, k, v, 0)
    o1, f1, buf, qkv4 = run(cfg, dev, q, k, v, POISON)
    assert not torch.isnan(o1).any() and not torch.isnan(f1).any()
    assert torch.equal(o0.view(torch.int16), o1.view(torch.int16)), name
    assert torch.equal(f0.view(torch.int16), f1.view(torch.int16)), name
    # every padded token of the quantised tensors was written by the prologue
    BH, N = cfg.B * cfg.H, cfg.N
    Np = (N + 127) // 128 * 128
    host = buf.cpu().numpy()
    base = buf.data_ptr()

    def field(ptr, count, dtype):
        off = ptr - base
        return host[off:off + count * np.dtype(dtype).itemsize].view(dtype)

    q4 = field(qkv4.q4, BH * Np * 64, np.uint8).reshape(BH, Np, 64)
    k4 = field(qkv4.k4, BH * Np * 64, np.uint8).reshape(BH, Np, 64)
    v4t = field(qkv4.v4t, BH * Np * 64, np.uint8).reshape(BH, Np // 128, 128, 64)
    sq = field(qkv4.sq, BH * (Np // 64), np.float32).reshape(BH, Np // 64)
    vsum = field(qkv4.vsum, BH * (Np // 64) * 128, np.int32).reshape(BH, Np // 64, 128)
    assert not q4[:, N:].any() and not k4[:, N:].any()
    tok = np.arange(Np)
    pad_tile, pad_byte = (tok[N:] // 128), (tok[N:] % 128) // 2
    lo_or_hi = tok[N:] % 2
    for t, byte, hi in zip(pad_tile, pad_byte, lo_or_hi):
        nib = (v4t[:, t, :, byte] >> (4 * hi)) & 0xF
        assert not nib.any(), (t, byte, hi)
    full_pad_blocks = np.arange((N + 63) // 64, Np // 64)
    assert not sq[:, full_pad_blocks].any()
    assert not vsum[:, full_pad_blocks].any()
