"""ra_int4_attention_host (host buffers in and out, copies overlapped with the
kernels over chunks of heads) against the device-buffer calls.

Every step of the path is independent per (b, h), so running the heads in
chunks as problems of their own must give the device-buffer result bit for
bit, whatever the chunk size: a tail chunk smaller than the others, B = 2
(heads flattened across the batch), one head per chunk, all heads in one
chunk, the ragged last KV tile of the Wan sequence, and two calls in a row
through the same staging buffer.
"""
import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.lib()
    return torch.device("cuda:0")


def device_path(cfg, dev, q, k, v):
    ra = api.RotateAttention(cfg, dev, fp16_path=False)
    qd, kd, vd = (torch.from_numpy(t).to(dev) for t in (q, k, v))
    out = ra.forward(qd, kd, vd, path="int4")
    ra.check()
    return ra, out.cpu().numpy()


CASES = [
    ("half", {}, (0, 3, 4, 1)),
    ("tiny", {"B": 2, "H": 3}, (0, 4, 6)),
    ("tiny", {"B": 2, "H": 20}, (0, 7)),    # default ramp 1, 2, 3, 4, 5, 5, ... over 40 heads
    ("wan", {"H": 5}, (2,)),                  # full Wan sequence, ragged last tile, tail of 1 head
    # the options ride along: caller pair blocks (Half), V Hadamard, symmetric P map
    ("half", {"rot": "blocks_half", "blocks": synth.random_pair_blocks(3), "v_rot": 1, "p_mode": "symmetric"},
     (0, 3)),
]


@pytest.mark.parametrize("name,over,chunks", CASES, ids=[f"{c[0]}{i}" for i, c in enumerate(CASES)])
def test_host_entry_equals_device_path(dev, name, over, chunks):
    cfg = synth.CONFIGS[name]
    if over:
        cfg = cfg.replace(name=f"{name}-{len(over)}", **over)
    q, k, v = synth.make_qkv(cfg)
    ra, ref = device_path(cfg, dev, q, k, v)
    qh, kh, vh = (torch.from_numpy(t).pin_memory() for t in (q, k, v))
    for per in chunks:
        for rep in range(2):                   # the staging buffer keeps the last call's contents
            oh = torch.full(ref.shape, float("nan"), dtype=torch.float16).pin_memory()
            ra.forward_host(qh, kh, vh, oh, heads_per_chunk=per)
            got = oh.numpy()
            assert np.array_equal(got.view(np.uint16), ref.view(np.uint16)), (name, per, rep)


def test_host_entry_accepts_pageable_buffers(dev):
    """Pageable host memory loses the overlap, not the result."""
    cfg = synth.CONFIGS["tiny"]
    q, k, v = synth.make_qkv(cfg)
    ra, ref = device_path(cfg, dev, q, k, v)
    oh = torch.empty(ref.shape, dtype=torch.float16)
    ra.forward_host(*(torch.from_numpy(t) for t in (q, k, v)), oh, heads_per_chunk=1)
    assert np.array_equal(oh.numpy().view(np.uint16), ref.view(np.uint16))
