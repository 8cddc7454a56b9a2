"""Worker of tests/test_gpu_bounds.py: runs every entry point of whichever
build RA_LIBRARY selects on the given configurations, with every buffer the
library reads or writes pre-filled with 0x77, and saves the outputs and the
status of ra_check_device_error to an .npz file.

    python tests/bounds_worker.py OUT.npz
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from int4_quantized_attention_b200 import api, synth  # noqa: E402

POISON = 0x77

CASES = {
    # N mod 128 = 66, text tokens
    "ragged_text": synth.Config("ragged_text", 1, 3, 3, 7, 9, 5, (44, 42, 42), "interleaved", "lognormal1", 11),
    # a text-only sequence with a second tile of 2 keys and a third of none
    "text_only": synth.Config("text_only", 1, 1, 0, 0, 0, 130, (44, 42, 42), "half", "outlier8", 14),
    # batch 2, one partial tile
    "norot_b2": synth.Config("norot_b2", 2, 2, 2, 5, 9, 0, (44, 42, 42), "none", "lognormal1", 13),
    # Full rotation and the V Hadamard, N mod 128 = 80
    "vrot_tail80": synth.Config("vrot_tail80", 1, 2, 2, 8, 13, 0, (16, 56, 56), "full", "lognormal1.5", 23, v_rot=1),
    # several tiles and a normaliser past 2^15 (the large-row rescale)
    "flat_long": synth.Config("flat_long", 1, 2, 4, 24, 50, 7, (44, 42, 42), "interleaved", "const0.3", 22),
    # the symmetric P map with caller pair blocks
    "blocks_sym": synth.Config("blocks_sym", 1, 2, 2, 9, 10, 40, (16, 56, 56), "blocks_half", "lognormal1.5", 21,
                               p_mode="symmetric", blocks=synth.random_pair_blocks(41)),
}


DETAILS = []


def status(fn):
    try:
        fn()
        return api.RA_OK
    except api.RotateAttnError as e:
        DETAILS.append(str(e))
        return e.status


def main(out_path):
    dev = torch.device("cuda:0")
    res = {}
    for name, cfg in CASES.items():
        p = api.problem(cfg)
        qh, kh, vh = synth.make_qkv(cfg)
        q, k, v = (torch.from_numpy(t).to(dev) for t in (qh, kh, vh))
        ws = torch.full((api.workspace_bytes(p, True),), POISON, dtype=torch.uint8, device=dev)
        buf = torch.full((api.qkv4_bytes(p),), POISON, dtype=torch.uint8, device=dev)
        qkv4 = api.qkv4_bind(p, buf)
        api.prepare(p, ws)
        o4 = torch.empty_like(q).view(torch.uint8).fill_(POISON).view(torch.float16)
        o16 = torch.empty_like(q).view(torch.uint8).fill_(POISON).view(torch.float16)
        api.rotate_quantize_qkv(p, q, k, v, qkv4, ws)
        api.int4_attention_fwd(p, qkv4, o4, ws)
        api.fp16_attention_fwd(p, q, k, v, o16, ws)
        res[f"{name}/status_device"] = status(lambda: api.check_device_error(ws))
        # host-buffer pipeline, chunks of one head
        oh = torch.empty(q.shape, dtype=torch.float16)
        staging = torch.full((api.host_staging_bytes(p, 1),), POISON, dtype=torch.uint8, device=dev)
        res[f"{name}/status_host"] = status(
            lambda: api.int4_attention_host(p, torch.from_numpy(qh), torch.from_numpy(kh), torch.from_numpy(vh), oh,
                                            staging, heads_per_chunk=1))
        # allocation-free prologue into a second poisoned buffer
        buf2 = torch.full((api.qkv4_bytes(p),), POISON, dtype=torch.uint8, device=dev)
        qkv4b = api.qkv4_bind(p, buf2)
        api.rotate_quantize_qkv_noalloc(p, q, k, v, qkv4b)
        res[f"{name}/status_noalloc"] = status(lambda: api.noalloc_check_device_error())
        torch.cuda.synchronize()
        res[f"{name}/o4"] = o4.cpu().numpy().view(np.uint16)
        res[f"{name}/o16"] = o16.cpu().numpy().view(np.uint16)
        res[f"{name}/o_host"] = oh.numpy().view(np.uint16)
        res[f"{name}/qkv4_noalloc"] = buf2.cpu().numpy()
        res[f"{name}/qkv4"] = buf.cpu().numpy()
    res["details"] = np.array(DETAILS if DETAILS else [""])
    np.savez(out_path, **res)


if __name__ == "__main__":
    main(sys.argv[1])
