"""Accuracy diagnostic: the GPU outputs against unquantised attention.

The pages' case for the method is accuracy: RoPE-aware rotations spread the
channel outliers before INT4 quantisation of Q and K ("What carries the
argument"; Fig. 3 caption) and the range-optimised map uses all 16 INT4 levels
for P (abstract; free-parameter ledger).  This module measures, on the
synthetic inputs, the cosine and relative L2 error of the INT4 path's output
against float64 attention on the unquantised inputs (RoPE and rotation in
fp32, then float64 softmax attention), next to the FP16 path's, per workload
and per rotation mode and P map.  These are reported numbers, not parity bars
(parity against the oracle is tests/test_gpu_parity.py); the assertions only
catch a broken path.  With RA_ACCURACY_REPORT set, the table is appended to
that file."""
import os

import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ROWS_LARGE = 512      # sampled query rows per head for the full-length workloads
HEADS_LARGE = 2       # heads of the full-length workloads (their own seeded draw)


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.lib()
    return torch.device("cuda:0")


def workload(name):
    cfg = synth.CONFIGS[name]
    if cfg.N > 4096:
        cfg = cfg.replace(H=HEADS_LARGE, name=f"{name}-H{HEADS_LARGE}")
    return cfg


def rows_of(cfg):
    if cfg.N <= 4096:
        return np.arange(cfg.N, dtype=np.int64)
    rng = np.random.default_rng(31)
    return np.unique(np.concatenate([rng.choice(cfg.N, ROWS_LARGE, replace=False), [cfg.N - 1]])).astype(np.int64)


def metrics(got, ref):
    g, r = got.ravel(), ref.ravel()
    cos = float(g @ r / (np.linalg.norm(g) * np.linalg.norm(r) + 1e-300))
    rel = float(np.linalg.norm(g - r) / (np.linalg.norm(r) + 1e-300))
    return cos, rel


def write(lines):
    text = "\n".join(lines)
    print("\n" + text)
    path = os.environ.get("RA_ACCURACY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(text + "\n\n")


def exact_rows(oracle_mod, cfg, q, k, v, rows):
    out = []
    for bh in range(cfg.B * cfg.H):
        b, h = divmod(bh, cfg.H)
        out.append(oracle_mod.exact_attention_rows(cfg, q[b, h], k[b, h], v[b, h], rows))
    return np.stack(out)


def gpu_rows(o, cfg, rows):
    o = o.cpu().numpy().reshape(cfg.B * cfg.H, cfg.N, cfg.d)
    return o[:, rows].astype(np.float64)


@pytest.mark.slow
def test_accuracy_per_workload(oracle_mod, dev):
    lines = ["| workload | rows | INT4 vs exact: cosine | rel. L2 | FP16 vs exact: cosine | rel. L2 |",
             "|---|---|---|---|---|---|"]
    for name in ("tiny", "half", "wan", "hunyuan"):
        cfg = workload(name)
        q, k, v = synth.make_qkv(cfg)
        rows = rows_of(cfg)
        ref = exact_rows(oracle_mod, cfg, q, k, v, rows)
        ra = api.RotateAttention(cfg, dev, fp16_path=True)
        qd, kd, vd = (torch.from_numpy(t).to(dev) for t in (q, k, v))
        c4, r4 = metrics(gpu_rows(ra.forward(qd, kd, vd, path="int4"), cfg, rows), ref)
        c16, r16 = metrics(gpu_rows(ra.forward(qd, kd, vd, path="fp16"), cfg, rows), ref)
        ra.check()
        lines.append(f"| {cfg.name} ({cfg.rot}) | {len(rows) * cfg.B * cfg.H} | {c4:.5f} | {r4:.4f} | "
                     f"{c16:.6f} | {r16:.5f} |")
        assert c16 >= 0.999, (name, c16)
        assert np.isfinite(c4) and c4 > 0.3, (name, c4)
    write(lines)


@pytest.mark.slow
def test_accuracy_per_rotation_and_p_map(oracle_mod, dev):
    lines = ["| workload | rows | rotation | P map | INT4 vs exact: cosine | rel. L2 |", "|---|---|---|---|---|---|"]
    for name in ("tiny", "half", "wan"):
        base = workload(name)
        q, k, v = synth.make_qkv(base)
        rows = rows_of(base)
        ref = exact_rows(oracle_mod, base, q, k, v, rows)
        qd, kd, vd = (torch.from_numpy(t).to(dev) for t in (q, k, v))
        cos = {}
        for rot in ("none", "interleaved", "half", "full"):
            for pm in ("range", "symmetric"):
                cfg = base.replace(rot=rot, p_mode=pm)
                ra = api.RotateAttention(cfg, dev, fp16_path=False)
                c, r = metrics(gpu_rows(ra.forward(qd, kd, vd, path="int4"), cfg, rows), ref)
                ra.check()
                cos[rot, pm] = c
                lines.append(f"| {base.name} | {len(rows) * base.B * base.H} | {rot} | {pm} | {c:.5f} | {r:.4f} |")
                assert np.isfinite(c) and c > 0.3, (name, rot, pm, c)
    write(lines)
