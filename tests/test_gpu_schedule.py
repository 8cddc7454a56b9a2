"""The mixed-precision schedule on the GPU: the pages' FP16 fallback on the
first and last sampling steps and DiT blocks, INT4 everywhere else
("RotateAttention" review page, Sec. 5.1 quoted in the circularity check;
free-parameter ledger).  The dispatch runs the same entry points as single
calls, so every call's output must be bit-identical to the single-path call
of its kind, and the share of INT4 calls must be the schedule's."""
import numpy as np
import pytest

from int4_quantized_attention_b200 import api, build, schedule, synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.lib()
    return torch.device("cuda:0")


@pytest.mark.parametrize("sched_name", ["BENCH_SCHEDULE_SHORT", "BENCH_SCHEDULE"])
def test_schedule_calls_equal_single_path_calls(dev, sched_name):
    sched = getattr(schedule, sched_name)
    cfg = synth.CONFIGS["half"]
    q, k, v = (torch.from_numpy(t).to(dev) for t in synth.make_qkv(cfg))
    ra = api.RotateAttention(cfg, dev, fp16_path=True)
    want = {"int4": ra.forward(q, k, v, path="int4").clone(), "fp16": ra.forward(q, k, v, path="fp16").clone()}
    ra.check()
    out = torch.empty_like(q)
    mismatches = []

    def on_call(i, kind, o):
        if not torch.equal(o.view(torch.int16), want[kind].view(torch.int16)):
            mismatches.append((i, kind))

    kinds, ms = schedule.run(ra, q, k, v, out, sched, on_call=on_call)
    ra.check()
    assert not mismatches, mismatches[:5]
    assert len(kinds) == sched.steps * sched.blocks
    assert kinds.count("int4") / len(kinds) == pytest.approx(schedule.BENCH_SCHEDULE.int4_fraction)
    assert all(t > 0 for t in ms)
    # the dispatch itself: FP16 exactly on the first/last steps and blocks
    for (s, b, kind), got in zip(sched.calls(), kinds):
        edge = (s < sched.first_steps or s >= sched.steps - sched.last_steps or b < sched.first_blocks
                or b >= sched.blocks - sched.last_blocks)
        assert got == ("fp16" if edge else "int4")
