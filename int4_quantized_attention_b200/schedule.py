"""Mixed-precision dispatch: which (denoising step, DiT block) pairs run the
FP16 attention path and which run the INT4 path.

"RotateAttention" review page, Sec. 5.1 (quoted in the circularity check) and
the free-parameter ledger: accuracy-sensitive attention stays in FP16 on the
first and last few sampling steps and on the first and last DiT blocks;
everything else runs the INT4 kernel.  Host logic only.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Schedule:
    steps: int
    blocks: int
    first_steps: int
    last_steps: int
    first_blocks: int
    last_blocks: int

    def is_fp16(self, step: int, block: int) -> bool:
        if not (0 <= step < self.steps and 0 <= block < self.blocks):
            raise IndexError("step or block out of range")
        return (step < self.first_steps or step >= self.steps - self.last_steps
                or block < self.first_blocks or block >= self.blocks - self.last_blocks)

    def calls(self):
        """(step, block, 'fp16' | 'int4') for every attention call, in order."""
        for s in range(self.steps):
            for b in range(self.blocks):
                yield s, b, ("fp16" if self.is_fp16(s, b) else "int4")

    @property
    def int4_fraction(self) -> float:
        n = sum(1 for _, _, k in self.calls() if k == "int4")
        return n / float(self.steps * self.blocks)


# The benchmarked schedule: Wan-shaped attention, 10 steps x 40 blocks, FP16 on
# the first/last 2 steps and the first/last 4 blocks (48 % INT4).
BENCH_SCHEDULE = Schedule(steps=10, blocks=40, first_steps=2, last_steps=2,
                          first_blocks=4, last_blocks=4)

# The same split on a quarter of the blocks (10 steps x 10 blocks, FP16 on the
# first/last 2 steps and the first/last block): (6/10) (8/10) = 48 % INT4 as
# well, in 100 calls instead of 400, for the default benchmark run.
BENCH_SCHEDULE_SHORT = Schedule(steps=10, blocks=10, first_steps=2, last_steps=2,
                                first_blocks=1, last_blocks=1)


def run(ra, q, k, v, out, schedule: Schedule, stream=None, time_calls: bool = True, on_call=None):
    """Run every attention call of `schedule` in order on one input set through
    RotateAttention `ra` (the FP16 or the INT4 entry points, as the schedule
    says), writing `out`.  Returns the kinds in call order and, with
    time_calls, each call's device time in ms (CUDA events on `stream`).
    on_call(index, kind, out), if given, runs after each call is enqueued."""
    import torch
    stream = torch.cuda.current_stream() if stream is None else stream
    kinds = [kind for _, _, kind in schedule.calls()]
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in kinds] \
        if time_calls else None
    for i, kind in enumerate(kinds):
        if evs:
            evs[i][0].record(stream)
        ra.forward(q, k, v, path=kind, out=out)
        if evs:
            evs[i][1].record(stream)
        if on_call is not None:
            on_call(i, kind, out)
    if not evs:
        return kinds, None
    torch.cuda.synchronize()
    return kinds, [a.elapsed_time(b) for a, b in evs]
