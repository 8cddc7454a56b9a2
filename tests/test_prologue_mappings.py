"""Index arithmetic of the Q/K prologue, emulated on the CPU for every split.

Two mappings decide which channels and table entries a thread touches:

- the Half rotations' register-local layout (used when every segment and
  half-segment boundary is a multiple of 4): thread g of a row takes the 4
  channels lo .. lo + 3 of the first half of a segment and their partners
  hi = lo + d_s/2 .. + 3, with segment s owning the next split[s] / 8 threads;
- the RoPE table slot of pair j in a position's block of segment s:
  (j mod 4) q_s + floor(j / 4), q_s = ceil(d_s / 8).

The GPU parity suite runs them on the pages' splits (44/42/42, 16/56/56);
these checks cover every split of head_dim 128 into three even segments.
"""

import pytest

D = 128


def splits(multiple):
    for s0 in range(multiple, D, multiple):
        for s1 in range(multiple, D - s0, multiple):
            s2 = D - s0 - s1
            if s2 > 0 and s2 % multiple == 0:
                yield (s0, s1, s2)


def half4(split):
    off = [0, split[0], split[0] + split[1]]
    return all(o % 4 == 0 and (s // 2) % 4 == 0 for o, s in zip(off, split))


def pairs_layout(split):
    """(lo, hi, segment) of each of the 16 threads of a row, as the kernel
    computes them from split[0] / 8 and split[1] / 8."""
    off = [0, split[0], split[0] + split[1]]
    q0, q1 = split[0] >> 3, split[1] >> 3
    out = []
    for g in range(16):
        seg = 0 if g < q0 else (1 if g < q0 + q1 else 2)
        start = (0, q0, q0 + q1)[seg]
        lo = off[seg] + 4 * (g - start)
        hi = lo + (split[seg] >> 1)
        out.append((lo, hi, seg))
    return out


@pytest.mark.parametrize("split", [s for s in splits(2) if half4(s)])
def test_half_pairs_layout_partitions_the_channels(split):
    off = [0, split[0], split[0] + split[1]]
    seen = []
    for lo, hi, seg in pairs_layout(split):
        h = split[seg] // 2
        # lo .. lo + 3 in the first half of its segment, hi .. hi + 3 their partners
        assert off[seg] <= lo and lo + 4 <= off[seg] + h
        assert hi == lo + h and hi + 4 <= off[seg] + split[seg]
        # the RoPE pairs (2j, 2j + 1) of the four channels stay inside the group
        assert lo % 2 == 0 and hi % 2 == 0
        seen += list(range(lo, lo + 4)) + list(range(hi, hi + 4))
    assert sorted(seen) == list(range(D))


def test_half4_holds_for_the_hunyuan_split_and_not_for_wan():
    assert half4((16, 56, 56))
    assert not half4((44, 42, 42))


@pytest.mark.parametrize("half", range(1, 65))
def test_table_slots_are_a_bijection_into_the_block(half):
    q = (half + 3) // 4
    slots = [(j % 4) * q + j // 4 for j in range(half)]
    assert len(set(slots)) == half and max(slots) < 4 * q


@pytest.mark.parametrize("split", [(44, 42, 42), (16, 56, 56), (2, 2, 124), (42, 44, 42)])
def test_table_reads_of_a_row_are_consecutive_per_pair(split):
    """For each of a thread's four pairs, the threads of a row whose pair lies
    in the same segment read consecutive slots (the point of the order)."""
    off = [0, split[0], split[0] + split[1]]
    for pp in range(4):
        by_seg = {}
        for g in range(16):
            c = 8 * g + 2 * pp
            s = 0 if c < off[1] else (1 if c < off[2] else 2)
            j = (c - off[s]) // 2
            q = (split[s] // 2 + 3) // 4
            by_seg.setdefault(s, []).append((j % 4) * q + j // 4)
        for s, slots in by_seg.items():
            # consecutive threads in one segment: one run of consecutive slots
            runs = sum(1 for a, b in zip(slots, slots[1:]) if b != a + 1) + 1
            assert runs <= 2, (split, pp, s, slots)
