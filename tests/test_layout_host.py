"""Host checks of the register layouts the linear kernels assume, against the
oracle's own (pinned) position function for the interleaved layout.

The forward decode kernel reads lane L's 16-byte slot as its m16n8k16 A
fragment (rows L/4, L/4 + 8; column pairs of L % 4).  The input-gradient
kernel reads the same tiles transposed: lane (g, t) (g = lane / 4,
t = lane % 4) takes the slots 4t + g % 4 (rows t, t + 8) and 4t + g % 4 + 16
(rows t + 4, t + 12) and, in every run of 16 columns, the columns
c = 2 (g % 4) + 8 (g / 4) (lower half-word) and c + 1 (upper half-word), the
code of the 8-row half h sitting at bit BITS h + 2 BITS (g / 4) of its half-word
-- after a further 8-bit shift for the second run of a 2-bit word.  These tests
restate those rules from the kernels' documentation and check every position
against the oracle."""
from __future__ import annotations

import pytest

from oracle import oracle as O


@pytest.mark.parametrize("bits", [4, 2])
def test_forward_fragment_slots(bits):
    T = 64 if bits == 4 else 128
    rows, cols = 16, T
    for lane in range(32):
        r, c = lane // 4, lane % 4
        for run in range(T // 16):
            for slot, (dr, dc) in enumerate(((0, 0), (8, 0), (0, 8), (8, 8))):
                for odd in range(2):
                    n, k = r + dr, 16 * run + 2 * c + dc + odd
                    byte, bit = O.code_position("interleaved", n, k, rows, cols, bits)
                    word = run if bits == 4 else run // 2
                    assert byte // 16 == lane and (byte % 16) // 4 == word
                    field = slot + 4 * odd if bits == 4 else 4 * (run % 2) + slot + 8 * odd
                    assert 8 * (byte % 4) + bit == bits * field, (lane, run, slot, odd)


@pytest.mark.parametrize("bits", [4, 2])
def test_transposed_fragment_slots(bits):
    """Every code of a 16-row tile is read by exactly one (lane, run, h,
    fragment) of the input-gradient kernel, at the position it assumes."""
    T = 64 if bits == 4 else 128
    rows, cols = 16, T
    seen = set()
    for lane in range(32):
        g, t = lane // 4, lane % 4
        hg = g // 4
        for run in range(T // 16):
            word = run if bits == 4 else run // 2
            extra = 8 * (run % 2) if bits == 2 else 0  # second run of a 2-bit word
            for h in range(2):
                for slot_base, row0 in ((4 * t + g % 4, t), (4 * t + g % 4 + 16, t + 4)):
                    for odd in range(2):
                        n = row0 + 8 * h
                        k = 16 * run + 2 * (g % 4) + 8 * hg + odd
                        byte, bit = O.code_position("interleaved", n, k, rows, cols, bits)
                        assert byte // 16 == slot_base, (lane, run, h, odd)
                        assert (byte % 16) // 4 == word
                        pos = 8 * (byte % 4) + bit - 16 * odd - extra
                        assert pos == bits * h + 2 * bits * hg, (lane, run, h, odd, pos)
                        seen.add((n, k))
    assert seen == {(n, k) for n in range(rows) for k in range(cols)}
