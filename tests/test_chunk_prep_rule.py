"""Host check of how a local chunked-prefill call splits the copy of the ring rows between
the CTAs of its prologue launch.

The attention of a local chunk needs the window - 1 ring rows that precede the chunk
(positions pos0 - window + 1 .. pos0 - 1), while the same launch writes the chunk's own
tokens into the ring.  Token i enters the ring when i >= T - window and takes slot
(pos0 + i) mod window.  Before it writes, it saves the row that slot held, which is row
(i mod window) - 1 of the copy (zeros before position 0), when i mod window >= 1.  A copy
CTA for row e skips the rows some entering token saves: when T >= window (every slot is
taken), else when e + 1 <= T - 1.  This test restates that partition (the kernel's rule, not
the oracle's arithmetic) and checks on a simulated ring that every row is written exactly
once with the position it must hold, and that no slot is read by a copy CTA while a token
CTA writes it.  The GPU chunk tests check the kernel itself against the oracle.
"""
import pytest


def _partition(T, W, p0):
    L = W - 1
    before = {q % W: q for q in range(max(0, p0 - W), p0)}   # slot -> position before the call
    written = {}
    taken = set()
    for i in range(T):                      # token CTAs that enter the ring
        if p0 < 0 or i < T - W:
            continue
        slot = (p0 + i) % W
        assert slot not in taken, "two tokens of one call take the same slot"
        taken.add(slot)
        r = i % W
        if r >= 1:
            q = p0 + r - W
            written.setdefault(r - 1, []).append(before.get(slot) if q >= 0 else 0)
    for e in range(L):                      # copy CTAs
        if p0 >= 0 and (T >= W or e + 1 <= T - 1):
            continue
        j = p0 - L + e
        if p0 >= 0 and j >= 0:
            assert j % W not in taken, "a copy CTA reads a slot a token CTA writes"
            written.setdefault(e, []).append(before.get(j % W))
        else:
            written.setdefault(e, []).append(0)
    return written


@pytest.mark.parametrize("W", [1, 2, 3, 7, 100, 512])
def test_every_ring_row_written_once_with_its_position(W):
    for T in sorted({1, 2, 3, 5, max(1, W - 1), W, W + 1, 2 * W - 1, 2 * W, 3 * W + 5, 700, 8192}):
        for p0 in (-1, 0, 1, 3, W - 1, W, W + 3, 1000, 57344):
            written = _partition(T, W, p0)
            for e in range(W - 1):
                vals = written.get(e, [])
                assert len(vals) == 1, (T, W, p0, e, vals)
                pos = p0 - (W - 1) + e
                expect = pos if (p0 >= 0 and pos >= 0) else 0
                assert vals[0] == expect, (T, W, p0, e, vals, expect)
