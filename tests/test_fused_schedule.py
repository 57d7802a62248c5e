"""The fused prefill's division of work among CTAs, modelled on the CPU.

The steps of all units (head pairs), unit-major, are cut into one contiguous range per CTA;
a CTA runs the piece at its range's end first (a unit's first blocks), then its whole
units, then the piece at its start (a unit's last blocks), whose start state the previous
CTA hands over.  This model restates that ordering (the kernel's StepSeq) and checks that
every (unit, block) step is run exactly once, that a piece starts mid-unit only at a range
start and ends mid-unit only at a range end (where the hand-offs are), and that with equal
step times every hand-off is ready before the CTA that needs it gets there, whenever a CTA
has at least a unit's worth of blocks.
"""
import pytest


def cta_steps(c, S, U, nb):
    """(step index, piece start, piece end) in the order CTA c runs them."""
    W = U * nb
    a, e = c * W // S, (c + 1) * W // S
    ua, ue, ka = a // nb, e // nb, a % nb
    if e <= (ua + 1) * nb:
        iv = [(a, e)]
    else:
        iv = [(ue * nb, e), ((ua + 1) * nb if ka else a, ue * nb), ((a, (ua + 1) * nb) if ka else (0, 0))]
    out = []
    for lo, hi in iv:
        for i in range(lo, hi):
            out.append((i, i == lo or i % nb == 0, i == hi - 1 or i % nb == nb - 1))
    return a, e, out


def check(U, nb, sms=148):
    S = min(U, sms)
    seen, produced, needed = set(), {}, {}
    for c in range(S):
        a, e, steps = cta_steps(c, S, U, nb)
        assert len(steps) == e - a
        for t, (i, first, last) in enumerate(steps):
            assert i not in seen
            seen.add(i)
            if first and i % nb:
                assert i == a                      # a mid-unit start is the range start
                needed[c] = t
            if last and i % nb != nb - 1:
                assert i == e - 1                  # a mid-unit end is the range end
                produced[c + 1] = t + 1
    assert seen == set(range(U * nb))
    for c, t in needed.items():
        assert c in produced
        if U * nb >= S * nb:                       # at least a unit of blocks per CTA
            assert produced[c] <= t, (c, produced[c], t)
    return max(len(cta_steps(c, S, U, nb)[2]) for c in range(S))


@pytest.mark.parametrize("U,nb", [(160, 128), (96, 16), (4, 3), (2, 1), (300, 5), (149, 2), (1000, 7),
                                  (150, 1), (148, 9), (333, 64)])
def test_every_step_once_and_handoffs_in_time(U, nb):
    check(U, nb)


def test_long_prefill_balance():
    # 2.7B-shaped long prefill: 4 batches x 40 head pairs, 128 blocks, on 148 SMs
    assert check(160, 128) == 139                  # one unit per CTA would take 2 x 128
