"""The dispatch kernels' dynamic token order, modelled on the host.

Thread 0 of each CTA claims tokens from one counter, one token ahead of the
token being loaded (`dispatch_fp8_bulk_kernel` / `dispatch_bf16_bulk_kernel`,
claim word given).  This plays every CTA's sequence of claims under random
interleavings and checks what the kernels and the CGL_ERANGE threshold rely on:
every token of [0, n) is dispatched exactly once, and a launch that starts from
zero hands out at most n + 2 G values, so no claim reaches n + 2 G (the kernels
flag n + 3 G and above as a scratch that was not zero).
"""

import random

import pytest


def _cta(n, claim):
    """One CTA's thread 0, as a generator: yields before every atomic claim,
    returns the tokens it dispatched.  Mirrors the kernels' control flow:
    two claims up front, a third when the second is a token, then one more
    per token while the one after next is a token."""
    clamp = lambda v: v if v < n else n
    done = []
    yield
    v1 = claim()
    yield
    v2 = claim()
    t = clamp(v1)
    tn = clamp(v2) if t < n else n
    pend = n
    if tn < n:
        yield
        pend = claim()
    while t < n:
        s = clamp(pend)                  # s_next: the claim made one token earlier
        done.append(t)                   # token t is quantised and copied
        tnn = s if tn < n else n
        if tnn < n:
            yield
            pend = claim()
        else:
            pend = n
        t, tn = tn, tnn
    return done


def _run(n, grid, seed):
    rng = random.Random(seed)
    counter = [0]
    values = []

    def claim():
        v = counter[0]
        counter[0] += 1
        values.append(v)
        return v

    ctas = [_cta(n, claim) for _ in range(grid)]
    dispatched, live = [], list(range(grid))
    while live:
        i = rng.choice(live)
        try:
            next(ctas[i])
        except StopIteration as stop:
            dispatched += stop.value
            live.remove(i)
    return sorted(dispatched), values


@pytest.mark.parametrize("n,grid", [(1, 2), (5, 3), (296, 296), (297, 296), (600, 296), (4096, 296),
                                    (4096, 37), (100, 7), (7, 100)])
def test_every_token_once_and_claims_below_bound(n, grid):
    for seed in range(20):
        dispatched, values = _run(n, grid, seed)
        assert dispatched == list(range(n))
        assert len(values) <= n + 2 * grid
        assert max(values) < n + 2 * grid
        assert len(set(values)) == len(values)


def test_skewed_schedules():
    """One CTA runs alone to the end while the others wait at their first claim."""
    n, grid = 50, 8
    counter = [0]
    values = []

    def claim():
        v = counter[0]
        counter[0] += 1
        values.append(v)
        return v

    ctas = [_cta(n, claim) for _ in range(grid)]
    dispatched = []
    for c in ctas[1:]:
        next(c)                          # parked before their first claim
    try:
        while True:
            next(ctas[0])
    except StopIteration as stop:
        dispatched += stop.value
    assert dispatched == list(range(n))  # the first CTA took every token
    for c in ctas[1:]:
        try:
            while True:
                next(c)
        except StopIteration as stop:
            assert stop.value == []
    assert max(values) < n + 2 * grid
