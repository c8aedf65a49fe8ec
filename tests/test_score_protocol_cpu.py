"""A dependency model of one CTA of the tcgen05 score kernel, run on the CPU.

The roles wait on one another through mbarriers:
- the producer writes the tile info of tile k once the MMAs of tile k - stages
  are done (its key stage is free), once the epilogue has handed back tile
  k - 16 (its tile-info slot is free) and, at the first tile of a request,
  once the query buffer it reuses is released;
- the MMA issuer, at the first tile of a request, releases the previous
  request's query buffer, then issues tile g once its keys are in and the
  epilogue has handed back tile g - nacc (its accumulator);
- epilogue group h takes tiles h, h + T, ...; before tile i it waits for the
  tile info of tile i + dist*T (the side-data prefetch), then for the MMAs
  of tile i, then hands tile i back.

The model fires every enabled event until nothing changes; a hand-back that
never happens is a deadlock (on the GPU, a bounded wait expiring).  The tests
check that the prefetch distance the kernel picks is safe in every launch
plan, over request layouts with many short requests, and that one more tile
of distance is not."""
import itertools
import random

import pytest


def kernel_distance(T, nacc, nq, stages):
    """The kernel's rule: the largest of 2, 1, 0 with d*T < nq + nacc and
    d*T < stages + nacc."""
    d = 2
    while d > 0 and not (d * T < nq + nacc and d * T < stages + nacc):
        d -= 1
    return d


def runs_to_completion(req, T, nacc, nq, stages, dist, aux=16):
    n = len(req)
    first = [k == 0 or req[k] != req[k - 1] for k in range(n)]
    riter = [r - 1 for r in itertools.accumulate(1 if f else 0 for f in first)]
    info, commit, handback = [False] * n, [False] * n, [False] * n
    released = set()                      # request iterations whose query buffer is free
    producer, mma = 0, 0
    nxt = {h: h for h in range(T)}        # next tile of each group
    ready = {h: False for h in range(T)}  # prefetch wait passed for that tile
    prologue = {h: dist == 0 for h in range(T)}
    changed = True
    while changed:
        changed = False
        if producer < n:
            k = producer
            ok = not (first[k] and riter[k] >= nq) or (riter[k] - nq) in released
            ok = ok and (k < stages or commit[k - stages]) and (k < aux or handback[k - aux])
            if ok:
                info[k] = True
                producer += 1
                changed = True
        if mma < n:
            g = mma
            if first[g] and riter[g] >= 1 and (riter[g] - 1) not in released:
                released.add(riter[g] - 1)
                changed = True
            if info[g] and (g < nacc or handback[g - nacc]):
                commit[g] = True
                mma += 1
                changed = True
        for h in range(T):
            i = nxt[h]
            if i >= n:
                continue
            if not prologue[h]:
                if all(info[x] for x in range(h, min(n, h + dist * T), T)):
                    prologue[h] = True
                    changed = True
                continue
            if not ready[h]:
                want = i if dist == 0 else i + dist * T
                if want >= n or info[want]:
                    ready[h] = True
                    changed = True
            if ready[h] and commit[i]:
                handback[i] = True
                nxt[h] = i + T
                ready[h] = False
                changed = True
    return all(handback)


def request_layouts(seed, count=250, n=64):
    rng = random.Random(seed)
    out = [[0] * n]
    for _ in range(count):
        req, r = [], 0
        while len(req) < n:
            req += [r] * rng.choice([1, 1, 1, 2, 3, 5, 8, 20])
            r += 1
        out.append(req[:n])
    return out


# (epilogue tile groups T, accumulators nacc, query buffers nq, key stages)
# of the launch plans: two CTAs per SM at N <= 64 and at 64 < N <= 128 (3 to
# 8 stages, as shared memory allows), one CTA per SM at N > 128 with two
# groups per tile (several rows) or one (a single row).
PLANS = ([(2, 4, 1, s) for s in range(3, 9)] + [(2, 2, 1, s) for s in range(3, 9)] +
         [(2, 2, 2, 8), (4, 2, 2, 8)])


@pytest.mark.parametrize("plan", PLANS)
def test_kernel_prefetch_distance_never_deadlocks(plan):
    T, nacc, nq, stages = plan
    d = kernel_distance(*plan)
    for req in request_layouts(stages * 10 + nacc):
        assert runs_to_completion(req, T, nacc, nq, stages, d), (plan, d, req)


@pytest.mark.parametrize("plan", [(2, 2, 1, 5), (2, 2, 2, 8), (4, 2, 2, 8), (2, 4, 1, 6)])
def test_one_more_tile_of_distance_can_deadlock(plan):
    # the rule is tight: with short requests, distance d + 1 stalls
    T, nacc, nq, stages = plan
    d = kernel_distance(*plan) + 1
    assert not all(runs_to_completion(req, T, nacc, nq, stages, d) for req in request_layouts(7))


def test_headline_plan_keeps_two_tiles_of_prefetch():
    assert kernel_distance(2, 4, 1, 6) == 2      # one row, N = 64, two CTAs per SM
    assert kernel_distance(2, 2, 2, 8) == 1      # MTP rows, N = 256
    assert kernel_distance(4, 2, 2, 8) == 0      # one row, N > 128
