"""A model, on the CPU, of how the block-scaled expert MLP's one GEMM launch
hands out its work, checked for the two properties its kernel relies on.

The launch's CTAs take work items from one counter in index order: every
gate/up item (token tile t, 128 weight rows) comes before every down item. A
CTA's producer takes the next item while the current item's last stages go
out. It then issues that item's copies. Before issuing a down item's copies
it waits until the tile's gate/up items have all finished, each having
raised the tile's count after its pieces of h were stored. The item
finishes later, in the CTA's order, whatever the producer does meanwhile
(its MMAs and epilogue need only the copies already issued).

The properties:
* every run ends, even when fewer CTAs can be resident than the grid holds
  (a CTA only becomes resident when another exits), so nothing assumes
  co-residency;
* no down item's copies are issued before its tile's gate/up items are done.

Durations are random; the model runs many seeds, grid sizes and residency
limits, down to one resident CTA.
"""
import heapq
import random

import pytest


def simulate(n_tiles, mt_gu, mt_dn, grid, resident, seed, down_first=False):
    rng = random.Random(seed)
    n_gu = n_tiles * mt_gu
    n_dn = n_tiles * mt_dn
    n_items = n_gu + n_dn

    def item_of(i):
        # (kind, tile): kind 0 = gate/up, 1 = down; the kernel's order puts
        # every gate/up item first (down_first: the order the kernel must not use)
        if down_first:
            return (1, i // mt_dn) if i < n_dn else (0, (i - n_dn) // mt_gu)
        if i < n_gu:
            return 0, i // mt_gu
        return 1, (i - n_gu) // mt_dn

    counter = 0
    done = [0] * n_tiles           # gate/up items finished per tile
    finished = set()
    issue_log = []                 # (time, item) when an item's copies are issued
    events = []                    # (time, seq, kind, payload)
    seq = 0

    def push(t, kind, payload):
        nonlocal seq
        heapq.heappush(events, (t, seq, kind, payload))
        seq += 1

    class Cta:
        def __init__(self, cid):
            self.cid = cid
            self.next = None          # item taken ahead of time
            self.busy_until = 0.0     # the CTA's MMAs and epilogue finish in order
            self.waiting = None       # down item whose tile is not done yet
            self.outstanding = 0      # issued items not finished yet

    def take():
        nonlocal counter
        i = counter
        counter += 1
        return i

    waiting = []   # CTAs blocked on a tile count

    def producer_step(cta, now):
        # the producer's next item: the one taken ahead, else a fresh take
        i = cta.next if cta.next is not None else take()
        cta.next = None
        if i >= n_items:
            if cta.outstanding == 0:
                push(now, "exit", cta)
            else:
                cta.exiting = True
            return
        kind, t = item_of(i)
        if kind == 1 and done[t] < mt_gu:
            cta.waiting = (i, t)
            waiting.append(cta)
            return
        issue(cta, i, now)

    def issue(cta, i, now):
        kind, t = item_of(i)
        if kind == 1:
            assert done[t] == mt_gu, "down item issued before its tile's gate/up items"
        issue_log.append((now, i))
        issue_time = rng.uniform(0.5, 1.5)
        # the next item is taken while this one's last stages go out
        cta.next = take()
        # this item finishes after its copies, behind the CTA's earlier items
        fin = max(cta.busy_until, now + issue_time) + rng.uniform(0.1, 2.0)
        cta.busy_until = fin
        cta.outstanding += 1
        push(fin, "finish", (cta, i))
        push(now + issue_time, "produce", cta)

    resident = min(resident, grid)
    ctas = [Cta(c) for c in range(grid)]
    for c in ctas:
        c.exiting = False
    pending = list(ctas[resident:])
    for c in ctas[:resident]:
        push(0.0, "produce", c)

    now = 0.0
    steps = 0
    while events:
        steps += 1
        assert steps < 10_000_000
        now, _, kind, payload = heapq.heappop(events)
        if kind == "produce":
            producer_step(payload, now)
        elif kind == "finish":
            cta, i = payload
            finished.add(i)
            cta.outstanding -= 1
            k, t = item_of(i)
            if k == 0:
                done[t] += 1
                if done[t] == mt_gu:
                    for w in [w for w in waiting if w.waiting[1] == t]:
                        waiting.remove(w)
                        i2, _ = w.waiting
                        w.waiting = None
                        issue(w, i2, now)
            if cta.exiting and cta.outstanding == 0:
                push(now, "exit", cta)
        elif kind == "exit":
            if pending:
                push(now, "produce", pending.pop(0))
    # every item was issued and finished, and nobody is left waiting
    assert not waiting, "a producer waits for ever"
    assert finished == set(range(n_items))
    return issue_log


@pytest.mark.parametrize("n_tiles,mt_gu,mt_dn", [(1, 3, 2), (5, 45, 23), (34, 45, 23), (7, 1, 1)])
@pytest.mark.parametrize("grid,resident", [(1, 1), (4, 1), (16, 3), (296, 296), (296, 40)])
def test_every_run_ends_and_down_items_follow_their_tiles(n_tiles, mt_gu, mt_dn, grid, resident):
    for seed in range(6):
        log = simulate(n_tiles, mt_gu, mt_dn, grid, resident, seed)
        # items are issued at most once each, every one of them
        issued = [i for _, i in log]
        assert sorted(issued) == list(range(n_tiles * (mt_gu + mt_dn)))


def test_a_wrong_order_is_caught():
    # the model does catch a broken rule: with the down items first in index
    # order and one resident CTA, the CTA takes a down item and waits on a
    # tile whose gate/up items nobody can take
    with pytest.raises(AssertionError, match="waits for ever"):
        simulate(2, 2, 1, grid=4, resident=1, seed=0, down_first=True)
