"""Shared pieces of the barrier-protocol model checks (test infrastructure).

An mbarrier is modelled by its arrival count and number of completed phases. A wait on
parity P passes while the number of completed phases has the other parity, the hardware's
rule, so a barrier two phases ahead of a waiter looks incomplete to it (phase aliasing).
Roles are Python generators that yield after each step; `schedule` interleaves them at random
with a per-role speed, and steps the asynchronous engines (tensor pipe, TMA) in between.
"""
import random


class Barrier:
    def __init__(self, count: int):
        self.count, self.arrived, self.completed = count, 0, 0

    def arrive(self):
        self.arrived += 1
        if self.arrived == self.count:
            self.arrived = 0
            self.completed += 1

    def test_parity(self, parity: int) -> bool:
        # mbarrier.try_wait.parity: passes once the phase of that parity has completed, i.e.
        # while the current (incomplete) phase has the other parity
        return (self.completed & 1) != parity


class Violation(AssertionError):
    pass


def schedule(rng: random.Random, roles, engines, max_steps: int = 200_000):
    """Run generator `roles` to completion, stepping the endless generator `engines` in
    between; raises Violation if the roles stop making progress."""
    live = list(range(len(roles)))
    speed = [rng.choice((1, 1, 2, 8)) for _ in roles]  # skewed speeds push roles apart
    for _ in range(max_steps):
        if not live:
            return
        if engines and rng.random() < 0.3:
            next(rng.choice(engines))
            continue
        k = rng.choices(live, weights=[speed[j] for j in live])[0]
        try:
            next(roles[k])
        except StopIteration:
            live.remove(k)
    raise Violation(f"no progress after {max_steps} steps (roles left: {live})")
