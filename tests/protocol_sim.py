"""Discrete-event machinery for the CPU models of the tcgen05 kernels' barrier protocols: an
mbarrier with a phase count (a wait names the phase it expects and asserts that the barrier is at
most one phase past it, since the hardware only tests parity), asynchronous completions after
random delays, and a scheduler that runs the roles (generators that yield the waits) in random
order and reports a deadlock when no role can run and nothing is in flight."""
import random


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, self.name
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, k):
        """Has phase k (0-based) completed? The kernel tests parity k & 1, which is only sound
        while the barrier is at most one phase past k."""
        assert self.phase <= k + 1, (f"{self.name}: phase {self.phase} while phase {k} is awaited "
                                     "(a parity wait would alias)")
        return self.phase > k


class Sim:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.events, self.time = [], 0

    def later(self, delay, fn):
        self.events.append((self.time + delay, fn))

    def pop_event(self):
        self.events.sort(key=lambda e: e[0])
        tm, fn = self.events.pop(0)
        self.time = max(self.time, tm)
        fn()

    def roles(self) -> dict:
        raise NotImplementedError

    def run(self):
        """Each role is a generator yielding (barrier, phase) waits, or None for a point where
        other roles may interleave."""
        roles = self.roles()
        blocked = {name: None for name in roles}
        finished = set()
        for _ in range(10 ** 6):
            if len(finished) == len(roles):
                break
            runnable = [r for r in roles if r not in finished and (blocked[r] is None or blocked[r][0].done(blocked[r][1]))]
            if not runnable or (self.events and self.rng.random() < 0.3):
                if not self.events:
                    waits = ", ".join(f"{r} on {b[0].name} phase {b[1]}" for r, b in blocked.items()
                                      if r not in finished and b)
                    raise AssertionError("deadlock: " + waits)
                self.pop_event()
                continue
            r = self.rng.choice(runnable)
            blocked[r] = None
            try:
                w = next(roles[r])
                if w is not None and not w[0].done(w[1]):
                    blocked[r] = w
            except StopIteration:
                finished.add(r)
        else:
            raise AssertionError("no progress")
        while self.events:
            self.pop_event()
