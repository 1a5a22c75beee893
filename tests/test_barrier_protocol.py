"""A model of the FP8 attention kernel's mbarrier protocol (csrc/attention.cu), run
under adversarial schedules on the CPU.

Agents, as in the kernel: the TMA producer (K/V ring of 4 stages), the MMA
issuer(s) -- one thread for both query tiles in a fixed order (coupled) or one
per tile (decoupled) --, four softmax warps per query tile, and the tensor pipe,
which runs MMAs in issue order; a commit arrives once every earlier MMA of its
thread is done. Every wait sees a barrier only through the parity of its
phase, as `mbarrier.try_wait.parity` does.

A softmax warp whose key tile has only zero probabilities may skip storing P
(its columns already hold zeros). The kernel's rule: that warp still waits for
the previous P.V (`o_ready`) before arriving on `p_full`. The model checks that
with this rule every schedule completes, for both issue orders, and that the
older rule -- wait only for the previous `p_full` phase -- can leave `p_full`
two phases ahead of a slow MMA thread, whose parity wait then never succeeds.
"""
import random

import pytest

STAGES = 4


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):
        """The phase with this parity has completed: what a parity wait can tell."""
        return (self.phase & 1) != parity


def run(n_tiles, decoupled, old_rule, seed, zero_p, slow_mma, max_steps=40000):
    """Returns "ok" if every agent finishes, "stuck" if none can move any more."""
    rnd = random.Random(seed)
    n_mma = 2 if decoupled else 1
    bar = {("k_full", i): Bar(1) for i in range(STAGES)}
    bar.update({("v_full", i): Bar(1) for i in range(STAGES)})
    bar.update({("kv_empty", i): Bar(n_mma) for i in range(STAGES)})
    for t in range(2):
        bar.update({("s_full", t): Bar(1), ("s_free", t): Bar(4), ("p_full", t): Bar(4), ("o_ready", t): Bar(1)})
    pipes = {}  # per MMA thread, in issue order: the barrier each commit arrives at once its earlier MMAs are done
    tma = []    # loads in flight: [delay, keys]

    def producer():
        for it in range(n_tiles):
            st = it % STAGES
            while not bar["kv_empty", st].done(((it // STAGES) & 1) ^ 1):
                yield False
            tma.append([rnd.randint(1, 6), [("k_full", st), ("v_full", st)]])
            yield True

    def wait(key, parity):
        while not bar[key].done(parity):
            yield False

    def mma(tiles):
        pipe = pipes.setdefault(tuple(tiles), [])
        yield from wait(("k_full", 0), 0)
        for t in tiles:
            pipe.append(("s_full", t))
        for it in range(n_tiles):
            st, nst = it % STAGES, (it + 1) % STAGES
            if it + 1 < n_tiles:
                yield from wait(("k_full", nst), ((it + 1) // STAGES) & 1)
            yield from wait(("v_full", st), (it // STAGES) & 1)
            for t in tiles:
                if it + 1 < n_tiles:
                    yield from wait(("s_free", t), it & 1)
                    pipe.append(("s_full", t))
                yield from wait(("p_full", t), it & 1)
                pipe.append(("o_ready", t))
            pipe.append(("kv_empty", st))
            yield True

    def softmax(t):
        p_zero = False
        for it in range(n_tiles):
            yield from wait(("s_full", t), it & 1)
            bar["s_free", t].arrive()
            zero = rnd.random() < zero_p
            if it > 0:
                if old_rule and zero and p_zero:
                    yield from wait(("p_full", t), (it - 1) & 1)
                else:
                    yield from wait(("o_ready", t), (it - 1) & 1)
            p_zero = zero
            bar["p_full", t].arrive()
            yield True

    agents = {"producer": producer()}
    if decoupled:
        agents["mma0"], agents["mma1"] = mma([0]), mma([1])
    else:
        agents["mma0"] = mma([0, 1])
    for t in range(2):
        for w in range(4):
            agents[("softmax", t, w)] = softmax(t)
    live = dict(agents)
    for _ in range(max_steps):
        moved = False
        order = list(live)
        rnd.shuffle(order)
        for name in order:
            if isinstance(name, str) and name.startswith("mma") and rnd.random() < slow_mma:
                continue  # the MMA thread is elsewhere (asleep, or busy with the other tile)
            try:
                moved |= bool(next(live[name]))
            except StopIteration:
                del live[name]
                moved = True
        busy = [q for q in pipes.values() if q]
        if busy and rnd.random() < 0.5:
            bar[rnd.choice(busy).pop(0)].arrive()  # threads' MMAs finish in issue order, not with each other
            moved = True
        for load in list(tma):
            load[0] -= 1
            if load[0] <= 0:
                for key in load[1]:
                    bar[key].arrive()
                tma.remove(load)
                moved = True
        if not live and not any(pipes.values()):
            return "ok"
        if not moved and not tma and not any(pipes.values()) and slow_mma == 0.0:
            return "stuck"
    return "stuck" if live else "ok"


@pytest.mark.parametrize("decoupled", [False, True])
def test_committed_rule_never_hangs(decoupled):
    for seed in range(60):
        for n in (1, 2, 5, 9, 17):
            zero_p = (0.0, 0.6, 0.95)[seed % 3]
            r = run(n, decoupled, old_rule=False, seed=seed, zero_p=zero_p, slow_mma=(0.0, 0.8, 0.97)[seed % 3])
            assert r == "ok", (decoupled, seed, n)


def test_old_rule_can_leave_p_full_two_phases_ahead():
    """With the old rule and a slow MMA thread, some schedule never finishes: the
    zero-tile warps complete two p_full phases before the MMA thread looks, so its
    parity wait for the first one never succeeds."""
    stuck = 0
    for seed in range(120):
        for decoupled in (False, True):
            stuck += run(9, decoupled, old_rule=True, seed=seed, zero_p=0.97, slow_mma=0.97,
                         max_steps=20000) == "stuck"
    assert stuck > 0
