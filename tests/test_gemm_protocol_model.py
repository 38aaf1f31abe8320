"""A model of the prefill GEMM's synchronisation protocol, checked on CPU.

The MMA warp of `gemm_i2_kernel` waits on hardware named barriers, which have
no timeout, so the kernel is hang-free only if every other role arrives
exactly once per barrier phase, in order, whatever its own bounded waits do.
This discrete-event model has the same roles as the kernel:
- 3 producer warps;
- 2 expander groups of 4 warps;
- 4 epilogue warps;
- 1 MMA warp.
It also has the same barriers:
- mbarriers full / empty (7 stages), aempty (4 TMEM A buffers) and accf
  (2 accumulators), completed by the copies and by the MMA's commits;
- named barriers AB[a] (4 expander warps + MMA warp) and ACC[b] (4 epilogue
  warps + MMA warp).

It runs them in random interleavings with random copy and MMA delays, with
and without one K block's copies withheld (the kernel's forced-stall test aid).
Checks:
- every role finishes (no hang);
- no named-barrier phase mixes arrivals of two K blocks or tiles;
- the timeout flag is raised exactly when a copy was withheld.
A planted mistake (expanders that do not wait for the MMA's commit before
reusing a buffer) must be caught.
"""
import random
import sys

import pytest

_SKIP_AEMPTY = False   # planted mistake, switched on by one test

K_STAGES, K_ABUFS, K_PROD = 7, 4, 3
STALL_BLOCK = 2


class MBar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.phase = name, count, count, 0   # phase = completed phases

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity_phase):          # has phase number k completed?
        return self.phase > parity_phase


class NBar:
    def __init__(self, name, warps):
        self.name, self.warps = name, warps
        self.arrived = 0
        self.tags = set()
        self.completed = 0
        self.sync_waiting = []

    def arrive(self, tag):
        self.arrived += 1
        self.tags.add(tag)
        if self.arrived == self.warps:
            assert len(self.tags) == 1, f"{self.name}: phase mixes {self.tags}"
            self.completed += 1
            self.arrived = 0
            self.tags = set()
            return True
        return False


def simulate(kblocks_per_tile, force_stall, seed, limit=60, long_limit=100000):
    rng = random.Random(seed)
    full = [MBar(f"full{s}", 1) for s in range(K_STAGES)]
    empty = [MBar(f"empty{s}", 1 + 4) for s in range(K_STAGES)]
    aempty = [MBar(f"aempty{a}", 1) for a in range(K_ABUFS)]
    accf = [MBar(f"accf{b}", 1) for b in range(2)]
    ab = [NBar(f"AB{a}", 5) for a in range(K_ABUFS)]
    acc = [NBar(f"ACC{b}", 5) for b in range(2)]
    state = {"abort": False, "t": 0, "events": [], "flag": False}
    seq = []   # (tile, kb) per it
    for t, kbs in enumerate(kblocks_per_tile):
        for kb in range(kbs):
            seq.append((t, kb))
    T = len(kblocks_per_tile)

    def later(delay, fn):
        state["events"].append((state["t"] + delay, fn))

    # a role is a generator yielding ("wait_mbar", bar, phase, kind) / ("nb_sync", nbar, tag) / ("nb_arrive", nbar, tag) / ("step",)
    def wait_mbar(bar, k, kind):
        # kind: "abort" (limit + abort flag), "progress" (long limit), "drain"
        start = state["t"]
        while True:
            if bar.done(k):
                return True
            if kind == "abort" and state["abort"]:
                return False
            lim = limit if kind == "abort" else long_limit
            if state["t"] - start > lim:
                return False
            yield ("block",)

    def fail():
        state["abort"] = True
        state["flag"] = True

    # tensor core: MMAs complete in order with delay; commits arrive after all prior MMAs complete
    tc = {"busy_until": 0}

    def tc_issue(commit_bars):
        tc["busy_until"] = max(tc["busy_until"], state["t"]) + rng.randint(1, 4)
        done_at = tc["busy_until"]
        for bar in commit_bars:
            later(done_at - state["t"], bar.arrive)

    def producer(pidx):
        it, last, ok, issued = 0, -1, True, []
        for (t, kb) in seq:
            if it % K_PROD == pidx:
                s, r = it % K_STAGES, it // K_STAGES
                if r > 0:
                    got = yield from wait_mbar(empty[s], r - 1, "abort")
                    if not got:
                        fail()
                        ok = False
                        break
                if not (force_stall and it == STALL_BLOCK):
                    later(rng.randint(1, 30), full[s].arrive)
                    issued.append(it)
                last = it
            it += 1
            yield ("step",)
        if not ok:
            for j in issued:
                if j > last - K_STAGES:
                    yield from wait_mbar(full[j % K_STAGES], j // K_STAGES, "progress")
        return "producer done"

    def mma():
        it, s, a = 0, 0, 0
        for t, kbs in enumerate(kblocks_per_tile):
            b = t & 1
            if t >= 2:
                yield ("nb_sync", acc[b], ("tile", t - 2))
            for kb in range(kbs):
                yield ("nb_sync", ab[a], ("it", it))
                tc_issue([empty[s], aempty[a]])
                it += 1
                s = (s + 1) % K_STAGES
                a = (a + 1) % K_ABUFS
                yield ("step",)
            tc_issue([accf[b]])
        for t in range(max(T - 2, 0), T):
            yield ("nb_sync", acc[t & 1], ("tile", t))
        return "mma done"

    def expander(grp, w):
        it, aborted = 0, False
        for (t, kb) in seq:
            if it % 2 == grp:
                s, a, ra = it % K_STAGES, it % K_ABUFS, it // K_ABUFS
                if not aborted:
                    got = yield from wait_mbar(full[s], it // K_STAGES, "abort")
                    if not got:
                        fail()
                        aborted = True
                empty[s].arrive()
                if ra > 0 and not _SKIP_AEMPTY:
                    got = yield from wait_mbar(aempty[a], ra - 1, "progress")
                    if not got:
                        raise AssertionError(f"expander progress wait failed at it={it}")
                yield ("nb_arrive", ab[a], ("it", it))
            it += 1
            yield ("step",)
        return "expander done"

    def epilogue(w):
        for t in range(T):
            b = t & 1
            got = yield from wait_mbar(accf[b], t >> 1, "progress")
            if not got:
                raise AssertionError(f"epilogue progress wait failed at tile {t}")
            yield ("nb_arrive", acc[b], ("tile", t))
        return "epilogue done"

    roles = {}
    for pi in range(K_PROD):
        roles[f"prod{pi}"] = producer(pi)
    roles["mma"] = mma()
    for g in range(2):
        for w in range(4):
            roles[f"exp{g}.{w}"] = expander(g, w)
    for w in range(4):
        roles[f"epi{w}"] = epilogue(w)
    waiting_nb = {}    # role -> (nbar, completed count at sync start)
    finished = set()
    pending_yield = {}
    steps = 0
    while len(finished) < len(roles):
        steps += 1
        if steps > 2_000_000:
            raise AssertionError("simulation did not finish (hang)")
        state["t"] += 1
        for ev in [e for e in state["events"] if e[0] <= state["t"]]:
            state["events"].remove(ev)
            ev[1]()
        order = [r for r in roles if r not in finished]
        rng.shuffle(order)
        progressed = False
        for name in order:
            if name in waiting_nb:
                nbar, c0 = waiting_nb[name]
                if nbar.completed > c0:
                    del waiting_nb[name]
                else:
                    continue
            try:
                y = next(roles[name])
            except StopIteration:
                finished.add(name)
                progressed = True
                continue
            if y[0] == "nb_arrive":
                y[1].arrive(y[2])
                progressed = True
            elif y[0] == "nb_sync":
                c0 = y[1].completed
                y[1].arrive(y[2])
                if y[1].completed == c0:
                    waiting_nb[name] = (y[1], c0)
                progressed = True
            elif y[0] == "step":
                progressed = True
        if not progressed and not state["events"] and all(n in waiting_nb or n in finished for n in roles):
            raise AssertionError(f"deadlock: waiting {sorted(waiting_nb)}")
    return state["flag"]




CONFIGS = [[3, 12, 1, 7, 2], [12] * 4, [71], [1], [2, 1], [13, 1, 1, 9]]


@pytest.mark.parametrize("cfg", CONFIGS, ids=[f"tiles{len(c)}" for c in CONFIGS])
@pytest.mark.parametrize("force_stall", [False, True])
def test_protocol_never_hangs_or_mixes_phases(cfg, force_stall):
    for seed in range(6):
        flag = simulate(cfg, force_stall, seed * 7919 + len(cfg))
        assert flag == (force_stall and sum(cfg) > STALL_BLOCK)


def test_model_catches_expanders_running_ahead(monkeypatch):
    """The check has teeth: without the wait for the MMA's commit, an expander
    group can arrive for a buffer's next use before the MMA warp consumed the
    previous one, and a barrier phase then mixes two K blocks."""
    global _SKIP_AEMPTY
    monkeypatch.setattr(sys.modules[__name__], "_SKIP_AEMPTY", True)
    with pytest.raises(AssertionError, match="phase mixes|hang|deadlock"):
        for seed in range(20):
            simulate([12] * 4, False, seed)
