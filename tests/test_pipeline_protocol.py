"""The barrier protocol of the bf16 attention kernel, checked on the host.

attn_tc_kernel's roles -- the TMA producer, the MMA issuer and the two softmax warpgroups --
coordinate through mbarriers that are waited on by phase parity.  This test restates each
role's sequence of waits, arrivals and commits in program order (with the phase index
each parity stands for), runs the roles under many random interleavings for every tile
count up to 40, and checks that:

* no interleaving deadlocks: some role can always proceed until all have finished;
* no wait can alias: when a role waits for phase k of a barrier, the barrier has not yet
  completed phase k + 1 (a parity wait cannot tell k from k + 2);
* no buffer is reused early: a K/V ring stage is reloaded only after every product that
  reads it has been issued, an S buffer is overwritten only after the softmax has handed
  over P from it and the PV products reading that P were issued, and O is read or
  rescaled by the softmax only after the previous PV into it was issued (tcgen05 products
  of one thread execute in issue order, and a commit tracks every earlier product).

Program order is the kernel's; MMA completion is modelled at the commit that tracks it.
"""
import random

import pytest

STAGES = 2


def producer(T):
    yield ("complete", "Q_FULL")
    for j in range(T):
        s = j % STAGES
        if j >= STAGES:
            yield ("wait", f"K_EMPTY{s}", j // STAGES - 1)
        yield ("load", "K", j)
        yield ("complete", f"K_FULL{s}")
        if j >= STAGES:
            yield ("wait", f"V_EMPTY{s}", j // STAGES - 1)
        yield ("load", "V", j)
        yield ("complete", f"V_FULL{s}")


def issuer(T):
    yield ("wait", "Q_FULL", 0)
    if T > 0:
        yield ("wait", "K_FULL0", 0)
        yield ("wait", "V_FULL0", 0)
        yield ("mma", "S", 0, 0)
        yield ("complete", "S_FULL0")
        yield ("mma", "S", 1, 0)
        yield ("complete", "S_FULL1")
        yield ("release", "K", 0)
        yield ("complete", "K_EMPTY0")
    for j in range(T):
        s, s1, more = j % STAGES, (j + 1) % STAGES, j + 1 < T
        yield ("wait", "P_LO0", j)
        yield ("mma", "PVlo", 0, j)
        if more:
            yield ("wait", f"K_FULL{s1}", (j + 1) // STAGES)
        yield ("wait", "P_HI0", j)
        yield ("mma", "PVhi", 0, j)
        yield ("complete", "O_DONE0")
        if more:
            yield ("mma", "S", 0, j + 1)
            yield ("complete", "S_FULL0")
        yield ("wait", "P_LO1", j)
        yield ("mma", "PVlo", 1, j)
        if more:
            yield ("wait", f"V_FULL{s1}", (j + 1) // STAGES)
        yield ("wait", "P_HI1", j)
        yield ("mma", "PVhi", 1, j)
        yield ("complete", "O_DONE1")
        yield ("release", "V", j)
        yield ("complete", f"V_EMPTY{s}")
        if more:
            yield ("mma", "S", 1, j + 1)
            yield ("complete", "S_FULL1")
            yield ("release", "K", j + 1)
            yield ("complete", f"K_EMPTY{s1}")


def softmax(x, T, first_tiles):
    for j in range(T):
        yield ("wait", f"S_FULL{x}", j)
        yield ("read_s", x, j)
        if j in first_tiles and j > 0:
            yield ("touch_o", x, j)             # epilogue of the previous partition
        yield ("touch_o", x, j)                 # a rescale may happen on any tile
        yield ("write_p", x, j)
        yield ("complete", f"P_LO{x}")
        yield ("complete", f"P_HI{x}")
    if T > 0:
        yield ("wait", f"O_DONE{x}", T - 1)
        yield ("touch_o", x, T)


class State:
    def __init__(self, T):
        self.T = T
        self.done = {}                  # barrier -> completed phases
        self.loaded = {}                # ("K"|"V", stage) -> tile
        self.readers = {}               # ("K"|"V", tile) -> products issued that read it
        self.s_tile = {0: None, 1: None}    # tile whose scores the S buffer holds
        self.p_ready = {0: -1, 1: -1}       # last tile whose P was handed over
        self.pv_issued = {0: -1, 1: -1}     # last tile whose PV hi was issued
        self.s_read = {0: -1, 1: -1}

    def check(self, op, role):
        kind = op[0]
        if kind == "load":
            _, kv, j = op
            stage = j % STAGES
            prev = self.loaded.get((kv, stage))
            if prev is not None:
                need = 2 if kv == "K" else 4    # S_a, S_b read K; PV lo/hi of a and b read V
                assert self.readers.get((kv, prev), 0) == need, f"{kv} stage {stage} reloaded early"
            self.loaded[(kv, stage)] = j
        elif kind == "mma":
            _, what, x, j = op
            if what == "S":
                assert self.loaded.get(("K", j % STAGES)) == j, "S issued before its K tile"
                if self.s_tile[x] is not None:
                    assert self.p_ready[x] >= self.s_tile[x], "S overwritten before P was handed over"
                    assert self.pv_issued[x] >= self.s_tile[x], "S overwritten before PV read P"
                self.s_tile[x] = j
                self.readers[("K", j)] = self.readers.get(("K", j), 0) + 1
            else:
                assert self.loaded.get(("V", j % STAGES)) == j, "PV issued before its V tile"
                assert self.p_ready[x] >= j if what == "PVhi" else True
                self.readers[("V", j)] = self.readers.get(("V", j), 0) + 1
                if what == "PVhi":
                    self.pv_issued[x] = j
        elif kind == "read_s":
            _, x, j = op
            assert self.s_tile[x] == j, "softmax read a score buffer holding another tile"
            self.s_read[x] = j
        elif kind == "write_p":
            _, x, j = op
            self.p_ready[x] = j
        elif kind == "touch_o":
            _, x, j = op
            assert self.pv_issued[x] >= j - 1, "O touched before the previous PV was issued"


def runnable(st, op):
    if op[0] != "wait":
        return True
    _, bar, k = op
    c = st.done.get(bar, 0)
    # a parity wait for phase k is only sound while phase k + 1 has not completed
    assert c <= k + 1, f"wait on {bar} phase {k} would alias (completed {c})"
    return c > k


def simulate(T, first_tiles, seed):
    rng = random.Random(seed)
    st = State(T)
    roles = {"producer": producer(T), "issuer": issuer(T),
             "softmax0": softmax(0, T, first_tiles), "softmax1": softmax(1, T, first_tiles)}
    pending = {name: next(g, None) for name, g in roles.items()}
    while any(op is not None for op in pending.values()):
        ready = [n for n, op in pending.items() if op is not None and runnable(st, op)]
        assert ready, f"deadlock at T={T}: " + str({n: op for n, op in pending.items() if op})
        name = rng.choice(ready)
        op = pending[name]
        if op[0] == "complete":
            st.done[op[1]] = st.done.get(op[1], 0) + 1
        else:
            st.check(op, name)
        pending[name] = next(roles[name], None)


@pytest.mark.parametrize("T", list(range(0, 41)))
def test_attention_pipeline_protocol(T):
    rng = random.Random(T)
    for seed in range(25):
        # partitions of 1..5 tiles: their first tiles trigger the epilogue
        firsts, j = set(), 0
        while j < T:
            firsts.add(j)
            j += rng.randint(1, 5)
        simulate(T, firsts, seed)
