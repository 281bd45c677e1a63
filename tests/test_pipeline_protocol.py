"""The barrier protocol of the bf16 attention kernel, checked on the host.

attn_tc_kernel's roles -- the TMA producer, the MMA issuer, the two softmax warpgroups and the
epilogue warpgroup -- coordinate through mbarriers that are waited on by phase parity.  This test restates each
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
  of one thread execute in issue order, and a commit tracks every earlier product);
* the epilogue reads O_x of a partition only after that partition's last PV product and
  before the next partition's first PV product (which overwrites O_x), and reads the
  (max, sum) slot of that partition before the softmax reuses the slot;
* no product reads a Q, K or V tile before its load has landed.

A CTA's work is a list of partition lengths in KV tiles.

Program order is the kernel's; MMA completion is modelled at the commit that tracks it.  A
TMA load completes (lands and arrives on its barrier) at any later step, in any order.
"""
import random

import pytest

STAGES = 2


class Work:
    """Tile structure of a CTA's work: parts = [tiles of each partition]."""

    def __init__(self, parts):
        self.T = sum(parts)
        self.first_tiles, j = set(), 0
        for n in parts:
            self.first_tiles.add(j)
            j += n
        self.last_tiles = {j for j in range(self.T) if j + 1 in self.first_tiles or j == self.T - 1}


def producer(w):
    yield ("tma", ("Q",), "Q_FULL")             # Q_a and Q_b, one barrier
    for j in range(w.T):
        s = j % STAGES
        if j >= STAGES:
            yield ("wait", f"K_EMPTY{s}", j // STAGES - 1)
        yield ("tma", ("K", j), f"K_FULL{s}")
        if j >= STAGES:
            yield ("wait", f"V_EMPTY{s}", j // STAGES - 1)
        yield ("tma", ("V", j), f"V_FULL{s}")


def issuer(w):
    T, first_tiles, last_tiles = w.T, w.first_tiles, w.last_tiles
    yield ("wait", "Q_FULL", 0)
    if T == 0:
        return
    yield ("wait", "K_FULL0", 0)
    yield ("wait", "V_FULL0", 0)
    yield ("mma", "S", 0, 0)
    yield ("complete", "S_FULL0")
    yield ("mma", "S", 1, 0)
    yield ("complete", "S_FULL1")
    yield ("release", "K", 0)
    yield ("complete", "K_EMPTY0")
    e = 0                                       # ordinal of the current partition
    for j in range(T):
        s, s1, more = j % STAGES, (j + 1) % STAGES, j + 1 < T
        need_free = j in first_tiles and e > 0
        if need_free:
            yield ("wait", "O_FREE0", e - 1)
        yield ("wait", "P_LO0", j)
        yield ("mma", "PVlo", 0, j, e)
        if more:
            yield ("wait", f"K_FULL{s1}", (j + 1) // STAGES)
        yield ("wait", "P_HI0", j)
        yield ("mma", "PVhi", 0, j, e)
        if j in last_tiles:
            yield ("complete", "O_FINAL0")
        if more:
            yield ("mma", "S", 0, j + 1)
            yield ("complete", "S_FULL0")
        if need_free:
            yield ("wait", "O_FREE1", e - 1)
        yield ("wait", "P_LO1", j)
        yield ("mma", "PVlo", 1, j, e)
        if more:
            yield ("wait", f"V_FULL{s1}", (j + 1) // STAGES)
        yield ("wait", "P_HI1", j)
        yield ("mma", "PVhi", 1, j, e)
        if j in last_tiles:
            yield ("complete", "O_FINAL1")
        yield ("release", "V", j)
        yield ("complete", f"V_EMPTY{s}")
        if more:
            yield ("mma", "S", 1, j + 1)
            yield ("complete", "S_FULL1")
            yield ("release", "K", j + 1)
            yield ("complete", f"K_EMPTY{s1}")
        if j in last_tiles:
            e += 1


def softmax(x, w):
    T, first_tiles, last_tiles = w.T, w.first_tiles, w.last_tiles
    e = 0
    for j in range(T):
        yield ("wait", f"S_FULL{x}", j)
        yield ("read_s", x, j)
        if j not in first_tiles:
            yield ("touch_o", x, j)             # a rescale may happen on any later tile
        yield ("write_p", x, j)
        yield ("complete", f"P_LO{x}")
        yield ("complete", f"P_HI{x}")
        if j in last_tiles:
            yield ("write_ml", x, e)
            yield ("complete", f"ML_FULL{x}{e & 1}")
            e += 1


def epilogue(w):
    for e in range(len(w.first_tiles)):
        for x in range(2):
            yield ("wait", f"O_FINAL{x}", e)
            yield ("wait", f"ML_FULL{x}{e & 1}", e >> 1)
            yield ("read_ml", x, e)
            yield ("read_o", x, e)
            yield ("complete", f"O_FREE{x}")


class State:
    def __init__(self, w):
        T = w.T
        self.T = T
        self.w = w
        firsts = sorted(w.first_tiles)
        self.part_first = firsts                            # partition -> first tile
        self.part_last = [f - 1 for f in firsts[1:]] + ([T - 1] if T > 0 else [])
        self.o_part = {0: None, 1: None}    # partition whose sums O_x accumulates
        self.o_read = {0: -1, 1: -1}        # last partition the epilogue read out of O_x
        self.ml_slot = {}                   # (x, slot) -> partition whose (max, sum) it holds
        self.ml_read = {0: -1, 1: -1}
        self.done = {}                  # barrier -> completed phases
        self.loaded = {}                # ("K"|"V", stage) -> tile
        self.landed = set()             # loads whose data has arrived
        self.readers = {}               # ("K"|"V", tile) -> products issued that read it
        self.s_tile = {0: None, 1: None}    # tile whose scores the S buffer holds
        self.p_ready = {0: -1, 1: -1}       # last tile whose P was handed over
        self.pv_issued = {0: -1, 1: -1}     # last tile whose PV hi was issued
        self.s_read = {0: -1, 1: -1}

    def check(self, op, role):
        kind = op[0]
        if kind == "tma" and op[1][0] in "KV":
            _, (kv, j), _ = op
            stage = j % STAGES
            prev = self.loaded.get((kv, stage))
            if prev is not None:
                need = 2 if kv == "K" else 4    # S_a, S_b read K; PV lo/hi of a and b read V
                assert self.readers.get((kv, prev), 0) == need, f"{kv} stage {stage} reloaded early"
            self.loaded[(kv, stage)] = j
        elif kind == "mma" and op[1] == "S":
            _, what, x, j = op
            assert ("Q",) in self.landed, "score product issued before Q landed"
            assert ("K", j) in self.landed, "score product issued before its K tile landed"
            assert self.loaded.get(("K", j % STAGES)) == j, "S issued before its K tile"
            if self.s_tile[x] is not None:
                assert self.p_ready[x] >= self.s_tile[x], "S overwritten before P was handed over"
                assert self.pv_issued[x] >= self.s_tile[x], "S overwritten before PV read P"
            self.s_tile[x] = j
            self.readers[("K", j)] = self.readers.get(("K", j), 0) + 1
        elif kind == "mma":
            _, what, x, j, e = op
            assert self.loaded.get(("V", j % STAGES)) == j, "PV issued before its V tile"
            assert ("V", j) in self.landed, "PV issued before its V tile landed"
            if self.o_part[x] != e:
                # the first product of partition e overwrites O_x
                assert what == "PVlo" and j == self.part_first[e], "O_x restarted mid-partition"
                assert self.o_read[x] == e - 1, "O_x overwritten before the epilogue read it"
                self.o_part[x] = e
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
        elif kind == "write_ml":
            _, x, e = op
            assert self.ml_read[x] >= e - 2, "(max, sum) slot reused before the epilogue read it"
            self.ml_slot[(x, e & 1)] = e
        elif kind == "read_ml":
            _, x, e = op
            assert self.ml_slot.get((x, e & 1)) == e, "epilogue read another partition's (max, sum)"
            self.ml_read[x] = e
        elif kind == "read_o":
            _, x, e = op
            assert self.o_part[x] == e, "epilogue read O of another partition"
            assert self.pv_issued[x] == self.part_last[e], "epilogue read O before its last PV"
            self.o_read[x] = e


def runnable(st, op):
    if op[0] != "wait":
        return True
    _, bar, k = op
    c = st.done.get(bar, 0)
    # a parity wait for phase k is only sound while phase k + 1 has not completed
    assert c <= k + 1, f"wait on {bar} phase {k} would alias (completed {c})"
    return c > k


def simulate(parts, seed):
    rng = random.Random(seed)
    w = Work(parts)
    T = w.T
    st = State(w)
    roles = {"producer": producer(w), "issuer": issuer(w),
             "softmax0": softmax(0, w), "softmax1": softmax(1, w), "epilogue": epilogue(w)}
    pending = {name: next(g, None) for name, g in roles.items()}
    in_flight = []                      # issued TMA loads: (what, barrier)
    land_p = (0.01, 0.1, 0.5)[seed % 3]   # slow loads stay in flight across many steps
    while any(op is not None for op in pending.values()) or in_flight:
        ready = [n for n, op in pending.items() if op is not None and runnable(st, op)]
        assert ready or in_flight, f"deadlock at T={T}: " + str({n: op for n, op in pending.items() if op})
        if in_flight and (not ready or rng.random() < land_p):
            # a load lands (any of those in flight) and arrives on its barrier
            what, bar = in_flight.pop(rng.randrange(len(in_flight)))
            st.landed.add(what)
            st.done[bar] = st.done.get(bar, 0) + 1
            continue
        name = rng.choice(ready)
        op = pending[name]
        if op[0] == "complete":
            st.done[op[1]] = st.done.get(op[1], 0) + 1
        else:
            st.check(op, name)
            if op[0] == "tma":
                in_flight.append((op[1], op[2]))
        pending[name] = next(roles[name], None)


def _partitions(rng, T):
    parts, j = [], 0
    while j < T:
        n = min(rng.randint(1, 5), T - j)
        parts.append(n)
        j += n
    return parts


@pytest.mark.parametrize("T", list(range(0, 41)))
def test_attention_pipeline_protocol(T):
    # partitions of 1..5 tiles, each partition end going through the epilogue
    rng = random.Random(T)
    for seed in range(25):
        simulate(_partitions(rng, T), seed)
