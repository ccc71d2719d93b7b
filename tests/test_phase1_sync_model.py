"""A randomized model of the synchronisation of phase1_tc_kernel (csrc/phase1_tc.cu),
checked on the CPU for the failures that would hang or corrupt the GPU kernel:
a waiter that misses an mbarrier phase (the hardware parity wait would then
spin until its time limit), a deadlock, or an MMA / TMA copy / softmax step
that touches data out of order.

The model follows the kernel's roles and barriers one to one:
  producer   Q once (q_full), then K(j) and V(j) into stage j & 1 after the
             stage's *_empty barrier (2-stage ring);
  issuer     QK_t(0) for both heads; per key tile j: wait P0(j) (p_full0) and
             V(j) (v_full), PV0(j), wait K(j+1), QK0(j+1); wait P1(j), PV1(j),
             release V(j), QK1(j+1), release K(j+1); MMAs run in issue order on
             one pipe and a commit arrives once every earlier MMA has finished;
  softmax t  wait S_t(j) (s_full_t), read S, write P over S, arrive p_full_t.
mbarriers keep an arrival count and a transaction count per phase; a parity
wait for phase k succeeds when the completed-phase count has the other parity
than k, exactly as mbarrier.try_wait.parity.  Copy latencies, MMA durations
and softmax times are random, so the runs cover many interleavings.  Two
planted protocol mistakes must be caught, which shows the model can see them.
The softmax step may also rescale O (the lazy rescale), so no PV of its head
may be in flight anywhere in that step.
"""
import random

import pytest


class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.done = count, 0, 0

    def arrive(self, n=1, expect_tx=0):
        self.tx += expect_tx
        self.pending -= n
        if self.pending < 0:
            raise AssertionError(f"{self.name}: more arrivals than its count in phase {self.done}")
        self._maybe()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe()

    def _maybe(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def ready(self, k):
        if self.done >= k + 2:
            raise AssertionError(f"missed phase: {self.name} completed phase {self.done - 1} "
                                 f"while a waiter still waits for phase {k}")
        return (self.done & 1) != (k & 1)


class Model:
    def __init__(self, seed, nkv, mutation=None):
        self.rng = random.Random(seed)
        self.nkv, self.mutation = nkv, mutation
        self.t, self.events, self.pipe_free = 0, [], 0
        self.bars = {"q_full": Bar("q_full", 1)}
        for s in (0, 1):
            for name in ("k_full", "k_empty", "v_full", "v_empty", "s_full", "o_final"):
                self.bars[f"{name}{s}"] = Bar(f"{name}{s}", 1)
            self.bars[f"p_full{s}"] = Bar(f"p_full{s}", 128)
        self.k_stage = [None, None]     # key tile held (landed) by each K stage
        self.v_stage = [None, None]
        self.k_readers = [0, 0]         # MMA groups in flight reading a stage
        self.v_readers = [0, 0]
        self.S = [None, None]           # TMEM S_t / P_t: ("S", j) or ("P", j)
        self.s_users = [0, 0]           # MMA groups in flight using S_t / P_t
        self.o_users = [0, 0]           # PV groups in flight accumulating into O_t

    def at(self, t, fn):
        self.events.append((t, fn))

    def copy(self, stage_list, st, j, bar):
        def land():
            stage_list[st] = j
            self.bars[bar].complete_tx(1)
        stage_list[st] = None
        self.bars[bar].arrive(expect_tx=1)
        self.at(self.t + self.rng.randint(1, 600), land)

    def mma_group(self, start_check, finish):
        start = max(self.t, self.pipe_free)
        self.pipe_free = start + self.rng.randint(20, 60)
        self.at(start, start_check)
        self.at(self.pipe_free, finish)

    def commit(self, bar):
        self.at(max(self.t, self.pipe_free), lambda: self.bars[bar].arrive())

    # ------------------------------------------------------------- roles
    def producer(self):
        b = self.bars
        b["q_full"].arrive(expect_tx=1)
        self.at(self.t + self.rng.randint(1, 100), lambda: b["q_full"].complete_tx(1))
        for j in range(self.nkv):
            st = j & 1
            if j >= 2:
                yield (f"k_empty{st}", (j >> 1) - 1)
            assert self.k_readers[st] == 0, f"K stage {st} refilled while an MMA reads it (tile {j})"
            self.copy(self.k_stage, st, j, f"k_full{st}")
            if j >= 2 and self.mutation != "v_no_empty_wait":
                yield (f"v_empty{st}", (j >> 1) - 1)
            assert self.v_readers[st] == 0, f"V stage {st} refilled while an MMA reads it (tile {j})"
            self.copy(self.v_stage, st, j, f"v_full{st}")

    def issuer(self):
        def qk(t, st, j):
            def start():
                assert self.k_stage[st] == j, f"QK{t}({j}) reads K stage {st} holding {self.k_stage[st]}"
                self.k_readers[st] += 1
                self.s_users[t] += 1

            def finish():
                self.k_readers[st] -= 1
                self.s_users[t] -= 1
                self.S[t] = ("S", j)
            self.mma_group(start, finish)

        def pv(t, st, j):
            def start():
                assert self.v_stage[st] == j, f"PV{t}({j}) reads V stage {st} holding {self.v_stage[st]}"
                assert self.S[t] == ("P", j), f"PV{t}({j}) reads {self.S[t]}"
                self.v_readers[st] += 1
                self.s_users[t] += 1
                self.o_users[t] += 1

            def finish():
                self.v_readers[st] -= 1
                self.s_users[t] -= 1
                self.o_users[t] -= 1
            self.mma_group(start, finish)

        yield ("q_full", 0)
        yield ("k_full0", 0)
        qk(0, 0, 0)
        self.commit("s_full0")
        qk(1, 0, 0)
        self.commit("s_full1")
        self.commit("k_empty0")
        nkv = self.nkv
        for j in range(nkv):
            st, st1 = j & 1, (j + 1) & 1
            yield ("p_full0", j)
            yield (f"v_full{st}", j >> 1)
            pv(0, st, j)
            if j == nkv - 1:
                self.commit("o_final0")
            if j + 1 < nkv:
                yield (f"k_full{st1}", (j + 1) >> 1)
                qk(0, st1, j + 1)
                self.commit("s_full0")
            if self.mutation != "pv1_without_p1":
                yield ("p_full1", j)
            pv(1, st, j)
            if j == nkv - 1:
                self.commit("o_final1")
            self.commit(f"v_empty{st}")
            if j + 1 < nkv:
                qk(1, st1, j + 1)
                self.commit("s_full1")
                self.commit(f"k_empty{st1}")

    def softmax(self, t):
        for j in range(self.nkv):
            yield (f"s_full{t}", j)
            assert self.S[t] == ("S", j), f"softmax{t}({j}) reads {self.S[t]}"
            assert self.s_users[t] == 0, f"softmax{t}({j}) reads S while an MMA uses it"
            # the lazy rescale of O may run anywhere in this step: no PV may be in flight
            assert self.o_users[t] == 0, f"softmax{t}({j}) may rescale O while a PV accumulates into it"
            yield ("sleep", self.rng.randint(1, 300))
            assert self.s_users[t] == 0, f"softmax{t}({j}) writes P while an MMA uses S"
            assert self.o_users[t] == 0, f"softmax{t}({j}) may rescale O while a PV accumulates into it"
            self.S[t] = ("P", j)
            self.bars[f"p_full{t}"].arrive(128)
        yield (f"o_final{t}", 0)

    # ---------------------------------------------------------- scheduler
    def run(self):
        actors = {"producer": self.producer(), "issuer": self.issuer(),
                  "softmax0": self.softmax(0), "softmax1": self.softmax(1)}
        waits = {a: None for a in actors}
        for _ in range(10 ** 6):
            if not actors:
                return
            ready = []
            for a in actors:
                w = waits[a]
                if w is None or (w[0] == "sleep" and self.t >= w[1]) or \
                        (w[0] != "sleep" and self.bars[w[0]].ready(w[1])):
                    ready.append(a)
            if ready:
                a = self.rng.choice(ready)
                try:
                    y = next(actors[a])
                except StopIteration:
                    del actors[a]
                    continue
                waits[a] = ("sleep", self.t + y[1]) if y[0] == "sleep" else y
                continue
            wakes = [waits[a][1] for a in actors if waits[a] is not None and waits[a][0] == "sleep"]
            self.events.sort(key=lambda e: e[0])
            nxt = ([self.events[0][0]] if self.events else []) + wakes
            if not nxt:
                raise AssertionError(f"deadlock: { {a: waits[a] for a in actors} }")
            self.t = max(self.t, min(nxt))
            while self.events and self.events[0][0] <= self.t:
                self.events.pop(0)[1]()
        raise AssertionError("no progress")


@pytest.mark.parametrize("nkv", [1, 2, 3, 4, 7])
def test_kernel_protocol_has_no_missed_phase_deadlock_or_race(nkv):
    for seed in range(400):
        Model(seed, nkv).run()


@pytest.mark.parametrize("mutation", ["v_no_empty_wait", "pv1_without_p1"])
def test_the_model_catches_planted_protocol_mistakes(mutation):
    caught = 0
    for seed in range(300):
        try:
            Model(seed, 5, mutation).run()
        except AssertionError:
            caught += 1
    assert caught > 0
