"""A randomized model of the synchronisation of the two tcgen05 attention
kernels, phase1_tc_kernel (csrc/phase1_tc.cu) and phase2_tc_kernel
(csrc/phase2_tc.cu), checked on the CPU for the failures that would hang or
corrupt the GPU kernel:
a waiter that misses an mbarrier phase (the hardware parity wait would then
spin until its time limit), a deadlock, or an MMA / TMA copy / softmax step
that touches data out of order.

The model follows the kernels' roles and barriers one to one:
  producer   Q once (q_full), then K(j) into stage j % KST and V(j) into stage
             j % VST after the stage's *_empty barrier (Phase 1: 2 and 2
             stages; Phase 2: 3 and 2 at d = 128, 4 and 4 at d = 64);
  converter  (Phase 2 only) after K(j) lands, convert the stage to fp16 in
             place and arrive k_conv; the issuer's QK^T waits for that;
  issuer     QK_t(0) for both heads; per key tile j: wait P0(j) (p_full0) and
             V(j) (v_full), PV0(j), wait K(j+1), QK0(j+1); wait P1(j), PV1(j),
             release V(j), QK1(j+1), release K(j+1); MMAs run in issue order on
             one pipe and a commit arrives once every earlier MMA has finished;
  softmax t  wait S_t(j) (s_full_t), read S, write P over S, arrive p_full_t
             (t is the head in Phase 1 and the 128-row tile in Phase 2).
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
    def __init__(self, seed, nkv, mutation=None, kst=2, vst=2, convert=False):
        self.rng = random.Random(seed)
        self.nkv, self.mutation = nkv, mutation
        self.kst, self.vst, self.convert = kst, vst, convert
        self.t, self.events, self.pipe_free = 0, [], 0
        self.bars = {"q_full": Bar("q_full", 1)}
        for s in range(kst):
            for name in ("k_full", "k_empty"):
                self.bars[f"{name}{s}"] = Bar(f"{name}{s}", 1)
            self.bars[f"k_conv{s}"] = Bar(f"k_conv{s}", 64)
        for s in range(vst):
            for name in ("v_full", "v_empty"):
                self.bars[f"{name}{s}"] = Bar(f"{name}{s}", 1)
        for t in (0, 1):
            for name in ("s_full", "o_final"):
                self.bars[f"{name}{t}"] = Bar(f"{name}{t}", 1)
            self.bars[f"p_full{t}"] = Bar(f"p_full{t}", 128)
        self.k_stage = [None] * kst     # key tile held (landed) by each K stage
        self.k_ready = [None] * kst     # key tile whose stage is ready for QK^T (converted in Phase 2)
        self.v_stage = [None] * vst
        self.k_readers = [0] * kst      # MMA groups in flight reading a stage
        self.v_readers = [0] * vst
        self.S = [None, None]           # TMEM S_t / P_t: ("S", j) or ("P", j)
        self.s_users = [0, 0]           # MMA groups in flight using S_t / P_t
        self.o_users = [0, 0]           # PV groups in flight accumulating into O_t

    def at(self, t, fn):
        self.events.append((t, fn))

    def copy(self, stage_list, st, j, bar):
        def land():
            stage_list[st] = j
            if stage_list is self.k_stage and not self.convert:
                self.k_ready[st] = j
            self.bars[bar].complete_tx(1)
        stage_list[st] = None
        if stage_list is self.k_stage:
            self.k_ready[st] = None
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
            sk, sv = j % self.kst, j % self.vst
            if j >= self.kst:
                yield (f"k_empty{sk}", j // self.kst - 1)
            assert self.k_readers[sk] == 0, f"K stage {sk} refilled while an MMA reads it (tile {j})"
            self.copy(self.k_stage, sk, j, f"k_full{sk}")
            if j >= self.vst and self.mutation != "v_no_empty_wait":
                yield (f"v_empty{sv}", j // self.vst - 1)
            assert self.v_readers[sv] == 0, f"V stage {sv} refilled while an MMA reads it (tile {j})"
            self.copy(self.v_stage, sv, j, f"v_full{sv}")

    def converter(self):
        for j in range(self.nkv):
            sk = j % self.kst
            if self.mutation != "convert_before_landing":
                yield (f"k_full{sk}", j // self.kst)
            assert self.k_stage[sk] == j, f"converter({j}) converts stage {sk} holding {self.k_stage[sk]}"
            assert self.k_readers[sk] == 0, f"converter({j}) rewrites stage {sk} while an MMA reads it"
            yield ("sleep", self.rng.randint(1, 200))
            assert self.k_stage[sk] == j and self.k_readers[sk] == 0
            self.k_ready[sk] = j
            self.bars[f"k_conv{sk}"].arrive(64)

    def issuer(self):
        def qk(t, st, j):
            def start():
                assert self.k_ready[st] == j, f"QK{t}({j}) reads K stage {st} holding {self.k_ready[st]}"
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

        kbar = "k_conv" if self.convert else "k_full"
        yield ("q_full", 0)
        yield (f"{kbar}0", 0)
        qk(0, 0, 0)
        self.commit("s_full0")
        qk(1, 0, 0)
        self.commit("s_full1")
        self.commit("k_empty0")
        nkv = self.nkv
        for j in range(nkv):
            sv, sk1 = j % self.vst, (j + 1) % self.kst
            yield ("p_full0", j)
            yield (f"v_full{sv}", j // self.vst)
            pv(0, sv, j)
            if j == nkv - 1:
                self.commit("o_final0")
            if j + 1 < nkv:
                yield (f"{kbar}{sk1}", (j + 1) // self.kst)
                qk(0, sk1, j + 1)
                self.commit("s_full0")
            if self.mutation != "pv1_without_p1":
                yield ("p_full1", j)
            pv(1, sv, j)
            if j == nkv - 1:
                self.commit("o_final1")
            self.commit(f"v_empty{sv}")
            if j + 1 < nkv:
                qk(1, sk1, j + 1)
                self.commit("s_full1")
                self.commit(f"k_empty{sk1}")

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
        if self.convert:
            actors["converter"] = self.converter()
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


KERNELS = {
    "phase1_tc": dict(kst=2, vst=2, convert=False),
    "phase2_tc_d128": dict(kst=3, vst=2, convert=True),
    "phase2_tc_d64": dict(kst=4, vst=4, convert=True),
}


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("nkv", [1, 2, 3, 4, 7])
def test_kernel_protocol_has_no_missed_phase_deadlock_or_race(kernel, nkv):
    for seed in range(300):
        Model(seed, nkv, **KERNELS[kernel]).run()


@pytest.mark.parametrize("kernel,mutation", [("phase1_tc", "v_no_empty_wait"), ("phase1_tc", "pv1_without_p1"),
                                             ("phase2_tc_d128", "convert_before_landing")])
def test_the_model_catches_planted_protocol_mistakes(kernel, mutation):
    caught = 0
    for seed in range(300):
        try:
            Model(seed, 5, mutation, **KERNELS[kernel]).run()
        except AssertionError:
            caught += 1
    assert caught > 0
