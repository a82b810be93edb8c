"""A randomized model check of the two-query-tile attention kernel's barrier protocol (CPU).

attn_gqa_tc2_kernel (attention_tc.cu) runs one TMA producer, one MMA-issuing thread, the tensor
pipe and two softmax warpgroups (one per query tile t, four warps each, one thread per tile row):

* ``q_full``: both query tiles loaded;
* ``k_full``/``k_empty`` and ``v_full``/``v_empty``: two-stage K and V rings (K tile i+1 is loaded
  before V tile i); K stages are freed after S_1 of the tile, V stages after P_1 V;
* ``s_full[t]``: committed after S_t = Q_t K_i^T, which the MMA thread issues after P_t V_{i-1};
* ``p_full[t]``: all 128 rows of tile t wrote P_t over the first half of S_t;
* ``o_full[t]``: committed after the last P_t V.

The roles are restated as Python generators and run under many random interleavings. A wait on
parity P passes while the number of completed phases has the other parity (the hardware's rule,
so a barrier two phases ahead of a waiter looks incomplete). The tensor pipe executes issued MMAs
in issue order, and a commit arrives once everything issued before it has run. Checked:

* S_t of tile i overwrites the S_t/P_t columns only after P_t V_{i-1} has read them;
* a softmax warp reads S_t of tile i (not older scores, not P, not newer scores);
* P_t V_i runs only after all four warps of tile t wrote P_{t,i}, reads the V stage holding
  tile i, and the P_t V run in order;
* a warp rescales O_t only between P_t V_{i-1} and P_t V_i;
* no TMA load overwrites a K or V stage before both query tiles' MMAs that read it have run;
* at the end every P_t V has run before the epilogue reads O_t.

Negative controls must fail: K stages freed after S_0 instead of S_1, V stages freed after P_0 V,
S_t issued before P_t V_{i-1}, and the O rescale done after releasing P.
"""
import random

import pytest

from protocol_model import Barrier, Violation, schedule

N_WARPS = 4   # softmax warps per query tile (one per TMEM lane quarter)
STAGES = 2


class Model:
    def __init__(self, n, grows, bug=None):
        self.n, self.grows, self.bug = n, grows, bug
        self.q_full = Barrier(1)
        self.k_full = [Barrier(1) for _ in range(STAGES)]
        self.v_full = [Barrier(1) for _ in range(STAGES)]
        self.k_empty = [Barrier(1) for _ in range(STAGES)]
        self.v_empty = [Barrier(1) for _ in range(STAGES)]
        self.s_full = [Barrier(1), Barrier(1)]
        self.p_full = [Barrier(N_WARPS), Barrier(N_WARPS)]
        self.o_full = [Barrier(1), Barrier(1)]
        self.fifo = []                               # issued tensor-pipe work, in order
        self.tma = []                                # in-flight loads
        self.k_stage = [None] * STAGES
        self.v_stage = [None] * STAGES
        self.q_loaded = False
        self.s_buf = [None, None]                    # ("S" | "P", tile) held by the S_t columns
        self.p_rows = [dict(), dict()]               # tile t -> {warp: tile whose P it wrote}
        self.pv_done = [[], []]                      # per query tile: key tiles whose P V ran
        self.s_done = set()                          # (t, i) of S_t = Q_t K_i^T that ran

    # ---- roles ------------------------------------------------------------------------------
    def producer(self):
        self.tma.append(("Q", 0, 0))
        yield

        def load(kind, i):
            st = i % STAGES
            empty = self.k_empty if kind == "K" else self.v_empty
            while not empty[st].test_parity(((i // STAGES) & 1) ^ 1):
                yield
            self.tma.append((kind, st, i))
            yield
        if self.n:
            yield from load("K", 0)
        for i in range(self.n):
            if i + 1 < self.n:
                yield from load("K", i + 1)
            yield from load("V", i)

    def mma_thread(self):
        def issue_pv(t, i):
            st = i % STAGES
            while not self.p_full[t].test_parity(i & 1):
                yield
            if t == 0:
                while not self.v_full[st].test_parity((i // STAGES) & 1):
                    yield
            self.fifo.append(("PV", t, i))
            if t == (0 if self.bug == "v_after_pv0" else 1):
                self.fifo.append(("COMMIT", self.v_empty[st]))
            yield

        while not self.q_full.test_parity(0):
            yield
        for i in range(self.n):
            st = i % STAGES
            while not self.k_full[st].test_parity((i // STAGES) & 1):
                yield
            for t in (0, 1):
                if self.bug == "s_before_pv":
                    self.fifo.append(("S", t, i))
                    if i > 0:
                        yield from issue_pv(t, i - 1)
                else:
                    if i > 0:
                        yield from issue_pv(t, i - 1)
                    self.fifo.append(("S", t, i))
                self.fifo.append(("COMMIT", self.s_full[t]))
                if self.bug == "k_after_s0" and t == 0:
                    self.fifo.append(("COMMIT", self.k_empty[st]))
                yield
            if self.bug != "k_after_s0":
                self.fifo.append(("COMMIT", self.k_empty[st]))
        for t in (0, 1):
            if self.n:
                yield from issue_pv(t, self.n - 1)
                self.fifo.append(("COMMIT", self.o_full[t]))

    def tma_engine(self):
        while True:
            if self.tma:
                kind, st, i = self.tma.pop(0)
                if kind == "Q":
                    self.q_loaded = True
                    self.q_full.arrive()
                elif kind == "K":
                    prev = i - STAGES
                    if prev >= 0 and not ((0, prev) in self.s_done and (1, prev) in self.s_done):
                        raise Violation(f"K_{i} overwrote stage {st} before both S of tile {prev} read it")
                    self.k_stage[st] = i
                    self.k_full[st].arrive()
                else:
                    prev = i - STAGES
                    if prev >= 0 and not (prev in self.pv_done[0] and prev in self.pv_done[1]):
                        raise Violation(f"V_{i} overwrote stage {st} before both P V of tile {prev} read it")
                    self.v_stage[st] = i
                    self.v_full[st].arrive()
            yield

    def tensor_pipe(self):
        while True:
            if not self.fifo:
                yield
                continue
            op = self.fifo.pop(0)
            if op[0] == "S":
                _, t, i = op
                if not self.q_loaded or self.k_stage[i % STAGES] != i:
                    raise Violation(f"S_{t} of tile {i} read K stage holding {self.k_stage[i % STAGES]}")
                if i > 0 and (i - 1) not in self.pv_done[t]:
                    raise Violation(f"S_{t} of tile {i} overwrote P_{t} of tile {i - 1} before P V read it")
                self.s_buf[t] = ("S", i)
                self.p_rows[t] = {}
                self.s_done.add((t, i))
            elif op[0] == "PV":
                _, t, i = op
                missing = [w for w in range(N_WARPS) if self.p_rows[t].get(w) != i]
                if missing or self.s_buf[t] != ("P", i):
                    raise Violation(f"P_{t} V of tile {i} ran with P rows {self.p_rows[t]}, buffer {self.s_buf[t]}")
                if self.v_stage[i % STAGES] != i:
                    raise Violation(f"P_{t} V of tile {i} read V stage holding {self.v_stage[i % STAGES]}")
                if self.pv_done[t] != list(range(i)):
                    raise Violation(f"P_{t} V of tile {i} ran out of order after {self.pv_done[t]}")
                self.pv_done[t].append(i)
            else:
                op[1].arrive()
            yield

    def softmax_warp(self, t, w):
        for i in range(self.n):
            while not self.s_full[t].test_parity(i & 1):
                yield
            if self.s_buf[t] not in (("S", i), ("P", i)) or (self.s_buf[t] == ("P", i) and w in self.p_rows[t]):
                raise Violation(f"warp {w} of tile {t} read {self.s_buf[t]} expecting S of tile {i}")
            yield
            self.p_rows[t][w] = i
            if len(self.p_rows[t]) == N_WARPS:
                self.s_buf[t] = ("P", i)
            yield

            def rescale():
                if i >= 1 and self.grows[(t, w, i)]:
                    if (i - 1) not in self.pv_done[t] or i in self.pv_done[t]:
                        raise Violation(f"warp {w} rescaled O_{t} at tile {i} with P V done for {self.pv_done[t]}")
            if self.bug != "rescale_after_release":
                rescale()
            self.p_full[t].arrive()
            yield
            if self.bug == "rescale_after_release":
                rescale()
        if self.n:
            while not self.o_full[t].test_parity(0):
                yield
            if self.pv_done[t] != list(range(self.n)):
                raise Violation(f"epilogue of tile {t} read O with P V done for {self.pv_done[t]}")


def run(n, seed, bug=None, max_steps=200_000):
    rng = random.Random(seed)
    grows = {(t, w, i): rng.random() < 0.3 for t in (0, 1) for w in range(N_WARPS) for i in range(n)}
    m = Model(n, grows, bug)
    roles = [m.producer(), m.mma_thread()] + [m.softmax_warp(t, w) for t in (0, 1) for w in range(N_WARPS)]
    schedule(rng, roles, [m.tensor_pipe(), m.tma_engine()], max_steps)
    return m


@pytest.mark.parametrize("n_tiles", [1, 2, 3, 8])
def test_protocol_holds_under_random_interleavings(n_tiles):
    for seed in range(300):
        m = run(n_tiles, seed)
        assert m.pv_done == [list(range(n_tiles))] * 2


@pytest.mark.parametrize("bug", ["k_after_s0", "v_after_pv0", "s_before_pv", "rescale_after_release"])
def test_broken_variants_are_caught(bug):
    for seed in range(400):
        try:
            run(6, seed, bug=bug, max_steps=50_000)
        except Violation:
            return
    pytest.fail(f"the {bug} variant passed every interleaving")
