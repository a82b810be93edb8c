"""A randomized model check of the attention kernel's barrier protocol (CPU).

The tensor-core attention kernel (attention_tc.cu) coordinates one MMA-issuing thread, the
tensor pipe and eight softmax warps (two per TMEM lane quarter) through mbarriers:

* ``s_full[i & 1]``: committed after S_i = Q K_i^T;
* ``p_full[i & 1]``: all softmax warps wrote P_i over their scores;
* ``pv_done[i & 1]``: committed after O += P_i V_i;
* ``k_full``/``k_empty`` and ``v_full``/``v_empty``: the two-stage K and V rings the TMA
  producer fills (K tile i+1 is loaded before V tile i).

Each softmax warp owns 16 rows (lanes) of its quarter, and both halves of each row's scores sit
in that warp (threads t and t + 16): it reads its rows' scores with one warp-collective load
and writes P over them, so the halves meet by shuffle, without a barrier. The model also keeps
the kernel's earlier layout ("columns"), in which the two warps of a quarter split every row's
columns and exchanged their row maxima through ``ex_bar[q]``: half 1's P lands on scores that
half 0 reads, so that layout needs the exchange.

This file restates those roles as Python generators and runs them under many random
interleavings. An mbarrier wait on parity P passes when the number of completed phases has the
other parity, exactly the hardware's rule, so a barrier that runs two phases ahead of a waiter
is mistaken for one that has not completed: the model reproduces that aliasing. The tensor
pipe executes issued MMAs in order, and a commit arrives once everything issued before it has
run. Checked invariants:

* P·V for tile i runs only after every warp wrote its part of P_i;
* QK^T and P·V read K and V stages that hold their tile, and no load overwrites a stage
  before the MMA that reads it has run;
* a score buffer is overwritten by QK^T only after the P·V that read its P;
* a warp reads S_i while the buffer still holds S_i, and the partner's row max of tile i;
* O is rescaled only between P·V_{i-1} and P·V_i;
* at the end every P·V has run, in order.

Three negative controls must fail: the same model with a single p_full barrier (the protocol
before consecutive tiles were split across two barriers), the column layout with its max
exchange skipped, and one that frees V stages after QK^T instead of after P·V.
"""
import random

import pytest

from protocol_model import Barrier, Violation, schedule

N_QUARTERS, N_HALVES = 4, 2
N_WARPS = N_QUARTERS * N_HALVES
KV_STAGES = 2


class Model:
    def __init__(self, n_tiles: int, grows, split_p_full: bool, exchange: bool = True, early_v_release: bool = False,
                 layout: str = "rows"):
        self.n = n_tiles
        self.grows = grows  # grows[(quarter, tile)]: the quarter's rows rescale O at that tile
        self.s_full = [Barrier(1), Barrier(1)]
        self.pv_done = [Barrier(1), Barrier(1)]
        nb = 2 if split_p_full else 1
        self.p_full = [Barrier(N_WARPS) for _ in range(nb)]
        self.split = split_p_full
        self.layout = layout              # "rows": warp owns 16 rows; "columns": warps split each row
        self.exchange = exchange          # columns layout, False: a warp skips its partner's max
        self.early_v_release = early_v_release  # True: V stages freed after QK^T, not after P·V
        self.ex_bar = [Barrier(N_HALVES) for _ in range(N_QUARTERS)]
        self.fifo = []                    # issued tensor-pipe work, executed in order
        self.s_buf = [None, None]         # tile whose scores (or P) the buffer holds
        self.p_written = [dict(), dict()]  # buffer -> {(q, h): tile}
        self.pv_applied = []              # tiles whose P·V ran, in order
        self.red_max = {}                 # (parity, q, h) -> tile
        self.read_scores = set()          # (tile, q, h): that half has read its scores
        # K/V rings of KV_STAGES stages each, filled by the TMA producer
        self.k_full = [Barrier(1) for _ in range(KV_STAGES)]
        self.v_full = [Barrier(1) for _ in range(KV_STAGES)]
        self.k_empty = [Barrier(1) for _ in range(KV_STAGES)]
        self.v_empty = [Barrier(1) for _ in range(KV_STAGES)]
        self.k_stage = [None] * KV_STAGES  # tile whose K the stage holds
        self.v_stage = [None] * KV_STAGES
        self.tma = []                      # in-flight loads: ("K" | "V", stage, tile)
        self.qk_done = set()

    def pfull(self, i):
        return self.p_full[i & 1] if self.split else self.p_full[0]

    def pfull_parity(self, i):
        return ((i >> 1) & 1) if self.split else (i & 1)

    # ---- roles -------------------------------------------------------------------------
    def mma_thread(self):
        def issue_pv(i):
            st = i % KV_STAGES
            while not self.pfull(i).test_parity(self.pfull_parity(i)):
                yield
            while not self.v_full[st].test_parity((i // KV_STAGES) & 1):
                yield
            self.fifo.append(("PV", i))
            self.fifo.append(("COMMIT", self.pv_done[i & 1]))
            if not self.early_v_release:
                self.fifo.append(("COMMIT", self.v_empty[st]))
            yield

        for i in range(self.n):
            st = i % KV_STAGES
            while not self.k_full[st].test_parity((i // KV_STAGES) & 1):
                yield
            self.fifo.append(("QK", i))
            self.fifo.append(("COMMIT", self.s_full[i & 1]))
            self.fifo.append(("COMMIT", self.k_empty[st]))
            if self.early_v_release:
                self.fifo.append(("COMMIT", self.v_empty[st]))
            yield
            if i >= 1:
                yield from issue_pv(i - 1)
        if self.n:
            yield from issue_pv(self.n - 1)

    def producer(self):
        # K tile i+1 is issued before V tile i: K stages free up after QK^T, V stages only
        # after P·V, so the K loads run a tile further ahead
        def load(kind, i):
            st = i % KV_STAGES
            empty = self.k_empty if kind == "K" else self.v_empty
            while not empty[st].test_parity(((i // KV_STAGES) & 1) ^ 1):
                yield
            self.tma.append((kind, st, i))
            yield

        if self.n:
            yield from load("K", 0)
        for i in range(self.n):
            if i + 1 < self.n:
                yield from load("K", i + 1)
            yield from load("V", i)

    def tma_engine(self):
        while True:
            if self.tma:
                kind, st, i = self.tma.pop(0)
                if kind == "K":
                    if i >= KV_STAGES and (i - KV_STAGES) not in self.qk_done:
                        raise Violation(f"K_{i} overwrote stage {st} before QK_{i - KV_STAGES} read it")
                    self.k_stage[st] = i
                    self.k_full[st].arrive()
                else:
                    if i >= KV_STAGES and (i - KV_STAGES) not in self.pv_applied:
                        raise Violation(f"V_{i} overwrote stage {st} before PV_{i - KV_STAGES} read it")
                    self.v_stage[st] = i
                    self.v_full[st].arrive()
            yield

    def tensor_pipe(self):
        while True:
            if not self.fifo:
                yield
                continue
            op = self.fifo.pop(0)
            if op[0] == "QK":
                i = op[1]
                if i >= 2 and (i - 2) not in self.pv_applied:
                    raise Violation(f"QK_{i} overwrote the score buffer before PV_{i - 2} read it")
                if self.k_stage[i % KV_STAGES] != i:
                    raise Violation(f"QK_{i} read K stage holding tile {self.k_stage[i % KV_STAGES]}")
                self.s_buf[i & 1] = i
                self.qk_done.add(i)
            elif op[0] == "PV":
                i = op[1]
                written = self.p_written[i & 1]
                missing = [k for k in written if written[k] != i] + \
                          [(q, h) for q in range(N_QUARTERS) for h in range(N_HALVES) if (q, h) not in written]
                if missing:
                    raise Violation(f"PV_{i} ran before P_{i} was written by warps {sorted(set(missing))}")
                if self.pv_applied != list(range(i)):
                    raise Violation(f"PV_{i} ran out of order after {self.pv_applied}")
                if self.v_stage[i % KV_STAGES] != i:
                    raise Violation(f"PV_{i} read V stage holding tile {self.v_stage[i % KV_STAGES]}")
                self.pv_applied.append(i)
            else:
                op[1].arrive()
            yield

    def softmax_warp(self, q: int, h: int):
        for i in range(self.n):
            while not self.s_full[i & 1].test_parity((i >> 1) & 1):
                yield
            if self.s_buf[i & 1] != i:
                raise Violation(f"warp ({q},{h}) read buffer {i & 1} holding tile {self.s_buf[i & 1]}, not {i}")
            self.read_scores.add((i, q, h))
            if self.layout == "rows":
                # one collective load read every score of this warp's rows; P goes over them
                yield
                if (i, q, h) not in self.read_scores:
                    raise Violation(f"warp ({q},{h}) wrote P_{i} over scores it did not read")
            else:
                self.red_max[(i & 1, q, h)] = i
                self.ex_bar[q].arrive()
                yield
                while self.exchange and not self.ex_bar[q].test_parity(i & 1):
                    yield
                if self.red_max.get((i & 1, q, 1 - h)) != i:
                    raise Violation(f"warp ({q},{h}) read its partner's max of tile "
                                    f"{self.red_max.get((i & 1, q, 1 - h))}")
                if (i, q, 1 - h) not in self.read_scores:
                    raise Violation(f"warp ({q},{h}) wrote P_{i} before its partner read the scores under it")
            self.p_written[i & 1][(q, h)] = i
            yield
            if i >= 1 and self.grows[(q, i)]:
                b = self.pv_done[(i - 1) & 1]
                while not b.test_parity(((i - 1) >> 1) & 1):
                    yield
                if (i - 1) not in self.pv_applied or i in self.pv_applied:
                    raise Violation(f"warp ({q},{h}) rescaled O at tile {i} with P·V done for {self.pv_applied}")
            self.pfull(i).arrive()
            yield
        if self.n:
            b = self.pv_done[(self.n - 1) & 1]
            while not b.test_parity(((self.n - 1) >> 1) & 1):
                yield
            if self.pv_applied != list(range(self.n)):
                raise Violation(f"warp ({q},{h}) read O with P·V done for {self.pv_applied}")


def run(n_tiles: int, seed: int, split_p_full: bool = True, exchange: bool = True, early_v_release: bool = False,
        max_steps: int = 200_000, layout: str = "rows"):
    rng = random.Random(seed)
    grows = {(q, i): rng.random() < 0.3 for q in range(N_QUARTERS) for i in range(n_tiles)}
    m = Model(n_tiles, grows, split_p_full, exchange, early_v_release, layout)
    roles = [m.producer(), m.mma_thread()] + [m.softmax_warp(q, h) for q in range(N_QUARTERS)
                                              for h in range(N_HALVES)]
    schedule(rng, roles, [m.tensor_pipe(), m.tma_engine()], max_steps)
    return m


@pytest.mark.parametrize("n_tiles", [1, 2, 3, 7])
def test_protocol_holds_under_random_interleavings(n_tiles):
    for seed in range(300):
        m = run(n_tiles, seed)
        assert m.pv_applied == list(range(n_tiles))


def test_the_column_layout_holds_with_its_max_exchange():
    for seed in range(200):
        m = run(5, seed, layout="columns")
        assert m.pv_applied == list(range(5))


def test_a_single_p_full_barrier_lets_a_fast_quarter_complete_a_slow_quarters_phase():
    failures = 0
    for seed in range(400):
        try:
            run(6, seed, split_p_full=False)
        except Violation:
            failures += 1
    assert failures > 0


def test_the_column_layout_without_the_max_exchange_is_caught():
    # there the exchange is also what keeps half 1's P off half 0's unread scores
    failures = 0
    for seed in range(200):
        try:
            run(4, seed, exchange=False, layout="columns")
        except Violation:
            failures += 1
    assert failures > 0


def test_releasing_v_stages_before_p_v_is_caught():
    for seed in range(200):
        try:
            run(6, seed, early_v_release=True, max_steps=50_000)
        except Violation:
            return
    pytest.fail("early V release passed every interleaving")
