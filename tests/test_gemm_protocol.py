"""A randomized model check of the persistent GEMM kernel's barrier protocol (CPU).

The tcgen05 GEMM (gemm_tcgen05.cu) runs, per CTA, a TMA producer thread, one MMA-issuing
thread and four epilogue warps (eight for the gated residual, two per TMEM lane quarter) over a
ring of shared-memory stages and two TMEM accumulators:

* ``full[s]`` completes when stage s's TMA loads have landed; ``empty[s]`` is committed after
  the MMAs that read stage s;
* ``tfull[a]`` is committed after a tile's last MMA into accumulator a; ``tempty[a]``
  completes when every epilogue warp has read accumulator a.

The producer waits ``empty`` with the flipped parity (the ring starts empty), the MMA thread
waits ``tempty`` with the flipped parity (both accumulators start free), as the kernel does.
This file restates the roles with the shared barrier model (hardware parity rule, in-order
tensor pipe, TMA loads that land later) and checks under random interleavings that:

* the MMA reads a stage only while it holds that (tile, k-block)'s data;
* the producer refills a stage only after the MMAs that read it have run;
* the epilogue reads an accumulator only when it holds the whole tile;
* the MMA starts a tile in an accumulator only after the epilogue of the tile before it
  there has finished.

Negative controls must fail: an empty-barrier wait without the parity flip, a tempty barrier
that expects one arrival where four warps arrive, and one that still expects four where the
residual's eight arrive.
"""
import random

import pytest

from protocol_model import Barrier, Violation, schedule

class Gemm:
    def __init__(self, tiles: int, nk: int, stages: int, flip_empty: bool = True, n_epi: int = 4,
                 tempty_count: int = None):
        self.tiles, self.nk, self.S = tiles, nk, stages
        self.n_epi = n_epi
        tempty_count = n_epi if tempty_count is None else tempty_count
        self.full = [Barrier(1) for _ in range(stages)]
        self.empty = [Barrier(1) for _ in range(stages)]
        self.tfull = [Barrier(1), Barrier(1)]
        self.tempty = [Barrier(tempty_count), Barrier(tempty_count)]
        self.flip_empty = flip_empty
        self.stage_data = [None] * stages      # (tile, kb) held by the stage
        self.stage_readers = [0] * stages      # MMAs issued on the stage and not yet run
        self.acc = [None, None]                # (tile, k-blocks accumulated)
        self.acc_reading = [0, 0]              # epilogue warps still reading
        self.tma = []                          # in-flight loads: (stage, tile, kb)
        self.pipe = []                         # issued tensor work, in order
        self.reads_done = {}                   # tile -> epilogue warps that finished reading it

    # ---- asynchronous engines ------------------------------------------------------------
    def tma_engine(self):
        while True:
            if self.tma:
                s, t, kb = self.tma.pop(0)
                if self.stage_readers[s]:
                    raise Violation(f"load of tile {t} k-block {kb} overwrote stage {s} under an unrun MMA")
                self.stage_data[s] = (t, kb)
                self.full[s].arrive()
            yield

    def tensor_pipe(self):
        while True:
            if self.pipe:
                op = self.pipe.pop(0)
                if op[0] == "MMA":
                    _, s, t, kb, a = op
                    if self.stage_data[s] != (t, kb):
                        raise Violation(f"MMA for tile {t} k-block {kb} read stage {s} holding {self.stage_data[s]}")
                    if self.acc[a] is None or self.acc[a][0] != t or self.acc[a][1] != kb:
                        raise Violation(f"MMA for tile {t} k-block {kb} found accumulator {a} at {self.acc[a]}")
                    if self.acc_reading[a]:
                        raise Violation(f"MMA for tile {t} wrote accumulator {a} while the epilogue read it")
                    self.acc[a] = (t, kb + 1)
                    self.stage_readers[s] -= 1
                else:
                    op[1].arrive()
            yield

    # ---- roles -----------------------------------------------------------------------------
    def producer(self):
        stage, phase = 0, 0
        for t in range(self.tiles):
            for kb in range(self.nk):
                want = phase ^ 1 if self.flip_empty else phase
                while not self.empty[stage].test_parity(want):
                    yield
                self.tma.append((stage, t, kb))
                yield
                stage += 1
                if stage == self.S:
                    stage, phase = 0, phase ^ 1

    def mma(self):
        stage, phase = 0, 0
        for t in range(self.tiles):
            a = t & 1
            while not self.tempty[a].test_parity(((t >> 1) & 1) ^ 1):
                yield
            prev = self.acc[a]
            if prev is not None and self.reads_done.get(prev[0], 0) != self.n_epi:
                raise Violation(f"tile {t} claimed accumulator {a} before all epilogue warps read tile {prev[0]}")
            self.acc[a] = (t, 0)
            for kb in range(self.nk):
                while not self.full[stage].test_parity(phase):
                    yield
                self.stage_readers[stage] += 1
                self.pipe.append(("MMA", stage, t, kb, a))
                self.pipe.append(("COMMIT", self.empty[stage]))
                yield
                stage += 1
                if stage == self.S:
                    stage, phase = 0, phase ^ 1
            self.pipe.append(("COMMIT", self.tfull[a]))
            yield

    def epilogue(self, w: int):
        for t in range(self.tiles):
            a = t & 1
            while not self.tfull[a].test_parity((t >> 1) & 1):
                yield
            if self.acc[a] != (t, self.nk):
                raise Violation(f"epilogue warp {w} read accumulator {a} at {self.acc[a]}, not tile {t} complete")
            self.acc_reading[a] += 1
            yield
            self.acc_reading[a] -= 1
            self.reads_done[t] = self.reads_done.get(t, 0) + 1
            self.tempty[a].arrive()
            yield


def run(tiles: int, nk: int, stages: int, seed: int, max_steps: int = 200_000, **kw):
    rng = random.Random(seed)
    g = Gemm(tiles, nk, stages, **kw)
    roles = [g.producer(), g.mma()] + [g.epilogue(w) for w in range(g.n_epi)]
    schedule(rng, roles, [g.tma_engine(), g.tensor_pipe()], max_steps)
    return g


@pytest.mark.parametrize("n_epi", [4, 8])
@pytest.mark.parametrize("tiles,nk,stages", [(1, 1, 4), (3, 5, 4), (6, 2, 4), (5, 7, 6), (4, 3, 1)])
def test_protocol_holds_under_random_interleavings(tiles, nk, stages, n_epi):
    for seed in range(200):
        run(tiles, nk, stages, seed, n_epi=n_epi)


@pytest.mark.parametrize("kw", [dict(flip_empty=False), dict(tempty_count=1), dict(n_epi=8, tempty_count=4)])
def test_broken_protocols_are_caught(kw):
    # a deadlock counts as a failure too (no progress within the step budget)
    for seed in range(200):
        try:
            run(5, 3, 2, seed, max_steps=20_000, **kw)
        except Violation:
            return
    pytest.fail("the broken protocol passed every interleaving")
