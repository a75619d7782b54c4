"""A model of the persistent GEMM's barrier protocol (gemm_tc.cu), run under random
timings on the CPU: no deadlock, and no data race on the shared-memory ring or on the
two tensor-memory accumulators.

Roles, as in the kernel: a TMA producer walks this CTA's tiles and their k-blocks
through a ring of `stages` slots (full / empty); one MMA thread takes tile number `it`
into accumulator it % 2 after waiting for it to be empty (tempty), consumes each
k-block (full), releases its slot with a commit (empty), and commits tfull when the
tile's last k-block is issued; the epilogue warps wait for tfull, read the accumulator
and arrive on tempty (256 threads). Tensor-core operations run in issue order; a commit
completes when everything issued before it has; TMA copies complete in any order."""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self, n=1):
        for _ in range(n):
            self.pending -= 1
            if self.pending == 0:
                self.phase ^= 1
                self.pending = self.count

    def ready(self, parity):
        return self.phase != parity


class Race(Exception):
    pass


def run(tiles, kblocks, stages, seed, wait_for_empty_acc=True):
    rnd = random.Random(seed)
    full = [Bar(1) for _ in range(stages)]
    empty = [Bar(1) for _ in range(stages)]
    tfull, tempty = [Bar(1), Bar(1)], [Bar(256), Bar(256)]
    slot = [None] * stages
    acc = [("free", None), ("free", None)]     # state of each accumulator
    tma, mma = [], []

    def producer():
        stage, phase = 0, 0
        for tile in range(tiles):
            for kb in range(kblocks):
                while not empty[stage].ready(phase ^ 1):
                    yield
                tma.append(((tile, kb), stage, full[stage]))
                yield
                stage += 1
                if stage == stages:
                    stage, phase = 0, phase ^ 1

    def mma_thread():
        stage, phase = 0, 0
        for it in range(tiles):
            a = it & 1
            while wait_for_empty_acc and not tempty[a].ready(((it >> 1) & 1) ^ 1):
                yield
            for kb in range(kblocks):
                while not full[stage].ready(phase):
                    yield
                mma.append(("mma", it, kb, stage, a))
                mma.append(("commit", empty[stage]))
                yield
                stage += 1
                if stage == stages:
                    stage, phase = 0, phase ^ 1
            mma.append(("commit", tfull[a]))
            yield

    done = [False]

    def epilogue():
        for it in range(tiles):
            a = it & 1
            while not tfull[a].ready((it >> 1) & 1):
                yield
            if acc[a] != ("done", it):
                raise Race(f"epilogue of tile {it} read accumulator {a} holding {acc[a]}")
            yield
            acc[a] = ("free", it)
            tempty[a].arrive(256)
            yield
        done[0] = True
        yield

    def execute(op):
        if op[0] == "commit":
            op[1].arrive()
            return
        _, it, kb, st, a = op
        if slot[st] != (it, kb):
            raise Race(f"MMA of tile {it}, k-block {kb} read slot {slot[st]}")
        if kb == 0:
            if acc[a][0] != "free":
                raise Race(f"tile {it} overwrote accumulator {a} holding {acc[a]}")
            acc[a] = ("partial", it)
        if kb == kblocks - 1:
            acc[a] = ("done", it)

    gens = [producer(), mma_thread(), epilogue()]
    alive = [True] * 3
    for _ in range(200000):
        i = rnd.randrange(3)
        if alive[i]:
            try:
                next(gens[i])
            except StopIteration:
                alive[i] = False
        if tma and rnd.random() < 0.3:
            lab, st, bar = tma.pop(rnd.randrange(len(tma)))
            slot[st] = lab
            bar.arrive()
        if mma and rnd.random() < 0.3:
            execute(mma.pop(0))
        if done[0] and not any(alive[:2]) and not mma:
            return True
    return False


@pytest.mark.parametrize("stages", [4, 6, 8])         # the rings of the BN = 256 / 128 / 64 tiles
def test_gemm_protocol_is_live_and_race_free(stages):
    for tiles in [1, 2, 3, 7]:
        for kblocks in [1, 2, 5, 24]:
            for seed in range(4):
                assert run(tiles, kblocks, stages, seed), f"deadlock: {tiles} tiles, {kblocks} k-blocks, {stages} stages"


def test_model_catches_a_missing_accumulator_wait():
    """Without the MMA thread's wait for an empty accumulator, tile it + 2 can overwrite
    tile it's result before the epilogue read it."""
    races = 0
    for seed in range(40):
        try:
            run(6, 2, 4, seed, wait_for_empty_acc=False)
        except Race:
            races += 1
    assert races > 0


# --------------------------------------------------------------------------------------
# The CTA-pair GEMM (gemm_bf16_pair_kernel): two CTAs, each with its own ring, producer
# and epilogue; the even CTA's MMA thread consumes both CTAs' slots. Each CTA's TMA
# copies complete on the even CTA's full[stage], which only the even producer arms
# (arrive + both CTAs' bytes); the MMA's commits release empty[stage] and signal
# tfull[acc] in both CTAs; both epilogues arrive on the even CTA's tempty[acc].
# --------------------------------------------------------------------------------------

class TxBar(Bar):
    """An mbarrier with a transaction count: a phase completes when its arrivals are in
    and its expected bytes have landed (bytes may land before they are expected)."""

    def __init__(self, count):
        super().__init__(count)
        self.tx = 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase ^= 1
            self.pending = self.count

    def arrive(self, n=1):
        for _ in range(n):
            self.pending -= 1
            self._check()

    def expect_and_arrive(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete(self, nbytes):
        self.tx -= nbytes
        self._check()


def run_pair(tiles, kblocks, stages, seed, armed_bytes=2):
    rnd = random.Random(seed)
    full0 = [TxBar(1) for _ in range(stages)]                  # the even CTA's full barriers
    empty = [[Bar(1) for _ in range(stages)] for _ in range(2)]
    tfull = [[Bar(1), Bar(1)] for _ in range(2)]
    tempty0 = [Bar(512), Bar(512)]
    slot = [[None] * stages for _ in range(2)]
    acc = [[("free", None), ("free", None)] for _ in range(2)]
    tma, mma = [], []

    def producer(r):
        stage, phase = 0, 0
        for tile in range(tiles):
            for kb in range(kblocks):
                while not empty[r][stage].ready(phase ^ 1):
                    yield
                if r == 0:
                    full0[stage].expect_and_arrive(armed_bytes)
                tma.append(((tile, kb), r, stage))
                yield
                stage += 1
                if stage == stages:
                    stage, phase = 0, phase ^ 1

    def mma_thread():
        stage, phase = 0, 0
        for it in range(tiles):
            a = it & 1
            while not tempty0[a].ready(((it >> 1) & 1) ^ 1):
                yield
            for kb in range(kblocks):
                while not full0[stage].ready(phase):
                    yield
                mma.append(("mma", it, kb, stage, a))
                mma.append(("commit", [empty[0][stage], empty[1][stage]]))
                yield
                stage += 1
                if stage == stages:
                    stage, phase = 0, phase ^ 1
            mma.append(("commit", [tfull[0][a], tfull[1][a]]))
            yield

    done = [False, False]

    def epilogue(r):
        for it in range(tiles):
            a = it & 1
            while not tfull[r][a].ready((it >> 1) & 1):
                yield
            if acc[r][a] != ("done", it):
                raise Race(f"CTA {r} epilogue of tile {it} read accumulator {a} holding {acc[r][a]}")
            yield
            acc[r][a] = ("free", it)
            tempty0[a].arrive(256)
            yield
        done[r] = True
        yield

    def execute(op):
        if op[0] == "commit":
            for bar in op[1]:
                bar.arrive()
            return
        _, it, kb, st, a = op
        for r in range(2):
            if slot[r][st] != (it, kb):
                raise Race(f"MMA of tile {it}, k-block {kb} read CTA {r}'s slot {slot[r][st]}")
            if kb == 0:
                if acc[r][a][0] != "free":
                    raise Race(f"tile {it} overwrote CTA {r}'s accumulator {a} holding {acc[r][a]}")
                acc[r][a] = ("partial", it)
            if kb == kblocks - 1:
                acc[r][a] = ("done", it)

    gens = [producer(0), producer(1), mma_thread(), epilogue(0), epilogue(1)]
    alive = [True] * 5
    for _ in range(400000):
        i = rnd.randrange(5)
        if alive[i]:
            try:
                next(gens[i])
            except StopIteration:
                alive[i] = False
        if tma and rnd.random() < 0.3:
            lab, r, st = tma.pop(rnd.randrange(len(tma)))
            slot[r][st] = lab
            full0[st].complete(1)
        if mma and rnd.random() < 0.3:
            execute(mma.pop(0))
        if all(done) and not any(alive[:3]) and not mma:
            return True
    return False


def test_pair_gemm_protocol_is_live_and_race_free():
    for tiles in [1, 2, 3, 6]:
        for kblocks in [1, 2, 5, 24]:
            for seed in range(4):
                assert run_pair(tiles, kblocks, 6, seed), f"deadlock: {tiles} tiles, {kblocks} k-blocks"


def test_pair_model_catches_a_full_barrier_armed_for_one_cta():
    """If the even producer expected only its own bytes, the MMA could start on a slot
    whose peer half has not landed."""
    races = 0
    for seed in range(40):
        try:
            run_pair(4, 3, 6, seed, armed_bytes=1)
        except Race:
            races += 1
    assert races > 0
