"""A model of the attention kernel's barrier protocol (attn_tc.cu), run under random
timings on the CPU: no deadlock, and no data race on the shared-memory K/V ring or on
tensor memory.

Roles, as in the kernel: a TMA producer loads Q once, then K_0, K_1, V_0, K_2, V_1, ...
through a ring of `stages` slots (kv_full / kv_empty); one MMA thread, for key tile j and
query tile t, waits for P_t(j-1) (p_full[t]), issues O_t += P_t(j-1) V_{j-1} and
S_t = Q_t K_j^T, and commits s_full[t]; each query tile's softmax waits for S_t(j),
rewrites it in place as P_t(j) and arrives on p_full[t]. Tensor-core operations run in
issue order; a commit completes when everything issued before it has; TMA copies
complete in any order. The checks: every operation reads the contents it expects (S_t(j)
for the softmax, K_j / V_j from the slot, P_t(j) for PV) and O_t is idle whenever the
softmax rescales it."""
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


def pos_k(j):
    return 0 if j == 0 else 2 * j - 1


def pos_v(j, n):
    return 2 * n - 1 if j == n - 1 else 2 * j + 2


def run(n, stages, seed, wait_for_p=True, units=1, qbufs=1, wait_q_empty=True, phase_per_unit=False):
    """One CTA over ``units`` units of ``n`` key tiles each (the persistent variant when
    units > 1: Q in ``qbufs`` buffers refilled after q_empty, every phase counted across
    units; ``phase_per_unit`` plants the mistake of restarting the softmax's S phase at
    each unit). The first PV of a unit relies on p_full alone: the softmax threads read
    the previous unit's O out before they finish that unit's first P. Returns True when
    all finish."""
    rnd = random.Random(seed)
    q_full, q_empty = [Bar(1) for _ in range(qbufs)], [Bar(1) for _ in range(qbufs)]
    kv_full = [Bar(1) for _ in range(stages)]
    kv_empty = [Bar(1) for _ in range(stages)]
    s_full, p_full, o_final = [Bar(1), Bar(1)], [Bar(128), Bar(128)], [Bar(1), Bar(1)]
    slot = [None] * stages           # contents of each ring slot
    qbuf = [None] * qbufs            # contents of each Q buffer
    S = [None, None]                 # contents of each query tile's S/P columns: (kind, unit, j)
    O = [None, None]                 # (unit, PVs accumulated) of each query tile's O columns
    read_out = [-1, -1]              # last unit whose O the epilogue has read
    tma, mma = [], []

    def producer():
        issued = 0
        for u in range(units):
            qb = u % qbufs
            if u >= qbufs:
                while wait_q_empty and not q_empty[qb].ready((u // qbufs - 1) & 1):
                    yield
            tma.append((("Q", u), ("q", qb), q_full[qb]))
            yield
            for ld in range(2 * n):
                st = issued % stages
                while not kv_empty[st].ready(((issued // stages) & 1) ^ 1):
                    yield
                if ld == 0:
                    lab = ("K", u, 0)
                elif ld == 2 * n - 1:
                    lab = ("V", u, n - 1)
                elif ld & 1:
                    lab = ("K", u, (ld + 1) >> 1)
                else:
                    lab = ("V", u, (ld >> 1) - 1)
                tma.append((lab, ("kv", st), kv_full[st]))
                issued += 1
                yield

    def mma_thread():
        def ready(pos):
            return kv_full[pos % stages].ready((pos // stages) & 1)
        for u in range(units):
            qb, base, tiles = u % qbufs, u * 2 * n, u * n
            while not q_full[qb].ready((u // qbufs) & 1):
                yield
            for j in range(n):
                pk = base + pos_k(j)
                while not ready(pk):
                    yield
                pvpos = None
                if j > 0:
                    pvpos = base + pos_v(j - 1, n)
                    while not ready(pvpos):
                        yield
                for t in range(2):
                    if j > 0:
                        while wait_for_p and not p_full[t].ready((tiles + j - 1) & 1):
                            yield
                        mma.append(("pv", t, u, j - 1, pvpos % stages))
                    mma.append(("qk", t, u, j, (pk % stages, qb)))
                    mma.append(("commit", s_full[t]))
                    yield
                mma.append(("commit", kv_empty[pk % stages]))
                if j > 0:
                    mma.append(("commit", kv_empty[pvpos % stages]))
                yield
            mma.append(("commit", q_empty[qb]))
            last = n - 1
            pvpos = base + pos_v(last, n)
            while not ready(pvpos):
                yield
            for t in range(2):
                while not p_full[t].ready((tiles + last) & 1):
                    yield
                mma.append(("pv", t, u, last, pvpos % stages))
                mma.append(("commit", o_final[t]))
                yield
            mma.append(("commit", kv_empty[pvpos % stages]))
            yield

    done = [False, False]

    def softmax(t):
        for u in range(units):
            tiles = 0 if phase_per_unit else u * n
            for j in range(n):
                while not s_full[t].ready((tiles + j) & 1):
                    yield
                if S[t] != ("S", u, j):
                    raise Race(f"softmax {t} read {S[t]} at unit {u} key tile {j}")
                if j > 0 and O[t] != (u, j):
                    raise Race(f"softmax {t} may rescale O while a PV is pending")
                yield
                S[t] = ("P", u, j)
                p_full[t].arrive(128)
                yield
            while not o_final[t].ready(u & 1):
                yield
            if O[t] != (u, n):
                raise Race(f"epilogue of unit {u} read O = {O[t]}")
            yield                        # the reads of O take a while
            if O[t] != (u, n):
                raise Race(f"O of unit {u} overwritten while the epilogue read it")
            read_out[t] = u
            yield
        done[t] = True
        yield

    def execute(op):
        if op[0] == "commit":
            op[1].arrive()
            return
        kind, t, u, j, where = op
        if kind == "qk":
            st, qb = where
            if slot[st] != ("K", u, j):
                raise Race(f"QK {t},{u},{j} read slot {slot[st]}")
            if qbuf[qb] != ("Q", u):
                raise Race(f"QK {t},{u},{j} read Q buffer {qbuf[qb]}")
            prev = ("P", u, j - 1) if j > 0 else (("P", u - 1, n - 1) if u > 0 else None)
            want_o = (u, j) if j > 0 else ((u - 1, n) if u > 0 else None)
            if S[t] != prev or O[t] != want_o:
                raise Race(f"QK {t},{u},{j} overwrote {S[t]} before its PV")
            S[t] = ("S", u, j)
        else:
            st = where
            if slot[st] != ("V", u, j):
                raise Race(f"PV {t},{u},{j} read slot {slot[st]}")
            if S[t] != ("P", u, j):
                raise Race(f"PV {t},{u},{j} read {S[t]}")
            if j == 0:
                if read_out[t] != u - 1:
                    raise Race(f"first PV of unit {u} overwrote O before the epilogue read unit {u - 1}")
            elif O[t] != (u, j):
                raise Race(f"PV {t},{u},{j} accumulated onto {O[t]}")
            O[t] = (u, j + 1)

    gens = [producer(), mma_thread(), softmax(0), softmax(1)]
    alive = [True] * 4
    for _ in range(400000):
        i = rnd.randrange(4)
        if alive[i]:
            try:
                next(gens[i])
            except StopIteration:
                alive[i] = False
        if tma and rnd.random() < 0.3:
            lab, (kind, idx), bar = tma.pop(rnd.randrange(len(tma)))
            if kind == "kv":
                slot[idx] = lab
            else:
                if qbuf[idx] is not None and any(op[0] == "qk" and op[4][1] == idx for op in mma):
                    raise Race(f"Q buffer {idx} refilled while a QK on it was pending")
                qbuf[idx] = lab
            bar.arrive()
        if mma and rnd.random() < 0.3:
            execute(mma.pop(0))
        if all(done):
            return True
    return False


@pytest.mark.parametrize("stages", [5, 8])          # the bf16 and E4M3 rings
def test_attention_protocol_is_live_and_race_free(stages):
    for n in [1, 2, 3, 5, 8, 17]:                    # key tiles per CTA (whole units and key-split halves)
        for seed in range(12):
            assert run(n, stages, seed), f"deadlock: {n} key tiles, {stages} stages, seed {seed}"


def test_model_catches_a_missing_wait():
    """The model is not vacuous: an MMA thread that issues PV without waiting for the
    softmax's P is caught as a race for some timing."""
    races = 0
    for seed in range(40):
        try:
            run(5, 5, seed, wait_for_p=False)
        except Race:
            races += 1
    assert races > 0


@pytest.mark.parametrize("n", [1, 2, 3, 4])           # key tiles per unit of the persistent variant
def test_persistent_protocol_is_live_and_race_free(n):
    """Several units per CTA (double-buffered Q, 3-slot ring, phases carried across
    units): every unit's output is read before the next unit overwrites it."""
    for units in [1, 2, 3, 5]:
        for seed in range(10):
            assert run(n, 3, seed, units=units, qbufs=2), f"deadlock: {n} tiles, {units} units, seed {seed}"


def test_persistent_model_catches_a_phase_restart():
    """A softmax that counts its S phases from zero at every unit (instead of across the
    units of the CTA) reads a stale S for some timing (odd key-tile counts)."""
    races = 0
    for seed in range(40):
        try:
            run(3, 3, seed, units=4, qbufs=2, phase_per_unit=True)
        except Race:
            races += 1
    assert races > 0


def test_persistent_protocol_without_the_q_buffer_wait_still_holds():
    """The Q refill wait is a guard, not a necessity, at these ring depths: the producer
    reaches unit u + 2's Q only after the ring has freed slots whose release followed
    unit u's last QK."""
    for n in [1, 2, 4]:
        for seed in range(20):
            assert run(n, 3, seed, units=5, qbufs=2, wait_q_empty=False)
