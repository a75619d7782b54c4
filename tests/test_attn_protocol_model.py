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


def run(n, stages, seed, wait_for_p=True):
    rnd = random.Random(seed)
    q_full = Bar(1)
    kv_full = [Bar(1) for _ in range(stages)]
    kv_empty = [Bar(1) for _ in range(stages)]
    s_full, p_full, o_final = [Bar(1), Bar(1)], [Bar(128), Bar(128)], [Bar(1), Bar(1)]
    slot = [None] * stages           # contents of each ring slot
    S = [None, None]                 # contents of each query tile's S/P columns
    pv_done = [0, 0]
    tma, mma = [], []

    def producer():
        tma.append((None, None, q_full))
        yield
        for ld in range(2 * n):
            st = ld % stages
            while not kv_empty[st].ready(((ld // stages) & 1) ^ 1):
                yield
            if ld == 0:
                lab = ("K", 0)
            elif ld == 2 * n - 1:
                lab = ("V", n - 1)
            elif ld & 1:
                lab = ("K", (ld + 1) >> 1)
            else:
                lab = ("V", (ld >> 1) - 1)
            tma.append((lab, st, kv_full[st]))
            yield

    def mma_thread():
        def ready(pos):
            return kv_full[pos % stages].ready((pos // stages) & 1)
        while not q_full.ready(0):
            yield
        for j in range(n):
            pk = pos_k(j)
            while not ready(pk):
                yield
            pvpos = None
            if j > 0:
                pvpos = pos_v(j - 1, n)
                while not ready(pvpos):
                    yield
            for t in range(2):
                if j > 0:
                    while wait_for_p and not p_full[t].ready((j - 1) & 1):
                        yield
                    mma.append(("pv", t, j - 1, pvpos % stages))
                mma.append(("qk", t, j, pk % stages))
                mma.append(("commit", s_full[t]))
                yield
            mma.append(("commit", kv_empty[pk % stages]))
            if j > 0:
                mma.append(("commit", kv_empty[pvpos % stages]))
            yield
        last = n - 1
        pvpos = pos_v(last, n)
        while not ready(pvpos):
            yield
        for t in range(2):
            while not p_full[t].ready(last & 1):
                yield
            mma.append(("pv", t, last, pvpos % stages))
            mma.append(("commit", o_final[t]))
            yield
        mma.append(("commit", kv_empty[pvpos % stages]))
        yield

    done = [False, False]

    def softmax(t):
        for j in range(n):
            while not s_full[t].ready(j & 1):
                yield
            if S[t] != ("S", j):
                raise Race(f"softmax {t} read {S[t]} at key tile {j}")
            if j > 0 and pv_done[t] != j:
                raise Race(f"softmax {t} may rescale O while a PV is pending")
            yield
            S[t] = ("P", j)
            p_full[t].arrive(128)
            yield
        while not o_final[t].ready(0):
            yield
        if pv_done[t] != n:
            raise Race("epilogue before the last PV")
        done[t] = True
        yield

    def execute(op):
        if op[0] == "commit":
            op[1].arrive()
            return
        kind, t, j, st = op
        if kind == "qk":
            if slot[st] != ("K", j):
                raise Race(f"QK {t},{j} read slot {slot[st]}")
            if j > 0 and (S[t] != ("P", j - 1) or pv_done[t] != j):
                raise Race(f"QK {t},{j} overwrote {S[t]} before its PV")
            S[t] = ("S", j)
        else:
            if slot[st] != ("V", j):
                raise Race(f"PV {t},{j} read slot {slot[st]}")
            if S[t] != ("P", j) or pv_done[t] != j:
                raise Race(f"PV {t},{j} read {S[t]}")
            pv_done[t] += 1

    gens = [producer(), mma_thread(), softmax(0), softmax(1)]
    alive = [True] * 4
    for _ in range(200000):
        i = rnd.randrange(4)
        if alive[i]:
            try:
                next(gens[i])
            except StopIteration:
                alive[i] = False
        if tma and rnd.random() < 0.3:
            lab, st, bar = tma.pop(rnd.randrange(len(tma)))
            if st is not None:
                slot[st] = lab
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
