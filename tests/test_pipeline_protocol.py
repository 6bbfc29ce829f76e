"""The mbarrier hand-off protocols of the persistent GEMMs, simulated on the CPU.

Each role of a kernel (TMA producer, MMA issuer, decoder warps, epilogue warps) is
written here as a sequence of the waits and arrivals it performs, with the counts,
parities and ring sizes of the kernel source (k_tc_gemm.cu, k_tc_gemm_mx8.cu).  A
scheduler runs the roles in random interleavings under mbarrier semantics (a phase
completes when its pending arrivals and transaction bytes reach zero; a parity wait on
phase parity P passes once the phase in progress has the other parity), and checks:
  * every role finishes (no deadlock);
  * a waiter never sees a barrier that has already run two phases past the one it waits
    for (the parity would then be ambiguous);
  * no producer overwrites a buffer (shared-memory stage, TMEM stage, accumulator) that a
    consumer of its previous contents has not released.
This checks the design of the counts and parities, not the compiled kernels.
"""
import random

import pytest


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self):
        assert self.pending > 0, self.name
        self.pending -= 1
        self._maybe_complete()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        assert self.tx >= nbytes, self.name
        self.tx -= nbytes
        self._maybe_complete()

    def passes(self, parity, want_phase):
        """try_wait.parity: the phase in progress has parity completed % 2."""
        ok = (self.completed % 2) != parity
        if ok:
            assert self.completed <= want_phase + 1, f"{self.name}: ran past phase {want_phase}"
        return ok


class Buffers:
    """Readers still owed per (buffer, slot); a producer may only fill a slot nobody reads."""

    def __init__(self):
        self.readers = {}

    def fill(self, key, n_readers):
        assert self.readers.get(key, 0) == 0, f"{key} overwritten while still being read"
        self.readers[key] = n_readers

    def release(self, key):
        assert self.readers.get(key, 0) > 0, f"{key} released twice"
        self.readers[key] -= 1


def wait(bar, parity, phase):
    """A role step: block until bar passes the parity wait (phase = index of the awaited
    completion, for the overrun check)."""
    return ("wait", bar, parity, phase)


class Async:
    """Work that completes later: TMA loads land in any order; the completions an MMA
    thread's commits report come in issue order (a commit tracks every earlier MMA)."""

    def __init__(self):
        self.loads, self.mma = [], []

    def __bool__(self):
        return bool(self.loads or self.mma)

    def step(self, rng):
        if self.mma and (not self.loads or rng.random() < 0.5):
            self.mma.pop(0)()
        else:
            self.loads.pop(rng.randrange(len(self.loads)))()


def run(roles, q, seed, max_steps=200000):
    """roles: name -> generator of steps; q: the Async the roles hand delayed completions to."""
    rng = random.Random(seed)
    blocked = {}
    live = dict(roles)
    for _ in range(max_steps):
        if not live and not q:
            return
        ready = []
        for name, gen in live.items():
            b = blocked.get(name)
            if b is None or b[1].passes(b[2], b[3]):
                ready.append(name)
        choices = ready + (["<async>"] if q else [])
        assert choices, f"deadlock: blocked {sorted((n, b[1].name) for n, b in blocked.items())}"
        pick = rng.choice(choices)
        if pick == "<async>":
            q.step(rng)
            continue
        blocked.pop(pick, None)
        try:
            step = next(live[pick])
        except StopIteration:
            del live[pick]
            continue
        if step is not None and step[0] == "wait":
            blocked[pick] = step
    raise AssertionError("no progress")


# ---------------------------------------------------------------- the bf16 GEMM (k_tc_gemm.cu)

def bf16_gemm(n_tiles, nkb, stages):
    full = [Barrier(f"full{s}", 1) for s in range(stages)]
    empty = [Barrier(f"empty{s}", 1) for s in range(stages)]
    acc_full = [Barrier(f"acc_full{b}", 1) for b in range(2)]
    acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(2)]
    bufs, q = Buffers(), Async()
    acc_done = {}

    def producer():
        it = 0
        for t in range(n_tiles):
            for kb in range(nkb):
                s = it % stages
                yield wait(empty[s], ((it // stages) & 1) ^ 1, it // stages - 1)
                bufs.fill(("smem", s), 1)
                full[s].arrive_expect_tx(64)
                q.loads.append(lambda s=s: full[s].complete_tx(64))
                it += 1

    def mma():
        it = 0
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_empty[buf], ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
            bufs.fill(("acc", buf), 4)
            acc_done[buf] = 0
            for kb in range(nkb):
                s = it % stages
                yield wait(full[s], (it // stages) & 1, it // stages)

                def done(s=s, buf=buf):
                    acc_done[buf] += 1
                    bufs.release(("smem", s))
                    empty[s].arrive()
                q.mma.append(done)
                it += 1
            q.mma.append(lambda b=buf: acc_full[b].arrive())

    def epilogue(w):
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_full[buf], (j >> 1) & 1, j >> 1)
            assert acc_done[buf] == nkb, "epilogue read an accumulator before its MMAs completed"
            bufs.release(("acc", buf))
            acc_empty[buf].arrive()

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"epi{w}": epilogue(w) for w in range(4)})
    return roles, q


# ---------------------------------------------------------------- the 8-bit GEMM (k_tc_gemm_mx8.cu)

def lowp_gemm(n_tiles, nkb, stages, t_stages=4, dec_warps=8):
    f_full = [Barrier(f"f_full{s}", 1) for s in range(stages)]
    f_empty = [Barrier(f"f_empty{s}", dec_warps + 1) for s in range(stages)]
    t_full = [Barrier(f"t_full{s}", dec_warps) for s in range(t_stages)]
    t_empty = [Barrier(f"t_empty{s}", 1) for s in range(t_stages)]
    acc_full = [Barrier(f"acc_full{b}", 1) for b in range(2)]
    acc_empty = [Barrier(f"acc_empty{b}", 4) for b in range(2)]
    bufs, q = Buffers(), Async()
    acc_done = {}

    def producer():
        it = 0
        for t in range(n_tiles):
            for kb in range(nkb):
                s = it % stages
                yield wait(f_empty[s], ((it // stages) & 1) ^ 1, it // stages - 1)
                bufs.fill(("smem", s), dec_warps + 1)  # the decoders read the codes, the MMAs the tokens
                f_full[s].arrive_expect_tx(96)
                q.loads.append(lambda s=s: f_full[s].complete_tx(96))
                it += 1

    def mma():
        it = 0
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_empty[buf], ((j >> 1) & 1) ^ 1, (j >> 1) - 1)
            bufs.fill(("acc", buf), 4)
            acc_done[buf] = 0
            for kb in range(nkb):
                s, ts = it % stages, it % t_stages
                yield wait(t_full[ts], (it // t_stages) & 1, it // t_stages)
                yield wait(f_full[s], (it // stages) & 1, it // stages)
                assert tmem_writes.get(ts) == (it, dec_warps), "MMA read a TMEM stage not fully written"

                def done(s=s, ts=ts, buf=buf):
                    acc_done[buf] += 1
                    bufs.release(("tmem", ts))
                    t_empty[ts].arrive()
                    bufs.release(("smem", s))
                    f_empty[s].arrive()
                q.mma.append(done)
                it += 1
            q.mma.append(lambda b=buf: acc_full[b].arrive())

    def decoder(w):
        it = 0
        for t in range(n_tiles):
            for kb in range(nkb):
                s, ts = it % stages, it % t_stages
                yield wait(f_full[s], (it // stages) & 1, it // stages)
                yield wait(t_empty[ts], ((it // t_stages) & 1) ^ 1, it // t_stages - 1)
                write_tmem(ts, it)
                bufs.release(("smem", s))
                f_empty[s].arrive()
                t_full[ts].arrive()
                it += 1

    tmem_writes = {}

    def write_tmem(ts, it):
        # each decoder warp writes its part of TMEM stage ts for iteration it; the first
        # write fills the stage (one reader: the MMA), the MMA checks all parts are there
        last, n = tmem_writes.get(ts, (None, 0))
        if last != it:
            bufs.fill(("tmem", ts), 1)
            tmem_writes[ts] = (it, 1)
        else:
            tmem_writes[ts] = (it, n + 1)

    def epilogue(w):
        for j in range(n_tiles):
            buf = j & 1
            yield wait(acc_full[buf], (j >> 1) & 1, j >> 1)
            assert acc_done[buf] == nkb, "epilogue read an accumulator before its MMAs completed"
            bufs.release(("acc", buf))
            acc_empty[buf].arrive()

    roles = {"tma": producer(), "mma": mma()}
    roles.update({f"dec{w}": decoder(w) for w in range(dec_warps)})
    roles.update({f"epi{w}": epilogue(w) for w in range(4)})
    return roles, q


@pytest.mark.parametrize("n_tiles,nkb,stages", [(1, 1, 2), (3, 1, 3), (2, 5, 3), (5, 4, 6), (4, 32, 3), (7, 3, 8)])
def test_bf16_gemm_protocol(n_tiles, nkb, stages):
    for seed in range(30):
        roles, q = bf16_gemm(n_tiles, nkb, stages)
        run(roles, q, seed)


@pytest.mark.parametrize("n_tiles,nkb,stages", [(1, 1, 2), (3, 1, 6), (2, 5, 3), (5, 4, 6), (3, 16, 6), (6, 3, 2),
                                                (4, 7, 8)])
def test_lowp_gemm_protocol(n_tiles, nkb, stages):
    for seed in range(30):
        roles, q = lowp_gemm(n_tiles, nkb, stages)
        run(roles, q, seed)


def _lowp_with_count(f_empty_count, seed):
    orig = Barrier.__init__

    def patched(self, name, count):
        orig(self, name, f_empty_count if name.startswith("f_empty") else count)
    Barrier.__init__ = patched
    try:
        roles, q = lowp_gemm(3, 5, 2, dec_warps=8)
    finally:
        Barrier.__init__ = orig
    run(roles, q, seed)


def test_the_checker_catches_a_wrong_count():
    """With f_empty counting the decoder warps only (the MMAs' release of the token tiles
    not awaited), some interleaving must be reported: a stage overwritten while read, a
    release without a reader, a barrier run past its waiter, or a deadlock."""
    caught = 0
    for seed in range(100):
        try:
            _lowp_with_count(8, seed)
        except AssertionError:
            caught += 1
    assert caught > 0
    for seed in range(20):       # and the kernel's count passes the same interleavings
        _lowp_with_count(9, seed)
